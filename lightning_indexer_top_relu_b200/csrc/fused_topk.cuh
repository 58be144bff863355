// Fused indexer -> top-k: the per-row threshold and the exact selection over
// candidate lists (sm_100a, CUDA cores + shared memory).
//
// The full F-layer score matrix is never stored.  For each query row the
// stack (1) scores a sample of the key tiles (every stride-th tile, the
// indexer's IDX_SAMPLE mode), (2) picks from those samples a threshold key
// that at least k of the row's scores reach with high probability
// (fused_threshold_kernel), (3) runs the whole indexer again storing only the
// scores at or above the threshold, as candidates (IDX_CAND mode), and
// (4) selects the row's top k among its candidates (fused_select_kernel).
// The result is exact whenever the row has at least k candidates and they
// all fit in its list: every score above the k-th largest is then at or
// above the threshold too, so the true top-k (ties included) is among the
// candidates.  Rows for which that fails flag their query block; the stack
// re-runs flagged blocks through the plain indexer + top-k, so the result is
// exact for every row whatever the threshold did (the kualia.ai review, "The
// Hidden Quadratic": the indexer's O(L^2) share of prefill; the fusion keeps
// its score matrix on chip).
//
// Candidates are 64-bit values (key << 32) | ~s, key the order-preserving
// key of the score: unsigned order is then (score descending, position
// ascending), the selection order of the top-k, and every value is distinct.
#pragma once

#include "common.cuh"

namespace ic {

constexpr int FT_THREADS = 128;        // threshold kernel: threads per row
constexpr int FS_THREADS = 256;        // select kernel: threads per row
constexpr int FT_MAX_SAMPLES = 4096;   // sampled scores per row at most (32 tiles)

// k-th largest (1-based, 1 <= kth <= n) of vals[0, n) in shared memory, by
// most-significant-digit radix selection with 8-bit digits.  hist: 256 words
// of shared memory; sc: 4 words; one: a slot for the value.  Every thread of
// the block calls it and gets the value.  When the digit bin holding the
// k-th value has a single member, one more pass reads that member and the
// remaining digits are skipped.
template <typename T, int NT>
__device__ T block_kth_largest(const T* vals, int n, int kth, uint32_t* hist, int* sc, T* one) {
    constexpr int BITS = (int)sizeof(T) * 8;
    T prefix = 0;
    int remaining = kth;
    for (int shift = BITS - 8; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += NT) hist[i] = 0u;
        __syncthreads();
        const T hmask = (shift + 8 >= BITS) ? T(0) : (~T(0) << (shift + 8));   // digits fixed so far
        for (int i = threadIdx.x; i < n; i += NT) {
            const T v = vals[i];
            if ((v & hmask) == (prefix & hmask)) atomicAdd(&hist[(uint32_t)(v >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane l holds bins 255 - 8l ... 248 - 8l (top bins first)
            const int lane = threadIdx.x;
            uint32_t h[8], sum = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                h[e] = hist[255 - 8 * lane - e];
                sum += h[e];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t above = incl - sum;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (above < (uint32_t)remaining && above + h[e] >= (uint32_t)remaining) {
                    sc[0] = 255 - 8 * lane - e;
                    sc[1] = (int)above;
                    sc[2] = (int)h[e];
                }
                above += h[e];
            }
        }
        __syncthreads();
        const int b = sc[0];
        remaining -= sc[1];
        const int members = sc[2];
        prefix |= (T)b << shift;
        __syncthreads();                          // sc and hist are rewritten below
        if (members == 1 && shift > 0) {
            const T m2 = ~T(0) << shift;
            for (int i = threadIdx.x; i < n; i += NT)
                if ((vals[i] & m2) == prefix) *one = vals[i];
            __syncthreads();
            const T v = *one;
            __syncthreads();
            return v;
        }
    }
    return prefix;
}

// Exclusive prefix sum of one value per thread over the block; total in *tot.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t* wsum, uint32_t* tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        before += (w < warp) ? wsum[w] : 0u;
        all += wsum[w];
    }
    if (threadIdx.x == 0) *tot = all;
    __syncthreads();
    return before + incl - x;
}

struct FusedArgs {
    long long row_base, n_rows;   // flattened rows [row_base, row_base + n_rows) of this chunk
    int Lq, Lk, q_offset, k;
    int cap;                      // candidates a row may keep; rows with n <= cap keep all
    int lstride;                  // list slots per row (cap + room for unused reserved slots)
    int stride;                   // sampled key tiles: m * stride
    int ns;                       // sample tiles per sample row (row stride ns * 128)
    float z;                      // threshold margin, in binomial standard deviations
    int QB, nqb;
    long long g0;                 // flattened query block of the chunk's first row
    long long n_blocks;           // query blocks of the chunk
    const float* samp;            // [n_rows, ns * 128] sampled scores (-inf past t)
    uint32_t* thr;                // [n_rows] threshold key
    uint32_t* cnt;                // [n_rows] candidates found
    const unsigned long long* cand;   // [n_rows, lstride]
    uint32_t* bflag;              // [n_blocks] block needs the exact fallback
    int* blist;                   // [n_blocks] flagged blocks (global block ids)
    int* list_count;              // number of flagged blocks
    int32_t* idx;                 // [B*Lq, k] output rows
    uint32_t* mask;               // bitmask rows of dense-masked rows, or null
    int Lq_d, W;
};

// Sampled key tiles m = 0, 1, ... visible to a row at position t hold
// min(128, t - m*stride*128 + 1) visible scores each.
__device__ __forceinline__ int visible_samples(int t, int stride, int ns) {
    const int span = stride * 128;
    const int tiles = min(ns, t / span + 1);
    int m = 0;
    for (int i = 0; i < tiles; ++i) m += min(128, t - i * span + 1);
    return m;
}

// Per row: the threshold key, and the row's candidate counter cleared.  Rows
// with n <= k visible positions keep them all and need no candidate (key
// 0xFFFFFFFF: no score reaches it); rows with at most cap take key 0 (every
// visible score is a candidate).  Other rows, with m visible
// samples and p = k / n, take the r-th largest sampled key,
// r = ceil(m p + z sqrt(m p (1-p))) + 1, so the row's share of scores at or
// above it exceeds p unless the sample is off by about z standard
// deviations.  Also clears the chunk's block flags and the flagged-block
// count.
__global__ void __launch_bounds__(FT_THREADS)
fused_threshold_kernel(const FusedArgs a) {
    __shared__ uint32_t vals[FT_MAX_SAMPLES];
    __shared__ uint32_t hist[256];
    __shared__ int sc[4];
    __shared__ uint32_t one;
    for (long long b = (long long)blockIdx.x * FT_THREADS + threadIdx.x; b < a.n_blocks;
         b += (long long)gridDim.x * FT_THREADS)
        a.bflag[b] = 0u;
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.list_count = 0;
    for (long long rr = blockIdx.x; rr < a.n_rows; rr += gridDim.x) {
        const long long r = a.row_base + rr;
        const int t = a.q_offset + (int)(r % a.Lq);
        const int n = min(t + 1, a.Lk);
        if (threadIdx.x == 0) a.cnt[rr] = 0u;
        if (n <= a.cap) {
            if (threadIdx.x == 0) a.thr[rr] = n <= a.k ? 0xFFFFFFFFu : 0u;
            continue;
        }
        const int span = a.stride * 128;
        const int tiles = min(a.ns, t / span + 1);
        int m = 0;
        const float* srow = a.samp + rr * (long long)a.ns * 128;
        __syncthreads();                          // vals of the previous row are consumed
        for (int i = threadIdx.x; i < tiles * 128; i += FT_THREADS) {
            const int s = (i >> 7) * span + (i & 127);
            if (s <= t) {
                // compact: visible samples of tile i>>7 start after the full
                // tiles before it (every tile but the last is fully visible)
                vals[i] = score_key(srow[i]);
            }
        }
        m = visible_samples(t, a.stride, a.ns);
        __syncthreads();
        const double p = (double)a.k / (double)n;
        const double mean = (double)m * p;
        long long want = (long long)ceil(mean + (double)a.z * sqrt(mean * (1.0 - p))) + 1;
        uint32_t key = 0u;
        if (want <= m) key = block_kth_largest<uint32_t, FT_THREADS>(vals, m, (int)want, hist, sc, &one);
        if (threadIdx.x == 0) a.thr[rr] = key;
    }
}

// Per row: the exact top-k over the row's candidates when there are at least
// k of them and none was dropped (the row's reserved slots, counted by the
// counter, fit in the list); otherwise the row's query block is flagged (and
// listed once) for the exact fallback.  Reserved slots the indexer left
// unused hold 0 and are not counted.  The selection is the k largest
// candidate values (key << 32 | ~s, all distinct).  Only the 32-bit score
// keys stay in shared memory (so four CTAs share an SM): the k-th largest key
// T is selected on them; every candidate with a larger key is kept, and of
// those whose key equals T the lowest positions are kept, as many as the top
// k needs (a second selection over the tied positions, only when ties are
// cut).  The positions come from a second read of the row's list, which is
// still in L2, and go through a bitmap of the row's visible positions that
// yields them in ascending order and is also the row's selection bitmask
// when the row attends dense-masked.
__global__ void __launch_bounds__(FS_THREADS)
fused_select_kernel(const FusedArgs a) {
    extern __shared__ __align__(16) uint8_t fs_smem[];
    uint32_t* hist = reinterpret_cast<uint32_t*>(fs_smem);                  // 256
    int* sc = reinterpret_cast<int*>(fs_smem + 1024);                       // 4
    uint32_t* wsum = reinterpret_cast<uint32_t*>(fs_smem + 1040);           // 8
    uint32_t* tot = wsum + FS_THREADS / 32;                                 // 1
    uint32_t* one = reinterpret_cast<uint32_t*>(fs_smem + 1088);
    uint32_t* nties = reinterpret_cast<uint32_t*>(fs_smem + 1092);
    uint32_t* keys = reinterpret_cast<uint32_t*>(fs_smem + 1152);                       // lstride
    uint32_t* bm = reinterpret_cast<uint32_t*>(fs_smem + 1152 + (size_t)a.lstride * 4); // words

    const int tid = threadIdx.x;
    const long long rr = a.n_rows - 1 - (long long)blockIdx.x;   // longest rows first
    const long long r = a.row_base + rr;
    const int i = (int)(r % a.Lq);
    const int t = a.q_offset + i;
    const int n = min(t + 1, a.Lk);
    const int nw = (n + 31) >> 5;
    int32_t* out = a.idx + r * (long long)a.k;
    uint32_t* mrow = nullptr;
    if (a.mask != nullptr && i < a.Lq_d) mrow = a.mask + ((r / a.Lq) * a.Lq_d + i) * (long long)a.W;

    if (n <= a.k) {
        for (int s = tid; s < a.k; s += FS_THREADS) out[s] = s < n ? s : -1;
        if (mrow != nullptr)
            for (int w = tid; w < a.W; w += FS_THREADS)
                mrow[w] = w >= nw ? 0u : ((32 * w + 32 <= n) ? 0xffffffffu : ((1u << (n - 32 * w)) - 1u));
        return;
    }
    const uint32_t c = __ldg(a.cnt + rr);
    const unsigned long long* crow = a.cand + rr * (long long)a.lstride;
    uint32_t valid = 0;
    if (c <= (uint32_t)a.lstride) {                 // uniform
        // The list in pairs (lstride is even, so a row starts 16-byte
        // aligned and the pair holding entry c-1 lies inside the row), four
        // independent 16-byte loads per thread in flight.
        const ulonglong2* crow2 = reinterpret_cast<const ulonglong2*>(crow);
        const uint32_t npair = (c + 1) / 2;
        uint32_t mine = 0;
        for (uint32_t p0 = tid; p0 < npair; p0 += 4 * FS_THREADS) {
            ulonglong2 x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (p0 + u * FS_THREADS < npair) x[u] = __ldg(crow2 + p0 + u * FS_THREADS);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t pj = p0 + u * FS_THREADS;
                if (pj < npair) {
                    keys[2 * pj] = (uint32_t)(x[u].x >> 32);
                    mine += x[u].x != 0ull;
                    if (2 * pj + 1 < c) {
                        keys[2 * pj + 1] = (uint32_t)(x[u].y >> 32);
                        mine += x[u].y != 0ull;
                    }
                }
            }
        }
        block_excl_scan<FS_THREADS>(mine, wsum, tot);
        valid = *tot;
    }
    if (c > (uint32_t)a.lstride || valid < (uint32_t)a.k) {
        if (tid == 0) {
            const long long g = (r / a.Lq) * a.nqb + i / a.QB;
            if (atomicExch(a.bflag + (g - a.g0), 1u) == 0u) {
                const int pos = atomicAdd(a.list_count, 1);
                a.blist[pos] = (int)g;
            }
        }
        return;
    }
    for (int w = tid; w < nw; w += FS_THREADS) bm[w] = 0u;
    if (tid == 0) *nties = 0u;
    __syncthreads();
    // Padding keys are 0, below every key of a finite score, so with at
    // least k candidates the k-th largest key T is a candidate's.
    const uint32_t T = block_kth_largest<uint32_t, FS_THREADS>(keys, (int)c, a.k, hist, sc, one);
    uint32_t gt = 0, eq = 0;
    for (uint32_t j = tid; j < c; j += FS_THREADS) {
        const uint32_t kk = keys[j];
        gt += kk > T;
        eq += kk == T;
    }
    block_excl_scan<FS_THREADS>(gt, wsum, tot);
    const uint32_t n_gt = *tot;
    __syncthreads();                                   // tot is rewritten below
    block_excl_scan<FS_THREADS>(eq, wsum, tot);
    const uint32_t n_eq = *tot;
    const uint32_t need = (uint32_t)a.k - n_gt;        // candidates with key T that are kept
    // Every candidate with key T is kept when exactly `need` of them exist
    // (T > 0: padding cannot share the key).  Otherwise the kept ones are the
    // `need` lowest positions: the need-th largest ~s among them.
    const bool all_ties = T != 0u && n_eq == need;     // uniform
    uint32_t cut = 0u;
    if (!all_ties) {
        __syncthreads();                               // keys[] is free: it collects ~s of the ties
        for (uint32_t j = tid; j < c; j += FS_THREADS) {
            const unsigned long long v = __ldg(crow + j);
            if (v != 0ull && (uint32_t)(v >> 32) == T) keys[atomicAdd(nties, 1u)] = (uint32_t)v;
        }
        __syncthreads();
        cut = block_kth_largest<uint32_t, FS_THREADS>(keys, (int)*nties, (int)need, hist, sc, one);
    }
    // positions from a second read of the list (in L2 since the first)
    for (uint32_t j = tid; j < c; j += FS_THREADS) {
        const unsigned long long v = __ldg(crow + j);
        const uint32_t kk = (uint32_t)(v >> 32), lo = (uint32_t)v;
        if (v != 0ull && (kk > T || (kk == T && (all_ties || lo >= cut)))) {
            const uint32_t s = ~lo;
            atomicOr(&bm[s >> 5], 1u << (s & 31));
        }
    }
    __syncthreads();
    // each thread owns a contiguous run of words; the scan of their bit
    // counts gives every run's first output slot
    const int per = (nw + FS_THREADS - 1) / FS_THREADS;
    const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
    uint32_t mine = 0;
    for (int w = w0; w < w1; ++w) mine += __popc(bm[w]);
    uint32_t slot = block_excl_scan<FS_THREADS>(mine, wsum, tot);
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = bm[w];
        while (bits) {
            const int bpos = __ffs(bits) - 1;
            bits &= bits - 1u;
            if (slot < (uint32_t)a.k) out[slot] = 32 * w + bpos;
            ++slot;
        }
    }
    if (mrow != nullptr)
        for (int w = tid; w < a.W; w += FS_THREADS) mrow[w] = w < nw ? bm[w] : 0u;
}

// Shared memory of fused_select_kernel for a list of lstride slots and a row
// length (bitmap words).
__host__ __device__ constexpr size_t fused_select_smem(int lstride, int Lk) {
    return 1152 + (size_t)lstride * 4 + (size_t)((Lk + 31) / 32) * 4;
}

}  // namespace ic
