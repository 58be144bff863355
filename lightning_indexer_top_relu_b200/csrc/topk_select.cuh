// Exact per-row top-k over fp32 scores (sm_100a, CUDA cores + shared memory).
//
// A row at absolute position t sees n = min(t+1, Lk) positions.  The result
// is the set of min(k, n) positions first in the order (score descending,
// position ascending), written in ascending position order and padded with -1
// (IndexCache: the F layer's indexer keeps the top-k positions per query,
// which later S layers reuse; the tie rule and the output order are this
// library's reading, the pages do not state them).
//
// Method: scores map to order-preserving 32-bit keys (-0 folded onto +0, so
// the order is the IEEE one).  Three radix passes (11, 11 and 10 bits, from
// the top) find the exact key T of the k-th largest element and how many of
// the k come from elements equal to T.  One last index-ordered pass emits
// every element > T plus the first `need` elements == T, each at its output
// slot found by a block-wide prefix count, so the output comes out sorted by
// position with no sort.  Rows that fit in shared memory are read from HBM
// once; longer rows are re-read from L2 on each pass.
#pragma once

#include "common.cuh"

namespace ic {

constexpr int TK_THREADS = 512;
constexpr int TK_WARPS = TK_THREADS / 32;
constexpr int TK_BINS = 2048;
constexpr int TK_ITEMS = 4;                                  // consecutive elements per thread
constexpr int TK_SMEM_FIXED = TK_BINS * 4 + 64 * 8 + 64;     // histogram + scan scratch
constexpr int TK_CACHE_MAX = 40960;                          // longest row kept in shared memory

__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u << 1) == 0u) u = 0u;                                // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of a 64-bit value; returns the exclusive prefix
// and sets `total`.  Every thread of the block must call it.
__device__ __forceinline__ unsigned long long tk_block_excl_scan(unsigned long long v,
                                                                 unsigned long long* scratch,
                                                                 unsigned long long& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        unsigned long long y = lane < TK_WARPS ? scratch[lane] : 0ull;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            unsigned long long z = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y += z;
        }
        if (lane < TK_WARPS) scratch[32 + lane] = y;
    }
    __syncthreads();
    const unsigned long long before = warp > 0 ? scratch[32 + warp - 1] : 0ull;
    total = scratch[32 + TK_WARPS - 1];
    __syncthreads();
    return before + x - v;
}

// Rows [row_base, row_base + n_rows) of a [B*Lq] flattened row space; score
// row r lives at scores + (r - row_base) * ld; output row r at idx + r * k.
template <bool CACHE>
__global__ void __launch_bounds__(TK_THREADS)
topk_select_kernel(const float* __restrict__ scores, long long ld, long long row_base,
                   long long n_rows, int Lq, int Lk, int q_offset, int k,
                   int32_t* __restrict__ idx) {
    extern __shared__ __align__(16) uint8_t tk_smem[];
    uint32_t* hist = reinterpret_cast<uint32_t*>(tk_smem);
    unsigned long long* scratch = reinterpret_cast<unsigned long long*>(tk_smem + TK_BINS * 4);
    int* found = reinterpret_cast<int*>(tk_smem + TK_BINS * 4 + 64 * 8);
    uint32_t* keys = reinterpret_cast<uint32_t*>(tk_smem + TK_SMEM_FIXED);

    const int tid = threadIdx.x;
    const long long rr = n_rows - 1 - (long long)blockIdx.x;   // longest rows first
    const long long r = row_base + rr;
    const int t = q_offset + (int)(r % Lq);
    const int n = min(t + 1, Lk);
    int32_t* out = idx + r * (long long)k;

    if (n <= k) {
        for (int i = tid; i < k; i += TK_THREADS) out[i] = i < n ? i : -1;
        return;
    }
    const float* src = scores + rr * ld;
    if (CACHE) {
        for (int i = tid; i < n; i += TK_THREADS) keys[i] = score_key(src[i]);
    }
    auto key_at = [&](int i) -> uint32_t { return CACHE ? keys[i] : score_key(__ldg(src + i)); };

    if (tid == 0) {
        found[0] = 0;
        found[1] = 0;
    }
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
        for (int b = tid; b < TK_BINS; b += TK_THREADS) hist[b] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += TK_THREADS) {
            const uint32_t key = key_at(i);
            if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
        }
        __syncthreads();
        // Thread tid owns bins [hi-3, hi] with hi = 2047 - 4*tid (top bins first).
        const int hi = TK_BINS - 1 - 4 * tid;
        uint32_t h[4];
        unsigned long long mine = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            h[e] = hist[hi - e];
            mine += h[e];
        }
        unsigned long long tot;
        unsigned long long above = tk_block_excl_scan(mine, scratch, tot);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (above < (unsigned long long)remaining && above + h[e] >= (unsigned long long)remaining) {
                found[0] = hi - e;
                found[1] = (int)above;
            }
            above += h[e];
        }
        __syncthreads();
        const uint32_t digit = (uint32_t)found[0];
        remaining -= found[1];
        prefix |= digit << shift;
        pmask |= dmask << shift;
        __syncthreads();
    }
    const uint32_t T = prefix;
    const int need = remaining;   // elements equal to T that are kept, lowest positions first

    long long base_gt = 0, base_eq = 0;
#pragma unroll 1
    for (int tile = 0; tile < n; tile += TK_THREADS * TK_ITEMS) {
        const int i0 = tile + tid * TK_ITEMS;
        uint32_t kk[TK_ITEMS];
        uint32_t cgt = 0, ceq = 0;
#pragma unroll
        for (int e = 0; e < TK_ITEMS; ++e) {
            const int i = i0 + e;
            kk[e] = i < n ? key_at(i) : 0u;
            if (i < n) {
                cgt += kk[e] > T;
                ceq += kk[e] == T;
            }
        }
        unsigned long long tot;
        const unsigned long long ex =
            tk_block_excl_scan(((unsigned long long)cgt << 32) | ceq, scratch, tot);
        long long g = base_gt + (long long)(ex >> 32);
        long long q = base_eq + (long long)(ex & 0xFFFFFFFFull);
#pragma unroll
        for (int e = 0; e < TK_ITEMS; ++e) {
            const int i = i0 + e;
            if (i >= n) break;
            if (kk[e] > T) {
                const long long pos = g + min(q, (long long)need);
                if (pos < k) out[pos] = i;
                ++g;
            } else if (kk[e] == T) {
                if (q < need && g + q < k) out[g + q] = i;
                ++q;
            }
        }
        base_gt += (long long)(tot >> 32);
        base_eq += (long long)(tot & 0xFFFFFFFFull);
    }
}

}  // namespace ic
