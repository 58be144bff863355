// Exact per-row top-k over fp32 scores (sm_100a, CUDA cores + shared memory).
//
// A row at absolute position t sees n = min(t+1, Lk) positions.  The result
// is the set of min(k, n) positions first in the order (score descending,
// position ascending), written in ascending position order and padded with -1
// (IndexCache: the F layer's indexer keeps the top-k positions per query,
// which later S layers reuse; the tie rule and the output order are this
// library's reading, the pages do not state them).
//
// Method (one CTA per row):
//   1. One pass over the row maps every score to an order-preserving 32-bit
//      key (-0 folded onto +0, so the order is the IEEE one), keeps the keys
//      in shared memory when the row fits, and histograms the top 11 bits.
//   2. A suffix scan of the 2048 bins finds the bin holding the k-th largest
//      key.  Only that bin's keys (typically a few percent of the row) are
//      gathered as candidates, with one shared atomic per warp (ballot +
//      popc).  Each candidate is tagged with the warp whose step-3 segment
//      holds it.  The same pass counts each segment's keys of higher bins,
//      all of which are kept.  Two more radix passes (11 + 10 bits) over the
//      candidates give the exact k-th key T and `need`, how many keys equal
//      to T are kept.  A bin of more than TK_CAND keys (long tied rows) gets
//      no candidate list; the radix passes and the counts of step 3 then
//      read the whole row.
//   3. A final pass in position order emits every key > T and the first
//      `need` keys == T.  Each warp owns a contiguous segment; its counts of
//      keys > T and == T come from the candidate list.  One block-wide scan
//      of the per-warp counts gives every warp's first output slot, and the
//      warp writes its selections at ballot-prefix offsets -- sorted output,
//      no sort.  Rows that attend dense-masked also get their selection as
//      a bitmask row: lane 0 stores each 32-position ballot as one word.
// Every pass loads a whole batch (up to TK_VB float4 per thread) before
// using any of it, so a row costs one memory latency per batch instead of
// one per element.  Rows too long for shared memory re-read their scores
// from L2 in steps 2-3, batched the same way.
#pragma once

#include "common.cuh"

namespace ic {

// Threads per row.  Rows longer than TK_CACHE_MAX re-read their scores from
// L2/HBM; measured at L=65536, eight 256-thread CTAs per SM beat 2 x 512 and
// 1 x 1024 threads (more rows in flight outweigh keeping them in L2).  The
// same holds from 16K positions down: 16K rows took 0.72 ms per layer
// re-reading (eight CTAs per SM) against 0.90 ms cached (64 KB a CTA, three
// per SM), while 8K rows are faster cached (0.19 vs 0.21 ms: four per SM).
constexpr int TK_THREADS = 256;
constexpr int TK_THREADS_LONG = 256;
constexpr int TK_THREADS_FEW = 1024;     // fewer rows than 2 x SMs (decode): more threads per row
constexpr int TK_BINS = 2048;
constexpr int TK_CAND = 2048;                                     // candidate keys kept in smem
// hist + candidate keys + candidate warp ids + scratch
constexpr int TK_SMEM_FIXED = TK_BINS * 4 + TK_CAND * 4 + TK_CAND + 1024;
#ifndef IC_TK_CACHE_MAX
#define IC_TK_CACHE_MAX 8192
#endif
constexpr int TK_CACHE_MAX = IC_TK_CACHE_MAX;                     // longest row kept in smem
constexpr int TK_CACHE_MAX_FEW = 45056;   // the same with few rows (one 1024-thread CTA per SM)
constexpr int TK_VB = 8;                                          // float4 loads in flight per thread

// Sum of vals[w] over the warps w < warp (NW <= 32 per-warp totals in shared
// memory): each warp scans the NW totals with shuffles.
template <int NW>
__device__ __forceinline__ uint32_t tk_warps_before(const uint32_t* vals, int warp, int lane) {
    static_assert(NW >= 1 && NW <= 32, "one warp scans the totals");
    uint32_t x = lane < NW ? vals[lane] : 0u;
#pragma unroll
    for (int o = 1; o < NW; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    // inclusive scan at lane warp - 1 = the exclusive prefix of warp
    const uint32_t incl = __shfl_sync(0xffffffffu, x, warp > 0 ? warp - 1 : 0);
    return warp > 0 ? incl : 0u;
}

// Suffix scan of the 2048-bin histogram: finds the bin b whose count makes
// the running total (from the top bin down) reach `remaining`.  Writes
// found[0] = b, found[1] = count of elements in bins above b.  All threads.
template <int NT>
__device__ __forceinline__ void tk_find_bin(const uint32_t* hist, int remaining, int* found,
                                            unsigned* wsum) {
    constexpr int PER = TK_BINS / NT;              // bins per thread, top bins first
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hi = TK_BINS - 1 - PER * tid;
    uint32_t h[PER];
    uint32_t mine = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        h[e] = hist[hi - e];
        mine += h[e];
    }
    uint32_t x = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    const uint32_t before = tk_warps_before<NT / 32>(wsum, warp, lane);
    uint32_t above = before + x - mine;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        if (above < (uint32_t)remaining && above + h[e] >= (uint32_t)remaining) {
            found[0] = hi - e;
            found[1] = (int)above;
        }
        above += h[e];
    }
    __syncthreads();
}

// Block list of the fused top-k's exact fallback: the launch covers the
// query blocks blk_list[list_off ...] (at most list_len of them, as many as
// *blk_count says on the device); score row (entry - list_off) * QB + q holds
// query q of that block.  blk_list == nullptr selects the plain row range.
struct TopkList {
    const int* blk_list;
    const int* blk_count;
    int list_off, list_len, QB, nqb;
};

// Rows [row_base, row_base + n_rows) of a [B*Lq] flattened row space; score
// row r lives at scores + (r - row_base) * ld; output row r at idx + r * k.
// With `mask` non-null, rows i < Lq_d of each sequence also write their
// selection as a bitmask: row b*Lq_d + i of `mask` ([*, W] words) gets bit s
// set for every selected position s (words past the row's visible positions
// are zero).  The emit pass builds it from the ballots it already takes.
// A CTA loops over rows (gridDim.x apart), so a persistent grid can take a
// block list whose length only the device knows.
template <int NT, bool CACHE>
__global__ void __launch_bounds__(NT)
topk_select_kernel(const float* __restrict__ scores, long long ld, long long row_base,
                   long long n_rows, int Lq, int Lk, int q_offset, int k,
                   int32_t* __restrict__ idx, uint32_t* __restrict__ mask, int Lq_d, int W,
                   const TopkList lst) {
    constexpr int NW = NT / 32;
    static_assert(4 + 6 * NW <= 256, "scratch words");
    extern __shared__ __align__(16) uint8_t tk_smem[];
    uint32_t* hist = reinterpret_cast<uint32_t*>(tk_smem);
    uint32_t* cand = reinterpret_cast<uint32_t*>(tk_smem + TK_BINS * 4);
    uint8_t* cand_w = tk_smem + TK_BINS * 4 + TK_CAND * 4;                       // warp of each candidate
    int* found = reinterpret_cast<int*>(tk_smem + TK_BINS * 4 + TK_CAND * 5);      // [0..3]
    unsigned* wsum = reinterpret_cast<unsigned*>(found + 4);                        // [NW]
    unsigned* wgt = wsum + NW;                                                // [NW] keys > T
    unsigned* weq = wgt + NW;                                                 // [NW] keys == T
    unsigned* wdef = weq + NW;                                                // [NW] bins above b1
    unsigned* cgt = wdef + NW;                                                // [NW] candidates > T
    unsigned* ceq = cgt + NW;                                                 // [NW] candidates == T
    uint32_t* keys = reinterpret_cast<uint32_t*>(tk_smem + TK_SMEM_FIXED);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    long long n_iter = n_rows;
    if (lst.blk_list != nullptr) {
        long long have = (long long)__ldg(lst.blk_count) - lst.list_off;
        have = have < 0 ? 0 : (have < lst.list_len ? have : lst.list_len);
        n_iter = have * lst.QB;
    }
    for (long long it = blockIdx.x; it < n_iter; it += gridDim.x) {
        __syncthreads();                                           // shared memory of the last row is free
        long long r;
        const float* src;
        if (lst.blk_list != nullptr) {
            const int g = __ldg(lst.blk_list + lst.list_off + it / lst.QB);
            const int i = (g % lst.nqb) * lst.QB + (int)(it % lst.QB);
            if (i >= Lq) continue;                                 // past the last query of the block
            r = (long long)(g / lst.nqb) * Lq + i;
            src = scores + it * ld;
        } else {
            const long long rr = n_rows - 1 - it;                  // longest rows first
            r = row_base + rr;
            src = scores + rr * ld;
        }
        const int t = q_offset + (int)(r % Lq);
        const int n = min(t + 1, Lk);
        int32_t* out = idx + r * (long long)k;
        uint32_t* mrow = nullptr;
        if (mask != nullptr && (int)(r % Lq) < Lq_d)
            mrow = mask + ((r / Lq) * Lq_d + r % Lq) * (long long)W;
        const int nw = (n + 31) >> 5;                                 // words with visible positions
        if (mrow != nullptr)
            for (int w = nw + tid; w < W; w += NT) mrow[w] = 0u;

        if (n <= k) {
            for (int i = tid; i < k; i += NT) out[i] = i < n ? i : -1;
            if (mrow != nullptr)
                for (int w = tid; w < nw && w < W; w += NT)
                    mrow[w] = (32 * w + 32 <= n) ? 0xffffffffu : ((1u << (n - 32 * w)) - 1u);
            continue;
        }
        auto key_at = [&](int i) -> uint32_t { return CACHE ? keys[i] : score_key(__ldg(src + i)); };

        // ---- 1. keys + top-11-bit histogram in one pass
        for (int b = tid; b < TK_BINS; b += NT) hist[b] = 0;
        if (tid == 0) found[2] = 0;                                // candidate count
        __syncthreads();
        const bool vec = ((reinterpret_cast<uintptr_t>(src) & 15) == 0);
        const int nv = vec ? (n & ~3) : 0;
        for (int base = 0; base < nv; base += NT * 4 * TK_VB) {
            float4 f[TK_VB];
#pragma unroll
            for (int u = 0; u < TK_VB; ++u) {           // all loads of the batch first
                const int i = base + (u * NT + tid) * 4;
                f[u] = i < nv ? __ldg(reinterpret_cast<const float4*>(src + i))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < TK_VB; ++u) {
                const int i = base + (u * NT + tid) * 4;
                if (i < nv) {
                    const uint32_t k0 = score_key(f[u].x), k1 = score_key(f[u].y),
                                   k2 = score_key(f[u].z), k3 = score_key(f[u].w);
                    if (CACHE) *reinterpret_cast<uint4*>(keys + i) = make_uint4(k0, k1, k2, k3);
                    atomicAdd(&hist[k0 >> 21], 1u);
                    atomicAdd(&hist[k1 >> 21], 1u);
                    atomicAdd(&hist[k2 >> 21], 1u);
                    atomicAdd(&hist[k3 >> 21], 1u);
                }
            }
        }
        for (int i = nv + tid; i < n; i += NT) {
            const uint32_t kk = score_key(__ldg(src + i));
            if (CACHE) keys[i] = kk;
            atomicAdd(&hist[kk >> 21], 1u);
        }
        __syncthreads();

        tk_find_bin<NT>(hist, k, found, wsum);
        const uint32_t b1 = (uint32_t)found[0];
        int remaining = k - found[1];
        const uint32_t cnt1 = hist[b1];
        __syncthreads();                                           // hist is reused below

        // ---- 2. candidates of the threshold bin, then two radix passes on them.
        // Warp w scans the positions [w*seg, (w+1)*seg) it also emits in step 3,
        // counting the keys of higher bins (all kept) and gathering the bin's
        // keys with its warp id, so that step 3 needs no counting pass.
        const int seg = ((n + NW * 32 - 1) / (NW * 32)) * 32;
        const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
        uint32_t prefix = b1 << 21;
        uint32_t pmask = 0x7FFu << 21;
        const bool use_cand = cnt1 <= (uint32_t)TK_CAND;
        if (use_cand) {
            unsigned cdef = 0;
            for (int gbase = s0; gbase < s1; gbase += 32 * TK_VB) {
                uint32_t kb[TK_VB];
#pragma unroll
                for (int u = 0; u < TK_VB; ++u) {
                    const int i = gbase + u * 32 + lane;
                    kb[u] = i < s1 ? key_at(i) : 0u;
                }
#pragma unroll
                for (int u = 0; u < TK_VB; ++u) {
                    const int i = gbase + u * 32 + lane;
                    cdef += __popc(__ballot_sync(0xffffffffu, i < s1 && (kb[u] >> 21) > b1));
                    const bool m = i < s1 && (kb[u] >> 21) == b1;
                    const unsigned bal = __ballot_sync(0xffffffffu, m);
                    if (bal) {
                        unsigned pos0 = 0;
                        if (lane == 0) pos0 = atomicAdd(reinterpret_cast<unsigned*>(&found[2]), __popc(bal));
                        pos0 = __shfl_sync(0xffffffffu, pos0, 0);
                        if (m) {
                            const unsigned c = pos0 + __popc(bal & ((1u << lane) - 1u));
                            cand[c] = kb[u];
                            cand_w[c] = (uint8_t)warp;
                        }
                    }
                }
            }
            if (lane == 0) {
                wdef[warp] = cdef;
                cgt[warp] = 0u;
                ceq[warp] = 0u;
            }
        }
        for (int pass = 1; pass < 3; ++pass) {
            const int shift = pass == 1 ? 10 : 0;
            const uint32_t dmask = pass == 1 ? 0x7FFu : 0x3FFu;
            for (int b = tid; b < TK_BINS; b += NT) hist[b] = 0;
            __syncthreads();
            if (use_cand) {
                for (int i = tid; i < (int)cnt1; i += NT) {
                    const uint32_t kk = cand[i];
                    if ((kk & pmask) == prefix) atomicAdd(&hist[(kk >> shift) & dmask], 1u);
                }
            } else {
                for (int base = 0; base < n; base += NT * TK_VB) {
                    uint32_t kb[TK_VB];
#pragma unroll
                    for (int u = 0; u < TK_VB; ++u) {
                        const int i = base + u * NT + tid;
                        kb[u] = i < n ? key_at(i) : 0u;
                    }
#pragma unroll
                    for (int u = 0; u < TK_VB; ++u) {
                        const int i = base + u * NT + tid;
                        if (i < n && (kb[u] & pmask) == prefix)
                            atomicAdd(&hist[(kb[u] >> shift) & dmask], 1u);
                    }
                }
            }
            __syncthreads();
            tk_find_bin<NT>(hist, remaining, found, wsum);
            remaining -= found[1];
            prefix |= (uint32_t)found[0] << shift;
            pmask |= dmask << shift;
            __syncthreads();
        }
        const uint32_t T = prefix;
        const int need = remaining;   // keys equal to T that are kept, lowest positions first

        // ---- 3. emit in position order: warp w owns [w*seg, (w+1)*seg).  Per
        // warp, keys > T = higher bins + candidates > T; keys == T = candidates
        // == T (from the candidate list), or one counting pass without it.
        if (use_cand) {
            for (int c = tid; c < (int)cnt1; c += NT) {
                const uint32_t kk = cand[c];
                if (kk > T) atomicAdd(&cgt[cand_w[c]], 1u);
                else if (kk == T) atomicAdd(&ceq[cand_w[c]], 1u);
            }
            __syncthreads();
            if (tid < NW) {
                wgt[tid] = wdef[tid] + cgt[tid];
                weq[tid] = ceq[tid];
            }
        } else {
            unsigned cg = 0, ce = 0;
            for (int gbase = s0; gbase < s1; gbase += 32 * TK_VB) {
                uint32_t kb[TK_VB];
#pragma unroll
                for (int u = 0; u < TK_VB; ++u) {
                    const int i = gbase + u * 32 + lane;
                    kb[u] = i < s1 ? key_at(i) : 0u;
                }
#pragma unroll
                for (int u = 0; u < TK_VB; ++u) {
                    const int i = gbase + u * 32 + lane;
                    cg += __popc(__ballot_sync(0xffffffffu, i < s1 && kb[u] > T));
                    ce += __popc(__ballot_sync(0xffffffffu, i < s1 && kb[u] == T));
                }
            }
            if (lane == 0) {
                wgt[warp] = cg;
                weq[warp] = ce;
            }
        }
        __syncthreads();
        unsigned g = tk_warps_before<NW>(wgt, warp, lane);
        unsigned e = tk_warps_before<NW>(weq, warp, lane);
        const unsigned lt = (1u << lane) - 1u;
        if (tk_warps_before<NW>(weq, NW, lane) == (unsigned)need) {
            // Every key equal to T is kept (the usual case: T is unique), so
            // the selection is {key >= T}, exactly k keys: one ballot per 32
            // positions gives both the output slots and the mask word.
            unsigned base = g + e;
            for (int gbase = s0; gbase < s1; gbase += 32 * TK_VB) {
                uint32_t kb[TK_VB];
#pragma unroll
                for (int u = 0; u < TK_VB; ++u) {
                    const int i = gbase + u * 32 + lane;
                    kb[u] = i < s1 ? key_at(i) : 0u;
                }
#pragma unroll
                for (int u = 0; u < TK_VB; ++u) {
                    const int i = gbase + u * 32 + lane;
                    const unsigned ms = __ballot_sync(0xffffffffu, i < s1 && kb[u] >= T);
                    if ((ms >> lane) & 1u) out[base + __popc(ms & lt)] = i;
                    if (mrow != nullptr) {
                        const int w0 = (gbase + u * 32) >> 5;
                        if (lane == 0 && gbase + u * 32 < s1 && w0 < W) mrow[w0] = ms;
                    }
                    base += __popc(ms);
                }
            }
            continue;
        }
        for (int gbase = s0; gbase < s1; gbase += 32 * TK_VB) {
            uint32_t kb[TK_VB];
#pragma unroll
            for (int u = 0; u < TK_VB; ++u) {
                const int i = gbase + u * 32 + lane;
                kb[u] = i < s1 ? key_at(i) : 0u;
            }
#pragma unroll
            for (int u = 0; u < TK_VB; ++u) {
                const int i = gbase + u * 32 + lane;
                const unsigned mg = __ballot_sync(0xffffffffu, i < s1 && kb[u] > T);
                const unsigned me = __ballot_sync(0xffffffffu, i < s1 && kb[u] == T);
                const unsigned gi = g + __popc(mg & lt);
                const unsigned ei = e + __popc(me & lt);
                bool sel = false;
                if ((mg >> lane) & 1u) {
                    const unsigned pos = gi + min(ei, (unsigned)need);
                    if (pos < (unsigned)k) {
                        out[pos] = i;
                        sel = true;
                    }
                } else if (((me >> lane) & 1u) && ei < (unsigned)need) {
                    const unsigned pos = gi + ei;
                    if (pos < (unsigned)k) {
                        out[pos] = i;
                        sel = true;
                    }
                }
                if (mrow != nullptr) {
                    // 32 consecutive positions starting at a multiple of 32
                    const unsigned word = __ballot_sync(0xffffffffu, sel);
                    const int w0 = (gbase + u * 32) >> 5;
                    if (lane == 0 && gbase + u * 32 < s1 && w0 < W) mrow[w0] = word;
                }
                g += __popc(mg);
                e += __popc(me);
            }
        }
    }   // rows
}

}  // namespace ic
