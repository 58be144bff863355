// Cross-layer overlap of two layers' index sets (sm_100a, CUDA cores).
//
// IndexCache rests on adjacent layers selecting largely the same positions
// (skill page, Step 1: compare consecutive layers' top-k sets per query
// position; kualia.ai review: adjacent layers share 70-100% of them).  Per
// row this kernel returns |A & B|, |A| and |B| of the two rows read as sets
// (-1 = empty slot, a repeated position counts once), from which the overlap
// fraction |A & B| / k and the Jaccard index |A & B| / |A | B| follow.
//
// Both rows become bitmaps over [0, Lk) in shared memory (one atomicOr per
// slot), then one pass of popcounts over the words counts |A|, |B| and
// |A & B|.  Up to OV_WARP_MAX_LK positions one warp handles a row (its two
// bitmaps in its own slice of shared memory, so a CTA has 8 rows in flight);
// longer rows take a whole CTA each.  Bound: HBM, 8 bytes read per slot pair.
#pragma once

#include "common.cuh"

namespace ic {

constexpr int OV_THREADS = 256;
constexpr int OV_MAX_LK = 262144;                  // two bitmaps of 32 KB
constexpr int OV_WARP_MAX_LK = 16384;              // per-warp bitmaps: 2 x 2 KB
constexpr int OV_VB = 8;                           // loads in flight per lane

// One warp per row (grid-stride over rows, 8 warps per CTA).
__global__ void __launch_bounds__(OV_THREADS)
index_overlap_warp_kernel(const int32_t* __restrict__ a, const int32_t* __restrict__ b,
                          long long n_rows, int k, int Lk, int32_t* __restrict__ counts) {
    extern __shared__ uint32_t ovw_smem[];
    const int W = (Lk + 31) >> 5;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t* bm_a = ovw_smem + warp * 2 * W;
    uint32_t* bm_b = bm_a + W;
    for (long long r = (long long)blockIdx.x * (OV_THREADS / 32) + warp; r < n_rows;
         r += (long long)gridDim.x * (OV_THREADS / 32)) {
        for (int w = lane; w < 2 * W; w += 32) bm_a[w] = 0u;
        __syncwarp();
        const int32_t* ra = a + r * (long long)k;
        const int32_t* rb = b + r * (long long)k;
        for (int s0 = 0; s0 < k; s0 += 32 * OV_VB) {
            int x[OV_VB], y[OV_VB];
#pragma unroll
            for (int u = 0; u < OV_VB; ++u) {          // the whole batch in flight first
                const int s = s0 + u * 32 + lane;
                x[u] = s < k ? __ldg(ra + s) : -1;
                y[u] = s < k ? __ldg(rb + s) : -1;
            }
#pragma unroll
            for (int u = 0; u < OV_VB; ++u) {
                if (x[u] >= 0 && x[u] < Lk) atomicOr(&bm_a[x[u] >> 5], 1u << (x[u] & 31));
                else if (x[u] != -1) report(DEV_ERR_BAD_INDEX);
                if (y[u] >= 0 && y[u] < Lk) atomicOr(&bm_b[y[u] >> 5], 1u << (y[u] & 31));
                else if (y[u] != -1) report(DEV_ERR_BAD_INDEX);
            }
        }
        __syncwarp();
        int both = 0, na = 0, nb = 0;
        for (int w = lane; w < W; w += 32) {
            const uint32_t u = bm_a[w], v = bm_b[w];
            na += __popc(u);
            nb += __popc(v);
            both += __popc(u & v);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            both += __shfl_xor_sync(0xffffffffu, both, o);
            na += __shfl_xor_sync(0xffffffffu, na, o);
            nb += __shfl_xor_sync(0xffffffffu, nb, o);
        }
        if (lane == 0) {
            counts[3 * r] = both;
            counts[3 * r + 1] = na;
            counts[3 * r + 2] = nb;
        }
        __syncwarp();
    }
}

// One CTA per row (grid-stride), for rows over more than OV_WARP_MAX_LK positions.

__global__ void __launch_bounds__(OV_THREADS)
index_overlap_kernel(const int32_t* __restrict__ a, const int32_t* __restrict__ b,
                     long long n_rows, int k, int Lk, int32_t* __restrict__ counts) {
    extern __shared__ uint32_t ov_smem[];
    const int W = (Lk + 31) >> 5;
    uint32_t* bm_a = ov_smem;
    uint32_t* bm_b = ov_smem + W;
    __shared__ int red[3][OV_THREADS / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (long long r = blockIdx.x; r < n_rows; r += gridDim.x) {
        for (int w = tid; w < 2 * W; w += OV_THREADS) ov_smem[w] = 0u;
        __syncthreads();
        const int32_t* ra = a + r * (long long)k;
        const int32_t* rb = b + r * (long long)k;
        for (int s = tid; s < k; s += OV_THREADS) {
            const int x = __ldg(ra + s), y = __ldg(rb + s);
            if (x >= 0 && x < Lk) atomicOr(&bm_a[x >> 5], 1u << (x & 31));
            else if (x != -1) report(DEV_ERR_BAD_INDEX);
            if (y >= 0 && y < Lk) atomicOr(&bm_b[y >> 5], 1u << (y & 31));
            else if (y != -1) report(DEV_ERR_BAD_INDEX);
        }
        __syncthreads();
        int both = 0, na = 0, nb = 0;
        for (int w = tid; w < W; w += OV_THREADS) {
            const uint32_t u = bm_a[w], v = bm_b[w];
            na += __popc(u);
            nb += __popc(v);
            both += __popc(u & v);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            both += __shfl_xor_sync(0xffffffffu, both, o);
            na += __shfl_xor_sync(0xffffffffu, na, o);
            nb += __shfl_xor_sync(0xffffffffu, nb, o);
        }
        if (lane == 0) {
            red[0][warp] = both;
            red[1][warp] = na;
            red[2][warp] = nb;
        }
        __syncthreads();
        if (tid < 3) {
            int sum = 0;
#pragma unroll
            for (int w = 0; w < OV_THREADS / 32; ++w) sum += red[tid][w];
            counts[3 * r + tid] = sum;
        }
        __syncthreads();
    }
}

}  // namespace ic
