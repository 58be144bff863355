// Cross-layer overlap of two layers' index sets (sm_100a, CUDA cores).
//
// IndexCache rests on adjacent layers selecting largely the same positions
// (skill page, Step 1: compare consecutive layers' top-k sets per query
// position; kualia.ai review: adjacent layers share 70-100% of them).  Per
// row this kernel returns |A & B|, |A| and |B| of the two rows read as sets
// (-1 = empty slot, a repeated position counts once), from which the overlap
// fraction |A & B| / k and the Jaccard index |A & B| / |A | B| follow.
//
// One CTA per row (grid-stride): both rows become bitmaps over [0, Lk) in
// shared memory (one atomicOr per slot), then one pass of popcounts over the
// words counts |A|, |B| and |A & B|.  Bound: HBM, 8 bytes read per slot pair.
#pragma once

#include "common.cuh"

namespace ic {

constexpr int OV_THREADS = 256;
constexpr int OV_MAX_LK = 262144;                  // two bitmaps of 32 KB

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
