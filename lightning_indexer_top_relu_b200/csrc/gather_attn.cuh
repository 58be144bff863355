// Sparse MQA attention over gathered K/V rows, loaded straight into tensor-core
// fragments (sm_100a).
//
// For query row t and head h, over the slots i whose index idx_i is valid:
//   z_i = scale * q[t,h] . K[idx_i],  out = sum_i softmax(z)_i V[idx_i]
// (IndexCache: every layer, F or S, attends sparsely over the k positions
// held in the index cache; all query heads share the one K/V head).
//
// The K/V rows a query selects are scattered over the layer's keys, so the
// kernel is bound by how fast rows can be gathered.  Rows are read with
// 16-byte global loads directly into registers, already in the register
// layout of the m16n8k16 tensor-core fragments, with no shared-memory
// staging:
//   * QK^T sums over the head dimension, so Q and K may both have their
//     dimension permuted the same way: thread (g, c) of a warp (g = lane/4,
//     c = lane%4) loads bytes [64u + 16c, +16) of each 128-byte unit u of a
//     row, four threads reading 64 contiguous bytes per load, and those
//     registers are exactly its B-fragment pairs of the permuted dimension;
//   * PV needs V with slots along the fragment's k axis: each 8 x 8 block of
//     V (8 slots x 8 dimensions, one register per thread) is transposed in
//     registers by movmatrix; with the same permutation, every thread's
//     output fragment covers 8 consecutive dimensions of two heads.
// A pair of warps shares each group of 16 slots: warp h of the pair holds
// dimension half h of Q, K, V and O, computes its half of the QK^T partial
// sums, and the two halves are added through shared memory (the same sum in
// both warps, so both run the same softmax).  Halving the dimension per warp
// halves the registers a warp holds per slot, which leaves room to keep the
// loads of the next two groups in flight while one is computed.
// The CTA's pairs take interleaved groups of the row's slots; their partial
// (max, sum, O) merge through shared memory at the end, and rows split over
// several CTAs (decode) write per-split partials for the combine kernel.
#pragma once

#include "common.cuh"
#include "sparse_attn.cuh"

namespace ic {

constexpr int GA_WARPS = 4;                       // 2 pairs per CTA, 3 CTAs per SM
constexpr int GA_PAIRS = GA_WARPS / 2;
constexpr int GA_THREADS = 32 * GA_WARPS;
constexpr int GA_GROUP = 16;                      // slots per pair iteration
constexpr int GA_NBUF = 3;                        // groups in registers: 1 computed, 2 loading

template <int D>
struct GaSmem {
    static constexpr int OFF_IDX = 0;                                     // SA_IDX_TILE ints
    static constexpr int OFF_X = OFF_IDX + SA_IDX_TILE * 4;               // S exchange
    static constexpr int X_BYTES = GA_PAIRS * 2 * 2 * 2 * 32 * 16;        // [pair][half][parity][chunk][lane] float4
    static constexpr int OFF_MO = OFF_X + X_BYTES;                        // [pair][16][D] f32
    static constexpr int OFF_ML = OFF_MO + GA_PAIRS * 16 * D * 4;         // [pair][16][2] f32
    static constexpr int BYTES = OFF_ML + GA_PAIRS * 16 * 2 * 4;
};

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

__device__ __forceinline__ uint4 ldg_nc16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

template <int D>
__global__ void __launch_bounds__(GA_THREADS, 3)
gather_attn_kernel(const SparseAttnArgs a) {
    using S = GaSmem<D>;
    constexpr int HALF = D / 2;                   // dimensions per warp
    constexpr int NU = HALF / 32;                 // 32-dimension units per half (2 or 1)
    constexpr int NR = 4 * NU;                    // registers per half-row per thread
    constexpr int KK = HALF / 16;                 // k-chunks of QK^T per half
    constexpr int NTO = HALF / 8;                 // n-tiles of O per half
    extern __shared__ __align__(128) uint8_t ga_smem[];
    int32_t* idx_s = reinterpret_cast<int32_t*>(ga_smem + S::OFF_IDX);
    float4* xbuf = reinterpret_cast<float4*>(ga_smem + S::OFF_X);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int pair = warp >> 1, half = warp & 1;
    const int g = lane >> 2, c = lane & 3;
    const long long pidx = a.n_rows - 1 - (long long)blockIdx.x;    // longest rows first
    const long long row = sa_row(a, pidx);
    const int split = blockIdx.y;
    const int b = (int)(row / a.Lq);
    const int t = a.q_offset + (int)(row % a.Lq);
    const int tmax = min(t, a.Lk - 1);
    const int kend = a.trim ? min(a.kslots, t + 1) : a.kslots;
    const int s0 = split * a.slots_per_split;
    const int s1 = min(s0 + a.slots_per_split, kend);

    // this thread's 16-byte pieces of a row: unit u at byte 64u + 16c of the half
    const int hoff = half * HALF * 2 + 16 * c;                         // bytes
    const uint8_t* kbase = reinterpret_cast<const uint8_t*>(a.k + (long long)b * a.Lk * D) + hoff;
    const uint8_t* vbase = reinterpret_cast<const uint8_t*>(a.v + (long long)b * a.Lk * D) + hoff;
    const int32_t* irow = a.idx + row * a.kslots;

    // Q fragments of heads g and g+8 (rows >= Hq are zero), permuted like K.
    uint32_t q0[NR], q1[NR];
    {
        const uint8_t* qrow = reinterpret_cast<const uint8_t*>(a.q + row * a.Hq * D) + hoff;
#pragma unroll
        for (int u = 0; u < NU; ++u) {
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
            if (g < a.Hq) v0 = *reinterpret_cast<const uint4*>(qrow + (long long)g * D * 2 + 64 * u);
            if (g + 8 < a.Hq) v1 = *reinterpret_cast<const uint4*>(qrow + (long long)(g + 8) * D * 2 + 64 * u);
            q0[4 * u] = v0.x; q0[4 * u + 1] = v0.y; q0[4 * u + 2] = v0.z; q0[4 * u + 3] = v0.w;
            q1[4 * u] = v1.x; q1[4 * u + 1] = v1.y; q1[4 * u + 2] = v1.z; q1[4 * u + 3] = v1.w;
        }
    }

    float o[NTO][4];
#pragma unroll
    for (int i = 0; i < NTO; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;

    // K and V registers of GA_NBUF groups: [buffer][slot g / g+8][NR]
    uint32_t kr[GA_NBUF][2][NR], vr[GA_NBUF][2][NR];
    uint32_t par = 0;                                // exchange buffer parity

    for (int tile0 = s0; tile0 < s1; tile0 += SA_IDX_TILE) {
        const int tile1 = min(tile0 + SA_IDX_TILE, s1);
        const int ntile = tile1 - tile0;
        __syncthreads();                  // previous tile fully consumed
        for (int i = tid; i < SA_IDX_TILE; i += GA_THREADS) {
            int id = -1;
            if (i < ntile) {
                id = __ldg(irow + tile0 + i);
                if (id != -1 && (id < 0 || id > tmax)) {
                    report(DEV_ERR_BAD_INDEX);
                    id = -1;
                }
            }
            idx_s[i] = id;
        }
        __syncthreads();
        const int ngrp = (ntile + GA_GROUP - 1) / GA_GROUP;
        // this pair's groups: pair, pair + GA_PAIRS, ...
        const int nit = ngrp > pair ? (ngrp - pair + GA_PAIRS - 1) / GA_PAIRS : 0;

        auto load = [&](int it, uint32_t (&kk_)[2][NR], uint32_t (&vv_)[2][NR]) {
            const int* ids = idx_s + (pair + GA_PAIRS * it) * GA_GROUP;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int id = ids[g + 8 * h];
                const long long off = (long long)(id >= 0 ? id : 0) * D * 2;
#pragma unroll
                for (int u = 0; u < NU; ++u) {
                    const uint4 kv = ldg_nc16(kbase + off + 64 * u);
                    const uint4 vv = ldg_nc16(vbase + off + 64 * u);
                    kk_[h][4 * u] = kv.x; kk_[h][4 * u + 1] = kv.y;
                    kk_[h][4 * u + 2] = kv.z; kk_[h][4 * u + 3] = kv.w;
                    vv_[h][4 * u] = vv.x; vv_[h][4 * u + 1] = vv.y;
                    vv_[h][4 * u + 2] = vv.z; vv_[h][4 * u + 3] = vv.w;
                }
            }
        };

        auto compute = [&](int it, const uint32_t (&kk_)[2][NR], const uint32_t (&vv_)[2][NR]) {
            // partial S over this warp's dimension half: slots 2c,2c+1 | 8+2c,8+2c+1
            float sc[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
#pragma unroll
                for (int k2 = 0; k2 < KK; ++k2) {
                    const uint32_t af[4] = {q0[2 * k2], q1[2 * k2], q0[2 * k2 + 1], q1[2 * k2 + 1]};
                    mma_bf16(sc[nt], af, kk_[nt][2 * k2], kk_[nt][2 * k2 + 1]);
                }
            }
            // add the partner warp's half (both warps form the same sum)
            float4* mine = xbuf + ((((pair * 2 + half) * 2 + (int)par) * 2) * 32);
            mine[lane] = make_float4(sc[0][0], sc[0][1], sc[0][2], sc[0][3]);
            mine[32 + lane] = make_float4(sc[1][0], sc[1][1], sc[1][2], sc[1][3]);
            named_bar(1 + pair, 64);
            const float4* other = xbuf + ((((pair * 2 + (half ^ 1)) * 2 + (int)par) * 2) * 32);
            const float4 x0 = other[lane], x1 = other[32 + lane];
            par ^= 1u;
            const float p0[4] = {x0.x, x0.y, x0.z, x0.w}, p1[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                // half 0's partial first in both warps: bit-identical sums
                sc[0][e] = half == 0 ? sc[0][e] + p0[e] : p0[e] + sc[0][e];
                sc[1][e] = half == 0 ? sc[1][e] + p1[e] : p1[e] + sc[1][e];
            }
            const int* ids = idx_s + (pair + GA_PAIRS * it) * GA_GROUP;
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool valid = ids[nt * 8 + 2 * c + e] >= 0;
                    sc[nt][e] = valid ? sc[nt][e] * a.scale_log2 : -INFINITY;
                    sc[nt][2 + e] = valid ? sc[nt][2 + e] * a.scale_log2 : -INFINITY;
                    mx0 = fmaxf(mx0, sc[nt][e]);
                    mx1 = fmaxf(mx1, sc[nt][2 + e]);
                }
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float base0 = mn0 == -INFINITY ? 0.0f : mn0;
            const float base1 = mn1 == -INFINITY ? 0.0f : mn1;
            const float al0 = exp2f(m0 - base0), al1 = exp2f(m1 - base1);
            m0 = mn0;
            m1 = mn1;
            float rs0 = 0.0f, rs1 = 0.0f;
            uint32_t pa[4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const float e0 = exp2f(sc[nt][0] - base0), e1 = exp2f(sc[nt][1] - base0);
                const float e2 = exp2f(sc[nt][2] - base1), e3 = exp2f(sc[nt][3] - base1);
                rs0 += e0 + e1;
                rs1 += e2 + e3;
                pa[2 * nt] = pack_bf16(e0, e1);
                pa[2 * nt + 1] = pack_bf16(e2, e3);
            }
            l0 = l0 * al0 + rs0;
            l1 = l1 * al1 + rs1;
            if (__any_sync(0xffffffffu, al0 != 1.0f || al1 != 1.0f)) {
#pragma unroll
                for (int i = 0; i < NTO; ++i) {
                    o[i][0] *= al0;
                    o[i][1] *= al0;
                    o[i][2] *= al1;
                    o[i][3] *= al1;
                }
            }
            // O += P V over this warp's dimension half: n-tile (u, v) holds
            // dimensions 32u + 8c' + 2v + {0,1} for c' = 0..3
#pragma unroll
            for (int j = 0; j < NR; ++j) {
                const uint32_t b0 = movmatrix_t(vv_[0][j]);
                const uint32_t b1 = movmatrix_t(vv_[1][j]);
                mma_bf16(o[j], pa, b0, b1);
            }
        };

        // GA_NBUF-deep register pipeline over this pair's groups
#pragma unroll
        for (int p = 0; p < GA_NBUF - 1; ++p)
            if (p < nit) load(p, kr[p], vr[p]);
        for (int it0 = 0; it0 < nit; it0 += GA_NBUF) {
#pragma unroll
            for (int bb = 0; bb < GA_NBUF; ++bb) {
                const int it = it0 + bb;
                if (it < nit) {
                    const int nx = it + GA_NBUF - 1;
                    if (nx < nit) load(nx, kr[(bb + GA_NBUF - 1) % GA_NBUF], vr[(bb + GA_NBUF - 1) % GA_NBUF]);
                    compute(it, kr[bb], vr[bb]);
                }
            }
        }
    }

    // Row sums were kept per thread; reduce over the quad.
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    float* mo = reinterpret_cast<float*>(ga_smem + S::OFF_MO);
    float* ml = reinterpret_cast<float*>(ga_smem + S::OFF_ML);
#pragma unroll
    for (int j = 0; j < NR; ++j) {
        // n-tile j = 4u + v: dimensions half*HALF + 32u + 8c + 2v + {0,1}
        const int dcol = half * HALF + 32 * (j >> 2) + 8 * c + 2 * (j & 3);
        float* r0 = mo + (pair * 16 + g) * D + dcol;
        float* r1 = mo + (pair * 16 + g + 8) * D + dcol;
        r0[0] = o[j][0];
        r0[1] = o[j][1];
        r1[0] = o[j][2];
        r1[1] = o[j][3];
    }
    if (half == 0 && c == 0) {
        ml[(pair * 16 + g) * 2 + 0] = m0;
        ml[(pair * 16 + g) * 2 + 1] = l0;
        ml[(pair * 16 + g + 8) * 2 + 0] = m1;
        ml[(pair * 16 + g + 8) * 2 + 1] = l1;
    }
    __syncthreads();

    for (int e = tid; e < a.Hq * D; e += GA_THREADS) {
        const int h = e / D, dcol = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int p = 0; p < GA_PAIRS; ++p) M = fmaxf(M, ml[(p * 16 + h) * 2]);
        float L = 0.0f, acc = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int p = 0; p < GA_PAIRS; ++p) {
                const float f = exp2f(ml[(p * 16 + h) * 2] - M);
                L += f * ml[(p * 16 + h) * 2 + 1];
                acc += f * mo[(p * 16 + h) * D + dcol];
            }
        }
        const float val = L > 0.0f ? acc / L : 0.0f;
        const float lse2 = L > 0.0f ? M + log2f(L) : -INFINITY;
        if (a.splits == 1) {
            a.out[(row * a.Hq + h) * D + dcol] = __float2bfloat16_rn(val);
            if (a.lse && dcol == 0) a.lse[row * a.Hq + h] = lse2 * LN2;
        } else {
            const long long pr = (pidx * a.splits + split) * a.Hq + h;
            a.part_o[pr * D + dcol] = val;
            if (dcol == 0) a.part_lse[pr] = lse2;
        }
    }
}

}  // namespace ic
