// Sparse MQA attention over the cached top-k positions (sm_100a).
//
// For query row t and head h, over the slots i whose index idx_i is valid:
//   z_i = scale * q[t,h] . K[idx_i],  out = sum_i softmax(z)_i V[idx_i]
// (IndexCache: every layer, F or S, runs its own sparse attention over the k
// positions held in the index cache; all query heads share the one K/V head).
//
// One CTA handles one query row (all heads) and one split of its slots.  Per
// 64-slot chunk the CTA gathers the 64 K rows and 64 V rows with 16-byte
// cp.async copies (a 128-bit, fully coalesced load per thread per piece, rows
// XOR-swizzled in shared memory so ldmatrix is bank-conflict free), double
// buffered.  Each of the 4 warps then takes 16 of the slots: S = Q K^T and
// O += P V run on the tensor cores (m16n8k16, bf16 in, fp32 accumulate), the
// softmax is online in fp32 (exp2 with the scale pre-multiplied by log2 e).
// The warps' partial (max, sum, O) merge through shared memory at the end.
// With several splits per row each split writes (O / l, log2-sum-exp) to the
// caller's workspace and a combine kernel merges them.
#pragma once

#include "common.cuh"

namespace ic {

constexpr int SA_THREADS = 128;
constexpr int SA_CHUNK = 64;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct SparseAttnArgs {
    const __nv_bfloat16* q;    // [B, Lq, Hq, D]
    const __nv_bfloat16* k;    // [B, Lk, D]
    const __nv_bfloat16* v;    // [B, Lk, D]
    const int32_t* idx;        // [B*Lq, kslots]
    __nv_bfloat16* out;        // [B, Lq, Hq, D]
    float* lse;                // [B, Lq, Hq] or null
    float* part_o;             // [rows, splits, Hq, D] (splits > 1)
    float* part_lse;           // [rows, splits, Hq]
    int Lq, Lk, Hq, kslots, q_offset;
    int splits, slots_per_split;
    int trim;                  // slots past min(k, t+1) are known empty
    float scale_log2;
    long long n_rows;
};

template <int D>
struct SaSmem {
    static constexpr int ROW = D * 2;                     // bytes per K/V/Q row
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 16 * ROW;
    static constexpr int OFF_V = OFF_K + 2 * SA_CHUNK * ROW;
    static constexpr int OFF_IDX = OFF_V + 2 * SA_CHUNK * ROW;
    static constexpr int BYTES = OFF_IDX + 2 * SA_CHUNK * 4;
    // merge buffers (reuse the K/V region after the main loop)
    static constexpr int MERGE_O = OFF_K;                                  // [4][16][D] f32
    static constexpr int MERGE_ML = OFF_K + 4 * 16 * D * 4;                // [4][16][2] f32
    static_assert(MERGE_ML + 4 * 16 * 2 * 4 <= OFF_IDX, "merge buffer overflow");
};

__device__ __forceinline__ uint32_t swz(int row, int chunk, int row_bytes) {
    return (uint32_t)(row * row_bytes + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                        uint32_t& d) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                          uint32_t& d) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

template <int D>
__global__ void __launch_bounds__(SA_THREADS)
sparse_attn_kernel(const SparseAttnArgs a) {
    using S = SaSmem<D>;
    constexpr int CPR = D / 8;                 // 16-byte pieces per row
    extern __shared__ __align__(128) uint8_t sa_smem[];
    const uint32_t sbase = smem_u32(sa_smem);
    int32_t* idx_s = reinterpret_cast<int32_t*>(sa_smem + S::OFF_IDX);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long row = a.n_rows - 1 - (long long)blockIdx.x;     // longest rows first
    const int split = blockIdx.y;
    const int b = (int)(row / a.Lq);
    const int t = a.q_offset + (int)(row % a.Lq);
    const int tmax = min(t, a.Lk - 1);
    const int kend = a.trim ? min(a.kslots, t + 1) : a.kslots;
    const int s0 = split * a.slots_per_split;
    const int s1 = min(s0 + a.slots_per_split, kend);
    const int nchunks = s1 > s0 ? (s1 - s0 + SA_CHUNK - 1) / SA_CHUNK : 0;

    const __nv_bfloat16* kb = a.k + (long long)b * a.Lk * D;
    const __nv_bfloat16* vb = a.v + (long long)b * a.Lk * D;
    const int32_t* irow = a.idx + row * a.kslots;

    // Q rows (heads) -> shared memory, rows >= Hq zero.
    {
        const uint4* qsrc = reinterpret_cast<const uint4*>(a.q + row * a.Hq * D);
        for (int p = tid; p < 16 * CPR; p += SA_THREADS) {
            const int h = p / CPR, c = p % CPR;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (h < a.Hq) val = qsrc[h * CPR + c];
            *reinterpret_cast<uint4*>(sa_smem + S::OFF_Q + swz(h, c, S::ROW)) = val;
        }
    }

    auto issue = [&](int chunk, int st) {
        const int base = s0 + chunk * SA_CHUNK;
        if (tid < SA_CHUNK) {
            const int slot = base + tid;
            int id = -1;
            if (slot < s1) {
                id = __ldg(irow + slot);
                if (id != -1 && (id < 0 || id > tmax)) {
                    report(DEV_ERR_BAD_INDEX);
                    id = -1;
                }
            }
            idx_s[st * SA_CHUNK + tid] = id;
        }
        for (int p = tid; p < SA_CHUNK * CPR; p += SA_THREADS) {
            const int r = p / CPR, c = p % CPR;
            const int slot = base + r;
            int id = slot < s1 ? __ldg(irow + slot) : -1;
            const bool ok = id >= 0 && id <= tmax;
            const long long off = (long long)(ok ? id : 0) * D + c * 8;
            const uint32_t dk = sbase + S::OFF_K + st * SA_CHUNK * S::ROW + swz(r, c, S::ROW);
            const uint32_t dv = sbase + S::OFF_V + st * SA_CHUNK * S::ROW + swz(r, c, S::ROW);
            cp_async16(dk, kb + off, ok);
            cp_async16(dv, vb + off, ok);
        }
        cp_async_commit();
    };

    if (nchunks > 0) issue(0, 0);
    __syncthreads();

    // Q fragments (A operand, m16 x k16 per k-step) stay in registers.
    uint32_t qf[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = 2 * kk + (lane >> 4);
        ldsm_x4(sbase + S::OFF_Q + swz(r, c, S::ROW), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;

    for (int ch = 0; ch < nchunks; ++ch) {
        const int st = ch & 1;
        if (ch + 1 < nchunks) {
            issue(ch + 1, st ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();

        const uint32_t kbase = sbase + S::OFF_K + st * SA_CHUNK * S::ROW;
        const uint32_t vbase = sbase + S::OFF_V + st * SA_CHUNK * S::ROW;
        const int key0 = warp * 16;
        float sc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int r = key0 + (lane & 7) + (lane >> 4) * 8;
            const int c = 2 * kk + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kbase + swz(r, c, S::ROW), b0, b1, b2, b3);
            mma_bf16(sc[0], qf[kk], b0, b1);
            mma_bf16(sc[1], qf[kk], b2, b3);
        }
        // mask + scale (log2 domain)
        const int* ids = idx_s + st * SA_CHUNK + key0;
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = nt * 8 + (lane & 3) * 2 + e;
                const bool ok = ids[col] >= 0;
                sc[nt][e] = ok ? sc[nt][e] * a.scale_log2 : -INFINITY;
                sc[nt][2 + e] = ok ? sc[nt][2 + e] * a.scale_log2 : -INFINITY;
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
        float p[2][4];
        float rs0 = 0.0f, rs1 = 0.0f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            p[nt][0] = exp2f(sc[nt][0] - base0);
            p[nt][1] = exp2f(sc[nt][1] - base0);
            p[nt][2] = exp2f(sc[nt][2] - base1);
            p[nt][3] = exp2f(sc[nt][3] - base1);
            rs0 += p[nt][0] + p[nt][1];
            rs1 += p[nt][2] + p[nt][3];
        }
        l0 = l0 * al0 + rs0;
        l1 = l1 * al1 + rs1;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            o[i][0] *= al0;
            o[i][1] *= al0;
            o[i][2] *= al1;
            o[i][3] *= al1;
        }
        uint32_t pa[4];
        pa[0] = pack_bf16(p[0][0], p[0][1]);
        pa[1] = pack_bf16(p[0][2], p[0][3]);
        pa[2] = pack_bf16(p[1][0], p[1][1]);
        pa[3] = pack_bf16(p[1][2], p[1][3]);
#pragma unroll
        for (int dn = 0; dn < D / 16; ++dn) {
            const int r = key0 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int c = 2 * dn + (lane >> 4);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vbase + swz(r, c, S::ROW), b0, b1, b2, b3);
            mma_bf16(o[2 * dn], pa, b0, b1);
            mma_bf16(o[2 * dn + 1], pa, b2, b3);
        }
        __syncthreads();
    }

    // Row sums were kept per thread; reduce over the quad.
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    // Merge the 4 warps through shared memory.
    float* mo = reinterpret_cast<float*>(sa_smem + S::MERGE_O);
    float* ml = reinterpret_cast<float*>(sa_smem + S::MERGE_ML);
    const int g = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
        float* r0 = mo + (warp * 16 + g) * D + i * 8 + cq;
        float* r1 = mo + (warp * 16 + g + 8) * D + i * 8 + cq;
        r0[0] = o[i][0];
        r0[1] = o[i][1];
        r1[0] = o[i][2];
        r1[1] = o[i][3];
    }
    if ((lane & 3) == 0) {
        ml[(warp * 16 + g) * 2 + 0] = m0;
        ml[(warp * 16 + g) * 2 + 1] = l0;
        ml[(warp * 16 + g + 8) * 2 + 0] = m1;
        ml[(warp * 16 + g + 8) * 2 + 1] = l1;
    }
    __syncthreads();

    for (int e = tid; e < a.Hq * D; e += SA_THREADS) {
        const int h = e / D, dcol = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, ml[(w * 16 + h) * 2]);
        float L = 0.0f, acc = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float f = exp2f(ml[(w * 16 + h) * 2] - M);
                L += f * ml[(w * 16 + h) * 2 + 1];
                acc += f * mo[(w * 16 + h) * D + dcol];
            }
        }
        const float val = L > 0.0f ? acc / L : 0.0f;
        const float lse2 = L > 0.0f ? M + log2f(L) : -INFINITY;
        if (a.splits == 1) {
            a.out[(row * a.Hq + h) * D + dcol] = __float2bfloat16_rn(val);
            if (a.lse && dcol == 0) a.lse[row * a.Hq + h] = lse2 * LN2;
        } else {
            const long long pr = (row * a.splits + split) * a.Hq + h;
            a.part_o[pr * D + dcol] = val;
            if (dcol == 0) a.part_lse[pr] = lse2;
        }
    }
}

// Merges the per-split partial results of each row (log2-sum-exp weights).
template <int D>
__global__ void sparse_attn_combine_kernel(const SparseAttnArgs a) {
    const long long row = blockIdx.x;
    for (int e = threadIdx.x; e < a.Hq * D; e += blockDim.x) {
        const int h = e / D, dcol = e % D;
        float M = -INFINITY;
        for (int s = 0; s < a.splits; ++s)
            M = fmaxf(M, a.part_lse[(row * a.splits + s) * a.Hq + h]);
        float W = 0.0f, acc = 0.0f;
        if (M != -INFINITY) {
            for (int s = 0; s < a.splits; ++s) {
                const long long pr = (row * a.splits + s) * a.Hq + h;
                const float f = exp2f(a.part_lse[pr] - M);
                W += f;
                acc += f * a.part_o[pr * D + dcol];
            }
        }
        a.out[(row * a.Hq + h) * D + dcol] = __float2bfloat16_rn(W > 0.0f ? acc / W : 0.0f);
        if (a.lse && dcol == 0) a.lse[row * a.Hq + h] = W > 0.0f ? (M + log2f(W)) * LN2 : -INFINITY;
    }
}

}  // namespace ic
