// Sparse MQA attention over the cached top-k positions (sm_100a).
//
// For query row t and head h, over the slots i whose index idx_i is valid:
//   z_i = scale * q[t,h] . K[idx_i],  out = sum_i softmax(z)_i V[idx_i]
// (IndexCache: every layer, F or S, attends sparsely over the k positions
// held in the index cache; all query heads share the one K/V head).
//
// One CTA handles one query row (all heads) and one split of its slots.  The
// CTA stages up to 2048 of the row's indices at a time in shared memory in
// one coalesced burst (validating them), so no copy ever waits on an index
// load.  Its 4 warps then work independently on interleaved blocks of 16
// slots (warp w takes blocks w, w+4, ...).  Three CTAs share an SM (168
// registers a thread, 72 KB of shared memory each): the kernel is bound by
// latency, and a third CTA beat a third pipeline stage.  Each warp runs its
// own 2-stage cp.async pipeline: 16
// lanes copy one 256-byte K row (or V row) per instruction, so every request
// is a full, coalesced 128-byte line pair; rows land XOR-swizzled in shared
// memory so the ldmatrix reads are bank-conflict free.  S = Q K^T and
// O += P V run on the tensor cores (m16n8k16, bf16 in, fp32 accumulate); the
// softmax is online in fp32 (exp2, the scale times log2 e folded into the
// exponent's FMA); the exponent base moves, and O is rescaled, only when a
// block's maximum passes it by more than 2^8, and a tile with no empty slot
// skips the masking.  The warps' partial (base, sum, O) merge through shared
// memory at the end, one weight per (head, warp).  With several splits per
// row (few rows: decode), up to 8 splits run as one thread-block cluster:
// each keeps its (O / l, log2-sum-exp) in shared memory and, after a cluster
// barrier, split r merges heads r, r + splits, ... from every split through
// distributed shared memory.  With more splits each writes its partial to
// the caller's workspace and a combine kernel merges them.
#pragma once

#include "common.cuh"

namespace ic {

#ifndef IC_SA_BLOCK
#define IC_SA_BLOCK 16
#endif
#ifndef IC_SA_WARPS
#define IC_SA_WARPS 4
#endif
#ifndef IC_SA_STAGES
#define IC_SA_STAGES 2
#endif
#ifndef IC_SA_MINB
#define IC_SA_MINB 3
#endif
constexpr int SA_BLOCK = IC_SA_BLOCK;        // slots per warp iteration (16, 32 or 64)
constexpr int SA_WARPS = IC_SA_WARPS;
constexpr int SA_THREADS = 32 * SA_WARPS;
constexpr int SA_STAGES = IC_SA_STAGES;
static_assert(SA_BLOCK == 16 || SA_BLOCK == 32 || SA_BLOCK == 64, "block of 16, 32 or 64 slots");
#ifndef IC_SA_IDX_TILE
#define IC_SA_IDX_TILE 2048
#endif
constexpr int SA_IDX_TILE = IC_SA_IDX_TILE;  // indices staged in shared memory at a time
constexpr float SA_RESCALE = 8.0f;           // log2 headroom before the exponent base moves

// 2^x on the special-function unit (subnormal results flush to 0).
__device__ __forceinline__ float sa_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct SparseAttnArgs {
    const __nv_bfloat16* q;    // [B, Lq, Hq, D]
    const __nv_bfloat16* k;    // [B, Lk, D]
    const __nv_bfloat16* v;    // [B, Lk, D]
    const int32_t* idx;        // [B*Lq, kslots]
    __nv_bfloat16* out;        // [B, Lq, Hq, D]
    float* lse;                // [B, Lq, Hq] or null
    float* part_o;             // [rows, splits, Hq, D] (splits > 1, not clustered)
    float* part_lse;           // [rows, splits, Hq]
    int cluster;               // the row's splits form one thread-block cluster (splits <= 8)
    int Lq, Lk, Hq, kslots, q_offset;
    int splits, slots_per_split;
    int trim;                  // slots past min(k, t+1) are known empty
    float scale_log2;
    long long n_rows;          // rows processed: B * rows_per_b
    int rows_per_b;            // rows i in [row_i0, row_i0 + rows_per_b) of each sequence
    int row_i0;
};

// Processing index p -> flattened query row b*Lq + i.
__device__ __forceinline__ long long sa_row(const SparseAttnArgs& a, long long p) {
    const long long b = p / a.rows_per_b;
    return b * a.Lq + a.row_i0 + (p % a.rows_per_b);
}

template <int D>
struct SaSmem {
    static constexpr int ROW = D * 2;                          // bytes per K/V/Q row
    static constexpr int BLK = SA_BLOCK * ROW;                 // one block of K (or V) rows
    static constexpr int STAGE = 2 * BLK;                      // K then V
    // The Q rows are read into registers once, before any ring stage is
    // written, so they share warp 0's first stage.
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = 0;
    static_assert(16 * ROW <= STAGE, "the Q rows fit in one ring stage");
    static constexpr int WARP_KV = SA_STAGES * STAGE;
    static constexpr int OFF_IDX = OFF_KV + SA_WARPS * WARP_KV;
    static constexpr int BYTES = OFF_IDX + SA_IDX_TILE * 4;
    // merge buffers reuse the K/V rings once every warp has finished
    static constexpr int MROW = D + 8;                                      // padded merge rows
    static constexpr int MERGE_O = OFF_KV;                                  // [4][16][MROW] f32
    static constexpr int MERGE_ML = OFF_KV + SA_WARPS * 16 * MROW * 4;      // [4][16][2] f32
    static constexpr int MERGE_W = MERGE_ML + SA_WARPS * 16 * 2 * 4;        // [16][4] + [16] f32
    static constexpr int FIN = MERGE_W + (16 * SA_WARPS + 16) * 4;          // [16][D] f32 (clustered)
    static_assert(FIN + 16 * D * 4 <= OFF_IDX, "merge buffer overflow");
};

// Byte offset of 16-byte chunk c of row r in a [rows][D] bf16 tile whose
// chunks are XOR-swizzled by (r mod 8).
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async16_full(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
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

// Thread-block cluster primitives: a barrier over the cluster's CTAs
// (release / acquire, so shared-memory writes before it are visible to the
// other CTAs after it) and a 32-bit load from another CTA's shared memory.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

template <int D>
__global__ void __launch_bounds__(SA_THREADS, IC_SA_MINB)
sparse_attn_kernel(const SparseAttnArgs a) {
    using S = SaSmem<D>;
    constexpr int CPR = D / 8;                 // 16-byte chunks per row (16 or 8)
    constexpr int RPI = 32 / CPR;              // rows copied per warp instruction (2 or 4)
    extern __shared__ __align__(128) uint8_t sa_smem[];
    const uint32_t sbase = smem_u32(sa_smem);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long pidx = a.n_rows - 1 - (long long)blockIdx.x;    // longest rows first
    const long long row = sa_row(a, pidx);
    const int split = blockIdx.y;
    const int b = (int)(row / a.Lq);
    const int t = a.q_offset + (int)(row % a.Lq);
    const int tmax = min(t, a.Lk - 1);
    const int kend = a.trim ? min(a.kslots, t + 1) : a.kslots;
    const int s0 = split * a.slots_per_split;
    const int s1 = min(s0 + a.slots_per_split, kend);

    const __nv_bfloat16* kb = a.k + (long long)b * a.Lk * D;
    const __nv_bfloat16* vb = a.v + (long long)b * a.Lk * D;
    const __nv_bfloat16* kl = kb + (lane % (D / 8)) * 8;     // this lane's 16-byte chunk
    const __nv_bfloat16* vl = vb + (lane % (D / 8)) * 8;
    const int32_t* irow = a.idx + row * a.kslots;
    const uint32_t kv_base = sbase + S::OFF_KV + warp * S::WARP_KV;
    int32_t* idx_s = reinterpret_cast<int32_t*>(sa_smem + S::OFF_IDX);

    // Q rows (heads) are loaded into registers here and stored to shared
    // memory (rows >= Hq zero) only after the first index tile's loads are
    // issued, so the two memory latencies overlap.
    constexpr int QPT = (16 * CPR + SA_THREADS - 1) / SA_THREADS;   // 16-byte chunks a thread
    uint4 qv[QPT];
    {
        const uint4* qsrc = reinterpret_cast<const uint4*>(a.q + row * a.Hq * D);
#pragma unroll
        for (int u = 0; u < QPT; ++u) {
            const int p = tid + u * SA_THREADS;
            qv[u] = make_uint4(0, 0, 0, 0);
            if (p < 16 * CPR && p / CPR < a.Hq) qv[u] = qsrc[p];
        }
    }

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;
    uint32_t qf[D / 16][4];

    // Slots [s0, s1) are processed in tiles of SA_IDX_TILE staged indices.
    for (int tile0 = s0; tile0 < s1 || (tile0 == s0 && s1 <= s0); tile0 += SA_IDX_TILE) {
        const int tile1 = min(tile0 + SA_IDX_TILE, s1);
        const int ntile = max(tile1 - tile0, 0);
        __syncthreads();                  // previous tile fully consumed
        const int nfill = (ntile + SA_BLOCK - 1) / SA_BLOCK * SA_BLOCK;   // slots the blocks read
        int empty = 0;
        for (int i = tid; i < SA_IDX_TILE; i += SA_THREADS) {
            int id = -1;
            if (i < ntile) {
                id = __ldg(irow + tile0 + i);
                if (id != -1 && (id < 0 || id > tmax)) {
                    report(DEV_ERR_BAD_INDEX);
                    id = -1;
                }
            }
            empty |= (id < 0) & (i < nfill);
            idx_s[i] = id;
        }
        if (tile0 == s0) {
#pragma unroll
            for (int u = 0; u < QPT; ++u) {
                const int p = tid + u * SA_THREADS;
                if (p < 16 * CPR)
                    *reinterpret_cast<uint4*>(sa_smem + S::OFF_Q + swz<D>(p / CPR, p % CPR)) = qv[u];
            }
        }
        // Tiles whose blocks hold no empty slot (every row with at least k
        // positions) skip the per-slot masking below.
        const bool masked = __syncthreads_or(empty) != 0;
        if (tile0 == s0) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
                const int c = 2 * kk + (lane >> 4);
                ldsm_x4(sbase + S::OFF_Q + swz<D>(r, c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
            }
            __syncthreads();              // every warp holds Q before warp 0's ring overwrites it
        }
        const int nblk = (ntile + SA_BLOCK - 1) / SA_BLOCK;
        const int niter = nblk > warp ? (nblk - warp + SA_WARPS - 1) / SA_WARPS : 0;

        // Copies block (warp + SA_WARPS * it) of this tile into stage `st`;
        // empty slots (only in masked tiles) are zero-filled.
        auto issue = [&](int it, int st) {
            const int* ids = idx_s + (warp + SA_WARPS * it) * SA_BLOCK;
            const uint32_t kdst = kv_base + st * S::STAGE;
            const uint32_t vdst = kdst + S::BLK;
            const int c = lane % CPR;
            if (masked) {
#pragma unroll
                for (int i = 0; i < SA_BLOCK / RPI; ++i) {
                    const int r = i * RPI + lane / CPR;
                    const int rid = ids[r];
                    const bool ok = rid >= 0;
                    const long long off = (long long)(ok ? rid : 0) * D + c * 8;
                    cp_async16(kdst + swz<D>(r, c), kb + off, ok);
                    cp_async16(vdst + swz<D>(r, c), vb + off, ok);
                }
            } else {
#pragma unroll
                for (int i = 0; i < SA_BLOCK / RPI; ++i) {
                    const int r = i * RPI + lane / CPR;
                    const uint32_t rid = (uint32_t)ids[r];
                    cp_async16_full(kdst + swz<D>(r, c), kl + (size_t)rid * D);
                    cp_async16_full(vdst + swz<D>(r, c), vl + (size_t)rid * D);
                }
            }
        };
#pragma unroll
        for (int p = 0; p < SA_STAGES - 1; ++p) {
            if (p < niter) issue(p, p);
            cp_async_commit();
        }

        for (int it = 0; it < niter; ++it) {
            const int nx = it + SA_STAGES - 1;
            if (nx < niter) issue(nx, nx % SA_STAGES);
            cp_async_commit();
            cp_async_wait<SA_STAGES - 1>();
            __syncwarp();
            const int st = it % SA_STAGES;
            const uint32_t kbase = kv_base + st * S::STAGE;
            const uint32_t vbase = kbase + S::BLK;
            constexpr int NT = SA_BLOCK / 8;            // S n-tiles of 8 slots
            constexpr int KS = SA_BLOCK / 16;           // P.V k-steps of 16 slots
            float sc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    const int r = np * 16 + (lane & 7) + (lane >> 4) * 8;
                    const int c = 2 * kk + ((lane >> 3) & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kbase + swz<D>(r, c), b0, b1, b2, b3);
                    mma_bf16(sc[2 * np], qf[kk], b0, b1);
                    mma_bf16(sc[2 * np + 1], qf[kk], b2, b3);
                }
            }
            // Raw scores; the scale (times log2 e) is applied inside the
            // exponent's FMA.  Empty slots score -inf.
            if (masked) {
                const int* ids = idx_s + (warp + SA_WARPS * it) * SA_BLOCK;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        if (ids[nt * 8 + (lane & 3) * 2 + e] < 0) sc[nt][e] = sc[nt][2 + e] = -INFINITY;
                    }
                }
            }
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
                mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            mx0 *= a.scale_log2;
            mx1 *= a.scale_log2;
            // The exponent base m moves only when the block's maximum passes
            // it by more than SA_RESCALE (log2 units): below that the
            // probabilities stay under 2^SA_RESCALE, and O and l, which share
            // the base, need no rescale.  The final O / l is the same.
            const bool up0 = mx0 > m0 + SA_RESCALE, up1 = mx1 > m1 + SA_RESCALE;
            if (__any_sync(0xffffffffu, up0 || up1)) {
                const float al0 = up0 ? sa_ex2(m0 - mx0) : 1.0f;    // 0 while m was -inf
                const float al1 = up1 ? sa_ex2(m1 - mx1) : 1.0f;
                if (up0) m0 = mx0;
                if (up1) m1 = mx1;
                l0 *= al0;
                l1 *= al1;
#pragma unroll
                for (int i = 0; i < D / 8; ++i) {
                    o[i][0] *= al0;
                    o[i][1] *= al0;
                    o[i][2] *= al1;
                    o[i][3] *= al1;
                }
            }
            const float nb0 = m0 == -INFINITY ? 0.0f : -m0;
            const float nb1 = m1 == -INFINITY ? 0.0f : -m1;
            float rs0 = 0.0f, rs1 = 0.0f;
            uint32_t pa[KS][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float p0 = sa_ex2(fmaf(sc[nt][0], a.scale_log2, nb0));
                const float p1 = sa_ex2(fmaf(sc[nt][1], a.scale_log2, nb0));
                const float p2 = sa_ex2(fmaf(sc[nt][2], a.scale_log2, nb1));
                const float p3 = sa_ex2(fmaf(sc[nt][3], a.scale_log2, nb1));
                rs0 += p0 + p1;
                rs1 += p2 + p3;
                pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p0, p1);
                pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p2, p3);
            }
            l0 += rs0;
            l1 += rs1;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
                for (int dn = 0; dn < D / 16; ++dn) {
                    const int r = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int c = 2 * dn + (lane >> 4);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vbase + swz<D>(r, c), b0, b1, b2, b3);
                    mma_bf16(o[2 * dn], pa[ks], b0, b1);
                    mma_bf16(o[2 * dn + 1], pa[ks], b2, b3);
                }
            }
            __syncwarp();      // every lane is done with this stage before it is refilled
        }
        cp_async_wait<0>();
        if (tile1 >= s1) break;
    }
    cp_async_wait<0>();

    // Row sums were kept per thread; reduce over the quad.
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    __syncthreads();       // all warps are past their rings: reuse them for the merge
    float* mo = reinterpret_cast<float*>(sa_smem + S::MERGE_O);
    float* ml = reinterpret_cast<float*>(sa_smem + S::MERGE_ML);
    float* mw = reinterpret_cast<float*>(sa_smem + S::MERGE_W);
    const int g = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
        // rows padded to D + 8 floats: the quad's float2 stores of 8 rows hit distinct banks
        *reinterpret_cast<float2*>(mo + (warp * 16 + g) * S::MROW + i * 8 + cq) = make_float2(o[i][0], o[i][1]);
        *reinterpret_cast<float2*>(mo + (warp * 16 + g + 8) * S::MROW + i * 8 + cq) = make_float2(o[i][2], o[i][3]);
    }
    if ((lane & 3) == 0) {
        ml[(warp * 16 + g) * 2 + 0] = m0;
        ml[(warp * 16 + g) * 2 + 1] = l0;
        ml[(warp * 16 + g + 8) * 2 + 0] = m1;
        ml[(warp * 16 + g + 8) * 2 + 1] = l1;
    }
    __syncthreads();
    // Per head: the warps' weights 2^(m_w - M) / L and the log2-sum-exp M + log2 L.
    if (tid < 16) {
        const int h = tid;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < SA_WARPS; ++w) M = fmaxf(M, ml[(w * 16 + h) * 2]);
        float f[SA_WARPS], L = 0.0f;
#pragma unroll
        for (int w = 0; w < SA_WARPS; ++w) {
            f[w] = M == -INFINITY ? 0.0f : sa_ex2(ml[(w * 16 + h) * 2] - M);
            L += f[w] * ml[(w * 16 + h) * 2 + 1];
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
        for (int w = 0; w < SA_WARPS; ++w) mw[h * SA_WARPS + w] = f[w] * inv;
        mw[16 * SA_WARPS + h] = L > 0.0f ? M + log2f(L) : -INFINITY;
    }
    __syncthreads();

    for (int e = tid; e < a.Hq * D; e += SA_THREADS) {
        const int h = e / D, dcol = e % D;
        float val = 0.0f;
#pragma unroll
        for (int w = 0; w < SA_WARPS; ++w) val = fmaf(mw[h * SA_WARPS + w], mo[(w * 16 + h) * S::MROW + dcol], val);
        const float lse2 = mw[16 * SA_WARPS + h];
        if (a.splits == 1) {
            a.out[(row * a.Hq + h) * D + dcol] = __float2bfloat16_rn(val);
            if (a.lse && dcol == 0) a.lse[row * a.Hq + h] = lse2 * LN2;
        } else if (a.cluster) {
            reinterpret_cast<float*>(sa_smem + S::FIN)[h * D + dcol] = val;
        } else {
            const long long pr = (pidx * a.splits + split) * a.Hq + h;
            a.part_o[pr * D + dcol] = val;
            if (dcol == 0) a.part_lse[pr] = lse2;
        }
    }
    if (a.splits > 1 && a.cluster) {
        // The row's splits are one cluster (rank = split).  Each split's
        // (O / l, log2-sum-exp) stays in its shared memory; rank r merges
        // heads r, r + splits, ... from every rank's copy, with the same
        // weights as the combine kernel.
        cluster_sync_all();
        const uint32_t fin_addr = sbase + (uint32_t)S::FIN;
        const uint32_t lse_addr = sbase + (uint32_t)(S::MERGE_W + 16 * SA_WARPS * 4);
        for (int h = split; h < a.Hq; h += a.splits) {
            float lr[8];
            float M = -INFINITY;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                lr[r] = r < a.splits ? ld_cluster_f32(lse_addr + (uint32_t)h * 4u, (uint32_t)r) : -INFINITY;
                M = fmaxf(M, lr[r]);
            }
            float W = 0.0f;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                lr[r] = M == -INFINITY ? 0.0f : sa_ex2(lr[r] - M);
                W += lr[r];
            }
            const float inv = W > 0.0f ? 1.0f / W : 0.0f;
            for (int dcol = tid; dcol < D; dcol += SA_THREADS) {
                float acc = 0.0f;
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    if (r < a.splits)
                        acc = fmaf(lr[r], ld_cluster_f32(fin_addr + (uint32_t)(h * D + dcol) * 4u, (uint32_t)r), acc);
                a.out[(row * a.Hq + h) * D + dcol] = __float2bfloat16_rn(acc * inv);
                if (a.lse && dcol == 0) a.lse[row * a.Hq + h] = W > 0.0f ? (M + log2f(W)) * LN2 : -INFINITY;
            }
        }
        cluster_sync_all();            // no CTA leaves while another may read its shared memory
    }
}

// Merges the per-split partial results of each row (log2-sum-exp weights).
// One CTA per (row, head), one thread per output column: the split weights
// are computed once per head in shared memory.
template <int D>
__global__ void __launch_bounds__(D)
sparse_attn_combine_kernel(const SparseAttnArgs a) {
    __shared__ float wgt[64];
    __shared__ float mw[2];
    const long long pidx = blockIdx.x;
    const int h = blockIdx.y, dcol = threadIdx.x;
    const long long row = sa_row(a, pidx);
    const long long base = pidx * a.splits * a.Hq + h;               // split s at base + s*Hq
    if (threadIdx.x < 32) {
        float M = -INFINITY;
        for (int s = threadIdx.x; s < a.splits; s += 32) M = fmaxf(M, a.part_lse[base + (long long)s * a.Hq]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float W = 0.0f;
        for (int s = threadIdx.x; s < a.splits; s += 32) {
            const float f = M == -INFINITY ? 0.0f : exp2f(a.part_lse[base + (long long)s * a.Hq] - M);
            wgt[s] = f;
            W += f;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        if (threadIdx.x == 0) {
            mw[0] = M;
            mw[1] = W;
        }
    }
    __syncthreads();
    const float M = mw[0], W = mw[1];
    float acc = 0.0f;
    for (int s = 0; s < a.splits; ++s)
        acc += wgt[s] * a.part_o[(base + (long long)s * a.Hq) * D + dcol];
    a.out[(row * a.Hq + h) * D + dcol] = __float2bfloat16_rn(W > 0.0f ? acc / W : 0.0f);
    if (a.lse && dcol == 0) a.lse[row * a.Hq + h] = W > 0.0f ? (M + log2f(W)) * LN2 : -INFINITY;
}

}  // namespace ic
