// Sparse MQA attention for rows whose top-k covers a large share of their
// visible positions, computed tile-dense on the tensor cores (sm_100a).
//
// The result is the same softmax over the selected positions as the gather
// kernel (sparse_attn.cuh): a row's selection becomes a bitmask, and every
// position outside it gets probability exactly 0.  When a row keeps k of
// t+1 <= ~8k visible positions, sharing each K/V tile between the 8 queries
// x 16 heads of a block and running the contractions on tcgen05 moves far
// fewer bytes and runs far more flops per byte than gathering k rows per
// query (IndexCache: every layer attends over the k cached positions; MQA).
//
// Per CTA: one block of 128/Hq queries x Hq heads = 128 rows (TMEM lanes);
// two CTAs share an SM so one's MMAs overlap the other's softmax.
//   warp 0      TMA: the Q block once; per 64-key tile K[keys, d] into a
//               2-stage K ring and V^T[d, keys] (a per-layer transposed copy)
//               into a 2-stage V ring.  One thread polls both rings and
//               refills whichever stage is released first.
//   warp 1      TMEM allocation + MMA issue.  S(j) = bias + Q K(j)^T (M=128,
//               N=64) goes to one of two TMEM score buffers, so S(j+1) is
//               computed while the softmax works on S(j).  The bias term is one
//               extra K=16 step: a one-hot matrix (row -> its query) times the
//               tile's bias matrix (key x query: 0 where the key is selected,
//               -2^100 where it is not), so unselected scores arrive at about
//               -2^100 and their probabilities are exactly 0.  O += P(j) V(j)
//               reads P from TMEM (A operand) and the V^T tile from shared
//               memory; O accumulates in TMEM.
//   warps 2..5  softmax: thread = row = TMEM lane.  Loads S(j) once into
//               registers, computes the probabilities against the running
//               max, and only then waits for P(j-1) V(j-1) to finish before
//               it writes P(j) as bf16 over the columns of S(j) it has read.
//               The running max is raised lazily: only when a tile's max
//               exceeds it by more than 8 (log2 units) is O rescaled in TMEM,
//               so P stays <= 2^8 and O / l is exact either way.  A tile whose
//               probabilities sum to at most 2^8 cannot hold a larger one, so
//               the tile max is only taken (and the tile redone) when the sum
//               is larger or no selected key has been seen yet.  Rows raise
//               their max independently, but tcgen05.ld/st are warp-collective,
//               so the rescale is warp-uniform: when any row of a warp raises,
//               every lane takes O through registers (the others with factor
//               1).  Likewise every wait before a TMEM access is voted across
//               the warp.  Each thread also writes its share of the bias matrix
//               two tiles ahead from the selection bitmask of its query.
// Scores are scaled in the log2 domain.
#pragma once

#include "common.cuh"

namespace ic {

constexpr int DA_THREADS = 192;                  // 2 control warps + 4 softmax warps
constexpr int DA_TILE = 64;                      // keys per tile
constexpr float DA_RESCALE = 8.0f;               // lazy-max threshold (log2 units)
constexpr uint16_t DA_BIAS_OFF = 0xF180u;        // bf16 -2^100: an unselected key's bias
constexpr float DA_NONE = -1.0e29f;              // scores below this are unselected

struct DenseAttnArgs {
    const uint32_t* mask;      // [B * Lq_d, W] bitmask of selected positions, row b*Lq_d + i
    __nv_bfloat16* out;        // [B, Lq, Hq, 128]
    float* lse;                // [B, Lq, Hq] or null
    int Lq, Lk, Hq, q_offset;
    int Lq_d;                  // rows i < Lq_d of each sequence take this path
    int QBD;                   // queries per block (128 / Hq)
    int nqb_d;                 // blocks per sequence on this path
    int W;                     // mask words per row
    int n_blocks;              // B * nqb_d
    float scale_log2;
};

// No-swizzle K-major operand of K = 16 bf16: 8-row x 16-byte core matrices,
// the two along K 128 bytes apart, 8-row groups 256 bytes apart.
constexpr int DA_NS_LBO = 128;
constexpr int DA_NS_SBO = 256;

__device__ __forceinline__ uint32_t ns_offset(int row, int col) {
    return (uint32_t)((row >> 3) * DA_NS_SBO + (col >> 3) * DA_NS_LBO + (row & 7) * 16 + (col & 7) * 2);
}

struct DenseSmem {
    static constexpr int Q_BYTES = 128 * 128 * 2;            // 128 rows x 128 d (two 64-col boxes)
    static constexpr int K_BYTES = 64 * 128 * 2;             // 64 keys x 128 d (two boxes)
    static constexpr int V_BYTES = 128 * 64 * 2;             // 128 d x 64 keys (one box)
    static constexpr int BIAS_BYTES = 64 * 16 * 2;           // 64 keys x 16 queries, no swizzle
    static constexpr int ONEHOT_BYTES = 128 * 16 * 2;        // 128 rows x 16 queries, no swizzle
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;            // 2 stages
    static constexpr int OFF_V = OFF_K + 2 * K_BYTES;        // 2 stages
    static constexpr int OFF_BIAS = OFF_V + 2 * V_BYTES;     // 2 stages
    static constexpr int OFF_ONEHOT = OFF_BIAS + 2 * BIAS_BYTES;
    static constexpr int OFF_BAR = OFF_ONEHOT + ONEHOT_BYTES;
    static constexpr int N_BARS = 16;
    static constexpr int OFF_SLOT = OFF_BAR + N_BARS * 8;
    static constexpr int BYTES = OFF_SLOT + 16;
    // Up to 1024 B of slack for the 1024-B alignment of the swizzled tiles,
    // capped so that two CTAs (plus their 1 KB reserved each) fit the SM's
    // 228 KB; the kernel checks that the aligned layout fits.
    static constexpr int PAIR_MAX = 233472 / 2 - 1024;
    static constexpr int ALLOC = (BYTES + 1024) < PAIR_MAX ? (BYTES + 1024) : PAIR_MAX;
    static_assert(BYTES <= PAIR_MAX, "two CTAs must fit one SM");
};

// TMEM columns of one CTA: two 64-column score buffers (P(j) overwrites the
// first 32 columns of S(j) as packed bf16 pairs), then O (128 columns).
constexpr uint32_t DA_TMEM_COLS = 256;
constexpr uint32_t DA_O_COL = 128;

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2^x on the MUFU unit (flush-to-zero; exactly 0 for x = -inf).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Shared-memory descriptor of a no-swizzle K-major operand (layout code 0).
__device__ __forceinline__ uint64_t ns_kmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(DA_NS_LBO >> 4) << 16;
    d |= (uint64_t)(DA_NS_SBO >> 4) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16; A is M x K bf16 in TMEM (lane =
// row, two K elements per 32-bit column).
__device__ __forceinline__ void tc_mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                  uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// tmap_q: q as 3-D {128, Lq*Hq, B}, box {64, 128, 1}; tmap_k: K as {128, Lk, B},
// box {64, 64, 1}; tmap_vt: V^T as {Lk_d, 128, B} (rows padded), box {64, 128, 1}.
__global__ void __launch_bounds__(DA_THREADS, 2)
dense_attn_kernel(const __grid_constant__ CUtensorMap tmap_q,
                  const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_vt, const DenseAttnArgs a) {
    using S = DenseSmem;
    extern __shared__ uint8_t da_raw[];
    uint8_t* smem = align_smem_1024(da_raw, S::BYTES);
    if (smem == nullptr) return;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;       // [2]
    uint64_t* k_empty = bars + 3;      // [2]
    uint64_t* v_full = bars + 5;       // [2]
    uint64_t* v_empty = bars + 7;      // [2]
    uint64_t* s_full = bars + 9;       // [2]
    uint64_t* p_full = bars + 11;
    uint64_t* o_full = bars + 12;
    uint64_t* mma_done = bars + 13;
    uint64_t* bias_full = bars + 14;   // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::OFF_SLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = a.n_blocks - 1 - (int)blockIdx.x;             // longest rows first
    const int b = g / a.nqb_d;
    const int i0 = (g % a.nqb_d) * a.QBD;
    const int t_last = a.q_offset + i0 + a.QBD - 1;
    const int nt = (min(t_last + 1, a.Lk) + DA_TILE - 1) / DA_TILE;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&bias_full[i], 128);
        }
        mbar_init(p_full, 128);
        mbar_init(o_full, 1);
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    // one-hot rows (row r -> query r / Hq) and zeroed bias stages (the query
    // columns past QBD stay 0)
    {
        uint32_t* z = reinterpret_cast<uint32_t*>(smem + S::OFF_BIAS);
        for (int i = threadIdx.x; i < (2 * S::BIAS_BYTES + S::ONEHOT_BYTES) / 4; i += DA_THREADS)
            z[i] = 0u;
        __syncthreads();
        if (threadIdx.x < 128) {
            const int r = threadIdx.x;
            *reinterpret_cast<uint16_t*>(smem + S::OFF_ONEHOT + ns_offset(r, r / a.Hq)) = 0x3F80u;
        }
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, DA_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_vt);
            mbar_arrive_expect_tx(q_full, (uint32_t)S::Q_BYTES);
            for (int kb = 0; kb < 2; ++kb)
                tma_load_3d(smem + S::OFF_Q + kb * 128 * 128, &tmap_q, q_full, kb * 64,
                            i0 * a.Hq, b);
            // Refill whichever ring frees a stage first; V never runs ahead of K.
            int jk = 0, jv = 0, spins = 0;
            unsigned long long t0 = global_ns();
            while (jk < nt || jv < nt) {
                bool moved = false;
                if (jk < nt && mbar_try_wait(&k_empty[jk & 1], ((jk >> 1) & 1) ^ 1)) {
                    uint8_t* dst = smem + S::OFF_K + (jk & 1) * S::K_BYTES;
                    mbar_arrive_expect_tx(&k_full[jk & 1], (uint32_t)S::K_BYTES);
                    for (int kb = 0; kb < 2; ++kb)
                        tma_load_3d(dst + kb * 64 * 128, &tmap_k, &k_full[jk & 1], kb * 64,
                                    jk * DA_TILE, b);
                    ++jk;
                    moved = true;
                }
                if (jv < jk && mbar_try_wait(&v_empty[jv & 1], ((jv >> 1) & 1) ^ 1)) {
                    mbar_arrive_expect_tx(&v_full[jv & 1], (uint32_t)S::V_BYTES);
                    tma_load_3d(smem + S::OFF_V + (jv & 1) * S::V_BYTES, &tmap_vt, &v_full[jv & 1],
                                jv * DA_TILE, 0, b);
                    ++jv;
                    moved = true;
                }
                if (moved) {
                    spins = 0;
                    t0 = global_ns();
                } else if (++spins == 64) {
                    spins = 0;
                    if (global_ns() - t0 > WAIT_LIMIT_NS) {
                        report(DEV_ERR_TIMEOUT);
                        break;
                    }
                }
            }
            // never leave with copies in flight
            mbar_wait(q_full, 0);
            for (int c = (jk > 2 ? jk - 2 : 0); c < jk; ++c) mbar_wait(&k_full[c & 1], (c >> 1) & 1);
            for (int c = (jv > 2 ? jv - 2 : 0); c < jv; ++c) mbar_wait(&v_full[c & 1], (c >> 1) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, DA_TILE);
            const uint32_t idesc_o = idesc_bf16_f32(128, 128);
            const uint32_t q_addr = smem_u32(smem + S::OFF_Q);
            const uint64_t onehot_desc = ns_kmajor_desc(smem_u32(smem + S::OFF_ONEHOT));
            bool ok = mbar_wait(q_full, 0);
            // iteration j issues S(j), then P(j-1) V(j-1).  S(j) overwrites the
            // buffer of S(j-2) and P(j-2): the softmax released S(j-2) with
            // P(j-2), and P(j-2) V(j-2), which reads P(j-2) from there, has
            // completed before S(j) is issued.
            for (int j = 0; j <= nt && ok; ++j) {
                if (j < nt) {
                    const int st = j & 1;
                    if (!(ok = mbar_wait(&k_full[st], (j >> 1) & 1))) break;
                    if (!(ok = mbar_wait(&bias_full[st], (j >> 1) & 1))) break;
                    if (j >= 2 && !(ok = mbar_wait(o_full, (j - 2) & 1))) break;
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(smem + S::OFF_K + st * S::K_BYTES);
                    const uint32_t s_col = tmem + (uint32_t)(st * DA_TILE);
                    tc_mma_f16(s_col, onehot_desc,
                               ns_kmajor_desc(smem_u32(smem + S::OFF_BIAS + st * S::BIAS_BYTES)),
                               idesc_s, 0u);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t qo = (uint32_t)((kk >> 2) * 128 * 128 + (kk & 3) * 32);
                        const uint32_t ko = (uint32_t)((kk >> 2) * 64 * 128 + (kk & 3) * 32);
                        tc_mma_f16(s_col, sw128_kmajor_desc(q_addr + qo),
                                   sw128_kmajor_desc(k_addr + ko), idesc_s, 1u);
                    }
                    tc_commit(&s_full[st]);
                    tc_commit(&k_empty[st]);
                }
                if (j > 0) {
                    const int jp = j - 1, st = jp & 1;
                    if (!(ok = mbar_wait(p_full, jp & 1))) break;
                    if (!(ok = mbar_wait(&v_full[st], (jp >> 1) & 1))) break;
                    tc_fence_after();
                    const uint32_t v_addr = smem_u32(smem + S::OFF_V + st * S::V_BYTES);
                    const uint32_t p_col = tmem + (uint32_t)(st * DA_TILE);
                    // O += P V   (A = P [rows x 64 keys] in TMEM, B = V^T tile [128 d x 64 keys])
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_f16_tmem_a(tmem + DA_O_COL, p_col + (uint32_t)(kk * 8),
                                          sw128_kmajor_desc(v_addr + (uint32_t)(kk * 32)), idesc_o,
                                          (jp > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(o_full);
                    tc_commit(&v_empty[st]);
                }
            }
            // the MMAs this thread issued are done before TMEM is freed
            tc_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else {
        // ---------------- softmax warps: thread = row r = (query r / Hq, head r % Hq)
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const int qi = r / a.Hq, h = r % a.Hq;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const bool row_ok = i0 + qi < a.Lq_d;
        const uint32_t* mrow = a.mask + (long long)(b * a.Lq_d + (row_ok ? i0 + qi : 0)) * a.W;
        const float sc = a.scale_log2;
        // bias share: keys [kb0, kb0 + kpt) of each tile for query qi
        const int kpt = DA_TILE / a.Hq;
        const int kb0 = h * kpt;
        auto bias_word = [&](int jj) -> uint32_t {
            const int wi = (jj * DA_TILE + kb0) >> 5;
            return (row_ok && wi < a.W) ? __ldg(mrow + wi) : 0u;
        };
        auto write_bias = [&](int jj, uint32_t word) {
            uint8_t* bt = smem + S::OFF_BIAS + (jj & 1) * S::BIAS_BYTES;
            const int sh = kb0 & 31;
            for (int e = 0; e < kpt; ++e)
                *reinterpret_cast<uint16_t*>(bt + ns_offset(kb0 + e, qi)) =
                    ((word >> (sh + e)) & 1u) ? (uint16_t)0u : DA_BIAS_OFF;
            fence_proxy_async_smem();
            mbar_arrive(&bias_full[jj & 1]);
        };
        float m_used = -INFINITY, l_run = 0.0f;
        bool ok = true;
        if (nt > 0) write_bias(0, bias_word(0));
        if (nt > 1) write_bias(1, bias_word(1));
        uint32_t nbw = nt > 2 ? bias_word(2) : 0u;
        for (int j = 0; j < nt; ++j) {
            // waits are warp-uniform: the TMEM accesses below are warp-collective
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1))) { ok = false; break; }
            tc_fence_after();
            // S(j+2) overwrites bias stage j&1 only after S(j) is complete
            if (j + 2 < nt) {
                write_bias(j + 2, nbw);
                if (j + 3 < nt) nbw = bias_word(j + 3);
            }
            const uint32_t sb = tmem + lane_base + (uint32_t)((j & 1) * DA_TILE);
            uint32_t v[64];
            {
                uint32_t (&v0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&v[0]);
                uint32_t (&v1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&v[32]);
                tmem_ld_32x32b_x32(sb, v0);
                tmem_ld_32x32b_x32(sb + 32, v1);
                tmem_ld_wait();
            }
            // probabilities (bf16 pairs) against `base`, and their sum
            uint32_t pk[32];
            float rs;
            auto softmax_tile = [&](float base) {
                float2 rs2[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
                const float2 sc2 = make_float2(sc, sc), nb2 = make_float2(-base, -base);
#pragma unroll
                for (int e = 0; e < 64; e += 2) {
                    const float2 x = __ffma2_rn(
                        make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), sc2, nb2);
                    const float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                    rs2[(e >> 1) & 3] = __fadd2_rn(rs2[(e >> 1) & 3], p);
                    __nv_bfloat162 pp = __floats2bfloat162_rn(p.x, p.y);
                    pk[e >> 1] = *reinterpret_cast<uint32_t*>(&pp);
                }
                const float2 r01 = __fadd2_rn(rs2[0], rs2[1]), r23 = __fadd2_rn(rs2[2], rs2[3]);
                const float2 rsum = __fadd2_rn(r01, r23);
                rs = rsum.x + rsum.y;
            };
            // Against the running max first: a sum <= 2^8 means every
            // probability is <= 2^8, so the running max stands (the lazy
            // rule).  Otherwise -- or before any selected key was seen -- take
            // the tile max (unselected keys sit near -2^100) and redo the tile.
            bool raise = false;
            float m_new = m_used;
            bool need_max = m_used == -INFINITY;
            if (!need_max) {
                softmax_tile(m_used);
                need_max = !(rs <= 256.0f);
            }
            if (need_max) {
                float mx[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    mx[e] = fmaxf(__uint_as_float(v[e]), __uint_as_float(v[e + 32]));
#pragma unroll
                for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
                    for (int e = 0; e < w; ++e) mx[e] = fmaxf(mx[e], mx[e + w]);
                const float mxs = mx[0] > DA_NONE ? mx[0] * sc : -INFINITY;
                raise = mxs > m_used + DA_RESCALE;
                m_new = raise ? mxs : m_used;
                softmax_tile(m_new == -INFINITY ? 0.0f : m_new);
            }
            // P(j-1) V(j-1) must be complete before O is rescaled
            if (j > 0) {
                if (!__all_sync(0xffffffffu, mbar_wait(o_full, (j - 1) & 1))) { ok = false; break; }
                tc_fence_after();
            }
            // Rows raise their max independently, but TMEM loads and stores
            // are warp-collective: when any row of the warp raises, every
            // lane takes O through registers, the others with factor 1.
            const float alpha = raise ? ex2_approx(m_used - m_new) : 1.0f;   // 0 on a first raise
            if (j > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(tmem + DA_O_COL + lane_base + c * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st_32x32b_x32(tmem + DA_O_COL + lane_base + c * 32, o);
                }
            }
            if (raise) {
                l_run *= alpha;
                m_used = m_new;
            }
            l_run += rs;
            // P(j) over the first 32 columns of S(j), already read
            tmem_st_32x32b_x32(sb, pk);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (ok && nt > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(o_full, (nt - 1) & 1));
            tc_fence_after();
        }
        if (ok) {                                   // uniform across the warp
            const bool row_in = i0 + qi < a.Lq;
            const long long orow = ((long long)b * a.Lq + i0 + qi) * a.Hq + h;
            const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
            uint4* dst = reinterpret_cast<uint4*>(a.out + orow * 128);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld_32x32b_x32(tmem + DA_O_COL + lane_base + c * 32, o);
                tmem_ld_wait();
                if (!row_in) continue;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 pp = __floats2bfloat162_rn(__uint_as_float(o[8 * u + 2 * e]) * inv,
                                                                  __uint_as_float(o[8 * u + 2 * e + 1]) * inv);
                        w[e] = *reinterpret_cast<uint32_t*>(&pp);
                    }
                    dst[c * 4 + u] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            if (a.lse && row_in) a.lse[orow] = l_run > 0.0f ? (m_used + log2f(l_run)) * LN2 : -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, DA_TMEM_COLS);
    }
}

// Bitmask of each row's selected positions: row p (= b*Lq_d + i, i < Lq_d)
// of `mask` gets bit s set for every index s in idx[b, i, :] with
// 0 <= s <= t = q_offset + i (-1 skipped; any other value is skipped and
// reported as DEV_ERR_BAD_INDEX, like the gather kernel does).
__global__ void build_mask_kernel(const int32_t* __restrict__ idx, int Lq, int k, int q_offset,
                                  int Lq_d, int W, uint32_t* __restrict__ mask, long long n_rows) {
    extern __shared__ uint32_t mk_smem[];
    for (long long p = blockIdx.x; p < n_rows; p += gridDim.x) {
        const long long b = p / Lq_d, i = p % Lq_d;
        const int t = q_offset + (int)i;
        const int32_t* ir = idx + (b * Lq + i) * (long long)k;
        for (int w = threadIdx.x; w < W; w += blockDim.x) mk_smem[w] = 0u;
        __syncthreads();
        for (int s = threadIdx.x; s < k; s += blockDim.x) {
            const int id = __ldg(ir + s);
            if (id >= 0 && id <= t && (id >> 5) < W)
                atomicOr(&mk_smem[id >> 5], 1u << (id & 31));
            else if (id != -1)
                report(DEV_ERR_BAD_INDEX);
        }
        __syncthreads();
        for (int w = threadIdx.x; w < W; w += blockDim.x) mask[p * W + w] = mk_smem[w];
        __syncthreads();
    }
}

// V [B, Lk, 128] -> V^T [B, 128, ldt] for keys < Lk_d (64 keys x 128 d per CTA).
__global__ void transpose_v_kernel(const __nv_bfloat16* __restrict__ v, int Lk, int Lk_d, int ldt,
                                   __nv_bfloat16* __restrict__ vt) {
    __shared__ __nv_bfloat16 tile[64][128 + 8];
    const int b = blockIdx.y, s0 = blockIdx.x * 64;
    const __nv_bfloat16* vb = v + (long long)b * Lk * 128;
    for (int e = threadIdx.x; e < 64 * 16; e += blockDim.x) {
        const int s = e / 16, c = e % 16;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (s0 + s < Lk_d) val = *reinterpret_cast<const uint4*>(vb + (long long)(s0 + s) * 128 + c * 8);
        *reinterpret_cast<uint4*>(&tile[s][c * 8]) = val;
    }
    __syncthreads();
    __nv_bfloat16* tb = vt + (long long)b * 128 * ldt;
    for (int e = threadIdx.x; e < 128 * 64; e += blockDim.x) {
        const int d = e / 64, s = e % 64;
        if (s0 + s < ldt) tb[(long long)d * ldt + s0 + s] = tile[s][d];
    }
}

}  // namespace ic
