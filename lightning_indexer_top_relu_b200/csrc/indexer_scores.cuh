// Lightning indexer scores on the 5th-generation tensor cores (sm_100a).
//
// Computes, for query rows t and visible keys s <= t,
//     score[t, s] = sum_j w[t, j] * max(0, q_I[t, j] . k_I[s])
// (the IndexCache papers describe the indexer as scoring every preceding
// token of the query; the score form is the standard lightning-indexer one,
// which the pages do not print).
//
// Tile mapping.  Keys sit on the MMA M axis (128 TMEM lanes) and
// (query, head) pairs on N: one tcgen05.mma of M=128, N=QB*H_I (<= 256),
// K=d_I computes q_I[t,j] . k_I[s] for 128 keys x QB queries x H_I heads.
// The epilogue thread that owns TMEM lane s then holds every head of every
// query of the block for key s, so the ReLU and the w-weighted head sum are
// a per-thread register reduction, and the score stores run along s
// (coalesced).
//
// Pipeline (one persistent CTA per SM, warp-specialised):
//   warp 0      TMA producer: the query block (B operand) and its head
//               weights w (bulk copy), once per work unit, double-buffered;
//               k_I tiles (A operand) through a 3-stage ring
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2..   epilogue (16 warps with 64 heads, and with 32 heads outside
//               the candidate pass; else 8): tcgen05.ld -> ReLU -> w-weighted
//               head sum -> causal mask -> output.  With 64+ heads the TMEM
//               reads use the 16x256b shape: a thread holds 2 keys x a
//               quarter of its columns, its quarter of the head weights stays
//               in registers for the unit, and a quad adds its partial sums
//               by shuffles.  Warp w reads TMEM lane quarter w % 4 and the
//               part (w-2) / 4 of the block's queries, so 4 (or 2) warps
//               share each SM sub-partition.  Two TMEM accumulators
//               (2 x 256 columns) let the epilogue of tile j overlap the MMA
//               of tile j+1; with 16x256b reads a tile's accumulator is
//               released as soon as its last read lands.
// A work unit is (query block, run of up to `tpu` key tiles); units are
// ordered split-major, longest causal rows first within a split, and dealt
// round-robin to the CTAs.
//
// Epilogue modes (a template parameter; the MMA and the score arithmetic are
// the same code in every mode, so a score is bit-identical whichever mode
// produced it):
//   IDX_SCORES  every score of the visited key tiles is stored (-inf where
//               s > t);
//   IDX_SAMPLE  only key tiles j = m * stride are visited, and their scores
//               are stored compactly at column m*128 + lane of a sample row;
//   IDX_CAND    nothing is stored but the scores whose order-preserving key
//               is at least the row's threshold key: each is appended to the
//               row's candidate list as (key << 32) | ~s, one 64-bit value
//               whose unsigned order is (score descending, position
//               ascending).  Warps reserve list slots in ranges of IDX_RES;
//               the row's counter counts every reserved slot, also those past
//               the list's capacity (whose candidates are dropped), and
//               reserved slots left unused hold 0.
// With a block list (the exact fallback of the fused top-k), the launch's
// query blocks are taken from a device array whose length is read on the
// device, and scores go to consecutive buffer rows of those blocks.
#pragma once

#include "common.cuh"

namespace ic {

constexpr int IDX_BM = 128;          // keys per tile = TMEM lanes
constexpr int IDX_NMAX = 256;        // max (query, head) columns per MMA
constexpr int IDX_STAGES = 3;        // k_I tile ring depth
enum : int { IDX_SCORES = 0, IDX_SAMPLE = 1, IDX_CAND = 2 };
#ifndef IC_IDX_EARLY_FREE
#define IC_IDX_EARLY_FREE 1
#endif
// 16x256b epilogue: a tile's TMEM accumulator is released as soon as its
// last read has landed, before the second lane half's arithmetic.
constexpr bool IDX_EARLY_FREE = IC_IDX_EARLY_FREE != 0;
#ifndef IC_IDX_EPI_WIDE
#define IC_IDX_EPI_WIDE 16
#endif
#ifndef IC_IDX_WIDE32
#define IC_IDX_WIDE32 1
#endif
// Epilogue warps: with 64 heads (a block of 4 queries) four warps per TMEM
// lane quarter, one query each, and likewise with 32 heads (8 queries, two
// per warp) except in the candidate pass, whose extra state would not fit the
// registers of 18 warps; otherwise two warps per quarter.
__host__ __device__ constexpr int idx_epi_warps(int H, int mode) {
    return (H == 64 || (IC_IDX_WIDE32 && H == 32 && mode != IDX_CAND)) ? IC_IDX_EPI_WIDE : 8;
}
__host__ __device__ constexpr int idx_threads(int H, int mode) { return 64 + 32 * idx_epi_warps(H, mode); }

constexpr unsigned IDX_RES = 32;              // IDX_CAND: list slots reserved per atomic
// One ballot takes up to 32 candidates, and what the current range cannot
// hold goes to the single range reserved ahead: a range holds at least a warp.
static_assert(IDX_RES >= 32, "a reserved range must hold one ballot's candidates");
constexpr uint32_t IDX_NONE = 0xFFFFFFFFu;    // IDX_CAND threshold: the row keeps no candidate

// 16 lanes x (16 x 8) 32-bit columns: repetition r covers columns
// [8r, 8r+8); thread i of the warp gets, in r[4r .. 4r+3], lane (base + i/4)
// columns 8r + 2(i%4) + {0, 1}, then lane (base + 8 + i/4), same columns.
__device__ __forceinline__ void tmem_ld_16x256b_x16(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
          "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
          "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
          "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]),
          "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]),
          "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
}

// The same shape with 8 repetitions (columns [0, 64)).
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

struct IndexerArgs {
    const float* w;        // [B, Lq, H]
    float* scores;         // IDX_SCORES / IDX_SAMPLE: row (flattened query row - row_base), stride ld
    long long ld;
    int B, Lq, Lk, q_offset;
    int QB;                // queries per block
    int N;                 // MMA N (QB*H rounded up to 16)
    int nqb;               // query blocks per batch element
    int g0, g1;            // flattened query-block range of this launch
    long long row_base;    // flattened row of the first row of block g0
    int tpu;               // key tiles per work unit
    int max_splits;        // work units per query block (some may be empty)
    int stride;            // IDX_SAMPLE: key tiles j = m * stride are visited (1 otherwise)
    // IDX_CAND: per row (flattened row - row_base)
    const uint32_t* thr;   // threshold key
    uint32_t* cnt;         // candidates found (may exceed cap)
    unsigned long long* cand;   // [rows, cap]
    int cap;
    // block list: when blk_list is non-null the launch covers list entries
    // [list_off, list_off + min(list_len, *blk_count - list_off)); score
    // rows are (entry - list_off) * QB + query
    const int* blk_list;
    const int* blk_count;
    int list_off, list_len;
};

template <int DI>
struct IndexerSmem {
    static constexpr int Q_BYTES = IDX_NMAX * DI * 2;     // one query block
    static constexpr int A_BYTES = IDX_BM * DI * 2;       // one k_I tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_A = OFF_Q + 2 * Q_BYTES;
    static constexpr int OFF_W = OFF_A + IDX_STAGES * A_BYTES;   // 2 x 256 fp32 head weights
    static constexpr int OFF_BAR = OFF_W + 2 * IDX_NMAX * 4;
    static constexpr int N_BARS = 2 + 2 + IDX_STAGES + IDX_STAGES + 2 + 2;
    static constexpr int OFF_SLOT = OFF_BAR + N_BARS * 8;
    static constexpr int BYTES = OFF_SLOT + 16;
    // Up to 1024 B of slack for the 1024-B alignment of the swizzled tiles
    // (capped at the 227 KB limit; the kernel checks the aligned layout
    // fits); never less than 120 KB so that two CTAs, each holding all 512
    // TMEM columns, can never share an SM and wait on each other's allocation.
    static constexpr int ALLOC_RAW = (BYTES + 1024) < MAX_DYN_SMEM ? (BYTES + 1024) : MAX_DYN_SMEM;
    static constexpr int ALLOC = ALLOC_RAW > 120 * 1024 ? ALLOC_RAW : 120 * 1024;
    static_assert(BYTES <= MAX_DYN_SMEM, "indexer shared-memory layout too large");
};

struct UnitInfo {
    int b, i0, nq, j0, j1;   // tiles visited: j0..j1-1 (sample index m in IDX_SAMPLE)
    long long row0;          // output row of the block's first query
};

// Query blocks of this launch (in block-list mode the length is read on the device).
__device__ __forceinline__ long long idx_blocks(const IndexerArgs& a) {
    long long nb = (long long)(a.g1 - a.g0);
    if (a.blk_list != nullptr) {
        const long long have = (long long)__ldg(a.blk_count) - a.list_off;
        nb = have < 0 ? 0 : (have < a.list_len ? have : a.list_len);
    }
    return nb;
}

// Unit u of nb * max_splits, split-major: every block's first run of key
// tiles (longest rows first), then every block's second run, and so on.
// Units dealt round-robin to the CTAs then come in windows of similar size;
// block-major order would give each CTA the same split of every block (with
// an even grid and two splits, half the CTAs would get only the short
// remainders).
template <int MODE>
__device__ __forceinline__ UnitInfo unit_info(const IndexerArgs& a, long long u, long long nb) {
    UnitInfo r;
    const int slot = (int)(u % nb);
    int g;
    if (a.blk_list != nullptr) {
        g = __ldg(a.blk_list + a.list_off + slot);
    } else {
        g = a.g1 - 1 - slot;
    }
    const int split = (int)(u / nb);
    r.b = g / a.nqb;
    r.i0 = (g % a.nqb) * a.QB;
    r.nq = min(a.QB, a.Lq - r.i0);
    r.row0 = a.blk_list != nullptr ? (long long)slot * a.QB
                                   : (long long)r.b * a.Lq + r.i0 - a.row_base;
    int t_last = a.q_offset + r.i0 + r.nq - 1;
    int n_vis = min(t_last + 1, a.Lk);
    int nt = (n_vis + IDX_BM - 1) / IDX_BM;
    if (MODE == IDX_SAMPLE) nt = (nt + a.stride - 1) / a.stride;
    r.j0 = split * a.tpu;
    r.j1 = min(r.j0 + a.tpu, nt);
    return r;
}

template <int H, int DI, int MODE>
__global__ void __launch_bounds__(idx_threads(H, MODE), 1)
indexer_scores_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k, const IndexerArgs args) {
    using S = IndexerSmem<DI>;
    constexpr int KBOX = DI / 64;                 // 64-element (128-byte) swizzle boxes along d_I
    constexpr int QBMAX = IDX_NMAX / H;
    constexpr int EPI = idx_epi_warps(H, MODE);
    constexpr int NG = EPI / 4;                   // epilogue warps per TMEM lane quarter

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw, S::BYTES);
    if (smem == nullptr) return;                  // uniform: every thread sees the same sizes
    uint8_t* q_s = smem + S::OFF_Q;
    uint8_t* a_s = smem + S::OFF_A;
    float* w_s = reinterpret_cast<float*>(smem + S::OFF_W);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 2;
    uint64_t* a_full = bars + 4;
    uint64_t* a_empty = a_full + IDX_STAGES;
    uint64_t* acc_full = a_empty + IDX_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::OFF_SLOT);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long n_blocks = idx_blocks(args);
    const long long n_units = n_blocks * args.max_splits;
    const int kstride = MODE == IDX_SAMPLE ? args.stride : 1;   // key tile = visited index * kstride

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            // freed by the MMA commit of the unit's last tile and by every
            // epilogue warp once it has read the unit's head weights
            mbar_init(&q_empty[i], 1 + EPI);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 32 * EPI);
        }
        for (int i = 0; i < IDX_STAGES; ++i) {
            mbar_init(&a_full[i], 1);
            mbar_init(&a_empty[i], 1);
        }
        fence_barrier_init();
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            const uint32_t q_bytes = (uint32_t)args.N * 128u * KBOX;
            const uint32_t a_bytes = (uint32_t)S::A_BYTES;
            uint32_t uq = 0, ta = 0;
            bool ok = true;
            for (long long u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                UnitInfo ui = unit_info<MODE>(args, u, n_blocks);
                if (ui.j0 >= ui.j1) continue;
                const int qb = uq & 1;
                if (!mbar_wait(&q_empty[qb], ((uq >> 1) & 1) ^ 1)) { ok = false; break; }
                const uint32_t w_bytes = (uint32_t)(ui.nq * H * 4);
                mbar_arrive_expect_tx(&q_full[qb], q_bytes + w_bytes);
                uint8_t* qdst = q_s + qb * S::Q_BYTES;
                for (int kb = 0; kb < KBOX; ++kb)
                    tma_load_3d(qdst + kb * args.N * 128, &tmap_q, &q_full[qb], kb * 64, ui.i0 * H,
                                ui.b);
                bulk_load(w_s + qb * IDX_NMAX, args.w + ((long long)ui.b * args.Lq + ui.i0) * H,
                          w_bytes, &q_full[qb]);
                ++uq;
                for (int j = ui.j0; j < ui.j1; ++j, ++ta) {
                    const int st = ta % IDX_STAGES;
                    if (!mbar_wait(&a_empty[st], ((ta / IDX_STAGES) & 1) ^ 1)) { ok = false; break; }
                    mbar_arrive_expect_tx(&a_full[st], a_bytes);
                    uint8_t* adst = a_s + st * S::A_BYTES;
                    for (int kb = 0; kb < KBOX; ++kb)
                        tma_load_3d(adst + kb * IDX_BM * 128, &tmap_k, &a_full[st], kb * 64,
                                    j * kstride * IDX_BM, ui.b);
                }
            }
            // Drain: every load issued has landed before the CTA may retire.
            for (uint32_t i = (uq > 2 ? uq - 2 : 0); i < uq; ++i)
                mbar_wait(&q_full[i & 1], (i >> 1) & 1);
            for (uint32_t i = (ta > IDX_STAGES ? ta - IDX_STAGES : 0); i < ta; ++i)
                mbar_wait(&a_full[i % IDX_STAGES], (i / IDX_STAGES) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            const uint32_t idesc = idesc_bf16_f32(IDX_BM, args.N);
            uint32_t uq = 0, ta = 0;
            bool ok = true;
            for (long long u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                UnitInfo ui = unit_info<MODE>(args, u, n_blocks);
                if (ui.j0 >= ui.j1) continue;
                const int qb = uq & 1;
                if (!mbar_wait(&q_full[qb], (uq >> 1) & 1)) { ok = false; break; }
                const uint32_t q_addr = smem_u32(q_s + qb * S::Q_BYTES);
                for (int j = ui.j0; j < ui.j1; ++j, ++ta) {
                    const int st = ta % IDX_STAGES;
                    const int ab = ta & 1;
                    if (!mbar_wait(&a_full[st], (ta / IDX_STAGES) & 1)) { ok = false; break; }
                    if (!mbar_wait(&acc_empty[ab], ((ta >> 1) & 1) ^ 1)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(a_s + st * S::A_BYTES);
                    const uint32_t d_tmem = tmem_base + (uint32_t)(ab * IDX_NMAX);
#pragma unroll
                    for (int kk = 0; kk < DI / 16; ++kk) {
                        const uint32_t koff = (uint32_t)((kk & 3) * 32);
                        const uint64_t ad =
                            sw128_kmajor_desc(a_addr + (kk >> 2) * IDX_BM * 128 + koff);
                        const uint64_t bd =
                            sw128_kmajor_desc(q_addr + (kk >> 2) * args.N * 128 + koff);
                        tc_mma_f16(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&a_empty[st]);
                    tc_commit(&acc_full[ab]);
                }
                if (!ok) break;
                tc_commit(&q_empty[qb]);
                ++uq;
            }
        }
    } else {
        // ---------------- epilogue (warps 2 .. 1 + EPI)
        const int wq = warp & 3;                  // TMEM lane quarter this warp may read
        const int cg = (warp - 2) >> 2;           // which part of the block's queries (of NG)
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        constexpr int QH = (QBMAX + NG - 1) / NG; // queries per part at most
        constexpr bool QUAD = H >= 64;            // 16x256b TMEM reads, weights in registers
        const unsigned lt = (1u << lane) - 1u;
        uint32_t ta = 0, uq = 0;
        bool ok = true;
        for (long long u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            UnitInfo ui = unit_info<MODE>(args, u, n_blocks);
            if (ui.j0 >= ui.j1) continue;
            const int qb = uq & 1;
            // queries [qlo, qhi) of this block belong to this warp
            const int qpart = (args.QB + NG - 1) / NG;
            const int qlo = cg * qpart;
            const int qhi = min(ui.nq, qlo + qpart);
            const int ncol = (qhi > qlo ? qhi - qlo : 0) * H;        // multiple of 4
            const int nchunk = (ncol + 31) / 32;
            // the unit's head weights are in w_s[qb] once q_full[qb] completed
            if (!mbar_wait(&q_full[qb], (uq >> 1) & 1)) { ok = false; break; }
            const float* wsm = w_s + qb * IDX_NMAX + qlo * H;
            const long long row0 = ui.row0 + qlo;
            // QUAD: this thread's head weights of the unit, heads 8m + 2(lane%4) + {0,1}
            float2 wr[QUAD ? QH : 1][QUAD ? H / 8 : 1];
            if constexpr (QUAD) {
#pragma unroll
                for (int q = 0; q < QH; ++q)
#pragma unroll
                    for (int m = 0; m < H / 8; ++m)
                        wr[q][m] = q < qhi - qlo
                                       ? *reinterpret_cast<const float2*>(wsm + q * H + 8 * m + 2 * (lane & 3))
                                       : make_float2(0.0f, 0.0f);
            }
            const int t0 = args.q_offset + ui.i0 + qlo;
            uint32_t thrk[QH];
            // IDX_CAND: list slots are reserved ahead of need.  Per query the
            // warp holds a current range of IDX_RES slots [cpos, cend) and the
            // result (lane 0) of the atomic that reserved the next range,
            // issued when the current range was taken; a tile waits on an
            // atomic only when it crosses into a new range.  Slots still
            // unused when the unit ends are filled with 0, a value no
            // candidate takes (it would need a NaN key and position
            // 0xFFFFFFFF); the selection skips them.
            unsigned cpos[QH], cend[QH], npend[QH];
            auto reserve_next = [&](int q) {
                if (lane == 0) npend[q] = atomicAdd(args.cnt + row0 + q, (unsigned)IDX_RES);
            };
            auto pad = [&](int q, unsigned from, unsigned to) {          // sentinel-fill [from, to)
                for (unsigned x = from + lane; x < to; x += 32)
                    if (x < (unsigned)args.cap) args.cand[(row0 + q) * args.cap + x] = 0ull;
            };
            if (MODE == IDX_CAND) {
#pragma unroll
                for (int q = 0; q < QH; ++q) {
                    thrk[q] = q < qhi - qlo ? __ldg(args.thr + row0 + q) : IDX_NONE;
                    cpos[q] = cend[q] = 0u;
                    npend[q] = 0u;
                    if (q < qhi - qlo && thrk[q] != IDX_NONE) reserve_next(q);
                }
            }
            for (int j = ui.j0; j < ui.j1; ++j, ++ta) {
                const int ab = ta & 1;
                if (!mbar_wait(&acc_full[ab], (ta >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
                // Head-weighted ReLU sums.
                //  H >= 16: TMEM is read with the 16x256b shape, so a thread
                //  holds two keys (rows j and j+8 of each 16-lane half) x two
                //  columns of every 8-column block and needs only a quarter of
                //  the head weights, kept in registers for the unit (no
                //  shared-memory reads per tile).  Each (key, query) sum runs in
                //  packed f32x2 chains over the thread's heads; the four threads
                //  of a quad then add their partial sums with two shuffles.
                //  Afterwards thread (j = lane/4, e = lane%4) holds key
                //  klane = 16(e/2) + 8(e%2) + j of the warp's 32.
                //  H <= 8 (many queries per warp): 32x32b loads, one key per
                //  thread over all heads, weights broadcast from shared memory.
                float acc[QH];
                int klane = lane;
                if constexpr (QUAD) {
                    float p[2][2][QH];                                    // [lane half][row][query]
#pragma unroll
                    for (int lh = 0; lh < 2; ++lh) {
                        float2 a2[2][QH];
#pragma unroll
                        for (int q = 0; q < QH; ++q) a2[0][q] = a2[1][q] = make_float2(0.0f, 0.0f);
                        if (qhi > qlo) {                                  // warp-uniform
                            constexpr int REPS = QH * H / 8;              // 8-column repetitions
                            static_assert(REPS == 8 || REPS == 16, "16x256b reads of 64 or 128 columns");
                            uint32_t v[4 * REPS];
                            const uint32_t ta16 = tmem_base + ((uint32_t)(wq * 32 + 16 * lh) << 16) +
                                                  (uint32_t)(ab * IDX_NMAX + qlo * H);
                            if constexpr (REPS == 16)
                                tmem_ld_16x256b_x16(ta16, *reinterpret_cast<uint32_t(*)[64]>(&v[0]));
                            else
                                tmem_ld_16x256b_x8(ta16, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                            tmem_ld_wait();
                            if (IDX_EARLY_FREE && lh == 1) {          // the tile's TMEM is read
                                tc_fence_before();
                                mbar_arrive(&acc_empty[ab]);
                            }
#pragma unroll
                            for (int r = 0; r < REPS; ++r) {
                                const int q = (8 * r) / H, m = ((8 * r) % H) / 8;
                                const float2 r0 = make_float2(fmaxf(__uint_as_float(v[4 * r]), 0.0f),
                                                              fmaxf(__uint_as_float(v[4 * r + 1]), 0.0f));
                                const float2 r1 = make_float2(fmaxf(__uint_as_float(v[4 * r + 2]), 0.0f),
                                                              fmaxf(__uint_as_float(v[4 * r + 3]), 0.0f));
                                a2[0][q] = __ffma2_rn(wr[q][m], r0, a2[0][q]);
                                a2[1][q] = __ffma2_rn(wr[q][m], r1, a2[1][q]);
                            }
                        }
                        if (IDX_EARLY_FREE && lh == 1 && qhi <= qlo) {
                            tc_fence_before();
                            mbar_arrive(&acc_empty[ab]);
                        }
#pragma unroll
                        for (int q = 0; q < QH; ++q) {
                            p[lh][0][q] = a2[0][q].x + a2[0][q].y;
                            p[lh][1][q] = a2[1][q].x + a2[1][q].y;
                        }
                    }
#pragma unroll
                    for (int lh = 0; lh < 2; ++lh)
#pragma unroll
                        for (int rw = 0; rw < 2; ++rw)
#pragma unroll
                            for (int q = 0; q < QH; ++q) {
                                float x = p[lh][rw][q];
                                x += __shfl_xor_sync(0xffffffffu, x, 1);
                                x += __shfl_xor_sync(0xffffffffu, x, 2);
                                p[lh][rw][q] = x;
                            }
                    const int e = lane & 3;
                    klane = 16 * (e >> 1) + 8 * (e & 1) + (lane >> 2);
#pragma unroll
                    for (int q = 0; q < QH; ++q)
                        acc[q] = e == 0 ? p[0][0][q] : e == 1 ? p[0][1][q] : e == 2 ? p[1][0][q] : p[1][1][q];
                } else {
                    const uint32_t taddr =
                        tmem_base + lane_base + (uint32_t)(ab * IDX_NMAX + qlo * H);
#pragma unroll
                    for (int q = 0; q < QH; ++q) acc[q] = 0.0f;
                    // 64 columns per batch: two 32-column TMEM loads, one wait, reduce.
#pragma unroll
                    for (int bt = 0; bt < (QH * H + 63) / 64; ++bt) {
                        if (bt * 2 < nchunk) {
                            uint32_t v[64];
                            tmem_ld_32x32b_x32(taddr + bt * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                            if (bt * 2 + 1 < nchunk)
                                tmem_ld_32x32b_x32(taddr + bt * 64 + 32,
                                                   *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                            tmem_ld_wait();
#pragma unroll
                            for (int jj = 0; jj < 64; jj += 4) {
                                const int c = bt * 64 + jj;
                                if (c < ncol) {
                                    // columns c..c+3 are four heads of one query (H % 4 == 0)
                                    const int q = c / H;
                                    const float4 wv = *reinterpret_cast<const float4*>(wsm + c);
                                    float& a = acc[q];
                                    a = fmaf(wv.x, fmaxf(__uint_as_float(v[jj]), 0.0f), a);
                                    a = fmaf(wv.y, fmaxf(__uint_as_float(v[jj + 1]), 0.0f), a);
                                    a = fmaf(wv.z, fmaxf(__uint_as_float(v[jj + 2]), 0.0f), a);
                                    a = fmaf(wv.w, fmaxf(__uint_as_float(v[jj + 3]), 0.0f), a);
                                }
                            }
                        }
                    }
                }
                if (!(QUAD && IDX_EARLY_FREE)) {
                    tc_fence_before();
                    mbar_arrive(&acc_empty[ab]);
                }
                const int s = j * kstride * IDX_BM + wq * 32 + klane;     // key position
                if (MODE == IDX_CAND) {
#pragma unroll
                    for (int q = 0; q < QH; ++q) {
                        if (q < qhi - qlo && thrk[q] != IDX_NONE) {       // warp-uniform
                            const uint32_t key = score_key(acc[q]);
                            const bool sel = s <= t0 + q && key >= thrk[q];
                            const unsigned bal = __ballot_sync(0xffffffffu, sel);
                            if (bal != 0u) {
                                const unsigned n = __popc(bal), rank = __popc(bal & lt);
                                const unsigned a = min(n, cend[q] - cpos[q]);
                                unsigned slot = cpos[q] + rank;
                                cpos[q] += a;
                                if (n > a) {                              // into the next range
                                    const unsigned nb = __shfl_sync(0xffffffffu, npend[q], 0);
                                    if (rank >= a) slot = nb + (rank - a);
                                    cpos[q] = nb + (n - a);
                                    cend[q] = nb + IDX_RES;
                                    reserve_next(q);
                                }
                                if (sel && slot < (unsigned)args.cap)
                                    args.cand[(row0 + q) * args.cap + slot] =
                                        ((unsigned long long)key << 32) | (uint32_t)(~(uint32_t)s);
                            }
                        }
                    }
                } else if (s < args.Lk) {
                    const long long col = MODE == IDX_SAMPLE ? (long long)j * IDX_BM + wq * 32 + klane
                                                             : (long long)s;
                    float* dst = args.scores + row0 * args.ld + col;
#pragma unroll
                    for (int q = 0; q < QH; ++q) {
                        if (q < qhi - qlo) {
                            const float val = (s <= t0 + q) ? acc[q] : -INFINITY;
                            dst[(long long)q * args.ld] = val;
                        }
                    }
                }
            }
            if (!ok) break;
            if (MODE == IDX_CAND) {                                       // unused reserved slots
#pragma unroll
                for (int q = 0; q < QH; ++q) {
                    if (q < qhi - qlo && thrk[q] != IDX_NONE) {
                        pad(q, cpos[q], cend[q]);
                        const unsigned nb = __shfl_sync(0xffffffffu, npend[q], 0);
                        pad(q, nb, nb + IDX_RES);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_empty[qb]);
            ++uq;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// Writes -inf into score columns [ntiles*128, Lk) of each row: the part of a
// row beyond the key tiles the indexer visited, all of it invisible.
__global__ void indexer_fill_masked_kernel(float* scores, long long ld, int Lq, int Lk,
                                           int q_offset, int QB, long long row_base,
                                           long long n_rows) {
    for (long long row = blockIdx.x; row < n_rows; row += gridDim.x) {
        long long fr = row_base + row;
        int i = (int)(fr % Lq);
        int i0 = (i / QB) * QB;
        int nq = min(QB, Lq - i0);
        int t_last = q_offset + i0 + nq - 1;
        int n_vis = min(t_last + 1, Lk);
        int start = ((n_vis + IDX_BM - 1) / IDX_BM) * IDX_BM;
        float* dst = scores + row * ld;
        for (int s = start + threadIdx.x; s < Lk; s += blockDim.x) dst[s] = -INFINITY;
    }
}

}  // namespace ic
