// libindexcache.so: the C ABI declared in include/indexcache.h.
//
// Host side only validates arguments, builds TMA descriptors, sizes grids and
// enqueues the sm_100a kernels on the caller's stream; every step of the
// computation runs in the kernels below.  Nothing is allocated and nothing is
// cached between calls except per-device launch attributes.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "indexcache.h"
#include "common.cuh"
#include "dense_attn.cuh"
#include "fused_topk.cuh"
#include "index_overlap.cuh"
#include "indexer_scores.cuh"
#include "sparse_attn.cuh"
#include "topk_select.cuh"

namespace {

thread_local char g_msg[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(IC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Kernel launches this library has issued, over the process (all devices).
std::atomic<unsigned long long> g_launches{0};

// Status of the launch just made; counts it when it went in.
int launched(cudaError_t e, const char* what) {
    if (e != cudaSuccess) return cuda_fail(e, what);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return IC_OK;
}

// An NVTX range around host work, for profilers (a no-op unless one is
// attached); the scope pops it on every return path.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// fp32 / int32 buffers read and written element by element
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// ---------------------------------------------------------------- device facts

constexpr int MAX_DEV = 64;
std::mutex g_mu;
int g_sms[MAX_DEV];
bool g_attr_done[MAX_DEV];
// 8-CTA clusters of the gather kernel fit on the device (checked at setup)
bool g_attn_cluster[MAX_DEV];

int device_setup(int* dev_out, int* sms_out);

// ---------------------------------------------------------------- TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
// Looked up once; host threads may race on the first lookup (they store the
// same pointer), so the slot is atomic.
std::atomic<EncodeTiledFn> g_encode_fn{nullptr};

int get_encode() {
    if (g_encode_fn.load(std::memory_order_acquire)) return IC_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return fail(IC_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    g_encode_fn.store(reinterpret_cast<EncodeTiledFn>(fn), std::memory_order_release);
    return IC_OK;
}

// Valid after get_encode() returned IC_OK.
EncodeTiledFn encoder() { return g_encode_fn.load(std::memory_order_acquire); }

// 3-D bf16 tensor {d0 (contiguous), d1, d2}, 128-byte swizzled boxes {64, box1, 1}.
int make_tmap_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint32_t box1) {
    int rc = get_encode();
    if (rc) return rc;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {64, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(IC_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return IC_OK;
}

// ---------------------------------------------------------------- indexer

struct IndexerGeom {
    int QB, N, nqb;
};

IndexerGeom indexer_geom(int Lq, int H) {
    IndexerGeom g;
    g.QB = std::min(ic::IDX_NMAX / H, Lq);
    g.N = ((g.QB * H + 15) / 16) * 16;
    g.nqb = (Lq + g.QB - 1) / g.QB;
    return g;
}

long long block_row_start(const IndexerGeom& g, int Lq, long long gb) {
    return (gb / g.nqb) * (long long)Lq + (gb % g.nqb) * (long long)g.QB;
}

template <int H, int DI>
void set_indexer_attr() {
    cudaFuncSetAttribute(ic::indexer_scores_kernel<H, DI, ic::IDX_SCORES>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, ic::IndexerSmem<DI>::ALLOC);
    cudaFuncSetAttribute(ic::indexer_scores_kernel<H, DI, ic::IDX_SAMPLE>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, ic::IndexerSmem<DI>::ALLOC);
    cudaFuncSetAttribute(ic::indexer_scores_kernel<H, DI, ic::IDX_CAND>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, ic::IndexerSmem<DI>::ALLOC);
}

template <int H, int DI>
cudaError_t launch_indexer_t(int mode, const CUtensorMap& tq, const CUtensorMap& tk,
                             const ic::IndexerArgs& a, int grid, cudaStream_t st) {
    constexpr int SM = ic::IndexerSmem<DI>::ALLOC;
    if (mode == ic::IDX_SAMPLE)
        ic::indexer_scores_kernel<H, DI, ic::IDX_SAMPLE><<<grid, ic::idx_threads(H, ic::IDX_SAMPLE), SM, st>>>(tq, tk, a);
    else if (mode == ic::IDX_CAND)
        ic::indexer_scores_kernel<H, DI, ic::IDX_CAND><<<grid, ic::idx_threads(H, ic::IDX_CAND), SM, st>>>(tq, tk, a);
    else
        ic::indexer_scores_kernel<H, DI, ic::IDX_SCORES><<<grid, ic::idx_threads(H, ic::IDX_SCORES), SM, st>>>(tq, tk, a);
    return cudaGetLastError();
}

template <int DI>
cudaError_t launch_indexer_h(int H, int mode, const CUtensorMap& tq, const CUtensorMap& tk,
                             const ic::IndexerArgs& a, int grid, cudaStream_t st) {
    switch (H) {
        case 4: return launch_indexer_t<4, DI>(mode, tq, tk, a, grid, st);
        case 8: return launch_indexer_t<8, DI>(mode, tq, tk, a, grid, st);
        case 16: return launch_indexer_t<16, DI>(mode, tq, tk, a, grid, st);
        case 32: return launch_indexer_t<32, DI>(mode, tq, tk, a, grid, st);
        case 64: return launch_indexer_t<64, DI>(mode, tq, tk, a, grid, st);
        case 128: return launch_indexer_t<128, DI>(mode, tq, tk, a, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

// What an indexer launch does besides storing every score of its blocks
// (the default): the sampled tiles only, candidates above per-row
// thresholds, and/or query blocks taken from a device list.
struct IdxExtra {
    int mode = ic::IDX_SCORES;
    int stride = 1;                       // IDX_SAMPLE
    const uint32_t* thr = nullptr;        // IDX_CAND
    uint32_t* cnt = nullptr;
    unsigned long long* cand = nullptr;
    int cap = 0;
    const int* blk_list = nullptr;        // block list (blocks of [g0, g1) only)
    const int* blk_count = nullptr;
    int list_off = 0, list_len = 0;
    int tpu = 0;                          // key tiles per work unit (0: sized from the work)
};

// Scores query blocks [g0, g1) into `scores` (row = flattened row - row of g0),
// or does what `x` asks instead (sampled tiles, candidates, a block list).
int launch_indexer(const uint16_t* q_idx, const uint16_t* k_idx, const float* w, int B, int Lq,
                   int Lk, int H, int dI, int q_offset, long long g0, long long g1, float* scores,
                   long long ld, bool fill_masked, int sms, cudaStream_t st,
                   const IdxExtra& x = IdxExtra()) {
    const IndexerGeom geo = indexer_geom(Lq, H);
    CUtensorMap tq, tk;
    int rc = make_tmap_3d(&tq, q_idx, (uint64_t)dI, (uint64_t)Lq * H, (uint64_t)B, (uint32_t)geo.N);
    if (rc) return rc;
    rc = make_tmap_3d(&tk, k_idx, (uint64_t)dI, (uint64_t)Lk, (uint64_t)B, (uint32_t)ic::IDX_BM);
    if (rc) return rc;

    // Key tiles visited over the range (every stride-th in IDX_SAMPLE), to size work units.
    const int stride = x.mode == ic::IDX_SAMPLE ? std::max(1, x.stride) : 1;
    long long total = 0;
    int max_nt = 0;
    for (long long gb = g0; gb < g1; ++gb) {
        const int i0 = (int)(gb % geo.nqb) * geo.QB;
        const int nq = std::min(geo.QB, Lq - i0);
        const int n_vis = std::min(q_offset + i0 + nq, Lk);
        const int nt = ((n_vis + ic::IDX_BM - 1) / ic::IDX_BM + stride - 1) / stride;
        total += nt;
        max_nt = std::max(max_nt, nt);
    }
    const bool listed = x.blk_list != nullptr;
    long long blocks = listed ? std::min<long long>(x.list_len, g1 - g0) : g1 - g0;
    if (listed) {
        // unknown until run time how many blocks are listed: units of a
        // few tiles, so that even one long block spreads over many CTAs
        total = (long long)blocks * max_nt;
    }
    int tpu = (int)std::min<long long>(64, std::max<long long>(4, total / (6LL * sms)));
    if (listed) tpu = std::max(4, std::min(tpu, max_nt / 8));
#ifndef IC_IDX_EVEN_UNITS
#define IC_IDX_EVEN_UNITS 1
#endif
    if (IC_IDX_EVEN_UNITS && !listed && total == blocks * (long long)max_nt && max_nt > 4) {
        // Every block has the same number of key tiles (decode: one row per
        // sequence, all at the same position), so every unit costs the same
        // and the busiest CTA sets the time: take the unit length that
        // minimises its tiles, counting one tile of overhead per unit.
        long long best = -1;
        for (int c = 4; c <= std::min(64, max_nt); ++c) {
            const long long units = blocks * (long long)((max_nt + c - 1) / c);
            const long long cost = (units + sms - 1) / sms * (long long)(c + 1);
            if (best < 0 || cost < best) {
                best = cost;
                tpu = c;
            }
        }
    }
    if (x.tpu > 0) tpu = x.tpu;
    tpu = std::min(tpu, std::max(1, max_nt));
    const int max_splits = (max_nt + tpu - 1) / tpu;

    ic::IndexerArgs a{};
    a.w = w;
    a.scores = scores;
    a.ld = ld;
    a.B = B;
    a.Lq = Lq;
    a.Lk = Lk;
    a.q_offset = q_offset;
    a.QB = geo.QB;
    a.N = geo.N;
    a.nqb = geo.nqb;
    a.g0 = (int)g0;
    a.g1 = (int)g1;
    a.row_base = block_row_start(geo, Lq, g0);
    a.tpu = tpu;
    a.max_splits = max_splits;
    a.stride = stride;
    a.thr = x.thr;
    a.cnt = x.cnt;
    a.cand = x.cand;
    a.cap = x.cap;
    a.blk_list = x.blk_list;
    a.blk_count = x.blk_count;
    a.list_off = x.list_off;
    a.list_len = (int)blocks;
    const long long n_units = blocks * (long long)max_splits;
    const int grid = (int)std::min<long long>(n_units, sms);
    if (grid <= 0) return IC_OK;
    cudaError_t e = dI == 64 ? launch_indexer_h<64>(H, x.mode, tq, tk, a, grid, st)
                             : launch_indexer_h<128>(H, x.mode, tq, tk, a, grid, st);
    if (launched(e, "indexer_scores launch")) return IC_ERR_CUDA;
    if (fill_masked) {
        const long long n_rows = block_row_start(geo, Lq, g1) - a.row_base;
        const int fg = (int)std::min<long long>(n_rows, 65535);
        ic::indexer_fill_masked_kernel<<<fg, 256, 0, st>>>(scores, ld, Lq, Lk, q_offset, geo.QB,
                                                           a.row_base, n_rows);
        e = cudaGetLastError();
        if (launched(e, "indexer fill launch")) return IC_ERR_CUDA;
    }
    return IC_OK;
}

// ---------------------------------------------------------------- top-k

// Rows [row_base, row_base + n_rows) of `scores`, or (lst.blk_list non-null)
// the rows of the listed blocks, whose scores sit in consecutive rows.
int launch_topk(const float* scores, long long ld, long long row_base, long long n_rows, int Lq,
                int Lk, int q_offset, int k, int32_t* idx, int sms, cudaStream_t st,
                uint32_t* mask = nullptr, int Lq_d = 0, int W = 0,
                const ic::TopkList& lst = ic::TopkList{}) {
    if (n_rows <= 0) return IC_OK;
    const int n_max = std::min(Lk, q_offset + Lq);
    // one CTA per row; a listed launch loops a persistent grid over its rows
    const unsigned grid = lst.blk_list != nullptr
                              ? (unsigned)std::min<long long>(n_rows, 8LL * sms)
                              : (unsigned)n_rows;
    cudaError_t e;
    if (n_rows < 2LL * sms && n_max > 4096) {
        // few long rows (decode): a 1024-thread CTA per row, one per SM
        if (n_max <= ic::TK_CACHE_MAX_FEW) {
            ic::topk_select_kernel<ic::TK_THREADS_FEW, true>
                <<<grid, ic::TK_THREADS_FEW, ic::TK_SMEM_FIXED + n_max * 4, st>>>(
                    scores, ld, row_base, n_rows, Lq, Lk, q_offset, k, idx, mask, Lq_d, W, lst);
        } else {
            ic::topk_select_kernel<ic::TK_THREADS_FEW, false>
                <<<grid, ic::TK_THREADS_FEW, ic::TK_SMEM_FIXED, st>>>(
                    scores, ld, row_base, n_rows, Lq, Lk, q_offset, k, idx, mask, Lq_d, W, lst);
        }
    } else if (n_max <= ic::TK_CACHE_MAX) {
        const int smem = ic::TK_SMEM_FIXED + n_max * 4;
        ic::topk_select_kernel<ic::TK_THREADS, true><<<grid, ic::TK_THREADS, smem, st>>>(
            scores, ld, row_base, n_rows, Lq, Lk, q_offset, k, idx, mask, Lq_d, W, lst);
    } else {
        ic::topk_select_kernel<ic::TK_THREADS_LONG, false>
            <<<grid, ic::TK_THREADS_LONG, ic::TK_SMEM_FIXED, st>>>(
                scores, ld, row_base, n_rows, Lq, Lk, q_offset, k, idx, mask, Lq_d, W, lst);
    }
    e = cudaGetLastError();
    if (launched(e, "topk_select launch")) return IC_ERR_CUDA;
    return IC_OK;
}

// ---------------------------------------------------------------- sparse attention

int attn_splits(long long n_rows, int k_slots, int sms) {
    // rows x splits CTAs fill two CTAs per SM in one wave (three fit: the
    // spare slot absorbs the ragged end of the wave)
    if (n_rows >= 2LL * sms) return 1;
    long long s = (2LL * sms) / n_rows;
    s = std::min<long long>(s, (k_slots + ic::SA_WARPS * ic::SA_BLOCK - 1) / (ic::SA_WARPS * ic::SA_BLOCK));
    s = std::min<long long>(s, 64);
    return (int)std::max<long long>(1, s);
}

// Splits of up to ATTN_CLUSTER_MAX CTAs run as one thread-block cluster per
// row and merge through distributed shared memory (no workspace, no combine
// launch); a one-wave split count up to 16 is trimmed to it.  Measured on
// decode rows of 2048 slots: 8 beats 4, 6 and 10.
#ifndef IC_ATTN_CLUSTER_MAX
#define IC_ATTN_CLUSTER_MAX 8
#endif
constexpr int ATTN_CLUSTER_MAX = IC_ATTN_CLUSTER_MAX;
static_assert(ATTN_CLUSTER_MAX >= 2 && ATTN_CLUSTER_MAX <= 8, "portable cluster sizes only");

template <int D>
bool attn_cluster_fits() {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, ATTN_CLUSTER_MAX, 1);
    cfg.blockDim = dim3(ic::SA_THREADS, 1, 1);
    cfg.dynamicSmemBytes = ic::SaSmem<D>::BYTES;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = ATTN_CLUSTER_MAX;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    return cudaOccupancyMaxActiveClusters(&n, ic::sparse_attn_kernel<D>, &cfg) == cudaSuccess && n > 0;
}

bool attn_cluster_available() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEV) return false;
    return g_attn_cluster[dev];
}

template <int D>
cudaError_t launch_attn_kernel(const ic::SparseAttnArgs& a, dim3 grid, bool cluster, cudaStream_t st) {
    if (!cluster) {
        ic::sparse_attn_kernel<D><<<grid, ic::SA_THREADS, ic::SaSmem<D>::BYTES, st>>>(a);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(ic::SA_THREADS, 1, 1);
    cfg.dynamicSmemBytes = ic::SaSmem<D>::BYTES;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = grid.y;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ic::sparse_attn_kernel<D>, a);
}

size_t attn_ws_bytes(long long n_rows, int splits, int Hq, int d) {
    if (splits <= 1) return 0;
    return (size_t)n_rows * splits * (size_t)Hq * (d + 1) * sizeof(float);
}

// Gather attention over rows i in [row_i0, row_i0 + rows_per_b) of every
// sequence (rows_per_b < 0: all rows).
int launch_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* idx,
                int B, int Lq, int Lk, int Hq, int d, int k_slots, int q_offset, float scale,
                uint16_t* out, float* lse, void* ws, size_t ws_bytes, bool trim, int sms,
                cudaStream_t st, int row_i0 = 0, int rows_per_b = -1) {
    if (rows_per_b < 0) rows_per_b = Lq - row_i0;
    const long long n_rows = (long long)B * rows_per_b;
    if (n_rows <= 0) return IC_OK;
    int splits = attn_splits(n_rows, k_slots, sms);
    const bool cluster = splits > 1 && splits <= 16 && attn_cluster_available();
    if (cluster) splits = std::min(splits, ATTN_CLUSTER_MAX);
    while (!cluster && splits > 1 && (ws == nullptr || attn_ws_bytes(n_rows, splits, Hq, d) > ws_bytes))
        splits = splits / 2;
    ic::SparseAttnArgs a;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.k = reinterpret_cast<const __nv_bfloat16*>(k);
    a.v = reinterpret_cast<const __nv_bfloat16*>(v);
    a.idx = idx;
    a.out = reinterpret_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.cluster = cluster ? 1 : 0;
    a.part_o = splits > 1 && !cluster ? reinterpret_cast<float*>(ws) : nullptr;
    a.part_lse = splits > 1 && !cluster ? reinterpret_cast<float*>(ws) + n_rows * splits * (long long)Hq * d
                                        : nullptr;
    a.Lq = Lq;
    a.Lk = Lk;
    a.Hq = Hq;
    a.kslots = k_slots;
    a.q_offset = q_offset;
    a.splits = splits;
    a.slots_per_split = (k_slots + splits - 1) / splits;
    a.trim = trim ? 1 : 0;
    const float sc = scale > 0.0f ? scale : 1.0f / std::sqrt((float)d);
    a.scale_log2 = sc * ic::LOG2E;
    a.n_rows = n_rows;
    a.rows_per_b = rows_per_b;
    a.row_i0 = row_i0;
    dim3 grid((unsigned)n_rows, (unsigned)splits);
    cudaError_t e = d == 64 ? launch_attn_kernel<64>(a, grid, cluster, st)
                            : launch_attn_kernel<128>(a, grid, cluster, st);
    if (launched(e, "sparse_attn launch")) return IC_ERR_CUDA;
    if (splits > 1 && !cluster) {
        const dim3 cg((unsigned)n_rows, (unsigned)Hq);
        if (d == 64)
            ic::sparse_attn_combine_kernel<64><<<cg, 64, 0, st>>>(a);
        else
            ic::sparse_attn_combine_kernel<128><<<cg, 128, 0, st>>>(a);
        e = cudaGetLastError();
        if (launched(e, "sparse_attn combine launch")) return IC_ERR_CUDA;
    }
    return IC_OK;
}

// ---------------------------------------------------------------- dense-masked attention

// Rows whose top-k covers at least 1/DENSE_FACTOR of their visible positions
// (t < DENSE_FACTOR * k) attend tile-dense on the tensor cores; the others
// gather.  Only used inside the layer stack, whose index rows hold distinct
// positions (a bitmask cannot count a repeated index twice).
// Measured on B200 at k = 2048, Hq = 16: a dense-masked row costs about
// 9.6 ps per visible position, a gathered row about 103 ns, so the two meet
// near t = 5.3k; a factor of 6 against 8 took the 64K step from 111.2 to
// 109.9 ms and a 32K layer from 10.90 to 10.72 ms (same box).
#ifndef IC_DENSE_FACTOR
#define IC_DENSE_FACTOR 6
#endif
constexpr int DENSE_FACTOR = IC_DENSE_FACTOR;
// Keys a dense-masked row may see (bounds the bitmask row: 8 KB of shared
// memory in the mask build, and the transposed V copy).
constexpr int DENSE_MAX_KEYS = 65536;

struct DenseGeom {
    bool on = false;
    int QBD = 0, Lq_d = 0, nqb_d = 0, W = 0, Lk_d = 0, ldt = 0;
    size_t mask_bytes = 0, vt_bytes = 0, total = 0;
};

DenseGeom dense_geom(const ic_dims& D) {
    DenseGeom g;
    if (D.d != 128 || (128 % D.Hq) != 0) return g;
    g.QBD = 128 / D.Hq;
    long long lim = (long long)DENSE_FACTOR * D.k - D.q_offset;     // rows i with t < 6k
    lim = std::min<long long>(lim, (long long)DENSE_MAX_KEYS - D.q_offset);
    lim = std::min<long long>(lim, D.Lq);
    if (lim < g.QBD) return g;
    g.Lq_d = (int)(lim / g.QBD) * g.QBD;
    g.nqb_d = g.Lq_d / g.QBD;
    g.Lk_d = std::min(D.Lk, D.q_offset + g.Lq_d);
    g.W = (g.Lk_d + 31) / 32;
    g.ldt = ((g.Lk_d + 63) / 64) * 64;
    g.mask_bytes = (((size_t)D.B * g.Lq_d * g.W * 4) + 1023) / 1024 * 1024;
    g.vt_bytes = (size_t)D.B * 128 * g.ldt * 2;
    g.total = g.mask_bytes + g.vt_bytes;
    g.on = true;
    return g;
}

int launch_build_mask(const DenseGeom& g, const ic_dims& D, const int32_t* idx, uint32_t* mask,
                      cudaStream_t st) {
    const long long n = (long long)D.B * g.Lq_d;
    const int grid = (int)std::min<long long>(n, 65535);
    ic::build_mask_kernel<<<grid, 256, g.W * 4, st>>>(idx, D.Lq, D.k, D.q_offset, g.Lq_d, g.W,
                                                       mask, n);
    cudaError_t e = cudaGetLastError();
    return launched(e, "build_mask launch");
}

int launch_dense_attn(const DenseGeom& g, const ic_dims& D, const ic_layer& L,
                      const uint32_t* mask, uint16_t* vt, cudaStream_t st) {
    // V^T of this layer's keys < Lk_d, zero-padded to ldt columns
    dim3 tg((unsigned)(g.ldt / 64), (unsigned)D.B);
    ic::transpose_v_kernel<<<tg, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(L.v), D.Lk,
                                                g.Lk_d, g.ldt, reinterpret_cast<__nv_bfloat16*>(vt));
    cudaError_t e = cudaGetLastError();
    if (launched(e, "transpose_v launch")) return IC_ERR_CUDA;
    CUtensorMap tq, tk, tv;
    int rc = make_tmap_3d(&tq, L.q, 128, (uint64_t)D.Lq * D.Hq, (uint64_t)D.B, 128);
    if (!rc) rc = make_tmap_3d(&tk, L.k, 128, (uint64_t)D.Lk, (uint64_t)D.B, ic::DA_TILE);
    if (!rc) rc = get_encode();
    if (rc) return rc;
    {
        cuuint64_t dims[3] = {(cuuint64_t)g.Lk_d, 128, (cuuint64_t)D.B};
        cuuint64_t strides[2] = {(cuuint64_t)g.ldt * 2, (cuuint64_t)g.ldt * 2 * 128};
        cuuint32_t box[3] = {64, 128, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = encoder()(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, vt, dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(IC_ERR_CUDA, "cuTensorMapEncodeTiled (V^T) failed (%d)", (int)r);
    }
    ic::DenseAttnArgs a;
    a.mask = mask;
    a.out = reinterpret_cast<__nv_bfloat16*>(L.out);
    a.lse = L.lse;
    a.Lq = D.Lq;
    a.Lk = D.Lk;
    a.Hq = D.Hq;
    a.q_offset = D.q_offset;
    a.Lq_d = g.Lq_d;
    a.QBD = g.QBD;
    a.nqb_d = g.nqb_d;
    a.W = g.W;
    a.n_blocks = D.B * g.nqb_d;
    const float sc = D.scale > 0.0f ? D.scale : 1.0f / std::sqrt(128.0f);
    a.scale_log2 = sc * ic::LOG2E;
    ic::dense_attn_kernel<<<a.n_blocks, ic::DA_THREADS, ic::DenseSmem::ALLOC, st>>>(tq, tk, tv, a);
    e = cudaGetLastError();
    return launched(e, "dense_attn launch");
}

// How the attention step treats rows with t < 6k.
enum AttnMode {
    ATTN_GATHER = 0,        // every row gathers
    ATTN_MASK_READY = 1,    // dense-masked; the workspace already holds the bitmask
    ATTN_BUILD_MASK = 2,    // dense-masked; build the bitmask from idx first
};

// Attention of one layer over index rows that hold each position at most
// once.  Dense modes (the caller checked dense_geom(D).on and that ws holds
// dense_geom(D).total bytes): rows with t < 6k, whole blocks, on the
// dense-masked kernel -- bitmask at ws, V^T after it, the gathered rows'
// split partials after both -- and the rest gathered.  `trim` says slots past
// min(k, t+1) are empty (top-k output); `mid` (may be null) is recorded
// between the two parts.
int attn_step(const ic_dims& D, const ic_layer& L, const int32_t* idx, AttnMode mode, bool trim,
              void* ws, size_t ws_bytes, int sms, cudaStream_t st, cudaEvent_t mid) {
    auto mark = [&]() -> int {
        if (!mid) return IC_OK;
        cudaError_t e = cudaEventRecord(mid, st);
        return e == cudaSuccess ? IC_OK : cuda_fail(e, "cudaEventRecord");
    };
    int rc;
    if (mode == ATTN_GATHER) {
        if ((rc = mark())) return rc;
        return launch_attn(L.q, L.k, L.v, idx, D.B, D.Lq, D.Lk, D.Hq, D.d, D.k, D.q_offset,
                           D.scale, L.out, L.lse, ws, ws_bytes, trim, sms, st);
    }
    const DenseGeom dg = dense_geom(D);
    uint32_t* dmask = reinterpret_cast<uint32_t*>(ws);
    uint16_t* dvt = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(ws) + dg.mask_bytes);
    if (mode == ATTN_BUILD_MASK && (rc = launch_build_mask(dg, D, idx, dmask, st))) return rc;
    if ((rc = launch_dense_attn(dg, D, L, dmask, dvt, st))) return rc;
    if ((rc = mark())) return rc;
    if (dg.Lq_d >= D.Lq) return IC_OK;
    return launch_attn(L.q, L.k, L.v, idx, D.B, D.Lq, D.Lk, D.Hq, D.d, D.k, D.q_offset, D.scale,
                       L.out, L.lse, reinterpret_cast<uint8_t*>(ws) + dg.total, ws_bytes - dg.total,
                       trim, sms, st, dg.Lq_d, D.Lq - dg.Lq_d);
}

// ---------------------------------------------------------------- fused indexer -> top-k

constexpr int FUSED_CAP_FACTOR = 4;     // list slots a row may use: 4k
constexpr float FUSED_Z = 4.0f;         // threshold margin in binomial standard deviations
constexpr int FUSED_FB_DIV = 8;         // fallback scores: 1/8 of a chunk's blocks per round
constexpr int FUSED_MAX_K = 4096;       // candidate list in shared memory: 4k x 8 bytes
constexpr int FUSED_MAX_LK = 262144;    // bitmap of a row's positions in shared memory
constexpr int FUSED_AUTO_MIN_ROWS = 1024;

// Sizes of the fused path for given dims (ok = false when it cannot run).
constexpr int FUSED_TPU = 64;           // key tiles per unit of the candidate pass

struct FusedGeom {
    bool ok = false;
    int stride = 1;          // sampled key tiles m * stride
    int ns = 0;              // sampled tiles per row at most (<= 32)
    int cap = 0;             // candidates a row may keep (4k); rows with n <= cap keep all
    int lstride = 0;         // list slots per row: cap + what reserved, unused slots may take
    int n_max = 0;           // longest row's visible positions
};

FusedGeom fused_geom(const ic_dims& D) {
    FusedGeom f;
    if (D.k > FUSED_MAX_K || D.Lk > FUSED_MAX_LK || D.Lq < 1) return f;
    f.n_max = std::min(D.Lk, D.q_offset + D.Lq);
    const int nt_max = (f.n_max + ic::IDX_BM - 1) / ic::IDX_BM;
    f.stride = std::max(1, nt_max / 16);
    f.ns = (nt_max + f.stride - 1) / f.stride;
    f.cap = FUSED_CAP_FACTOR * D.k;
    // Each writer of a row's list (4 warp lane quarters x the candidate
    // pass's units of FUSED_TPU key tiles) leaves fewer than 2 reserved ranges
    // unused.
    const int splits = (nt_max + FUSED_TPU - 1) / FUSED_TPU;
    f.lstride = f.cap + 2 * (int)ic::IDX_RES * 4 * splits;
    f.ok = f.ns * ic::IDX_BM <= ic::FT_MAX_SAMPLES &&
           ic::fused_select_smem(f.lstride, D.Lk) <= (size_t)ic::MAX_DYN_SMEM;
    return f;
}

// Whether the stack fuses the top-k into the indexer: `mode` 1 asks for it,
// 0 refuses it, -1 leaves it to the library, which fuses when the longest
// row is over twice the candidate capacity and there are many rows (prefill).
bool fused_wanted(const FusedGeom& f, const ic_dims& D, int mode) {
    if (!f.ok || mode == 0) return false;
    if (mode == 1) return true;
    return f.n_max > 2 * f.cap && (long long)D.B * D.Lq >= FUSED_AUTO_MIN_ROWS;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace layout of one chunk of `blocks` query blocks on the fused path.
struct FusedLayout {
    size_t samp = 0, cand = 0, thr = 0, cnt = 0, flag = 0, list = 0, lcount = 0, fb = 0, total = 0;
    long long fb_blocks = 0;
};

FusedLayout fused_layout(const FusedGeom& f, long long blocks, int QB, int Lk) {
    FusedLayout L;
    const size_t rows = (size_t)blocks * QB;
    L.fb_blocks = (blocks + FUSED_FB_DIV - 1) / FUSED_FB_DIV;
    size_t o = 0;
    L.samp = o;   o = align256(o + rows * (size_t)f.ns * ic::IDX_BM * 4);
    L.cand = o;   o = align256(o + rows * (size_t)f.lstride * 8);
    L.thr = o;    o = align256(o + rows * 4);
    L.cnt = o;    o = align256(o + rows * 4);
    L.flag = o;   o = align256(o + (size_t)blocks * 4);
    L.list = o;   o = align256(o + (size_t)blocks * 4);
    L.lcount = o; o = align256(o + 16);
    L.fb = o;     o = align256(o + (size_t)L.fb_blocks * QB * (size_t)Lk * 4);
    L.total = o;
    return L;
}

// Most query blocks per chunk whose fused layout fits in `avail` bytes (0 if none).
long long fused_blocks_fitting(const FusedGeom& f, long long n_blocks, int QB, int Lk,
                               size_t avail) {
    const FusedLayout one = fused_layout(f, 1, QB, Lk);
    if (one.total > avail) return 0;
    long long lo = 1, hi = n_blocks;
    while (lo < hi) {                      // largest count that fits
        const long long mid = lo + (hi - lo + 1) / 2;
        if (fused_layout(f, mid, QB, Lk).total <= avail) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// One F layer's index rows of query blocks [g0, g1) on the fused path: the
// sampled scores, the thresholds, the candidates, the exact selection, and
// the fallback rounds over the flagged blocks (each round scores up to
// lay.fb_blocks listed blocks into the fallback buffer and runs the plain
// top-k on them; rounds past the list's length do nothing).  `mid` (may be
// null) is recorded after the candidate pass.
int fused_chunk(const ic_dims& D, const ic_layer& Lr, const IndexerGeom& geo, const FusedGeom& f,
                long long g0, long long g1, uint8_t* base, int32_t* idx, uint32_t* dmask,
                const DenseGeom& dg, float z, int sms, cudaStream_t st, cudaEvent_t mid) {
    const FusedLayout lay = fused_layout(f, g1 - g0, geo.QB, D.Lk);
    const long long r0 = block_row_start(geo, D.Lq, g0);
    const long long r1 = block_row_start(geo, D.Lq, g1);
    ic::FusedArgs fa{};
    fa.row_base = r0;
    fa.n_rows = r1 - r0;
    fa.Lq = D.Lq;
    fa.Lk = D.Lk;
    fa.q_offset = D.q_offset;
    fa.k = D.k;
    fa.cap = f.cap;
    fa.lstride = f.lstride;
    fa.stride = f.stride;
    fa.ns = f.ns;
    fa.z = z;
    fa.QB = geo.QB;
    fa.nqb = geo.nqb;
    fa.g0 = g0;
    fa.n_blocks = g1 - g0;
    fa.samp = reinterpret_cast<const float*>(base + lay.samp);
    fa.thr = reinterpret_cast<uint32_t*>(base + lay.thr);
    fa.cnt = reinterpret_cast<uint32_t*>(base + lay.cnt);
    fa.cand = reinterpret_cast<const unsigned long long*>(base + lay.cand);
    fa.bflag = reinterpret_cast<uint32_t*>(base + lay.flag);
    fa.blist = reinterpret_cast<int*>(base + lay.list);
    fa.list_count = reinterpret_cast<int*>(base + lay.lcount);
    fa.idx = idx;
    fa.mask = dmask;
    fa.Lq_d = dg.Lq_d;
    fa.W = dg.W;

    IdxExtra xs;
    xs.mode = ic::IDX_SAMPLE;
    xs.stride = f.stride;
    int rc = launch_indexer(Lr.q_idx, Lr.k_idx, Lr.w, D.B, D.Lq, D.Lk, D.H_I, D.d_I, D.q_offset,
                            g0, g1, reinterpret_cast<float*>(base + lay.samp),
                            (long long)f.ns * ic::IDX_BM, false, sms, st, xs);
    if (rc) return rc;
    const int tgrid = (int)std::min<long long>(fa.n_rows, 16LL * sms);
    ic::fused_threshold_kernel<<<tgrid, ic::FT_THREADS, 0, st>>>(fa);
    if (launched(cudaGetLastError(), "fused_threshold launch")) return IC_ERR_CUDA;
    IdxExtra xc;
    xc.mode = ic::IDX_CAND;
    xc.thr = fa.thr;
    xc.cnt = fa.cnt;
    xc.cand = reinterpret_cast<unsigned long long*>(base + lay.cand);
    xc.cap = f.lstride;
    xc.tpu = FUSED_TPU;
    rc = launch_indexer(Lr.q_idx, Lr.k_idx, Lr.w, D.B, D.Lq, D.Lk, D.H_I, D.d_I, D.q_offset, g0,
                        g1, nullptr, 0, false, sms, st, xc);
    if (rc) return rc;
    if (mid) {
        cudaError_t e = cudaEventRecord(mid, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    ic::fused_select_kernel<<<(unsigned)fa.n_rows, ic::FS_THREADS,
                              ic::fused_select_smem(f.lstride, D.Lk), st>>>(fa);
    if (launched(cudaGetLastError(), "fused_select launch")) return IC_ERR_CUDA;
    float* fb = reinterpret_cast<float*>(base + lay.fb);
    for (long long off = 0; off < g1 - g0; off += lay.fb_blocks) {
        IdxExtra xl;
        xl.blk_list = fa.blist;
        xl.blk_count = fa.list_count;
        xl.list_off = (int)off;
        xl.list_len = (int)lay.fb_blocks;
        rc = launch_indexer(Lr.q_idx, Lr.k_idx, Lr.w, D.B, D.Lq, D.Lk, D.H_I, D.d_I, D.q_offset,
                            g0, g1, fb, D.Lk, false, sms, st, xl);
        if (rc) return rc;
        ic::TopkList tl{fa.blist, fa.list_count, (int)off, (int)lay.fb_blocks, geo.QB, geo.nqb};
        rc = launch_topk(fb, D.Lk, 0, lay.fb_blocks * geo.QB, D.Lq, D.Lk, D.q_offset, D.k, idx,
                         sms, st, dmask, dg.Lq_d, dg.W, tl);
        if (rc) return rc;
    }
    return IC_OK;
}

// ---------------------------------------------------------------- per-device setup

int device_setup(int* dev_out, int* sms_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= MAX_DEV) return fail(IC_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_attr_done[dev]) {
        int major = 0, minor = 0, sms = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        if (major != 10 || minor != 0)
            return fail(IC_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                        dev, major, minor);
        set_indexer_attr<4, 64>();   set_indexer_attr<4, 128>();
        set_indexer_attr<8, 64>();   set_indexer_attr<8, 128>();
        set_indexer_attr<16, 64>();  set_indexer_attr<16, 128>();
        set_indexer_attr<32, 64>();  set_indexer_attr<32, 128>();
        set_indexer_attr<64, 64>();  set_indexer_attr<64, 128>();
        set_indexer_attr<128, 64>(); set_indexer_attr<128, 128>();
        cudaFuncSetAttribute(ic::topk_select_kernel<ic::TK_THREADS_FEW, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ic::TK_SMEM_FIXED + ic::TK_CACHE_MAX_FEW * 4);
        cudaFuncSetAttribute(ic::topk_select_kernel<ic::TK_THREADS, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ic::TK_SMEM_FIXED + ic::TK_CACHE_MAX * 4);
        cudaFuncSetAttribute(ic::dense_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ic::DenseSmem::ALLOC);
        cudaFuncSetAttribute(ic::fused_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ic::MAX_DYN_SMEM);
        cudaFuncSetAttribute(ic::index_overlap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             2 * (ic::OV_MAX_LK / 32) * 4);
        cudaFuncSetAttribute(ic::index_overlap_warp_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (ic::OV_THREADS / 32) * 2 * (ic::OV_WARP_MAX_LK / 32) * 4);
        cudaFuncSetAttribute(ic::sparse_attn_kernel<64>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ic::SaSmem<64>::BYTES);
        cudaFuncSetAttribute(ic::sparse_attn_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ic::SaSmem<128>::BYTES);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        g_attn_cluster[dev] = attn_cluster_fits<64>() && attn_cluster_fits<128>();
        cudaGetLastError();                         // a refused query only disables clusters
        g_sms[dev] = sms;
        g_attr_done[dev] = true;
    }
    *dev_out = dev;
    *sms_out = g_sms[dev];
    return IC_OK;
}

// ---------------------------------------------------------------- validation

int check_indexer_shape(int H, int dI) {
    if (dI != 64 && dI != 128) return fail(IC_ERR_UNSUPPORTED, "d_I=%d (supported: 64, 128)", dI);
    if (!pow2(H) || H < 4 || H > 128)
        return fail(IC_ERR_UNSUPPORTED, "H_I=%d (supported: powers of two in [4, 128])", H);
    return IC_OK;
}

int check_attn_shape(int Hq, int Hkv, int d) {
    if (Hkv != 1) return fail(IC_ERR_UNSUPPORTED, "Hkv=%d (only MQA, Hkv=1)", Hkv);
    if (d != 64 && d != 128) return fail(IC_ERR_UNSUPPORTED, "d=%d (supported: 64, 128)", d);
    if (Hq != 8 && Hq != 16) return fail(IC_ERR_UNSUPPORTED, "Hq=%d (supported: 8, 16)", Hq);
    return IC_OK;
}

int check_positions(int B, int Lq, int Lk, int q_offset) {
    if (B < 0 || Lq < 0 || Lk < 0 || q_offset < 0)
        return fail(IC_ERR_INVALID_ARG, "negative size (B=%d Lq=%d Lk=%d q_offset=%d)", B, Lq, Lk,
                    q_offset);
    if ((long long)q_offset + Lq > Lk)
        return fail(IC_ERR_INVALID_ARG, "q_offset + Lq = %lld exceeds Lk = %d",
                    (long long)q_offset + Lq, Lk);
    return IC_OK;
}

}  // namespace

// Scratch for ic_sparse_attn_no_alloc: the per-split partial results (O / l and
// the log2-sum-exp of each row, split and head) live in this fixed device
// array instead of a caller workspace.  Every GPU that loads the library holds
// it until the process exits.  Host code must never hand the symbol itself to
// a kernel (on the host it is only a stand-in); the device address comes from
// cudaGetSymbolAddress, looked up once per device.
constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)4 << 20;   // 4 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[MAX_DEV];

// Device address of g_noalloc_scratch on the current device (looked up on the
// first call per device, with that device current).
int noalloc_scratch(int dev, void** out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return IC_OK;
}
}  // namespace

// ======================================================================= C ABI

extern "C" {

const char* ic_status_string(int status) {
    switch (status) {
        case IC_OK: return "IC_OK";
        case IC_ERR_INVALID_ARG: return "IC_ERR_INVALID_ARG";
        case IC_ERR_UNSUPPORTED: return "IC_ERR_UNSUPPORTED";
        case IC_ERR_NO_CACHED_INDICES: return "IC_ERR_NO_CACHED_INDICES";
        case IC_ERR_WORKSPACE_TOO_SMALL: return "IC_ERR_WORKSPACE_TOO_SMALL";
        case IC_ERR_CUDA: return "IC_ERR_CUDA";
        case IC_ERR_TIMEOUT: return "IC_ERR_TIMEOUT";
        default: return "IC_ERR_UNKNOWN";
    }
}

const char* ic_last_error_message(void) { return g_msg; }

int ic_get_last_device_error(ic_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int v = 0;
    e = cudaMemcpyFromSymbol(&v, ic::g_dev_error, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    if (v) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(ic::g_dev_error, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    }
    if (v & ic::DEV_ERR_TIMEOUT) return fail(IC_ERR_TIMEOUT, "a kernel wait timed out");
    if (v & ic::DEV_ERR_SMEM)
        return fail(IC_ERR_CUDA, "a kernel's aligned shared-memory layout did not fit; it did no work");
    if (v & ic::DEV_ERR_BAD_INDEX)
        return fail(IC_ERR_INVALID_ARG, "an attention index outside [0, t] was skipped");
    return IC_OK;
}

unsigned long long ic_kernel_launch_count(void) {
    return g_launches.load(std::memory_order_relaxed);
}

int ic_selftest_wait_timeout(int timeout_us, ic_stream_t stream) {
    int dev, sms;
    int rc = device_setup(&dev, &sms);
    if (rc) return rc;
    const long long us = std::min(2000000, std::max(1, timeout_us));
    ic::selftest_wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)us * 1000ull);
    cudaError_t e = cudaGetLastError();
    if (launched(e, "selftest launch")) return IC_ERR_CUDA;
    return IC_OK;
}

int ic_indexer_scores(const uint16_t* q_idx, const uint16_t* k_idx, const float* w, int B,
                      int Lq, int Lk, int H_I, int d_I, int q_offset, float* scores,
                      ic_stream_t stream) {
    int rc = check_positions(B, Lq, Lk, q_offset);
    if (rc) return rc;
    if ((rc = check_indexer_shape(H_I, d_I))) return rc;
    if (B == 0 || Lq == 0) return IC_OK;
    if (!q_idx || !k_idx || !w || !scores) return fail(IC_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w))
        return fail(IC_ERR_UNSUPPORTED, "q_idx, k_idx and w must be 16-byte aligned");
    if (!aligned4(scores)) return fail(IC_ERR_UNSUPPORTED, "scores must be 4-byte aligned");
    if ((long long)Lq * H_I > (1LL << 31)) return fail(IC_ERR_UNSUPPORTED, "Lq*H_I too large");
    int dev, sms;
    if ((rc = device_setup(&dev, &sms))) return rc;
    const IndexerGeom geo = indexer_geom(Lq, H_I);
    return launch_indexer(q_idx, k_idx, w, B, Lq, Lk, H_I, d_I, q_offset, 0,
                          (long long)B * geo.nqb, scores, Lk, true, sms,
                          reinterpret_cast<cudaStream_t>(stream));
}

int ic_topk_select(const float* scores, int B, int Lq, int Lk, int q_offset, int k, int32_t* idx,
                   ic_stream_t stream) {
    int rc = check_positions(B, Lq, Lk, q_offset);
    if (rc) return rc;
    if (k < 1) return fail(IC_ERR_INVALID_ARG, "k=%d", k);
    if (B == 0 || Lq == 0) return IC_OK;
    if (!scores || !idx) return fail(IC_ERR_INVALID_ARG, "null pointer");
    if (!aligned4(scores) || !aligned4(idx))
        return fail(IC_ERR_UNSUPPORTED, "scores and idx must be 4-byte aligned");
    int dev, sms;
    if ((rc = device_setup(&dev, &sms))) return rc;
    return launch_topk(scores, Lk, 0, (long long)B * Lq, Lq, Lk, q_offset, k, idx, sms,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t ic_sparse_attn_workspace_bytes(int B, int Lq, int Hq, int d, int k_slots) {
    if (B <= 0 || Lq <= 0 || Hq <= 0 || d <= 0 || k_slots <= 0) return 0;
    int dev, sms;
    if (device_setup(&dev, &sms)) sms = 148;
    const long long n_rows = (long long)B * Lq;
    return attn_ws_bytes(n_rows, attn_splits(n_rows, k_slots, sms), Hq, d);
}

int ic_sparse_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* idx,
                   int B, int Lq, int Lk, int Hq, int Hkv, int d, int k_slots, int q_offset,
                   float scale, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                   ic_stream_t stream) {
    int rc = check_positions(B, Lq, Lk, q_offset);
    if (rc) return rc;
    if ((rc = check_attn_shape(Hq, Hkv, d))) return rc;
    if (k_slots < 1) return fail(IC_ERR_INVALID_ARG, "k=%d", k_slots);
    if (B == 0 || Lq == 0) return IC_OK;
    if (!q || !k || !v || !idx || !out) return fail(IC_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(IC_ERR_UNSUPPORTED, "q, k, v and out must be 16-byte aligned");
    if (!aligned4(idx) || (lse && !aligned4(lse)))
        return fail(IC_ERR_UNSUPPORTED, "idx and lse must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(IC_ERR_INVALID_ARG, "scale is not finite");
    if (ws && !aligned16(ws)) return fail(IC_ERR_UNSUPPORTED, "ws must be 16-byte aligned");
    int dev, sms;
    if ((rc = device_setup(&dev, &sms))) return rc;
    return launch_attn(q, k, v, idx, B, Lq, Lk, Hq, d, k_slots, q_offset, scale, out, lse, ws,
                       ws_bytes, false, sms, reinterpret_cast<cudaStream_t>(stream));
}

int ic_sparse_attn_no_alloc(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            const int32_t* idx, int B, int Lq, int Lk, int Hq, int Hkv, int d,
                            int k_slots, int q_offset, float scale, uint16_t* out, float* lse,
                            ic_stream_t stream) {
    int rc = check_positions(B, Lq, Lk, q_offset);
    if (rc) return rc;
    if ((rc = check_attn_shape(Hq, Hkv, d))) return rc;
    if (k_slots < 1) return fail(IC_ERR_INVALID_ARG, "k=%d", k_slots);
    if (B == 0 || Lq == 0) return IC_OK;
    if (!q || !k || !v || !idx || !out) return fail(IC_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(IC_ERR_UNSUPPORTED, "q, k, v and out must be 16-byte aligned");
    if (!aligned4(idx) || (lse && !aligned4(lse)))
        return fail(IC_ERR_UNSUPPORTED, "idx and lse must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(IC_ERR_INVALID_ARG, "scale is not finite");
    int dev, sms;
    if ((rc = device_setup(&dev, &sms))) return rc;
    void* scratch = nullptr;
    if ((rc = noalloc_scratch(dev, &scratch))) return rc;
    // launch_attn halves the slot split until its partials fit the scratch
    // (one split needs none), so every valid call runs.
    return launch_attn(q, k, v, idx, B, Lq, Lk, Hq, d, k_slots, q_offset, scale, out, lse, scratch,
                       NOALLOC_SCRATCH_BYTES, false, sms, reinterpret_cast<cudaStream_t>(stream));
}

size_t ic_sparse_attn_unique_workspace_bytes(int B, int Lq, int Lk, int q_offset, int Hq, int d,
                                             int k_slots) {
    if (B <= 0 || Lq <= 0 || Hq <= 0 || d <= 0 || k_slots <= 0) return 0;
    if (check_positions(B, Lq, Lk, q_offset)) return 0;
    ic_dims D{};
    D.B = B; D.Lq = Lq; D.Lk = Lk; D.q_offset = q_offset; D.Hq = Hq; D.Hkv = 1; D.d = d;
    D.k = k_slots;
    const DenseGeom dg = dense_geom(D);
    if (!dg.on) return ic_sparse_attn_workspace_bytes(B, Lq, Hq, d, k_slots);
    const int rows_g = Lq - dg.Lq_d;            // rows that still gather (t >= 6k)
    return dg.total + (rows_g > 0 ? ic_sparse_attn_workspace_bytes(B, rows_g, Hq, d, k_slots) : 0);
}

int ic_sparse_attn_unique(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          const int32_t* idx, int B, int Lq, int Lk, int Hq, int Hkv, int d,
                          int k_slots, int q_offset, float scale, uint16_t* out, float* lse,
                          void* ws, size_t ws_bytes, ic_stream_t stream) {
    int rc = check_positions(B, Lq, Lk, q_offset);
    if (rc) return rc;
    if ((rc = check_attn_shape(Hq, Hkv, d))) return rc;
    if (k_slots < 1) return fail(IC_ERR_INVALID_ARG, "k=%d", k_slots);
    if (B == 0 || Lq == 0) return IC_OK;
    if (!q || !k || !v || !idx || !out) return fail(IC_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(IC_ERR_UNSUPPORTED, "q, k, v and out must be 16-byte aligned");
    if (!aligned4(idx) || (lse && !aligned4(lse)))
        return fail(IC_ERR_UNSUPPORTED, "idx and lse must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(IC_ERR_INVALID_ARG, "scale is not finite");
    if (ws_bytes > 0 && !ws) return fail(IC_ERR_INVALID_ARG, "ws is NULL but ws_bytes > 0");
    if (ws && !aligned16(ws)) return fail(IC_ERR_UNSUPPORTED, "ws must be 16-byte aligned");
    int dev, sms;
    if ((rc = device_setup(&dev, &sms))) return rc;
    ic_dims D{};
    D.B = B; D.Lq = Lq; D.Lk = Lk; D.q_offset = q_offset; D.Hq = Hq; D.Hkv = Hkv; D.d = d;
    D.k = k_slots; D.scale = scale;
    ic_layer L{};
    L.q = q; L.k = k; L.v = v; L.out = out; L.lse = lse;
    const DenseGeom dg = dense_geom(D);
    const AttnMode mode = (dg.on && dg.total <= ws_bytes) ? ATTN_BUILD_MASK : ATTN_GATHER;
    return attn_step(D, L, idx, mode, false, ws, ws_bytes, sms,
                     reinterpret_cast<cudaStream_t>(stream), nullptr);
}

int ic_index_overlap(const int32_t* idx_a, const int32_t* idx_b, long long n_rows, int k, int Lk,
                     int32_t* counts, ic_stream_t stream) {
    if (n_rows < 0 || k < 1) return fail(IC_ERR_INVALID_ARG, "n_rows=%lld k=%d", n_rows, k);
    if (Lk < 1 || Lk > ic::OV_MAX_LK)
        return fail(IC_ERR_UNSUPPORTED, "Lk=%d (supported: 1..%d)", Lk, ic::OV_MAX_LK);
    if (n_rows == 0) return IC_OK;
    if (!idx_a || !idx_b || !counts) return fail(IC_ERR_INVALID_ARG, "null pointer");
    if (!aligned4(idx_a) || !aligned4(idx_b) || !aligned4(counts))
        return fail(IC_ERR_UNSUPPORTED, "idx_a, idx_b and counts must be 4-byte aligned");
    int dev, sms;
    int rc = device_setup(&dev, &sms);
    if (rc) return rc;
    const int W = (Lk + 31) / 32;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (Lk <= ic::OV_WARP_MAX_LK) {
        const long long per_cta = ic::OV_THREADS / 32;
        const int grid = (int)std::min<long long>((n_rows + per_cta - 1) / per_cta, (long long)sms * 8);
        ic::index_overlap_warp_kernel<<<grid, ic::OV_THREADS, per_cta * 2 * W * 4, st>>>(
            idx_a, idx_b, n_rows, k, Lk, counts);
    } else {
        const int grid = (int)std::min<long long>(n_rows, (long long)sms * 8);
        ic::index_overlap_kernel<<<grid, ic::OV_THREADS, 2 * W * 4, st>>>(idx_a, idx_b, n_rows, k,
                                                                          Lk, counts);
    }
    return launched(cudaGetLastError(), "index_overlap launch");
}

int ic_layer_stack_dense_rows(const ic_dims* dims, size_t ws_bytes) {
    if (!dims || check_positions(dims->B, dims->Lq, dims->Lk, dims->q_offset) ||
        check_indexer_shape(dims->H_I, dims->d_I) || dims->k < 1 || dims->Lq < 1)
        return 0;
    const DenseGeom dg = dense_geom(*dims);
    if (!dg.on) return 0;
    // the same test stack_forward applies to its workspace
    const IndexerGeom geo = indexer_geom(dims->Lq, dims->H_I);
    const size_t block_bytes = (size_t)geo.QB * (size_t)dims->Lk * sizeof(float);
    if (ws_bytes < dg.mask_bytes + std::max(block_bytes, dg.vt_bytes)) return 0;
    return dg.Lq_d;
}

size_t ic_layer_stack_workspace_bytes(const ic_dims* dims, int n_layers, long long rows_per_chunk) {
    if (!dims || n_layers < 1) return 0;
    if (check_positions(dims->B, dims->Lq, dims->Lk, dims->q_offset) ||
        check_indexer_shape(dims->H_I, dims->d_I) || dims->k < 1)
        return 0;
    const IndexerGeom geo = indexer_geom(std::max(dims->Lq, 1), dims->H_I);
    const long long n_rows = (long long)dims->B * dims->Lq;
    long long blocks = (long long)dims->B * geo.nqb;
    if (rows_per_chunk > 0)
        blocks = std::min(blocks, std::max(1LL, (rows_per_chunk + geo.QB - 1) / geo.QB));
    size_t scores = (size_t)blocks * geo.QB * (size_t)dims->Lk * sizeof(float);
    // the fused top-k's chunk (candidate lists, fallback buffer) in place of
    // the score chunk, when the fused path can run for these dims
    const FusedGeom fgeo = fused_geom(*dims);
    if (fgeo.ok) scores = std::max(scores, fused_layout(fgeo, blocks, geo.QB, dims->Lk).total);
    const size_t attn = ic_sparse_attn_workspace_bytes(dims->B, dims->Lq, dims->Hq, dims->d, dims->k);
    const DenseGeom dg = dense_geom(*dims);
    (void)n_rows;
    // dense-masked rows: the bitmask (written by the top-k) sits before the
    // score chunk; V^T and the split partials of the rows that still gather
    // (t >= 6k) reuse the score region
    if (dg.on) {
        const int rows_g = dims->Lq - dg.Lq_d;
        const size_t attn_g =
            rows_g > 0 ? ic_sparse_attn_workspace_bytes(dims->B, rows_g, dims->Hq, dims->d, dims->k)
                       : 0;
        return std::max(dg.mask_bytes + scores, dg.total + attn_g);
    }
    return std::max(scores, attn);
}

static int stack_forward(const char* pattern, int n_layers, const ic_layer* layers,
                         const ic_dims* dims, const ic_stack_options* opts, int32_t* idx_cache,
                         void* ws, size_t ws_bytes, ic_stream_t stream, void* const* events) {
    if (!pattern || !layers || !dims || !idx_cache || n_layers < 1)
        return fail(IC_ERR_INVALID_ARG, "null argument or n_layers < 1");
    if ((int)strnlen(pattern, (size_t)n_layers + 1) != n_layers)
        return fail(IC_ERR_INVALID_ARG, "pattern length differs from n_layers=%d", n_layers);
    for (int l = 0; l < n_layers; ++l) {
        const char c = pattern[l];
        if (c != 'F' && c != '1' && c != 'S' && c != '0')
            return fail(IC_ERR_INVALID_ARG, "pattern[%d]='%c' is neither F/1 nor S/0", l, c);
    }
    if (pattern[0] == 'S' || pattern[0] == '0')
        return fail(IC_ERR_NO_CACHED_INDICES,
                    "layer 0 is Shared: the index cache is empty until a Full layer has run");
    const ic_dims& D = *dims;
    int rc = check_positions(D.B, D.Lq, D.Lk, D.q_offset);
    if (rc) return rc;
    if ((rc = check_indexer_shape(D.H_I, D.d_I))) return rc;
    if ((rc = check_attn_shape(D.Hq, D.Hkv, D.d))) return rc;
    if (D.k < 1 || D.k > D.Lk) return fail(IC_ERR_INVALID_ARG, "k=%d outside [1, Lk]", D.k);
    if (!std::isfinite(D.scale)) return fail(IC_ERR_INVALID_ARG, "scale is not finite");
    const int fuse_mode = opts ? opts->fused_topk : -1;
    const FusedGeom fgeo = fused_geom(D);
    if (fuse_mode == 1 && !fgeo.ok)
        return fail(IC_ERR_UNSUPPORTED, "the fused top-k needs k <= %d and Lk <= %d",
                    FUSED_MAX_K, FUSED_MAX_LK);
    for (int l = 0; l < n_layers; ++l) {
        const ic_layer& L = layers[l];
        const bool full = pattern[l] == 'F' || pattern[l] == '1';
        if (!L.q || !L.k || !L.v || !L.out)
            return fail(IC_ERR_INVALID_ARG, "layer %d: null q/k/v/out", l);
        if (!aligned16(L.q) || !aligned16(L.k) || !aligned16(L.v) || !aligned16(L.out))
            return fail(IC_ERR_UNSUPPORTED, "layer %d: q, k, v, out must be 16-byte aligned", l);
        if (L.lse && !aligned4(L.lse))
            return fail(IC_ERR_UNSUPPORTED, "layer %d: lse must be 4-byte aligned", l);
        if (full) {
            if (!L.q_idx || !L.k_idx || !L.w)
                return fail(IC_ERR_INVALID_ARG, "layer %d is F but q_idx/k_idx/w is null", l);
            if (!aligned16(L.q_idx) || !aligned16(L.k_idx) || !aligned16(L.w))
                return fail(IC_ERR_UNSUPPORTED, "layer %d: q_idx, k_idx, w must be 16-byte aligned",
                            l);
        }
    }
    if (!aligned4(idx_cache)) return fail(IC_ERR_UNSUPPORTED, "idx_cache must be 4-byte aligned");
    if (ws && !aligned16(ws)) return fail(IC_ERR_UNSUPPORTED, "ws must be 16-byte aligned");
    if (D.B == 0 || D.Lq == 0) return IC_OK;
    if ((long long)D.Lq * D.H_I > (1LL << 31)) return fail(IC_ERR_UNSUPPORTED, "Lq*H_I too large");
    int dev, sms;
    if ((rc = device_setup(&dev, &sms))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    const IndexerGeom geo = indexer_geom(D.Lq, D.H_I);
    const long long n_blocks = (long long)D.B * geo.nqb;
    const long long n_rows = (long long)D.B * D.Lq;
    const size_t block_bytes = (size_t)geo.QB * (size_t)D.Lk * sizeof(float);
    if (!ws || ws_bytes < block_bytes)
        return fail(IC_ERR_WORKSPACE_TOO_SMALL,
                    "workspace of %zu bytes is below one query block of scores (%zu bytes)",
                    ws_bytes, block_bytes);
    // Rows with t < 6k attend dense-masked when the workspace holds the
    // bitmask (which the top-k writes, ahead of the score chunk) plus one
    // block of scores, and V^T (which, like the gathered rows' partials,
    // reuses the score region once the layer's top-k is done).  The bitmask
    // of an F layer is read by the S layers after it.
    const DenseGeom dg = dense_geom(D);
    const bool dense = dg.on && ws_bytes >= dg.mask_bytes + std::max(block_bytes, dg.vt_bytes);
    const size_t sc_off = dense ? dg.mask_bytes : 0;
    long long blocks_per_chunk =
        std::min<long long>(n_blocks, (long long)((ws_bytes - sc_off) / block_bytes));
    // Fused indexer -> top-k: chunks as large as the workspace holds their
    // candidate lists and fallback buffer; the score matrix is never stored.
    const float z = (opts && opts->z > 0.0f) ? opts->z : FUSED_Z;
    bool fused = fused_wanted(fgeo, D, fuse_mode);
    if (fused) {
        const long long fb =
            fused_blocks_fitting(fgeo, n_blocks, geo.QB, D.Lk, ws_bytes - sc_off);
        if (fb < 1) {
            if (fuse_mode == 1)
                return fail(IC_ERR_WORKSPACE_TOO_SMALL,
                            "workspace of %zu bytes holds no query block of the fused top-k",
                            ws_bytes);
            fused = false;
        } else {
            blocks_per_chunk = fb;
        }
    }
    float* sc = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + sc_off);
    uint32_t* dmask = dense ? reinterpret_cast<uint32_t*>(ws) : nullptr;

    auto mark = [&](int l, int slot) -> int {
        if (!events || !events[IC_MARKS_PER_LAYER * l + slot]) return IC_OK;
        cudaError_t e = cudaEventRecord(
            reinterpret_cast<cudaEvent_t>(events[IC_MARKS_PER_LAYER * l + slot]), st);
        return e == cudaSuccess ? IC_OK : cuda_fail(e, "cudaEventRecord");
    };
    const bool one_chunk = blocks_per_chunk >= n_blocks;
    for (int l = 0; l < n_layers; ++l) {
        const ic_layer& L = layers[l];
        const bool full = pattern[l] == 'F' || pattern[l] == '1';
        char label[32];
        snprintf(label, sizeof label, "layer %d %c", l, full ? 'F' : 'S');
        const NvtxRange layer_range(label);
        if ((rc = mark(l, 0))) return rc;
        if (full) {
            const NvtxRange r("indexer + top-k");
            for (long long g0 = 0; g0 < n_blocks; g0 += blocks_per_chunk) {
                const long long g1 = std::min(n_blocks, g0 + blocks_per_chunk);
                if (fused) {
                    cudaEvent_t m1 = nullptr;
                    if (one_chunk && events)
                        m1 = reinterpret_cast<cudaEvent_t>(events[IC_MARKS_PER_LAYER * l + 1]);
                    rc = fused_chunk(D, L, geo, fgeo, g0, g1, reinterpret_cast<uint8_t*>(sc),
                                     idx_cache, dmask, dg, z, sms, st, m1);
                    if (rc) return rc;
                    continue;
                }
                rc = launch_indexer(L.q_idx, L.k_idx, L.w, D.B, D.Lq, D.Lk, D.H_I, D.d_I,
                                    D.q_offset, g0, g1, sc, D.Lk, false, sms, st);
                if (rc) return rc;
                if (one_chunk && (rc = mark(l, 1))) return rc;
                const long long r0 = block_row_start(geo, D.Lq, g0);
                const long long r1 = block_row_start(geo, D.Lq, g1);
                rc = launch_topk(sc, D.Lk, r0, r1 - r0, D.Lq, D.Lk, D.q_offset, D.k, idx_cache, sms,
                                 st, dmask, dg.Lq_d, dg.W);
                if (rc) return rc;
            }
        }
        if (!(full && one_chunk) && (rc = mark(l, 1))) return rc;
        if ((rc = mark(l, 2))) return rc;
        cudaEvent_t mid = events ? reinterpret_cast<cudaEvent_t>(events[IC_MARKS_PER_LAYER * l + 3])
                                 : nullptr;
        {
            const NvtxRange r("attention");
            rc = attn_step(D, L, idx_cache, dense ? ATTN_MASK_READY : ATTN_GATHER, true, ws,
                           ws_bytes, sms, st, mid);
        }
        if (rc) return rc;
        if ((rc = mark(l, 4))) return rc;
        if (L.idx_dump) {
            cudaError_t e = cudaMemcpyAsync(L.idx_dump, idx_cache,
                                            (size_t)n_rows * D.k * sizeof(int32_t),
                                            cudaMemcpyDeviceToDevice, st);
            if (e != cudaSuccess) return cuda_fail(e, "idx_dump copy");
        }
    }
    return IC_OK;
}

int ic_layer_stack_forward(const char* pattern, int n_layers, const ic_layer* layers,
                           const ic_dims* dims, int32_t* idx_cache, void* ws, size_t ws_bytes,
                           ic_stream_t stream) {
    return stack_forward(pattern, n_layers, layers, dims, nullptr, idx_cache, ws, ws_bytes, stream,
                         nullptr);
}

int ic_layer_stack_forward_events(const char* pattern, int n_layers, const ic_layer* layers,
                                  const ic_dims* dims, int32_t* idx_cache, void* ws,
                                  size_t ws_bytes, ic_stream_t stream, void* const* events) {
    return stack_forward(pattern, n_layers, layers, dims, nullptr, idx_cache, ws, ws_bytes, stream,
                         events);
}

int ic_layer_stack_forward_opts(const char* pattern, int n_layers, const ic_layer* layers,
                                const ic_dims* dims, const ic_stack_options* opts,
                                int32_t* idx_cache, void* ws, size_t ws_bytes,
                                ic_stream_t stream, void* const* events) {
    if (opts && (opts->fused_topk < -1 || opts->fused_topk > 1 || !std::isfinite(opts->z)))
        return fail(IC_ERR_INVALID_ARG, "options: fused_topk=%d z=%g", opts->fused_topk,
                    (double)opts->z);
    return stack_forward(pattern, n_layers, layers, dims, opts, idx_cache, ws, ws_bytes, stream,
                         events);
}

int ic_layer_stack_fused_fallback_blocks(const ic_dims* dims, const ic_stack_options* opts,
                                         const void* ws, size_t ws_bytes, ic_stream_t stream,
                                         int* blocks) {
    if (!dims || !ws || !blocks) return fail(IC_ERR_INVALID_ARG, "null argument");
    if (check_positions(dims->B, dims->Lq, dims->Lk, dims->q_offset) ||
        check_indexer_shape(dims->H_I, dims->d_I) || dims->k < 1 || dims->Lq < 1)
        return fail(IC_ERR_INVALID_ARG, "invalid dims");
    const ic_dims& D = *dims;
    const IndexerGeom geo = indexer_geom(D.Lq, D.H_I);
    const long long n_blocks = (long long)D.B * geo.nqb;
    const size_t block_bytes = (size_t)geo.QB * (size_t)D.Lk * sizeof(float);
    const DenseGeom dg = dense_geom(D);
    const bool dense = dg.on && ws_bytes >= dg.mask_bytes + std::max(block_bytes, dg.vt_bytes);
    const size_t sc_off = dense ? dg.mask_bytes : 0;
    const FusedGeom fgeo = fused_geom(D);
    if (!fused_wanted(fgeo, D, opts ? opts->fused_topk : -1) || ws_bytes < sc_off)
        return fail(IC_ERR_INVALID_ARG, "the stack does not fuse the top-k for these dims");
    const long long fb = fused_blocks_fitting(fgeo, n_blocks, geo.QB, D.Lk, ws_bytes - sc_off);
    if (fb < 1) return fail(IC_ERR_WORKSPACE_TOO_SMALL, "no fused chunk fits the workspace");
    const long long g_last = ((n_blocks - 1) / fb) * fb;          // the last chunk's first block
    const FusedLayout lay = fused_layout(fgeo, std::min(fb, n_blocks - g_last), geo.QB, D.Lk);
    int v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, reinterpret_cast<const uint8_t*>(ws) + sc_off + lay.lcount,
                                    sizeof v, cudaMemcpyDeviceToHost,
                                    reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "read the fallback block count");
    *blocks = v;
    return IC_OK;
}

}  // extern "C"
