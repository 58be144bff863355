/*
 * indexcache.h — C ABI of libindexcache.so: a DSA-style sparse-attention
 * layer stack with IndexCache cross-layer index reuse, for NVIDIA B200
 * (sm_100a).
 *
 * Sources.  "IndexCache: Accelerating Sparse Attention via Cross-Layer Index
 * Reuse" (arXiv 2603.12201), as described by:
 *   - the fugumt digest, Abstract: per query, a lightning indexer ranks the
 *     earlier tokens and only the k best-ranked enter core attention, which
 *     then costs O(Lk) per sequence rather than O(L^2); a Full layer keeps its indexer, a
 *     Shared layer takes the index set of the closest Full layer above it;
 *   - the kualia.ai review, "The Redundancy That Was Sitting There": the
 *     cache is one scratch tensor of indices that each F layer replaces;
 *   - the skill page, Step 3 (IndexCacheManager.get_indices_for_layer): an S
 *     layer with nothing cached is an error;
 *   - the knowledge note "Cross-Layer Index Reuse", How It Works: the anchor
 *     layer scores the visible positions and stores its selection; each
 *     layer after it attends sparsely over that stored selection.
 * The pages print no indexer formula; this library computes the standard
 * lightning-indexer score s[t,s] = sum_j w[t,j] * max(0, q_I[t,j] . k_I[s]).
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers to caller-owned, contiguous, row-major
 *     buffers (shapes below).  bf16 tensors are passed as uint16_t bit
 *     patterns.  The library allocates nothing and keeps no state from one
 *     call to the next (so no index cache can leak between sequences).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously.  Argument errors are detected on the
 *     host and returned before anything is launched.
 *   - Query row i of batch b sits at absolute position t = q_offset + i and
 *     sees key positions s <= t.  Requirement: q_offset + Lq <= Lk.
 *     Prefill: q_offset = 0, Lq = Lk.  Decode: Lq = 1, q_offset = Lk - 1.
 *   - Supported shapes: d_I in {64, 128}; H_I a power of two in [4, 128];
 *     d in {64, 128}; Hq in {8, 16}; Hkv == 1 (MQA); 1 <= k <= Lk.  Other
 *     shapes return IC_ERR_UNSUPPORTED.  Alignment:
 *       - bf16 buffers, the indexer's head weights w and every workspace
 *         must be 16-byte aligned: kernels read them with 16-byte vector,
 *         bulk or TMA copies;
 *       - the other fp32 / int32 buffers (scores, idx, lse, counts) must be
 *         4-byte aligned.
 *     A misaligned pointer returns IC_ERR_UNSUPPORTED before any launch.
 *   - Device-side faults are never raised on purpose: kernels report an
 *     out-of-range attention index or a timed-out wait into a device error
 *     word that ic_get_last_device_error() reads.
 */
#ifndef INDEXCACHE_H
#define INDEXCACHE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *ic_stream_t;

typedef enum {
    IC_OK = 0,
    IC_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad pattern character */
    IC_ERR_UNSUPPORTED = 2,        /* shape outside the supported set, misaligned pointer */
    IC_ERR_NO_CACHED_INDICES = 3,  /* an S layer precedes every F layer */
    IC_ERR_WORKSPACE_TOO_SMALL = 4,
    IC_ERR_CUDA = 5,               /* a CUDA runtime/driver call or launch failed */
    IC_ERR_TIMEOUT = 6             /* a kernel's bounded wait gave up (device error word) */
} ic_status;

/* Static text for a status code. */
const char *ic_status_string(int status);

/* Detail text of the last failing call on this host thread ("" if none). */
const char *ic_last_error_message(void);

/* Synchronises `stream`, reads and clears the current device's error word.
 * Returns IC_OK, IC_ERR_TIMEOUT (a bounded wait expired) or
 * IC_ERR_INVALID_ARG (an attention index outside [0, t] was skipped), or
 * IC_ERR_CUDA if the synchronisation itself failed. */
int ic_get_last_device_error(ic_stream_t stream);

/*
 * Failure-detection self test.  Launches one CTA whose thread waits on an
 * mbarrier that nothing ever arrives on, for at most timeout_us microseconds
 * (clamped to [1, 2000000]).  The bounded wait gives up, the kernel records a
 * timeout in the device error word and returns, so the next
 * ic_get_last_device_error() returns IC_ERR_TIMEOUT and the CUDA context stays
 * usable.  It exercises the same bounded wait every pipelined kernel uses.
 */
int ic_selftest_wait_timeout(int timeout_us, ic_stream_t stream);

/*
 * Lightning indexer scores (digest Abstract; review Introduction:
 * one indexer pass rates every earlier token of each query).
 *   q_idx  [B, Lq, H_I, d_I] bf16     k_idx [B, Lk, d_I] bf16
 *   w      [B, Lq, H_I]      fp32     scores [B, Lq, Lk] fp32 (written)
 * scores[b,i,s] = sum_j w[b,i,j] * max(0, q_idx[b,i,j,:] . k_idx[b,s,:]) for
 * s <= t = q_offset + i, and -INFINITY for t < s < Lk.  bf16 products,
 * fp32 accumulation (tcgen05 tensor cores).
 */
int ic_indexer_scores(const uint16_t *q_idx, const uint16_t *k_idx, const float *w, int B,
                      int Lq, int Lk, int H_I, int d_I, int q_offset, float *scores,
                      ic_stream_t stream);

/*
 * Per-row top-k (digest Abstract: k tokens are kept per query).
 *   scores [B, Lq, Lk] fp32 (only s <= t is read)   idx [B, Lq, k] int32 (written)
 * Row (b, i) keeps the min(k, t+1) visible positions first in the order
 * (score descending, position ascending), written in ascending position
 * order; the remaining slots are -1.  Scores compare as IEEE floats (-0 ==
 * +0); NaN scores are outside the contract.  Exact (bit-for-bit
 * deterministic).
 */
int ic_topk_select(const float *scores, int B, int Lq, int Lk, int q_offset, int k,
                   int32_t *idx, ic_stream_t stream);

/*
 * Sparse attention over the cached positions (digest Abstract:
 * core attention over k tokens; knowledge note: every later layer attends
 * sparsely over the stored set).  MQA: Hkv must be 1.
 *   q [B, Lq, Hq, d] bf16   k, v [B, Lk, Hkv, d] bf16   idx [B, Lq, k] int32
 *   out [B, Lq, Hq, d] bf16 (written)   lse [B, Lq, Hq] fp32 (written; may be NULL)
 * For each (b, i, h) over the slots whose index lies in [0, t]:
 *   z = scale * q . K[idx], out = sum softmax(z) * V[idx], lse = ln sum e^z.
 * Slots holding -1 are empty.  A slot outside [0, t] is skipped and flags
 * IC_ERR_INVALID_ARG in the device error word.  A row with no valid slot
 * gives out = 0, lse = -INFINITY.  scale <= 0 selects 1/sqrt(d).
 * ws/ws_bytes: optional device workspace.  When there are few rows (decode)
 * each row splits its slots over several CTAs.  Up to 8 splits of a row run
 * as one thread-block cluster and merge through distributed shared memory,
 * with no workspace.  More splits (fewer than about 19 rows on a 148-SM
 * B200) need ic_sparse_attn_workspace_bytes(...) bytes for their partials;
 * with less, fewer splits run and the results are the same.  ws may be NULL
 * (ws_bytes 0).
 */
int ic_sparse_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *idx,
                   int B, int Lq, int Lk, int Hq, int Hkv, int d, int k_slots, int q_offset,
                   float scale, uint16_t *out, float *lse, void *ws, size_t ws_bytes,
                   ic_stream_t stream);

/* Workspace that lets ic_sparse_attn use its preferred slot split. */
size_t ic_sparse_attn_workspace_bytes(int B, int Lq, int Hq, int d, int k_slots);

/*
 * ic_sparse_attn without a workspace argument and without any allocation.
 * The paper has no counterpart: this entry point exists for callers that
 * cannot allocate device memory — for example a host framework that owns all
 * GPU memory and hands a plugin only its inputs and outputs, or a decode loop
 * that must not call cudaMalloc (it can synchronise the device and its cost is
 * unpredictable).  Same arguments, semantics and results as ic_sparse_attn.
 * Rows that split their slots over more CTAs than one 8-CTA cluster holds
 * (decode with fewer than about 19 rows) keep the per-split partial results
 * in a fixed 4 MiB array inside the library instead of a workspace; every
 * GPU that loads the library holds that array until the process exits.  Up
 * to 8 splits merge inside their cluster and use no array.
 *   - Rows split their slots only while rows x splits stays within two CTAs
 *     per SM, so with the supported Hq <= 16 and d <= 128 the partials take
 *     at most 2 x SMs x 16 x 129 x 4 bytes (2.4 MB on a 148-SM B200) and the
 *     preferred split always fits.  On a GPU with more SMs the call would run
 *     with fewer splits (one split needs no scratch); results are the same.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any
 *     stream capture.  The library keeps that address, and its per-device
 *     kernel attributes, for the life of the process: do not use it again on
 *     a device after cudaDeviceReset.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Every partial a call reads is written by the same call first, so nothing
 *     needs clearing, but calls that overlap on the GPU (different streams,
 *     or different host threads) race on the array: serialise them.
 */
int ic_sparse_attn_no_alloc(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const int32_t *idx, int B, int Lq, int Lk, int Hq, int Hkv, int d,
                            int k_slots, int q_offset, float scale, uint16_t *out, float *lse,
                            ic_stream_t stream);

/*
 * The sparse attention step as the layer stack runs it, for index rows that hold every position
 * at most once (top-k output always does).  Same arguments, layout and
 * results as ic_sparse_attn, except that a position repeated within a row
 * counts once here (ic_sparse_attn counts every slot).  Rows whose selection
 * covers a sixth of their visible positions or more (t < 6k, in whole blocks of
 * 128/Hq queries; d = 128 and Hq dividing 128; at most 65536 visible keys)
 * attend tile-dense on the tensor cores under a bitmask of the selection --
 * probability exactly 0 outside it -- when ws holds at least
 * ic_sparse_attn_unique_workspace_bytes(...) bytes; the other rows, and all
 * rows with a smaller workspace, gather.  Slots outside [0, t] are skipped and
 * flag IC_ERR_INVALID_ARG in the device error word, as in ic_sparse_attn.
 */
int ic_sparse_attn_unique(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const int32_t *idx, int B, int Lq, int Lk, int Hq, int Hkv, int d,
                          int k_slots, int q_offset, float scale, uint16_t *out, float *lse,
                          void *ws, size_t ws_bytes, ic_stream_t stream);

/* Workspace with which ic_sparse_attn_unique takes the dense-masked path
 * where it applies (0 for invalid sizes). */
size_t ic_sparse_attn_unique_workspace_bytes(int B, int Lq, int Lk, int q_offset, int Hq, int d,
                                             int k_slots);

/* One layer of the stack.  S layers may leave q_idx, k_idx and w NULL. */
typedef struct {
    const uint16_t *q;      /* [B, Lq, Hq, d] bf16 */
    const uint16_t *k;      /* [B, Lk, Hkv, d] bf16 */
    const uint16_t *v;      /* [B, Lk, Hkv, d] bf16 */
    const uint16_t *q_idx;  /* [B, Lq, H_I, d_I] bf16 (F layers) */
    const uint16_t *k_idx;  /* [B, Lk, d_I] bf16 (F layers) */
    const float *w;         /* [B, Lq, H_I] fp32 (F layers) */
    uint16_t *out;          /* [B, Lq, Hq, d] bf16, written */
    float *lse;             /* [B, Lq, Hq] fp32, written; may be NULL */
    int32_t *idx_dump;      /* [B, Lq, k] int32: copy of the indices this layer used; may be NULL */
} ic_layer;

typedef struct {
    int B, Lq, Lk, q_offset;
    int H_I, d_I;
    int Hq, Hkv, d;
    int k;
    float scale;            /* <= 0 -> 1/sqrt(d) */
} ic_dims;

/*
 * Workspace for ic_layer_stack_forward.  rows_per_chunk <= 0 asks for the
 * size that scores every query row of an F layer in one pass; a positive
 * value asks for the size of chunks of that many rows (rounded up to the
 * indexer's query block).  Returns 0 for invalid dims.
 */
size_t ic_layer_stack_workspace_bytes(const ic_dims *dims, int n_layers, long long rows_per_chunk);

/*
 * Rows per sequence (the first ones, i < returned value) that
 * ic_layer_stack_forward sends to the dense-masked attention for these dims
 * and a workspace of ws_bytes: rows with t < 6k in whole blocks of 128/Hq
 * queries, when d = 128, Hq divides 128, at most 65536 keys are visible and
 * the workspace holds the selection bitmask next to one block of scores and
 * the transposed V.  The other rows gather.  0 for invalid dims.
 */
int ic_layer_stack_dense_rows(const ic_dims *dims, size_t ws_bytes);

/*
 * The IndexCache layer loop (skill page Step 3; technical
 * summary, Methodologie; review, "The Redundancy That Was Sitting There": the
 * loop gains one branch per layer).
 * pattern: n_layers characters, 'F' or '1' = Full layer, 'S' or '0' = Shared.
 * For layer l: if F, the indexer scores and the top-k overwrite idx_cache
 * ([B, Lq, k] int32, caller-owned, the one index cache); then every layer
 * attends over idx_cache.  An S layer therefore uses exactly the indices of
 * the nearest preceding F layer.  pattern[0] must be F
 * (IC_ERR_NO_CACHED_INDICES otherwise, before any launch).
 * ws: device workspace of ws_bytes; F-layer scores are produced in row
 * chunks that fit in it; fewer than one query block of rows returns
 * IC_ERR_WORKSPACE_TOO_SMALL.  Each layer is an NVTX range ("layer <l> F" or
 * "layer <l> S", with nested ranges for the indexer + top-k and the
 * attention) for profilers.  Nothing inside synchronises the host or
 * allocates, so the call is meant to be capturable into a CUDA graph; no
 * test captures it yet.
 */
int ic_layer_stack_forward(const char *pattern, int n_layers, const ic_layer *layers,
                           const ic_dims *dims, int32_t *idx_cache, void *ws, size_t ws_bytes,
                           ic_stream_t stream);

/* Timing marks ic_layer_stack_forward_events records per layer. */
#define IC_MARKS_PER_LAYER 5

/*
 * ic_layer_stack_forward with per-layer timing marks: the same launches,
 * plus cudaEventRecord on `stream` of events[IC_MARKS_PER_LAYER*l + j] (each
 * a cudaEvent_t; NULL entries are skipped) at
 *   j=0 layer start,
 *   j=1 after the indexer (when the layer's scores take one chunk; otherwise
 *       after indexer + top-k),
 *   j=2 before the attention (after the top-k and, on F layers whose rows
 *       take the dense-masked path, the bitmask build),
 *   j=3 after the dense-masked attention of the rows with t < 6k (the
 *       transposed V copy included; equal to j=2 when no row takes it),
 *   j=4 after the attention.
 * For S layers j=0..2 coincide.  events holds IC_MARKS_PER_LAYER*n_layers
 * entries.
 */
int ic_layer_stack_forward_events(const char *pattern, int n_layers, const ic_layer *layers,
                                  const ic_dims *dims, int32_t *idx_cache, void *ws,
                                  size_t ws_bytes, ic_stream_t stream, void *const *events);

/*
 * Options of ic_layer_stack_forward_opts (NULL = all defaults).
 *   fused_topk  how an F layer turns scores into index rows (the kualia.ai
 *               review, "The Hidden Quadratic": the indexer's
 *               O(L^2) work and its L x L score matrix dominate long
 *               prefills):
 *                 0  store each chunk's causal scores in the workspace, then
 *                    run the top-k over them;
 *                 1  fused: never store the score matrix.  A pass over every
 *                    stride-th key tile (stride = max(1, key tiles / 16))
 *                    gives each row a threshold -- the r-th largest sampled
 *                    score, r = ceil(m p + z sqrt(m p (1 - p))) + 1 for m
 *                    visible samples and p = k / (t + 1) -- then the indexer
 *                    runs again keeping only scores at or above it, in a list
 *                    of 4k slots per row (rows with at most 2k visible
 *                    positions keep them all; rows with at most k need no
 *                    list), and an exact selection runs on those candidates.
 *                    A row with fewer than k candidates, or whose reserved
 *                    slots overflow its list, has its query block re-run the
 *                    way of mode 0, so the index rows equal mode 0's bit for
 *                    bit in every case.  Needs k <= 4096 and Lk <= 262144
 *                    (IC_ERR_UNSUPPORTED otherwise);
 *                -1  (default) the library's choice: fused when the longest
 *                    row sees more than 8k positions and there are at least
 *                    1024 query rows, else mode 0.
 *   z           the threshold's margin in binomial standard deviations
 *               (<= 0: 4).  Larger keeps more candidates and falls back less
 *               often; the index rows do not depend on it.
 */
typedef struct {
    int fused_topk;
    float z;
} ic_stack_options;

/*
 * ic_layer_stack_forward_events with options (opts may be NULL; events may be
 * NULL).  On the fused path, timing mark j=1 is recorded after the candidate
 * pass (sampled scores, thresholds and candidates), and j=2 after the exact
 * selection and the fallback rounds.  The workspace from
 * ic_layer_stack_workspace_bytes holds the fused path's chunk too; a smaller
 * one is split into more chunks, and fused_topk = 1 with a workspace that
 * holds no fused chunk returns IC_ERR_WORKSPACE_TOO_SMALL.
 */
int ic_layer_stack_forward_opts(const char *pattern, int n_layers, const ic_layer *layers,
                                const ic_dims *dims, const ic_stack_options *opts,
                                int32_t *idx_cache, void *ws, size_t ws_bytes,
                                ic_stream_t stream, void *const *events);

/*
 * Diagnostic of the fused path: synchronises `stream` and writes to *blocks
 * how many query blocks of the last F layer's last row chunk fell back to
 * the plain indexer + top-k (read from the workspace of the last
 * ic_layer_stack_forward_opts call with the same dims, options and
 * workspace).  IC_ERR_INVALID_ARG when the stack does not fuse for them.
 */
int ic_layer_stack_fused_fallback_blocks(const ic_dims *dims, const ic_stack_options *opts,
                                         const void *ws, size_t ws_bytes, ic_stream_t stream,
                                         int *blocks);

/*
 * Cross-layer overlap of two layers' index sets (skill page,
 * Step 1 "Analyze Index Correlation Across Layers": top-k sets of
 * consecutive layers compared per query position; kualia.ai review: in
 * adjacent layers 70-100% of the k picks coincide).
 *   idx_a, idx_b [n_rows, k] int32 (device; -1 = empty slot; every other
 *   entry in [0, Lk))   counts [n_rows, 3] int32 (device, written)
 * Row r gets counts[r] = { |A & B|, |A|, |B| } with each row read as the set
 * of its valid entries (a position repeated in a row counts once); the
 * overlap fraction is |A & B| / k and the Jaccard index |A & B| / |A | B|.
 * Entries outside [-1, Lk) are skipped and flag IC_ERR_INVALID_ARG in the
 * device error word.  Lk up to 262144.  Asynchronous on `stream`.
 */
int ic_index_overlap(const int32_t *idx_a, const int32_t *idx_b, long long n_rows, int k, int Lk,
                     int32_t *counts, ic_stream_t stream);

/*
 * Kernel launches this library has issued in this process so far (every
 * entry point, every device).  A host-side counter: reading it never
 * synchronises.  Callers take the difference around a region to count the
 * launches inside it.
 */
unsigned long long ic_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* INDEXCACHE_H */
