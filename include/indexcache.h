/*
 * indexcache.h -- C ABI of the IndexCache hot path on NVIDIA B200 (sm_100a).
 *
 * IndexCache ("IndexCache: Accelerating Sparse Attention via Cross-Layer
 * Index Reuse", summarised on gist.science) splits a stack of DeepSeek
 * sparse-attention (DSA) layers into F and S layers by a binary pattern:
 *   - an F ("Full") layer runs its lightning indexer over every causal key of
 *     every query, keeps the top-k key positions per query and stores them in
 *     a temporary index cache;
 *   - an S ("Shared") layer has no indexer and reuses the cached indices of
 *     the nearest preceding F layer;
 *   - every layer runs sparse attention over its query's selected keys only.
 * (es page, section 2 "Arquitectura del Método"; pt page, section 2
 * "Arquitetura"; de page, section 2 "Methodik: IndexCache".)
 *
 * Conventions shared by every call:
 *   - All array arguments are DEVICE pointers unless stated otherwise.  The
 *     caller owns every buffer; the library never allocates device memory and
 *     keeps no per-call state on the device.
 *   - Arrays are dense, row-major, with the layouts stated per argument.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronise, except ic_read_status and
 *     ic_check_status.  Calls over at most 256 query rows (decode) launch
 *     their kernels with programmatic stream serialization: a kernel may be
 *     scheduled, and run its on-chip setup, while the previous kernel on the
 *     stream finishes, but it touches no global memory before that kernel
 *     has completed.  Stream order holds as for plain launches, inside CUDA
 *     graph capture too.
 *   - Argument errors are returned before anything is launched.  A failed
 *     launch returns IC_ERR_CUDA.  Errors the kernels detect themselves (an
 *     index outside its row's causal range, a wait that ran out of time) are
 *     recorded as bits of a status word at the start of the workspace and
 *     read back with ic_read_status.  No kernel traps or asserts.
 *   - Workspace: every call takes `ws`/`ws_bytes`.  The first
 *     IC_STATUS_BYTES bytes hold the status word; zero them once with
 *     ic_workspace_init.  `ws` must be 256-byte aligned.  The size a call
 *     needs is given by its *_workspace_size function.
 *   - Causality: query row i of sequence b sits at absolute position
 *     t = q_start + i and its candidate keys are s = 0..t (its own key
 *     included).  A decode step is Lq = 1, q_start = T - 1.
 */
#ifndef INDEXCACHE_H
#define INDEXCACHE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define IC_STATUS_BYTES 256

typedef enum {
    IC_OK = 0,
    IC_ERR_INVALID_ARG = -1,  /* null pointer, bad size, stride or alignment        */
    IC_ERR_PATTERN = -2,      /* pattern not of 'F'/'S', wrong length, or starts 'S' */
    IC_ERR_UNSUPPORTED = -3,  /* dtype / shape combination not implemented          */
    IC_ERR_WORKSPACE = -4,    /* ws too small or misaligned                         */
    IC_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed                */
    IC_ERR_INDEX_RANGE = -6,  /* (device) an index was outside [0, t] and skipped   */
    IC_ERR_TIMEOUT = -7       /* (device) a pipeline wait ran out of time            */
} ic_status;

typedef enum {
    IC_F32 = 0,       /* IEEE float32                                   */
    IC_BF16 = 1,      /* bfloat16                                       */
    IC_FP8_E4M3 = 2   /* OCP E4M3 "FN" byte codes with per-token scale  */
} ic_dtype;

/* Rows of a call: B sequences, Lq query rows each starting at absolute
 * position q_start, T keys per sequence.  Requires q_start + Lq <= T. */
typedef struct {
    int B;
    int Lq;
    int q_start;
    int T;
} ic_rows;

/* ------------------------------------------------------------------------ */
/* Status and workspace                                                      */
/* ------------------------------------------------------------------------ */

/* Human-readable name of a status code (static string, never NULL). */
const char* ic_status_string(ic_status st);

/* Text of the last CUDA failure seen by a call of this library on the
 * calling thread ("<source>: <CUDA error string>"), behind the most recent
 * IC_ERR_CUDA; "" if none.  Per-thread static storage, valid until the next
 * failing call on the same thread; never NULL. */
const char* ic_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int ic_version(void);

/* Zero the status word at the start of `ws` (asynchronous memset on stream).
 * ws_bytes must be >= IC_STATUS_BYTES. */
ic_status ic_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, read the status word of `ws` into *device_status
 * (host pointer; bit 0 = index out of range, bit 1 = wait timeout) and clear
 * it.  Returns IC_OK when no bit was set, else the error of the lowest bit. */
ic_status ic_read_status(void* ws, void* stream, int32_t* device_status);

/* ic_read_status without the raw bits: synchronise `stream`, clear the
 * status word of `ws` and return IC_OK, IC_ERR_INDEX_RANGE or IC_ERR_TIMEOUT
 * (the error of the lowest set bit). */
ic_status ic_check_status(void* ws, void* stream);

/* Failure-path self-test: launches one CTA whose pipeline wait (the
 * library's bounded mbarrier wait) never completes.  After about 1 s the
 * wait gives up, bit 1 (wait timeout) of the status word of `ws` is set and
 * the kernel returns normally; read it with ic_read_status.  Faults and
 * hangs nothing; the context stays usable.  ws_bytes >= IC_STATUS_BYTES. */
ic_status ic_selftest_wait_timeout(void* ws, size_t ws_bytes, void* stream);

/* Number of kernels this library has launched in this process, by kind:
 * 0 = all, 1 = indexer, 2 = top-k, 3 = attention, 4 = split-k combine,
 * 5 = indexer launches that took the tensor-core path, 6 = attention
 * launches that took the tensor-core path, 7 = fused decode key selections
 * (each also counted once under 1 and once under 2).  A host-side diagnostic
 * counter (thread-safe). */
uint64_t ic_kernel_launches(int kind);

/* ------------------------------------------------------------------------ */
/* a1  Lightning indexer scores (F layers)                                   */
/* ------------------------------------------------------------------------ */
/*
 * The indexer scores every preceding token of each query so the top-k most
 * relevant can be kept; it is O(L^2) per layer (es page, section 1
 * "El Problema"; pt page, section 1 "O Gargalo do Indexador").  The score
 * form is not printed on the pages; this library computes
 *     scores[b,i,s] = sum_h w[b,i,h] * max(0, q_I[b,i,h,:] . k_I[b,s,:])
 * for s <= t = q_start + i.  Entries s > t of a row are NOT written.
 *
 *   q_idx   [B, Lq, H_I, d_I] of dt   (IC_F32, IC_BF16 or IC_FP8_E4M3 codes)
 *   q_scale [B, Lq] float32, one non-negative scale per query token
 *           (IC_FP8_E4M3 only; NULL otherwise): q value = e4m3(code)*scale
 *   w       [B, Lq, H_I] float32 head weights
 *   k_idx   [B, T, d_I] of dt
 *   k_scale [B, T] float32 (IC_FP8_E4M3 only; NULL otherwise)
 *   scores  [B, Lq, ld_scores] float32; ld_scores >= T, ld_scores % 4 == 0
 * Accumulation is float32.  With FP8 operands the scales are applied after
 * the head-sum (exact for non-negative scales, ReLU being positively
 * homogeneous).  Supported: H_I in [1,128]; d_I in [1,256].  The tensor-core
 * path is used for IC_BF16 / IC_FP8_E4M3 with d_I == 128 and H_I in
 * {16,32,64,128}; other shapes and IC_F32 use a CUDA-core path.
 */
size_t ic_indexer_workspace_size(ic_rows r, int H_I, int d_I, ic_dtype dt);
ic_status ic_indexer_scores(const void* q_idx, const float* q_scale, const float* w,
                            const void* k_idx, const float* k_scale, ic_dtype dt,
                            ic_rows r, int H_I, int d_I,
                            float* scores, int64_t ld_scores,
                            void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* a2  Top-k selection (F layers)                                            */
/* ------------------------------------------------------------------------ */
/*
 * DSA keeps the k most relevant keys of each query (es page, section 1).
 * Row t keeps the min(k, t+1) candidates s <= t with the largest score,
 * ordered by (score descending, position ascending): equal scores go to the
 * smaller position, -0.0 counts as +0.0.  The kept positions are written in
 * ASCENDING order, followed by -1 up to k entries.
 *
 *   scores [B, Lq, ld_scores] float32 (only s <= t of each row is read;
 *          ld_scores >= T, ld_scores % 4 == 0); must not hold NaN
 *   idx    [B, Lq, k] int32 (output)
 *   k      in [1, 16384]
 */
size_t ic_topk_workspace_size(ic_rows r, int k);
ic_status ic_topk(const float* scores, int64_t ld_scores, ic_rows r, int k, int32_t* idx,
                  void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* a1 + a2 in one call: an F layer's key selection                           */
/* ------------------------------------------------------------------------ */
/*
 * The indexer scores of ic_indexer_scores followed by the top-k of ic_topk,
 * with the same inputs, layouts and rules: the same indices, bit for bit
 * (the scores are computed by the same arithmetic in the same order).  For
 * decode-shaped rows (Lq <= 2, at most one row per SM, more than 4096
 * candidates) on the tensor-core shapes, when the row clusters together
 * cover most of the SMs, the two run as ONE kernel: one thread-block
 * cluster per row keeps the row's scores in shared memory and selects from
 * there, so no score row is written to memory.  Otherwise (fewer rows: the
 * stand-alone indexer on every SM is faster) the scores go through the
 * workspace.  (IndexCache's F layer computes exactly
 * this selection and caches it: es page, section 2 "Arquitectura del Método".)
 *   idx  [B, Lq, k] int32 (output), as ic_topk
 * Workspace: ic_indexer_topk_workspace_size.
 */
size_t ic_indexer_topk_workspace_size(ic_rows r, int H_I, int d_I, ic_dtype dt, int k);
ic_status ic_indexer_topk(const void* q_idx, const float* q_scale, const float* w,
                          const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r,
                          int H_I, int d_I, int k, int32_t* idx, void* ws, size_t ws_bytes,
                          void* stream);

/* ------------------------------------------------------------------------ */
/* a4/a5  Sparse multi-query attention (every layer)                         */
/* ------------------------------------------------------------------------ */
/*
 * Core attention restricted to the selected keys, O(Lk) (es page,
 * section 1; de page, section 1).  For row (b,i), head h and the entries j
 * of idx[b,i,:] that are >= 0:
 *     p_j = softmax_j(scale * q[b,i,h,0:d_qk] . K[b,j,0:d_qk])
 *     out[b,i,h,0:d_v] = sum_j p_j * V[b,j,0:d_v]
 * All Hq heads share the same key/value rows (multi-query attention).
 *
 *   q    [B, Lq, Hq, d_qk] of dt (IC_F32 or IC_BF16)
 *   kmat key row (b,s) starts at kmat + (b*T + s) * k_row_stride elements
 *   vmat value row (b,s) starts at vmat + (b*T + s) * v_row_stride elements
 *        (a latent KV cache passes the same pointer twice: K = the whole
 *        576-wide row, V = its first 512 columns)
 *   idx  [B, Lq, k] int32: positions in [0, t] or -1 (skipped, anywhere in
 *        the row).  An entry outside [0, t] and not -1 is never
 *        dereferenced: the row is computed without it and the status bit
 *        IC_ERR_INDEX_RANGE is set.
 *   out  [B, Lq, Hq, d_v] of dt.  A row with no valid index gets zeros.
 * Supported: Hq in [1,128], d_qk, d_v in [1,576].  The tensor-core path is
 * used for IC_BF16 with Hq == 128, d_qk == 576, d_v == 512 and kmat == vmat
 * (the latent MQA layout); other shapes use a CUDA-core path.  Rows with few
 * query rows per call (decode) are split over the k keys and merged by a
 * log-sum-exp combine (a5), which needs workspace.
 */
size_t ic_sparse_attn_workspace_size(ic_rows r, int k, int Hq, int d_qk, int d_v, ic_dtype dt);
ic_status ic_sparse_attn(const void* q, const void* kmat, int64_t k_row_stride,
                         const void* vmat, int64_t v_row_stride, const int32_t* idx, int k,
                         ic_dtype dt, ic_rows r, int Hq, int d_qk, int d_v, float scale,
                         void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Workspace-free variant of ic_sparse_attn for the latent MQA layout
 * (IC_BF16, Hq = 128, d_qk = 576, d_v = 512, K and V rows in one 576-wide
 * KV row: kv + (b*T + s)*576).  The IndexCache pages have no counterpart of
 * this call; it exists for callers that may not allocate device memory where
 * they run attention (an engine whose memory pool owns the whole GPU, a
 * plugin that only receives input and output buffers, a step where a
 * cudaMalloc and its possible device synchronisation are not acceptable).
 *
 * Same arguments, layouts and results as ic_sparse_attn with
 * kmat = vmat = kv and row strides 576, except that the split-k partials of
 * decode live in a fixed device array inside the library of
 * IC_NOALLOC_SCRATCH_BYTES bytes (about 8 MiB; every GPU that loads the
 * library holds it until the process exits), room for 64 partial rows
 * (query rows x splits).  Among its split counts this call only considers
 * those that keep B*Lq*splits <= 64, so it may split less finely than
 * ic_sparse_attn (same results within the attention tolerance, maybe
 * slower).  A row needs at least ceil(k / 2048) splits, so the call is
 * refused with IC_ERR_WORKSPACE, before launching anything, exactly when
 * k > 2048 and B*Lq*ceil(k / 2048) > 64; use ic_sparse_attn with a
 * workspace instead.  This function allocates nothing.
 *   device_status  NULL, or a DEVICE int32 that receives the call's status
 *                  bits (as ic_read_status reports them) when it completes.
 * The array's device address is looked up on the first call on a device
 * (with that device current) and again when the device's CUDA context has
 * changed since (after a cudaDeviceReset); make the first call on each
 * device, and the first after a reset, before any stream capture.  All calls
 * share the array and it keeps the last call's contents (the status word is
 * cleared at the start of each call): calls whose kernels overlap on the GPU
 * race on it, so serialise them (one stream, one thread).
 */
#define IC_NOALLOC_SCRATCH_BYTES ((8u << 20) + (128u << 10) + 512u)
ic_status ic_sparse_attn_noalloc(const void* q, const void* kv, const int32_t* idx, int k,
                                 ic_rows r, float scale, void* out, int32_t* device_status,
                                 void* stream);

/* ------------------------------------------------------------------------ */
/* a3  The layer stack with the F/S branch                                   */
/* ------------------------------------------------------------------------ */
typedef struct {
    ic_rows rows;
    int H_I, d_I;          /* indexer heads and width                          */
    ic_dtype idx_dtype;    /* dtype of q_idx / k_idx                           */
    int k;                 /* top-k                                            */
    int Hq, d_qk, d_v;     /* attention heads and widths                       */
    ic_dtype attn_dtype;   /* dtype of q, kmat, vmat, out                      */
    int64_t k_row_stride;  /* elements between consecutive key rows           */
    int64_t v_row_stride;  /* elements between consecutive value rows         */
    float scale;           /* softmax scale                                    */
} ic_stack_shape;

/* Per-layer device buffers, same layouts as the single calls above.  The
 * indexer fields (q_idx, q_scale, w, k_idx, k_scale) are ignored, and may be
 * NULL, on S layers. */
typedef struct {
    const void* q_idx;
    const float* q_scale;
    const float* w;
    const void* k_idx;
    const float* k_scale;
    const void* q;
    const void* kmat;
    const void* vmat;
    void* out;
} ic_layer_io;

/*
 * Run n_layers layers in order.  pattern is a NUL-terminated string of
 * exactly n_layers characters 'F' or 'S' whose first character is 'F'
 * (an S layer inherits from the nearest PRECEDING F layer, so a leading S
 * has nothing to inherit); anything else returns IC_ERR_PATTERN.
 *   F layer: indexer -> scores (workspace) -> top-k -> idx_buf
 *   S layer: idx_buf is used unchanged (no copy, no indexer launch)
 *   every layer: sparse attention over idx_buf -> layers[l].out
 * idx_buf [B, Lq, k] int32 is the single index cache.  idx_out is either
 * NULL or a HOST array of n_layers device pointers, each NULL or an
 * [B, Lq, k] int32 buffer that receives a copy of the indices layer l used
 * (for checking; costs one device copy per non-NULL entry).
 * ws_bytes >= ic_workspace_size(shape).
 */
size_t ic_workspace_size(const ic_stack_shape* shape);
ic_status ic_layer_stack_forward(const char* pattern, int n_layers, const ic_layer_io* layers,
                                 const ic_stack_shape* shape, int32_t* idx_buf,
                                 int32_t* const* idx_out, void* ws, size_t ws_bytes,
                                 void* stream);

/* ------------------------------------------------------------------------ */
/* Variable-length batches over a paged KV cache                             */
/* ------------------------------------------------------------------------ */
/*
 * The decode batch of a serving engine: every sequence has its own length,
 * and every per-key cache (the indexer keys k_I, their FP8 scales, the
 * latent KV rows) lives in fixed-size pages shared by all sequences, so a
 * sequence grows by pages without moving data.  This is the layout behind
 * the pages' throughput figure with the KV cache saturated (es page,
 * section 3 "Resultados Clave"; de page, section 3 "Wichtige Ergebnisse");
 * the pages do not describe the layout itself, and the serving system
 * around it is not part of this library.
 *
 *   B            sequences; Lq query rows per sequence (1 for decode)
 *   seq_lens     [B] int32, DEVICE: keys of sequence b (its context,
 *                including the query rows' own keys); Lq <= seq_lens[b] <= T_max
 *                (a length outside this range makes the sequence's rows
 *                empty: no index, zero output, status bit IC_ERR_INDEX_RANGE)
 *   T_max        upper bound of seq_lens (sizes the score rows and grids;
 *                the host never reads seq_lens)
 *   block_table  [B, max_pages] int32, DEVICE: physical page of logical page
 *                j of sequence b.  Key position s of sequence b lives in
 *                physical row block_table[b*max_pages + s/page_size] *
 *                page_size + s % page_size of every paged cache.
 *   page_size    rows per page: a multiple of 128
 *   num_pages    pages of each paged cache (physical rows = num_pages*page_size)
 * Query row i of sequence b sits at t = seq_lens[b] - Lq + i and its
 * candidate keys are the logical positions 0..t.  Indices (top-k outputs and
 * attention inputs) are LOGICAL positions.
 */
typedef struct {
    int B;
    int Lq;
    int T_max;
    const int32_t* seq_lens;
    const int32_t* block_table;
    int max_pages;
    int page_size;
    int num_pages;
} ic_paged_rows;

/* a1 over paged keys: scores[b,i,s] for logical s <= t as ic_indexer_scores.
 *   k_pages        [num_pages*page_size, d_I] of dt (IC_BF16 or IC_FP8_E4M3)
 *   k_scale_pages  [num_pages*page_size] float32 (IC_FP8_E4M3 only)
 *   scores         [B, Lq, ld_scores] float32, ld_scores >= T_max, % 4 == 0
 * Tensor-core shapes only: d_I == 128, H_I in {16,32,64,128}; other shapes
 * and IC_F32 return IC_ERR_UNSUPPORTED.  Workspace: ic_indexer_workspace_size. */
ic_status ic_indexer_scores_paged(const void* q_idx, const float* q_scale, const float* w,
                                  const void* k_pages, const float* k_scale_pages, ic_dtype dt,
                                  const ic_paged_rows* pr, int H_I, int d_I,
                                  float* scores, int64_t ld_scores,
                                  void* ws, size_t ws_bytes, void* stream);

/* a1 + a2 over paged keys: the indices of ic_indexer_scores_paged followed
 * by ic_topk_varlen, bit for bit (one fused kernel for decode-shaped rows, as
 * ic_indexer_topk).  Workspace: ic_indexer_topk_paged_workspace_size. */
size_t ic_indexer_topk_paged_workspace_size(const ic_paged_rows* pr, int k);
ic_status ic_indexer_topk_paged(const void* q_idx, const float* q_scale, const float* w,
                                const void* k_pages, const float* k_scale_pages, ic_dtype dt,
                                const ic_paged_rows* pr, int H_I, int d_I, int k, int32_t* idx,
                                void* ws, size_t ws_bytes, void* stream);

/* a2 with per-sequence lengths: row (b, i) keeps the min(k, t+1) best of
 * its t+1 candidates, t = seq_lens[b] - Lq + i, as ic_topk.  Only seq_lens,
 * B, Lq and T_max of pr are read.  Workspace: ic_topk_varlen_workspace_size. */
size_t ic_topk_varlen_workspace_size(const ic_paged_rows* pr, int k);
ic_status ic_topk_varlen(const float* scores, int64_t ld_scores, const ic_paged_rows* pr, int k,
                         int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/* a4/a5 over paged latent KV rows (IC_BF16, Hq = 128, d_qk = 576, d_v = 512):
 *   q         [B, Lq, 128, 576] bf16
 *   kv_pages  [num_pages*page_size, 576] bf16 (V = the first 512 columns)
 *   idx       [B, Lq, k] int32 logical positions in [0, t] or -1
 *   out       [B, Lq, 128, 512] bf16
 * Workspace: ic_sparse_attn_paged_workspace_size. */
size_t ic_sparse_attn_paged_workspace_size(const ic_paged_rows* pr, int k);
ic_status ic_sparse_attn_paged(const void* q, const void* kv_pages, const int32_t* idx, int k,
                               const ic_paged_rows* pr, float scale, void* out,
                               void* ws, size_t ws_bytes, void* stream);

/* a3 over paged caches: ic_layer_stack_forward with every layer's k_idx,
 * k_scale, kmat (== vmat) pointing at that layer's paged caches.  shape->rows
 * is ignored (pr gives the rows); shape must name the tensor-core shapes
 * (idx_dtype IC_BF16 or IC_FP8_E4M3, d_I 128; attn IC_BF16, 128 heads, 576 /
 * 512, row strides 576). */
size_t ic_paged_workspace_size(const ic_stack_shape* shape, const ic_paged_rows* pr);
ic_status ic_layer_stack_forward_paged(const char* pattern, int n_layers,
                                       const ic_layer_io* layers, const ic_stack_shape* shape,
                                       const ic_paged_rows* pr, int32_t* idx_buf,
                                       int32_t* const* idx_out, void* ws, size_t ws_bytes,
                                       void* stream);

#ifdef __cplusplus
}
#endif

#endif /* INDEXCACHE_H */
