// api.cu -- the C ABI of the IndexCache library (see include/indexcache.h).
//
// Argument validation, workspace layout, dispatch between the tensor-core and
// CUDA-core kernels, and the layer stack with IndexCache's F/S branch:
// F layers run indexer -> top-k into the single index cache, S layers reuse
// the cache unchanged, every layer runs sparse attention (IndexCache summary,
// es page, section 2 "Arquitectura del Método"; it page, section 2
// "Architettura e Funzionamento").
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>

#include "common.cuh"

namespace ic {

static std::atomic<uint64_t> g_launches[IC_LK_KINDS];

void count_launch(int kind) {
    g_launches[IC_LK_ALL].fetch_add(1, std::memory_order_relaxed);
    if (kind == IC_LK_INDEXER_TC) g_launches[IC_LK_INDEXER].fetch_add(1, std::memory_order_relaxed);
    if (kind == IC_LK_ATTN_TC) g_launches[IC_LK_ATTN].fetch_add(1, std::memory_order_relaxed);
    if (kind == IC_LK_SELECT) {  // one fused launch does an F layer's indexer and top-k
        g_launches[IC_LK_INDEXER].fetch_add(1, std::memory_order_relaxed);
        g_launches[IC_LK_TOPK].fetch_add(1, std::memory_order_relaxed);
    }
    if (kind > 0 && kind < IC_LK_KINDS) g_launches[kind].fetch_add(1, std::memory_order_relaxed);
}

namespace {
thread_local char tl_error[256] = "";
}

const char* tl_error_text() { return tl_error; }

ic_status cuda_error(const char* where) {
    const cudaError_t e = cudaGetLastError();
    snprintf(tl_error, sizeof(tl_error), "%s: %s", where,
             e == cudaSuccess ? "CUDA driver call failed" : cudaGetErrorString(e));
    return IC_ERR_CUDA;
}

ic_status last_launch_status() {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return IC_OK;
    snprintf(tl_error, sizeof(tl_error), "kernel launch: %s", cudaGetErrorString(e));
    return IC_ERR_CUDA;
}

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool rows_ok(const ic_rows& r) {
    if (r.B < 0 || r.Lq < 0 || r.q_start < 0 || r.T < 0) return false;
    return (int64_t)r.q_start + r.Lq <= r.T;
}
bool rows_empty(const ic_rows& r) { return r.B == 0 || r.Lq == 0; }

bool ws_ok(const void* ws, size_t bytes, size_t need) {
    return ws != nullptr && bytes >= need && ((uintptr_t)ws % kAlign) == 0;
}

uint32_t* status_of(void* ws) { return static_cast<uint32_t*>(ws); }
char* scratch_of(void* ws) { return static_cast<char*>(ws) + IC_STATUS_BYTES; }

size_t scores_bytes(const ic_rows& r) {
    const int64_t ld = ((int64_t)r.T + 3) / 4 * 4;
    return (size_t)r.B * r.Lq * ld * sizeof(float);
}

bool attn_args_ok(ic_dtype dt, int Hq, int d_qk, int d_v, int k) {
    return (dt == IC_F32 || dt == IC_BF16) && Hq >= 1 && Hq <= 128 && d_qk >= 1 && d_qk <= 576 &&
           d_v >= 1 && d_v <= 576 && k >= 1 && k <= 16384;
}

bool indexer_args_ok(ic_dtype dt, int H_I, int d_I) {
    return (dt == IC_F32 || dt == IC_BF16 || dt == IC_FP8_E4M3) && H_I >= 1 && H_I <= 128 &&
           d_I >= 1 && d_I <= 256;
}

size_t attn_scratch(const ic_rows& r, int k, int Hq, int d_qk, int d_v, ic_dtype dt) {
    // the tensor-core path may be taken when the shapes match; size for it
    if (dt == IC_BF16 && Hq == 128 && d_qk == 576 && d_v == 512) return attn_tc_scratch_bytes(r, k);
    return 0;
}

// A paged batch: sizes consistent, device arrays present, every sequence's
// logical pages addressable by its block-table row.
bool paged_ok(const ic_paged_rows* pr, bool need_pages) {
    if (pr == nullptr || pr->B < 0 || pr->Lq < 1 || pr->T_max < pr->Lq) return false;
    if (pr->B > 0 && pr->seq_lens == nullptr) return false;
    if (!need_pages) return true;
    if (pr->page_size < 128 || pr->page_size % 128 != 0 || pr->num_pages < 1) return false;
    if ((int64_t)pr->num_pages * pr->page_size >= 0x7fffffffLL) return false;
    if ((int64_t)pr->max_pages * pr->page_size < pr->T_max) return false;
    return pr->B == 0 || pr->block_table != nullptr;
}

// Planning rows of a paged batch: every sequence as long as T_max.
// Every score row starts on a 16-byte boundary (the cluster and multi-CTA
// top-k kernels read rows as 16-byte vectors).
bool rows_16b_aligned(const float* scores, int64_t ld) {
    return ((uintptr_t)scores & 15) == 0 && (ld & 3) == 0;
}

ic_rows plan_rows(const ic_paged_rows* pr) { return ic_rows{pr->B, pr->Lq, pr->T_max - pr->Lq, pr->T_max}; }

ic_status run_topk_varlen(const float* scores, int64_t ld, const ic_paged_rows* pr, int k,
                          int32_t* idx, cudaStream_t s) {
    const ic_rows r = plan_rows(pr);
    if (topk_cluster_applies(r, k) && rows_16b_aligned(scores, ld))
        return launch_topk_cluster(scores, ld, r, k, idx, s, pr->seq_lens);
    return launch_topk_rows(scores, ld, r, k, idx, s, pr->seq_lens);
}

bool latent_tc_shape(const ic_stack_shape* sh) {
    return indexer_tc_supported(sh->idx_dtype, sh->H_I, sh->d_I) && sh->attn_dtype == IC_BF16 &&
           sh->Hq == 128 && sh->d_qk == 576 && sh->d_v == 512 && sh->k_row_stride == 576 &&
           sh->v_row_stride == 576;
}

ic_status run_indexer(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                      const float* k_scale, ic_dtype dt, ic_rows r, int H_I, int d_I,
                      float* scores, int64_t ld, uint32_t* status, cudaStream_t s) {
    if (indexer_tc_supported(dt, H_I, d_I))
        return launch_indexer_tc(q_idx, q_scale, w, k_idx, k_scale, dt, r, H_I, d_I, scores, ld,
                                 status, s);
    return launch_indexer_simt(q_idx, q_scale, w, k_idx, k_scale, dt, r, H_I, d_I, scores, ld, s);
}

ic_status run_topk(const float* scores, int64_t ld, ic_rows r, int k, int32_t* idx, void* scratch,
                   size_t scratch_bytes, cudaStream_t s) {
    // the cluster and multi-CTA paths read 16-byte vectors: they need 16-byte
    // aligned rows.  Few long rows (decode): one cluster per row, one launch;
    // rows too long for the cluster's shared memory: three launches.
    if (topk_cluster_applies(r, k) && rows_16b_aligned(scores, ld))
        return launch_topk_cluster(scores, ld, r, k, idx, s);
    if (topk_multi_applies(r, k) && scratch != nullptr && rows_16b_aligned(scores, ld) &&
        scratch_bytes >= topk_multi_scratch_bytes(r, k))
        return launch_topk_multi(scores, ld, r, k, idx, scratch, s);
    return launch_topk_rows(scores, ld, r, k, idx, s);
}

// An F layer's key selection: fused for decode shapes, else indexer scores
// into `scores` then top-k.
ic_status run_select(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                     const float* k_scale, ic_dtype dt, ic_rows r, int H_I, int d_I, int k,
                     int32_t* idx, float* scores, int64_t ld, uint32_t* status, void* scratch,
                     size_t scratch_bytes, cudaStream_t s) {
    if (select_fused_applies(dt, H_I, d_I, r, k)) {
        const ic_status st = launch_select_fused(q_idx, q_scale, w, k_idx, k_scale, dt, r, H_I, k,
                                                 idx, status, s);
        if (st != IC_ERR_UNSUPPORTED) return st;
    }
    ic_status st = run_indexer(q_idx, q_scale, w, k_idx, k_scale, dt, r, H_I, d_I, scores, ld,
                               status, s);
    if (st != IC_OK) return st;
    return run_topk(scores, ld, r, k, idx, scratch, scratch_bytes, s);
}

ic_status run_attn(const void* q, const void* kmat, int64_t ks, const void* vmat, int64_t vs,
                   const int32_t* idx, int k, ic_dtype dt, ic_rows r, int Hq, int d_qk, int d_v,
                   float scale, void* out, uint32_t* status, void* scratch, size_t scratch_bytes,
                   cudaStream_t s) {
    if (attn_tc_supported(kmat, vmat, ks, vs, dt, Hq, d_qk, d_v) &&
        scratch_bytes >= attn_tc_scratch_bytes(r, k))
        return launch_attn_tc(q, kmat, ks, idx, k, r, scale, out, status, scratch, scratch_bytes, s);
    return launch_attn_simt(q, kmat, ks, vmat, vs, idx, k, dt, r, Hq, d_qk, d_v, scale, out,
                            status, s);
}

}  // namespace
}  // namespace ic

using namespace ic;

extern "C" {

const char* ic_last_error(void) { return ic::tl_error_text(); }

const char* ic_status_string(ic_status st) {
    switch (st) {
        case IC_OK: return "IC_OK";
        case IC_ERR_INVALID_ARG: return "IC_ERR_INVALID_ARG";
        case IC_ERR_PATTERN: return "IC_ERR_PATTERN";
        case IC_ERR_UNSUPPORTED: return "IC_ERR_UNSUPPORTED";
        case IC_ERR_WORKSPACE: return "IC_ERR_WORKSPACE";
        case IC_ERR_CUDA: return "IC_ERR_CUDA";
        case IC_ERR_INDEX_RANGE: return "IC_ERR_INDEX_RANGE";
        case IC_ERR_TIMEOUT: return "IC_ERR_TIMEOUT";
    }
    return "IC_ERR_UNKNOWN";
}

int ic_version(void) { return 10000; }

uint64_t ic_kernel_launches(int kind) {
    if (kind < 0 || kind >= IC_LK_KINDS) return 0;
    return g_launches[kind].load(std::memory_order_relaxed);
}

ic_status ic_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws_ok(ws, ws_bytes, IC_STATUS_BYTES)) return IC_ERR_WORKSPACE;
    if (cudaMemsetAsync(ws, 0, IC_STATUS_BYTES, (cudaStream_t)stream) != cudaSuccess)
        return cuda_error("api");
    return IC_OK;
}

ic_status ic_read_status(void* ws, void* stream, int32_t* device_status) {
    if (ws == nullptr || device_status == nullptr) return IC_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return cuda_error("api");
    if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_error("api");
    if (v != 0) {
        if (cudaMemsetAsync(ws, 0, sizeof(v), s) != cudaSuccess) return cuda_error("api");
        if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_error("api");
    }
    *device_status = (int32_t)v;
    if (v & IC_DEV_INDEX_RANGE) return IC_ERR_INDEX_RANGE;
    if (v & IC_DEV_TIMEOUT) return IC_ERR_TIMEOUT;
    return IC_OK;
}

ic_status ic_check_status(void* ws, void* stream) {
    if (ws == nullptr) return IC_ERR_INVALID_ARG;
    int32_t bits = 0;
    return ic_read_status(ws, stream, &bits);
}

size_t ic_indexer_workspace_size(ic_rows r, int H_I, int d_I, ic_dtype dt) {
    (void)r; (void)H_I; (void)d_I; (void)dt;
    return IC_STATUS_BYTES;
}

ic_status ic_indexer_scores(const void* q_idx, const float* q_scale, const float* w,
                            const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r,
                            int H_I, int d_I, float* scores, int64_t ld_scores, void* ws,
                            size_t ws_bytes, void* stream) {
    if (!rows_ok(r) || !indexer_args_ok(dt, H_I, d_I)) return IC_ERR_INVALID_ARG;
    if (ld_scores < r.T || ld_scores % 4 != 0) return IC_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, ic_indexer_workspace_size(r, H_I, d_I, dt))) return IC_ERR_WORKSPACE;
    if (rows_empty(r)) return IC_OK;
    if (!q_idx || !w || !k_idx || !scores) return IC_ERR_INVALID_ARG;
    if (dt == IC_FP8_E4M3 && (!q_scale || !k_scale)) return IC_ERR_INVALID_ARG;
    if (dt != IC_FP8_E4M3 && (q_scale || k_scale)) return IC_ERR_INVALID_ARG;
    return run_indexer(q_idx, q_scale, w, k_idx, k_scale, dt, r, H_I, d_I, scores, ld_scores,
                       status_of(ws), (cudaStream_t)stream);
}

size_t ic_topk_workspace_size(ic_rows r, int k) {
    return IC_STATUS_BYTES + align_up(topk_multi_scratch_bytes(r, k));
}

ic_status ic_topk(const float* scores, int64_t ld_scores, ic_rows r, int k, int32_t* idx,
                  void* ws, size_t ws_bytes, void* stream) {
    if (!rows_ok(r) || k < 1 || k > 16384) return IC_ERR_INVALID_ARG;
    if (ld_scores < r.T || ld_scores % 4 != 0) return IC_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, ic_topk_workspace_size(r, k))) return IC_ERR_WORKSPACE;
    if (rows_empty(r)) return IC_OK;
    if (!scores || !idx) return IC_ERR_INVALID_ARG;
    return run_topk(scores, ld_scores, r, k, idx, scratch_of(ws), ws_bytes - IC_STATUS_BYTES,
                    (cudaStream_t)stream);
}

size_t ic_indexer_topk_workspace_size(ic_rows r, int H_I, int d_I, ic_dtype dt, int k) {
    (void)H_I; (void)d_I; (void)dt;
    return IC_STATUS_BYTES + align_up(scores_bytes(r)) + align_up(topk_multi_scratch_bytes(r, k));
}

ic_status ic_indexer_topk(const void* q_idx, const float* q_scale, const float* w,
                          const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r, int H_I,
                          int d_I, int k, int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
    if (!rows_ok(r) || !indexer_args_ok(dt, H_I, d_I) || k < 1 || k > 16384)
        return IC_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, ic_indexer_topk_workspace_size(r, H_I, d_I, dt, k)))
        return IC_ERR_WORKSPACE;
    if (rows_empty(r)) return IC_OK;
    if (!q_idx || !w || !k_idx || !idx) return IC_ERR_INVALID_ARG;
    if (dt == IC_FP8_E4M3 && (!q_scale || !k_scale)) return IC_ERR_INVALID_ARG;
    if (dt != IC_FP8_E4M3 && (q_scale || k_scale)) return IC_ERR_INVALID_ARG;
    float* scores = reinterpret_cast<float*>(scratch_of(ws));
    const int64_t ld = ((int64_t)r.T + 3) / 4 * 4;
    char* tail = scratch_of(ws) + align_up(scores_bytes(r));
    return run_select(q_idx, q_scale, w, k_idx, k_scale, dt, r, H_I, d_I, k, idx, scores, ld,
                      status_of(ws), tail, ws_bytes - IC_STATUS_BYTES - align_up(scores_bytes(r)),
                      (cudaStream_t)stream);
}

size_t ic_sparse_attn_workspace_size(ic_rows r, int k, int Hq, int d_qk, int d_v, ic_dtype dt) {
    return IC_STATUS_BYTES + align_up(attn_scratch(r, k, Hq, d_qk, d_v, dt));
}

ic_status ic_sparse_attn(const void* q, const void* kmat, int64_t k_row_stride, const void* vmat,
                         int64_t v_row_stride, const int32_t* idx, int k, ic_dtype dt, ic_rows r,
                         int Hq, int d_qk, int d_v, float scale, void* out, void* ws,
                         size_t ws_bytes, void* stream) {
    if (!rows_ok(r) || !attn_args_ok(dt, Hq, d_qk, d_v, k)) return IC_ERR_INVALID_ARG;
    if (k_row_stride < d_qk || v_row_stride < d_v) return IC_ERR_INVALID_ARG;
    const size_t need = ic_sparse_attn_workspace_size(r, k, Hq, d_qk, d_v, dt);
    if (!ws_ok(ws, ws_bytes, need)) return IC_ERR_WORKSPACE;
    if (rows_empty(r)) return IC_OK;
    if (!q || !kmat || !vmat || !idx || !out) return IC_ERR_INVALID_ARG;
    return run_attn(q, kmat, k_row_stride, vmat, v_row_stride, idx, k, dt, r, Hq, d_qk, d_v, scale,
                    out, status_of(ws), scratch_of(ws), ws_bytes - IC_STATUS_BYTES,
                    (cudaStream_t)stream);
}

size_t ic_workspace_size(const ic_stack_shape* sh) {
    if (sh == nullptr) return 0;
    const ic_rows& r = sh->rows;
    // top-k and attention run one after the other: they share the scratch region
    const size_t tail = std::max(align_up(attn_scratch(r, sh->k, sh->Hq, sh->d_qk, sh->d_v, sh->attn_dtype)),
                                 align_up(topk_multi_scratch_bytes(r, sh->k)));
    return IC_STATUS_BYTES + align_up(scores_bytes(r)) + tail;
}

ic_status ic_layer_stack_forward(const char* pattern, int n_layers, const ic_layer_io* layers,
                                 const ic_stack_shape* sh, int32_t* idx_buf,
                                 int32_t* const* idx_out, void* ws, size_t ws_bytes,
                                 void* stream) {
    if (pattern == nullptr || n_layers < 0) return IC_ERR_PATTERN;
    if (strlen(pattern) != (size_t)n_layers) return IC_ERR_PATTERN;
    for (int l = 0; l < n_layers; ++l)
        if (pattern[l] != 'F' && pattern[l] != 'S') return IC_ERR_PATTERN;
    if (n_layers > 0 && pattern[0] != 'F') return IC_ERR_PATTERN;
    if (sh == nullptr || (n_layers > 0 && layers == nullptr)) return IC_ERR_INVALID_ARG;
    const ic_rows r = sh->rows;
    if (!rows_ok(r) || !indexer_args_ok(sh->idx_dtype, sh->H_I, sh->d_I) ||
        !attn_args_ok(sh->attn_dtype, sh->Hq, sh->d_qk, sh->d_v, sh->k))
        return IC_ERR_INVALID_ARG;
    if (sh->k_row_stride < sh->d_qk || sh->v_row_stride < sh->d_v) return IC_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, ic_workspace_size(sh))) return IC_ERR_WORKSPACE;
    if (rows_empty(r) || n_layers == 0) return IC_OK;
    if (idx_buf == nullptr) return IC_ERR_INVALID_ARG;
    // validate every layer's pointers before launching anything
    for (int l = 0; l < n_layers; ++l) {
        const ic_layer_io& L = layers[l];
        if (!L.q || !L.kmat || !L.vmat || !L.out) return IC_ERR_INVALID_ARG;
        if (pattern[l] == 'F') {
            if (!L.q_idx || !L.w || !L.k_idx) return IC_ERR_INVALID_ARG;
            const bool fp8 = sh->idx_dtype == IC_FP8_E4M3;
            if (fp8 != (L.q_scale != nullptr) || fp8 != (L.k_scale != nullptr))
                return IC_ERR_INVALID_ARG;
        }
    }
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t* status = status_of(ws);
    float* scores = reinterpret_cast<float*>(scratch_of(ws));
    const int64_t ld = ((int64_t)r.T + 3) / 4 * 4;
    char* attn_ws = scratch_of(ws) + align_up(scores_bytes(r));
    const size_t attn_ws_bytes = ws_bytes - IC_STATUS_BYTES - align_up(scores_bytes(r));
    const size_t idx_bytes = (size_t)r.B * r.Lq * sh->k * sizeof(int32_t);

    for (int l = 0; l < n_layers; ++l) {
        const ic_layer_io& L = layers[l];
        if (pattern[l] == 'F') {  // the one conditional branch of IndexCache
            const ic_status st = run_select(L.q_idx, L.q_scale, L.w, L.k_idx, L.k_scale,
                                            sh->idx_dtype, r, sh->H_I, sh->d_I, sh->k, idx_buf,
                                            scores, ld, status, attn_ws, attn_ws_bytes, s);
            if (st != IC_OK) return st;
        }
        ic_status st = run_attn(L.q, L.kmat, sh->k_row_stride, L.vmat, sh->v_row_stride, idx_buf,
                                sh->k, sh->attn_dtype, r, sh->Hq, sh->d_qk, sh->d_v, sh->scale,
                                L.out, status, attn_ws, attn_ws_bytes, s);
        if (st != IC_OK) return st;
        if (idx_out != nullptr && idx_out[l] != nullptr) {
            if (cudaMemcpyAsync(idx_out[l], idx_buf, idx_bytes, cudaMemcpyDeviceToDevice, s) !=
                cudaSuccess)
                return cuda_error("api");
        }
    }
    return IC_OK;
}

// ------------------------------------------------------------------ paged / varlen
ic_status ic_indexer_scores_paged(const void* q_idx, const float* q_scale, const float* w,
                                  const void* k_pages, const float* k_scale_pages, ic_dtype dt,
                                  const ic_paged_rows* pr, int H_I, int d_I, float* scores,
                                  int64_t ld_scores, void* ws, size_t ws_bytes, void* stream) {
    if (!paged_ok(pr, true) || !indexer_args_ok(dt, H_I, d_I)) return IC_ERR_INVALID_ARG;
    if (!indexer_tc_supported(dt, H_I, d_I)) return IC_ERR_UNSUPPORTED;
    if (ld_scores < pr->T_max || ld_scores % 4 != 0) return IC_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, IC_STATUS_BYTES)) return IC_ERR_WORKSPACE;
    if (pr->B == 0) return IC_OK;
    if (!q_idx || !w || !k_pages || !scores) return IC_ERR_INVALID_ARG;
    if (dt == IC_FP8_E4M3 && (!q_scale || !k_scale_pages)) return IC_ERR_INVALID_ARG;
    if (dt != IC_FP8_E4M3 && (q_scale || k_scale_pages)) return IC_ERR_INVALID_ARG;
    return launch_indexer_tc_paged(q_idx, q_scale, w, k_pages, k_scale_pages, dt, *pr, H_I, d_I,
                                   scores, ld_scores, status_of(ws), (cudaStream_t)stream);
}

size_t ic_indexer_topk_paged_workspace_size(const ic_paged_rows* pr, int k) {
    (void)k;
    if (pr == nullptr) return IC_STATUS_BYTES;
    return IC_STATUS_BYTES + align_up(scores_bytes(plan_rows(pr)));
}

ic_status ic_indexer_topk_paged(const void* q_idx, const float* q_scale, const float* w,
                                const void* k_pages, const float* k_scale_pages, ic_dtype dt,
                                const ic_paged_rows* pr, int H_I, int d_I, int k, int32_t* idx,
                                void* ws, size_t ws_bytes, void* stream) {
    if (!paged_ok(pr, true) || !indexer_args_ok(dt, H_I, d_I) || k < 1 || k > 16384)
        return IC_ERR_INVALID_ARG;
    if (!indexer_tc_supported(dt, H_I, d_I)) return IC_ERR_UNSUPPORTED;
    if (!ws_ok(ws, ws_bytes, ic_indexer_topk_paged_workspace_size(pr, k))) return IC_ERR_WORKSPACE;
    if (pr->B == 0) return IC_OK;
    if (!q_idx || !w || !k_pages || !idx) return IC_ERR_INVALID_ARG;
    if (dt == IC_FP8_E4M3 && (!q_scale || !k_scale_pages)) return IC_ERR_INVALID_ARG;
    if (dt != IC_FP8_E4M3 && (q_scale || k_scale_pages)) return IC_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const ic_rows r = plan_rows(pr);
    if (select_fused_applies(dt, H_I, d_I, r, k)) {
        const ic_status st = launch_select_fused_paged(q_idx, q_scale, w, k_pages, k_scale_pages,
                                                       dt, *pr, H_I, k, idx, status_of(ws), s);
        if (st != IC_ERR_UNSUPPORTED) return st;
    }
    float* scores = reinterpret_cast<float*>(scratch_of(ws));
    const int64_t ld = ((int64_t)r.T + 3) / 4 * 4;
    const ic_status st = launch_indexer_tc_paged(q_idx, q_scale, w, k_pages, k_scale_pages, dt, *pr,
                                                 H_I, d_I, scores, ld, status_of(ws), s);
    if (st != IC_OK) return st;
    return run_topk_varlen(scores, ld, pr, k, idx, s);
}

size_t ic_topk_varlen_workspace_size(const ic_paged_rows* pr, int k) {
    (void)pr; (void)k;
    return IC_STATUS_BYTES;
}

ic_status ic_topk_varlen(const float* scores, int64_t ld_scores, const ic_paged_rows* pr, int k,
                         int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
    if (!paged_ok(pr, false) || k < 1 || k > 16384) return IC_ERR_INVALID_ARG;
    if (ld_scores < pr->T_max || ld_scores % 4 != 0) return IC_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, ic_topk_varlen_workspace_size(pr, k))) return IC_ERR_WORKSPACE;
    if (pr->B == 0) return IC_OK;
    if (!scores || !idx) return IC_ERR_INVALID_ARG;
    return run_topk_varlen(scores, ld_scores, pr, k, idx, (cudaStream_t)stream);
}

size_t ic_sparse_attn_paged_workspace_size(const ic_paged_rows* pr, int k) {
    if (pr == nullptr || k < 1) return IC_STATUS_BYTES;
    return IC_STATUS_BYTES + align_up(attn_tc_scratch_bytes(plan_rows(pr), k));
}

ic_status ic_sparse_attn_paged(const void* q, const void* kv_pages, const int32_t* idx, int k,
                               const ic_paged_rows* pr, float scale, void* out, void* ws,
                               size_t ws_bytes, void* stream) {
    if (!paged_ok(pr, true) || k < 1 || k > 16384) return IC_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, ic_sparse_attn_paged_workspace_size(pr, k))) return IC_ERR_WORKSPACE;
    if (pr->B == 0) return IC_OK;
    if (!q || !kv_pages || !idx || !out) return IC_ERR_INVALID_ARG;
    return launch_attn_tc_paged(q, kv_pages, idx, k, *pr, scale, out, status_of(ws),
                                scratch_of(ws), ws_bytes - IC_STATUS_BYTES, (cudaStream_t)stream);
}

size_t ic_paged_workspace_size(const ic_stack_shape* sh, const ic_paged_rows* pr) {
    if (sh == nullptr || pr == nullptr) return 0;
    const ic_rows r = plan_rows(pr);
    return IC_STATUS_BYTES + align_up(scores_bytes(r)) + align_up(attn_tc_scratch_bytes(r, sh->k));
}

ic_status ic_layer_stack_forward_paged(const char* pattern, int n_layers, const ic_layer_io* layers,
                                       const ic_stack_shape* sh, const ic_paged_rows* pr,
                                       int32_t* idx_buf, int32_t* const* idx_out, void* ws,
                                       size_t ws_bytes, void* stream) {
    if (pattern == nullptr || n_layers < 0) return IC_ERR_PATTERN;
    if (strlen(pattern) != (size_t)n_layers) return IC_ERR_PATTERN;
    for (int l = 0; l < n_layers; ++l)
        if (pattern[l] != 'F' && pattern[l] != 'S') return IC_ERR_PATTERN;
    if (n_layers > 0 && pattern[0] != 'F') return IC_ERR_PATTERN;
    if (sh == nullptr || (n_layers > 0 && layers == nullptr)) return IC_ERR_INVALID_ARG;
    if (!paged_ok(pr, true) || sh->k < 1 || sh->k > 16384) return IC_ERR_INVALID_ARG;
    if (!latent_tc_shape(sh)) return IC_ERR_UNSUPPORTED;
    if (!ws_ok(ws, ws_bytes, ic_paged_workspace_size(sh, pr))) return IC_ERR_WORKSPACE;
    if (pr->B == 0 || n_layers == 0) return IC_OK;
    if (idx_buf == nullptr) return IC_ERR_INVALID_ARG;
    for (int l = 0; l < n_layers; ++l) {
        const ic_layer_io& L = layers[l];
        if (!L.q || !L.kmat || !L.out || (L.vmat && L.vmat != L.kmat)) return IC_ERR_INVALID_ARG;
        if (pattern[l] == 'F') {
            if (!L.q_idx || !L.w || !L.k_idx) return IC_ERR_INVALID_ARG;
            const bool fp8 = sh->idx_dtype == IC_FP8_E4M3;
            if (fp8 != (L.q_scale != nullptr) || fp8 != (L.k_scale != nullptr))
                return IC_ERR_INVALID_ARG;
        }
    }
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t* status = status_of(ws);
    const ic_rows r = plan_rows(pr);
    float* scores = reinterpret_cast<float*>(scratch_of(ws));
    const int64_t ld = ((int64_t)r.T + 3) / 4 * 4;
    char* attn_ws = scratch_of(ws) + align_up(scores_bytes(r));
    const size_t attn_ws_bytes = ws_bytes - IC_STATUS_BYTES - align_up(scores_bytes(r));
    const size_t idx_bytes = (size_t)pr->B * pr->Lq * sh->k * sizeof(int32_t);
    for (int l = 0; l < n_layers; ++l) {
        const ic_layer_io& L = layers[l];
        if (pattern[l] == 'F') {  // the one conditional branch of IndexCache
            ic_status st = IC_ERR_UNSUPPORTED;
            if (select_fused_applies(sh->idx_dtype, sh->H_I, sh->d_I, r, sh->k))
                st = launch_select_fused_paged(L.q_idx, L.q_scale, L.w, L.k_idx, L.k_scale,
                                               sh->idx_dtype, *pr, sh->H_I, sh->k, idx_buf, status,
                                               s);
            if (st == IC_ERR_UNSUPPORTED) {
                st = launch_indexer_tc_paged(L.q_idx, L.q_scale, L.w, L.k_idx, L.k_scale,
                                             sh->idx_dtype, *pr, sh->H_I, sh->d_I, scores, ld,
                                             status, s);
                if (st != IC_OK) return st;
                st = run_topk_varlen(scores, ld, pr, sh->k, idx_buf, s);
            }
            if (st != IC_OK) return st;
        }
        ic_status st = launch_attn_tc_paged(L.q, L.kmat, idx_buf, sh->k, *pr, sh->scale, L.out,
                                            status, attn_ws, attn_ws_bytes, s);
        if (st != IC_OK) return st;
        if (idx_out != nullptr && idx_out[l] != nullptr) {
            if (cudaMemcpyAsync(idx_out[l], idx_buf, idx_bytes, cudaMemcpyDeviceToDevice, s) !=
                cudaSuccess)
                return cuda_error("api");
        }
    }
    return IC_OK;
}

}  // extern "C"
