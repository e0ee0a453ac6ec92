// indexer_tc.cu -- lightning-indexer scores to global memory on the tcgen05
// tensor cores (the pipeline itself is in indexer_pipeline.cuh).
//
// Persistent CTAs, one per SM; work item = (sequence b, group of NTOK query
// rows, chunk of key tiles), ordered heaviest group first and strided over
// the CTAs.  Key tiles above a group's last causal key are never loaded.
// Dense keys, or paged keys with per-sequence lengths (ic_paged_rows).
#include "indexer_pipeline.cuh"

namespace ic {
namespace {

using namespace idx;

template <int H, int NTOK, bool FP8>
__global__ void __launch_bounds__(N_THREADS, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                  const float* __restrict__ w, const float* __restrict__ q_scale,
                  const float* __restrict__ k_scale, float* __restrict__ scores, int64_t ld, int B,
                  int Lq, int q_start, int T, Work wk, Paging pg, uint32_t* status) {
    using C = Cfg<H, NTOK, FP8>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const PersistentSched sched(wk, B, Lq, q_start, T, pg, NTOK);
    const GlobalSink sink{scores, ld, Lq};
    indexer_pipeline<H, NTOK, FP8, C>(&map_k, &map_q, smem, w, q_scale, k_scale, Lq, T, pg, sched,
                                      sink, status);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2D map over a [rows, 128-element] row-major matrix, box = 128 bytes x box_rows,
// 128-byte swizzle (the UMMA K-major canonical layout).
bool make_map(CUtensorMap* map, const void* base, int64_t rows, bool fp8, int box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const int esz = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)D_I, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D_I * esz};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int H, int NTOK, bool FP8>
ic_status launch_cfg(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                     const float* k_scale, ic_rows r, float* scores, int64_t ld, uint32_t* status,
                     cudaStream_t s, const Paging& pg, int64_t key_rows) {
    using C = Cfg<H, NTOK, FP8>;
    CUtensorMap map_k, map_q;
    if (!make_map(&map_k, k_idx, key_rows, FP8, BM)) return cuda_error("indexer_tc");
    if (!make_map(&map_q, q_idx, (int64_t)r.B * r.Lq * H, FP8, C::N)) return cuda_error("indexer_tc");
    Work wk;
    wk.n_groups = ceil_div(r.Lq, NTOK);
    // dense: the last row's candidates; paged: the longest possible sequence
    const int max_tiles = ceil_div(r.q_start + r.Lq, BM);
    const int base_items = r.B * wk.n_groups;
    const int sms = num_sms();
    int split = 1;
    if (base_items < 2 * sms) split = ceil_div(2 * sms, base_items);
    wk.chunk_tiles = ceil_div(max_tiles, split);
    wk.n_chunks = ceil_div(max_tiles, wk.chunk_tiles);
    const int64_t items = (int64_t)base_items * wk.n_chunks;
    if (items > 0x7fffffff) return IC_ERR_UNSUPPORTED;
    wk.n_items = (int)items;
    const size_t smem = 1024 + pipeline_smem_bytes<C, H>();
    auto kern = indexer_tc_kernel<H, NTOK, FP8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return cuda_error("indexer_tc");
    const int grid = (int)std::min<int64_t>(items, sms);
    if (launch_ex(kern, dim3(grid), dim3(N_THREADS), smem, s, pdl_rows((int64_t)r.B * r.Lq), 0,
                  map_k, map_q, w, q_scale, k_scale, scores, ld, r.B, r.Lq, r.q_start, r.T, wk, pg,
                  status) != cudaSuccess)
        return cuda_error("indexer_tc");
    count_launch(IC_LK_INDEXER_TC);
    return last_launch_status();
}

template <int H, bool FP8>
ic_status launch_h(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                   const float* k_scale, ic_rows r, float* scores, int64_t ld, uint32_t* status,
                   cudaStream_t s, const Paging& pg, int64_t key_rows) {
    constexpr int NT_WIDE = 256 / H;
    if (r.Lq <= 2)  // decode: one token per accumulator, the scan is HBM-bound
        return launch_cfg<H, 1, FP8>(q_idx, q_scale, w, k_idx, k_scale, r, scores, ld, status, s,
                                     pg, key_rows);
    return launch_cfg<H, NT_WIDE, FP8>(q_idx, q_scale, w, k_idx, k_scale, r, scores, ld, status,
                                       s, pg, key_rows);
}

ic_status launch_any(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                     const float* k_scale, ic_dtype dt, ic_rows r, int H_I, float* scores,
                     int64_t ld, uint32_t* status, cudaStream_t s, const Paging& pg,
                     int64_t key_rows) {
    const bool fp8 = dt == IC_FP8_E4M3;
#define IC_IDX_CASE(HH)                                                                         \
    case HH:                                                                                    \
        return fp8 ? launch_h<HH, true>(q_idx, q_scale, w, k_idx, k_scale, r, scores, ld,      \
                                        status, s, pg, key_rows)                                \
                   : launch_h<HH, false>(q_idx, q_scale, w, k_idx, k_scale, r, scores, ld,     \
                                         status, s, pg, key_rows);
    switch (H_I) {
        IC_IDX_CASE(16)
        IC_IDX_CASE(32)
        IC_IDX_CASE(64)
        IC_IDX_CASE(128)
    }
#undef IC_IDX_CASE
    return IC_ERR_UNSUPPORTED;
}

}  // namespace

bool indexer_tc_supported(ic_dtype dt, int H_I, int d_I) {
    return (dt == IC_BF16 || dt == IC_FP8_E4M3) && d_I == D_I &&
           (H_I == 16 || H_I == 32 || H_I == 64 || H_I == 128);
}

ic_status launch_indexer_tc(const void* q_idx, const float* q_scale, const float* w,
                            const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r,
                            int H_I, int d_I, float* scores, int64_t ld, uint32_t* status,
                            cudaStream_t s) {
    if (!indexer_tc_supported(dt, H_I, d_I)) return IC_ERR_UNSUPPORTED;
    if (((uintptr_t)q_idx & 15) || ((uintptr_t)k_idx & 15)) return IC_ERR_INVALID_ARG;
    const Paging dense = {nullptr, nullptr, 0, 0, 0, (int64_t)r.B * r.T};
    return launch_any(q_idx, q_scale, w, k_idx, k_scale, dt, r, H_I, scores, ld, status, s, dense,
                      (int64_t)r.B * r.T);
}

ic_status launch_indexer_tc_paged(const void* q_idx, const float* q_scale, const float* w,
                                  const void* k_pages, const float* k_scale_pages, ic_dtype dt,
                                  const ic_paged_rows& pr, int H_I, int d_I, float* scores,
                                  int64_t ld, uint32_t* status, cudaStream_t s) {
    if (!indexer_tc_supported(dt, H_I, d_I)) return IC_ERR_UNSUPPORTED;
    if (((uintptr_t)q_idx & 15) || ((uintptr_t)k_pages & 15)) return IC_ERR_INVALID_ARG;
    const Paging pg = {pr.seq_lens, pr.block_table, pr.max_pages, pr.page_size, pr.T_max,
                       (int64_t)pr.num_pages * pr.page_size};
    // planning rows: every sequence as long as T_max
    const ic_rows r = {pr.B, pr.Lq, pr.T_max - pr.Lq, pr.T_max};
    return launch_any(q_idx, q_scale, w, k_pages, k_scale_pages, dt, r, H_I, scores, ld, status, s,
                      pg, (int64_t)pr.num_pages * pr.page_size);
}

}  // namespace ic
