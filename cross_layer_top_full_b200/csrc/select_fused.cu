// select_fused.cu -- decode key selection in ONE kernel: the lightning
// indexer's scores of a decode row are computed on the tensor cores and kept
// in shared memory, and the row's exact top-k is taken from there; no score
// row reaches global memory.
//
// DSA selects, per query, the k keys its lightning indexer scores highest
// (IndexCache summary, es page, section 1 "El Problema"); an F layer of
// IndexCache runs exactly this and caches the result (es page, section 2).
// In decode the indexer is a scan of every cached key (HBM-bound) and its
// score row is short-lived: this kernel never writes it out.
//
// One thread-block cluster per query row (CL CTAs, 1..16).  CTA r owns the
// key segment [r*seg, (r+1)*seg) of the row (seg a multiple of the 128-key
// tile):
//   1. indexer pipeline (indexer_pipeline.cuh) over the segment's key tiles,
//      every score written into shared memory as an order-preserving key;
//   2. cluster_select (cluster_select.cuh): the exact top-k of the row from
//      the CL cached segments, with cluster barriers only.
// Dense keys, or paged keys with per-sequence lengths.
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "cluster_select.cuh"
#include "indexer_pipeline.cuh"

namespace ic {
namespace {

using namespace idx;
using csel::ClusterSmem;

constexpr int CL_MAX = 16;

// shared memory for the key-tile ring and query block: 5 FP8 or 3 bf16 stages
template <bool FP8>
constexpr int budget() { return FP8 ? 90 * 1024 : 114 * 1024; }

template <int H, bool FP8>
using FusedCfg = Cfg<H, 1, FP8, budget<FP8>()>;

constexpr size_t kSmemMax = 232448;   // dynamic shared memory per CTA (227 KB)

// the cluster-select state follows the pipeline's region on a 16-byte boundary
template <int H, bool FP8>
constexpr size_t select_offset() {
    return (pipeline_smem_bytes<FusedCfg<H, FP8>, H>() + 15) / 16 * 16;
}

template <int H, bool FP8>
constexpr size_t fixed_smem() {
    return 1024 + select_offset<H, FP8>() + sizeof(ClusterSmem<N_THREADS / 32>);
}

// Order keys of the segment [s0, s1) of the row, in shared memory.
struct KeySink {
    uint32_t* keys;
    int s0, s1;
    __device__ __forceinline__ void put(int, int, int s, float v) const {
        if (s >= s0 && s < s1) keys[s - s0] = order_key(v);
    }
};

template <int H, bool FP8>
__global__ void __launch_bounds__(N_THREADS, 1)
select_fused_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                    const float* __restrict__ w, const float* __restrict__ q_scale,
                    const float* __restrict__ k_scale, int Lq, int q_start, int T, Paging pg, int k,
                    int32_t* __restrict__ idx, uint32_t* status) {
    using C = FusedCfg<H, FP8>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    ClusterSmem<N_THREADS / 32>& S =
        *reinterpret_cast<ClusterSmem<N_THREADS / 32>*>(smem + select_offset<H, FP8>());
    uint32_t* keys = reinterpret_cast<uint32_t*>(&S + 1);

    // No early trigger: the attention kernel that follows launches when this
    // grid has finished (measured faster on the 32-sequence decode step,
    // 579 -> 572 us, than letting it start beside the selection).
    pdl_wait();
    const uint32_t CL = csel::cluster_ctas();
    const uint32_t rank = csel::cta_rank();
    const int64_t row = blockIdx.x / CL;
    const int b = (int)(row / Lq), i = (int)(row % Lq);
    int qs, Tb;
    const bool seq_ok = seq_extent(pg, b, Lq, q_start, T, qs, Tb);
    if (!seq_ok && rank == 0 && threadIdx.x == 0) flag_status(status, IC_DEV_INDEX_RANGE);
    const int n = seq_ok ? qs + i + 1 : 0;
    int32_t* dst = idx + row * (int64_t)k;
    if (n <= k) {  // every candidate is kept: no score is needed (same in every CTA)
        if (rank == 0)
            for (int j = threadIdx.x; j < k; j += N_THREADS) dst[j] = j < n ? j : -1;
        return;
    }
    const int seg = ((n + (int)CL - 1) / (int)CL + BM - 1) / BM * BM;
    const int s0 = min(n, (int)rank * seg);
    const int s1 = min(n, s0 + seg);
    const int m = s1 - s0;
    SingleSched sched;
    sched.item = Item{b, i, s0 / BM, (s1 + BM - 1) / BM, qs, Tb};
    sched.has = m > 0;
    const KeySink sink{keys, s0, s1};
    indexer_pipeline<H, 1, FP8, C, false>(&map_k, &map_q, smem, w, q_scale, k_scale, Lq, T, pg,
                                          sched, sink, status);
    __syncthreads();   // the segment's keys are complete
    csel::cluster_select<N_THREADS>(S, keys, m, s0, k, dst, CL, rank);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool make_map(CUtensorMap* map, const void* base, int64_t rows, bool fp8, int box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const int esz = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)D_I, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D_I * esz};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_total() {
    int n = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <int H, bool FP8>
size_t seg_capacity() {
    return (kSmemMax - fixed_smem<H, FP8>()) / sizeof(uint32_t) / BM * BM;
}

// Co-resident clusters of size cl for this kernel (0 if none fits).
template <int H, bool FP8>
int active_clusters(int cl, size_t smem) {
    auto kern = select_fused_kernel<H, FP8>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cl, 1, 1);
    cfg.blockDim = dim3(N_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

// Cluster size: the one that minimises (waves of clusters) x (keys per CTA),
// among the sizes whose segment fits in shared memory.  0 if none does.
template <int H, bool FP8>
int choose_cluster_uncached(int64_t rows, int n_max, size_t& smem_out) {
    auto kern = select_fused_kernel<H, FP8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    const size_t cap = seg_capacity<H, FP8>();
    int best = 0;
    double best_cost = 1e300;
    for (int cl = 1; cl <= CL_MAX; cl *= 2) {
        const int64_t seg = ((n_max + cl - 1) / cl + BM - 1) / BM * BM;
        if ((size_t)seg > cap) continue;
        const size_t smem = fixed_smem<H, FP8>() + (size_t)seg * sizeof(uint32_t);
        const int act = active_clusters<H, FP8>(cl, smem);
        if (act <= 0) continue;
        const double cost = (double)((rows + act - 1) / act) * (double)seg;
        if (cost < best_cost * 0.999) {
            best_cost = cost;
            best = cl;
            smem_out = smem;
        }
    }
    return best;
}

// The same, one answer per (device, rows, n_max): the occupancy queries cost
// host time on every launch otherwise.
template <int H, bool FP8>
int choose_cluster(int64_t rows, int n_max, size_t& smem_out) {
    int dev = 0;
    cudaGetDevice(&dev);
    static std::mutex mu;
    static std::map<std::tuple<int, int64_t, int>, std::pair<int, size_t>> cache;
    const auto key = std::make_tuple(dev, rows, n_max);
    {
        std::lock_guard<std::mutex> lock(mu);
        const auto it = cache.find(key);
        if (it != cache.end()) {
            smem_out = it->second.second;
            return it->second.first;
        }
    }
    size_t smem = 0;
    const int cl = choose_cluster_uncached<H, FP8>(rows, n_max, smem);
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = std::make_pair(cl, smem);
    smem_out = smem;
    return cl;
}

template <int H, bool FP8>
ic_status launch_h(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                   const float* k_scale, ic_rows r, const Paging& pg, int64_t key_rows, int k,
                   int32_t* idx, uint32_t* status, cudaStream_t s) {
    using C = FusedCfg<H, FP8>;
    auto kern = select_fused_kernel<H, FP8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return cuda_error("select_fused");
    const int64_t rows = (int64_t)r.B * r.Lq;
    size_t smem = 0;
    const int cl = choose_cluster<H, FP8>(rows, r.q_start + r.Lq, smem);
    if (cl == 0) return IC_ERR_UNSUPPORTED;
    CUtensorMap map_k, map_q;
    if (!make_map(&map_k, k_idx, key_rows, FP8, BM)) return cuda_error("select_fused");
    if (!make_map(&map_q, q_idx, rows * H, FP8, C::N)) return cuda_error("select_fused");
    if (launch_ex(kern, dim3((unsigned)(rows * cl)), dim3(N_THREADS), smem, s, pdl_rows(rows),
                  (unsigned)cl, map_k, map_q, w, q_scale, k_scale, r.Lq, r.q_start, r.T, pg, k, idx,
                  status) !=
        cudaSuccess)
        return cuda_error("select_fused");
    count_launch(IC_LK_SELECT);
    return last_launch_status();
}

ic_status launch_any(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                     const float* k_scale, ic_dtype dt, ic_rows r, int H_I, const Paging& pg,
                     int64_t key_rows, int k, int32_t* idx, uint32_t* status, cudaStream_t s) {
    if (((uintptr_t)q_idx & 15) || ((uintptr_t)k_idx & 15)) return IC_ERR_INVALID_ARG;
    const bool fp8 = dt == IC_FP8_E4M3;
#define IC_SEL_CASE(HH)                                                                           \
    case HH:                                                                                      \
        return fp8 ? launch_h<HH, true>(q_idx, q_scale, w, k_idx, k_scale, r, pg, key_rows, k,   \
                                        idx, status, s)                                           \
                   : launch_h<HH, false>(q_idx, q_scale, w, k_idx, k_scale, r, pg, key_rows, k,  \
                                         idx, status, s);
    switch (H_I) {
        IC_SEL_CASE(16)
        IC_SEL_CASE(32)
        IC_SEL_CASE(64)
        IC_SEL_CASE(128)
    }
#undef IC_SEL_CASE
    return IC_ERR_UNSUPPORTED;
}

}  // namespace

// Decode-shaped rows (few rows, each more candidates than fit one CTA's
// worth of work) on the tensor-core indexer shapes.
bool select_fused_applies(ic_dtype dt, int H_I, int d_I, ic_rows r, int k) {
    if (!indexer_tc_supported(dt, H_I, d_I)) return false;
    const int64_t rows = (int64_t)r.B * r.Lq;
    const int n_max = r.q_start + r.Lq;
    if (r.Lq > 2 || rows < 1 || rows > sm_total() || n_max <= k || n_max < 4096) return false;
    // (the largest head count leaves the least room for keys)
    const size_t cap = dt == IC_FP8_E4M3 ? seg_capacity<128, true>() : seg_capacity<128, false>();
    if ((size_t)((n_max + CL_MAX - 1) / CL_MAX) > cap) return false;
    // The fused kernel scans the keys with rows x CL CTAs, one row per
    // cluster.  With few rows the co-resident clusters of the largest sizes
    // run in more than one wave, and the stand-alone indexer on every SM
    // followed by the one-launch top-k is faster: measured on a B200, 8 rows
    // of 200K keys took 175 us fused against 55 + 38 us; 32 rows of 32K keys
    // 74 us fused against 61 + 26 us.  So: at least 16 rows, and CTAs on at
    // least 85 % of the SMs.
    if (rows < 16) return false;
    size_t smem = 0;
    int cl = 0;
    const bool fp8 = dt == IC_FP8_E4M3;
    switch (H_I) {
        case 16: cl = fp8 ? choose_cluster<16, true>(rows, n_max, smem) : choose_cluster<16, false>(rows, n_max, smem); break;
        case 32: cl = fp8 ? choose_cluster<32, true>(rows, n_max, smem) : choose_cluster<32, false>(rows, n_max, smem); break;
        case 64: cl = fp8 ? choose_cluster<64, true>(rows, n_max, smem) : choose_cluster<64, false>(rows, n_max, smem); break;
        case 128: cl = fp8 ? choose_cluster<128, true>(rows, n_max, smem) : choose_cluster<128, false>(rows, n_max, smem); break;
        default: return false;
    }
    return cl > 0 && rows * cl * 100 >= (int64_t)sm_total() * 85;
}

ic_status launch_select_fused(const void* q_idx, const float* q_scale, const float* w,
                              const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r,
                              int H_I, int k, int32_t* idx, uint32_t* status, cudaStream_t s) {
    const Paging dense = {nullptr, nullptr, 0, 0, 0, (int64_t)r.B * r.T};
    return launch_any(q_idx, q_scale, w, k_idx, k_scale, dt, r, H_I, dense, (int64_t)r.B * r.T, k,
                      idx, status, s);
}

ic_status launch_select_fused_paged(const void* q_idx, const float* q_scale, const float* w,
                                    const void* k_pages, const float* k_scale_pages, ic_dtype dt,
                                    const ic_paged_rows& pr, int H_I, int k, int32_t* idx,
                                    uint32_t* status, cudaStream_t s) {
    const int64_t key_rows = (int64_t)pr.num_pages * pr.page_size;
    const Paging pg = {pr.seq_lens, pr.block_table, pr.max_pages, pr.page_size, pr.T_max, key_rows};
    const ic_rows r = {pr.B, pr.Lq, pr.T_max - pr.Lq, pr.T_max};
    return launch_any(q_idx, q_scale, w, k_pages, k_scale_pages, dt, r, H_I, pg, key_rows, k, idx,
                      status, s);
}

}  // namespace ic
