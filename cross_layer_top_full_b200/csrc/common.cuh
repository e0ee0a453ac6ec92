// common.cuh -- shared definitions of the IndexCache CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <utility>

#include "indexcache.h"

// Bits of the device status word at the start of every workspace.
#define IC_DEV_INDEX_RANGE 1u
#define IC_DEV_TIMEOUT 2u

// Launch kinds counted by ic_kernel_launches.
enum {
    IC_LK_ALL = 0, IC_LK_INDEXER = 1, IC_LK_TOPK = 2, IC_LK_ATTN = 3, IC_LK_COMBINE = 4,
    IC_LK_INDEXER_TC = 5, IC_LK_ATTN_TC = 6, IC_LK_SELECT = 7, IC_LK_KINDS = 8
};

namespace ic {

// Host: count one launch of a kind (also counted under IC_LK_ALL).
void count_launch(int kind);

// Host: map the last CUDA error to a status.
ic_status last_launch_status();
// Records the pending CUDA runtime error (or, for a failed driver call, the
// site alone) as this thread's last error text and returns IC_ERR_CUDA.
ic_status cuda_error(const char* where);
const char* tl_error_text();

// Programmatic dependent launch.  A kernel launched by launch_ex with `pdl`
// may begin while the previous kernel on its stream is still running:
//  - pdl_trigger(): this CTA lets the stream's next kernel launch (it does
//    once every CTA of this grid has triggered or exited).  A kernel that
//    allocates tensor memory triggers only after its allocation, so that a
//    dependent CTA placed beside it can never hold columns it still needs;
//  - pdl_wait(): returns once the previous kernel has completed and its
//    memory operations are visible.  Every kernel launched by launch_ex calls
//    it before its first global load or store.
// Both are no-ops in a kernel launched without the attribute.
#ifndef IC_PDL
#define IC_PDL 1
#endif
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Host: whether a call over `rows` query rows launches with programmatic
// stream serialization.  Few-row (decode) calls run dozens of short kernels
// per step, where the early launch removes most of each kernel boundary:
// measured on B200, 2199 -> 2125 us for the 48-layer decode step of 8
// sequences of 200K keys.  Many-row calls do not: the same early launch made
// the 8K prefill step 2% slower (26.28 -> 26.85 ms).  The cost appears only
// when the attention grid is launched while the previous kernel's CTAs
// drain, probably because its 2-CTA clusters are then placed on whichever
// SMs free up first rather than on neighbouring ones.
constexpr int64_t kPdlMaxRows = 256;
inline bool pdl_rows(int64_t rows) { return IC_PDL && rows <= kPdlMaxRows; }

// Host: launch `kern` on stream s, with programmatic stream serialization
// when `pdl` holds and, for cluster > 0, that many CTAs per cluster.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                      bool pdl, unsigned cluster, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    ++n;
    if (cluster > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

__device__ __forceinline__ void flag_status(uint32_t* status, uint32_t bit) {
    if (status) atomicOr(status, bit);
}

// Element loads of the supported storage types, as float.
__device__ __forceinline__ float load_as_float(const float* p) { return *p; }
__device__ __forceinline__ float load_as_float(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float load_as_float(const __nv_fp8_e4m3* p) { return float(*p); }

__device__ __forceinline__ void store_from_float(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_from_float(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

__host__ __device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace ic

// Internal launchers (one per kernel family).  `status` points at the
// device status word; `scratch` is call-specific workspace after it.
namespace ic {

ic_status launch_indexer_simt(const void* q_idx, const float* q_scale, const float* w,
                              const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r,
                              int H_I, int d_I, float* scores, int64_t ld, cudaStream_t s);

bool indexer_tc_supported(ic_dtype dt, int H_I, int d_I);
ic_status launch_indexer_tc(const void* q_idx, const float* q_scale, const float* w,
                            const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r,
                            int H_I, int d_I, float* scores, int64_t ld, uint32_t* status,
                            cudaStream_t s);

// seq_lens: nullptr (every row of sequence b has q_start + i + 1 candidates)
// or [B] per-sequence key counts (row i: seq_lens[b] - Lq + i + 1; r.T is
// then the upper bound T_max and r.q_start = T_max - Lq).
ic_status launch_topk_rows(const float* scores, int64_t ld, ic_rows r, int k, int32_t* idx,
                           cudaStream_t s, const int32_t* seq_lens = nullptr);
bool topk_cluster_applies(ic_rows r, int k);
ic_status launch_topk_cluster(const float* scores, int64_t ld, ic_rows r, int k, int32_t* idx,
                              cudaStream_t s, const int32_t* seq_lens = nullptr);
bool topk_multi_applies(ic_rows r, int k);
size_t topk_multi_scratch_bytes(ic_rows r, int k);
ic_status launch_topk_multi(const float* scores, int64_t ld, ic_rows r, int k, int32_t* idx,
                            void* scratch, cudaStream_t s);

ic_status launch_attn_simt(const void* q, const void* kmat, int64_t ks, const void* vmat,
                           int64_t vs, const int32_t* idx, int k, ic_dtype dt, ic_rows r, int Hq,
                           int d_qk, int d_v, float scale, void* out, uint32_t* status,
                           cudaStream_t s);

bool attn_tc_supported(const void* kmat, const void* vmat, int64_t ks, int64_t vs, ic_dtype dt,
                       int Hq, int d_qk, int d_v);
// max_units caps the split-k plan's units (rows x splits); the smallest
// split count is kept even above it, so callers with a fixed limit check
// attn_tc_units against it first.
constexpr int64_t kNoUnitLimit = INT64_MAX;
int64_t attn_tc_units(ic_rows r, int k, int64_t max_units = kNoUnitLimit);
size_t attn_tc_scratch_bytes(ic_rows r, int k, int64_t max_units = kNoUnitLimit);
ic_status launch_attn_tc(const void* q, const void* kv, int64_t ks, const int32_t* idx, int k,
                         ic_rows r, float scale, void* out, uint32_t* status, void* scratch,
                         size_t scratch_bytes, cudaStream_t s, int64_t max_units = kNoUnitLimit);

// Fused decode key selection (indexer scores kept in shared memory + top-k).
bool select_fused_applies(ic_dtype dt, int H_I, int d_I, ic_rows r, int k);
ic_status launch_select_fused(const void* q_idx, const float* q_scale, const float* w,
                              const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r,
                              int H_I, int k, int32_t* idx, uint32_t* status, cudaStream_t s);
ic_status launch_select_fused_paged(const void* q_idx, const float* q_scale, const float* w,
                                    const void* k_pages, const float* k_scale_pages, ic_dtype dt,
                                    const ic_paged_rows& pr, int H_I, int k, int32_t* idx,
                                    uint32_t* status, cudaStream_t s);

// Paged / variable-length variants (ic_paged_rows: per-sequence lengths and a
// block table; see include/indexcache.h).
ic_status launch_indexer_tc_paged(const void* q_idx, const float* q_scale, const float* w,
                                  const void* k_pages, const float* k_scale_pages, ic_dtype dt,
                                  const ic_paged_rows& pr, int H_I, int d_I, float* scores,
                                  int64_t ld, uint32_t* status, cudaStream_t s);
ic_status launch_attn_tc_paged(const void* q, const void* kv_pages, const int32_t* idx, int k,
                               const ic_paged_rows& pr, float scale, void* out, uint32_t* status,
                               void* scratch, size_t scratch_bytes, cudaStream_t s);

}  // namespace ic
