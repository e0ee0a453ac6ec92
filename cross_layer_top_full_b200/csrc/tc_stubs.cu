// tc_stubs.cu -- placeholders until the tensor-core kernels land.
#include "common.cuh"
namespace ic {
bool indexer_tc_supported(ic_dtype, int, int) { return false; }
ic_status launch_indexer_tc(const void*, const float*, const float*, const void*, const float*,
                            ic_dtype, ic_rows, int, int, float*, int64_t, uint32_t*, cudaStream_t) {
    return IC_ERR_UNSUPPORTED;
}
bool attn_tc_supported(const void*, const void*, int64_t, int64_t, ic_dtype, int, int, int) {
    return false;
}
size_t attn_tc_scratch_bytes(ic_rows, int) { return 0; }
ic_status launch_attn_tc(const void*, const void*, int64_t, const int32_t*, int, ic_rows, float,
                         void*, uint32_t*, void*, size_t, cudaStream_t) {
    return IC_ERR_UNSUPPORTED;
}
}  // namespace ic
