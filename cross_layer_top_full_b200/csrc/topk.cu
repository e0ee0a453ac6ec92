// topk.cu -- per-row top-k of the indexer scores by radix select (one CTA
// per row; the many-row path of prefill).  topk_multi.cu holds the path for
// few long rows (decode), which spreads each row over many CTAs.
//
// DSA keeps the k most relevant keys per query (IndexCache summary, es page,
// section 1).  Row t keeps the min(k, t+1) candidates s <= t with the largest
// score; equal scores go to the smaller position and -0.0 counts as +0.0; the
// kept positions are written in ascending order and padded with -1.
//
// Method: each float becomes an order-preserving 32-bit key (flip all bits of
// negatives, set the sign bit of non-negatives; -0.0 is first mapped to
// +0.0).  Four 8-bit radix passes, most significant digit first, find the
// key tau of the k-th largest element and how many elements equal to tau
// must be kept ("need").  A final pass in position order keeps every key >
// tau and the first `need` keys == tau, which is exactly the smaller-position
// tie-break, and writes them with a block-wide prefix count, so the output is
// ascending without a sort.
//
// A row whose keys fit in shared memory is read from HBM once; longer rows
// are re-read (from L2 in practice) on every pass.  Histograms use
// warp-aggregated shared-memory atomics (__match_any_sync) so clustered
// digits do not serialise.
#include "topk_common.cuh"

namespace ic {
namespace {

constexpr int NT = 512;              // threads per CTA
constexpr int SMEM_KEYS_MAX = 40960; // keys cached in shared memory (160 KB)

__global__ void __launch_bounds__(NT)
topk_radix_kernel(const float* __restrict__ scores, int64_t ld, int Lq, int q_start, int k,
                  int32_t* __restrict__ idx, int cache_keys) {
    const int64_t row = blockIdx.x;
    const int i = (int)(row % Lq);
    const int t = q_start + i;
    extern __shared__ uint32_t keys_s[];
    __shared__ SelectState<NT / 32> st;
    select_row<NT>(scores + row * ld, t + 1, k, idx + row * (int64_t)k, keys_s, cache_keys, st);
}

}  // namespace

ic_status launch_topk_rows(const float* scores, int64_t ld, ic_rows r, int k, int32_t* idx,
                           cudaStream_t s) {
    const int n_max = r.q_start + r.Lq;  // candidates of the last row
    const int cache = n_max <= SMEM_KEYS_MAX ? n_max : 0;
    const size_t smem = (size_t)cache * sizeof(uint32_t);
    // the default dynamic limit leaves room for the static SelectState: opt in
    // whenever static + dynamic could pass 48 KB
    if (smem + sizeof(SelectState<NT / 32>) > 48 * 1024) {
        if (cudaFuncSetAttribute(topk_radix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return cuda_error("topk");
    }
    const int64_t rows = (int64_t)r.B * r.Lq;
    topk_radix_kernel<<<(unsigned)rows, NT, smem, s>>>(scores, ld, r.Lq, r.q_start, k, idx, cache);
    count_launch(IC_LK_TOPK);
    return last_launch_status();
}

}  // namespace ic
