// topk.cu -- per-row top-k of the indexer scores by radix select.
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
// One CTA per row.  A row whose keys fit in shared memory is read from HBM
// once; longer rows are re-read (from L2 in practice) on every pass.
// Histograms use warp-aggregated shared-memory atomics (__match_any_sync) so
// clustered digits do not serialise.
#include "common.cuh"

namespace ic {
namespace {

constexpr int NT = 512;              // threads per CTA
constexpr int NW = NT / 32;
constexpr int SMEM_KEYS_MAX = 40960; // keys cached in shared memory (160 KB)

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelectState {
    uint32_t hist[256];
    uint32_t warp_cnt[2][NW];
    uint32_t prefix;      // digits chosen so far
    uint32_t need;        // elements equal to the final tau still to keep
};

// Pick the digit holding the need-th largest element: scan bins from 255
// down.  Executed by warp 0; lane L owns bins 255-8L .. 248-8L.
__device__ __forceinline__ void choose_digit(SelectState& st, int shift) {
    const int lane = threadIdx.x & 31;
    uint32_t c[8];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        c[j] = st.hist[255 - 8 * lane - j];
        sum += c[j];
    }
    // inclusive scan of the lane sums in descending-bin order
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const uint32_t need = st.need;
    const uint32_t hit = __ballot_sync(0xffffffffu, incl >= need);
    const int src = __ffs(hit) - 1;  // first lane reaching need (always exists)
    if (lane == src) {
        uint32_t before = incl - sum;  // elements in higher bins
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (before + c[j] >= need) {
                st.prefix = (st.prefix << 8) | (uint32_t)(255 - 8 * lane - j);
                st.need = need - before;
                break;
            }
            before += c[j];
        }
    }
    (void)shift;
}

__global__ void __launch_bounds__(NT)
topk_radix_kernel(const float* __restrict__ scores, int64_t ld, int Lq, int q_start, int k,
                  int32_t* __restrict__ idx, int cache_keys) {
    const int64_t row = blockIdx.x;
    const int i = (int)(row % Lq);
    const int t = q_start + i;
    const int n = t + 1;
    const float* src = scores + row * ld;
    int32_t* dst = idx + row * (int64_t)k;

    if (n <= k) {  // every candidate is kept
        for (int j = threadIdx.x; j < k; j += NT) dst[j] = j < n ? j : -1;
        return;
    }

    extern __shared__ uint32_t keys_s[];
    __shared__ SelectState st;
    const bool cached = n <= cache_keys;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) { st.prefix = 0; st.need = (uint32_t)k; }

    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int j = threadIdx.x; j < 256; j += NT) st.hist[j] = 0;
        __syncthreads();
        const uint32_t prefix = st.prefix;
        // round the loop up to whole warps so __match_any_sync sees full warps
        const int n_round = (n + 31) & ~31;
        for (int j = threadIdx.x; j < n_round; j += NT) {
            bool live = j < n;
            uint32_t key = 0;
            if (live) {
                if (pass == 0) {
                    key = order_key(src[j]);
                    if (cached) keys_s[j] = key;
                } else {
                    key = cached ? keys_s[j] : order_key(src[j]);
                }
                live = pass == 0 || (key >> (shift + 8)) == prefix;
            }
            const uint32_t digit = live ? ((key >> shift) & 255u) : 256u;
            const uint32_t peers = __match_any_sync(0xffffffffu, digit);
            if (live && lane == __ffs(peers) - 1) atomicAdd(&st.hist[digit], __popc(peers));
        }
        __syncthreads();
        if (warp == 0) choose_digit(st, shift);
        __syncthreads();
    }

    const uint32_t tau = st.prefix;
    const uint32_t need_eq = st.need;
    // Compaction in position order: keep key > tau, and key == tau while
    // fewer than need_eq equal keys precede it.
    uint32_t run_gt = 0, run_eq = 0;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int n_round = (n + NT - 1) / NT * NT;
    for (int base = 0; base < n_round; base += NT) {
        const int j = base + threadIdx.x;
        uint32_t key = 0;
        if (j < n) key = cached ? keys_s[j] : order_key(src[j]);
        const bool gt = j < n && key > tau;
        const bool eq = j < n && key == tau;
        const uint32_t bg = __ballot_sync(0xffffffffu, gt);
        const uint32_t be = __ballot_sync(0xffffffffu, eq);
        const int buf = (base / NT) & 1;
        if (lane == 0) { st.warp_cnt[buf][warp] = __popc(bg) | ((uint32_t)__popc(be) << 16); }
        __syncthreads();
        uint32_t pre_gt = 0, pre_eq = 0, tot_gt = 0, tot_eq = 0;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) {
            const uint32_t v = st.warp_cnt[buf][w2];
            if (w2 < warp) { pre_gt += v & 0xffffu; pre_eq += v >> 16; }
            tot_gt += v & 0xffffu;
            tot_eq += v >> 16;
        }
        const uint32_t gt_before = run_gt + pre_gt + __popc(bg & lt_mask);
        const uint32_t eq_before = run_eq + pre_eq + __popc(be & lt_mask);
        if (gt || (eq && eq_before < need_eq)) {
            dst[gt_before + min(eq_before, need_eq)] = j;
        }
        run_gt += tot_gt;
        run_eq += tot_eq;
        // warp_cnt is double-buffered, so one barrier per chunk suffices
    }
}

}  // namespace

ic_status launch_topk(const float* scores, int64_t ld, ic_rows r, int k, int32_t* idx,
                      cudaStream_t s) {
    const int n_max = r.q_start + r.Lq;  // candidates of the last row
    const int cache = n_max <= SMEM_KEYS_MAX ? n_max : 0;
    const size_t smem = (size_t)cache * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(topk_radix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return IC_ERR_CUDA;
    }
    const int64_t rows = (int64_t)r.B * r.Lq;
    topk_radix_kernel<<<(unsigned)rows, NT, smem, s>>>(scores, ld, r.Lq, r.q_start, k, idx, cache);
    count_launch(IC_LK_TOPK);
    return last_launch_status();
}

}  // namespace ic
