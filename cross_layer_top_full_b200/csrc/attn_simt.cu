// attn_simt.cu -- sparse multi-query attention on the CUDA cores.
//
// For row (b,i), head h and the valid entries j of idx[b,i,:]:
//   p_j = softmax_j(scale * q[b,i,h,:d_qk] . K[b,j,:d_qk]);  out = sum_j p_j V[b,j,:d_v]
// (core attention over the k selected keys only, O(Lk): IndexCache summary,
// es page, section 1; de page, section 1).  This is the exact-float32 path and
// the path for shapes outside the tensor-core kernel (attn_tc.cu).
//
// One CTA = one query row x 4 heads, one warp per head.  Keys are taken 16
// at a time: the CTA stages the 16 selected K/V rows in shared memory as
// float; each lane owns a strided slice of d_qk / d_v, partial dot products
// are reduced across the warp, and the online softmax (running max m, sum l)
// rescales the lane's slice of the output.  An index outside [0, t] is never
// dereferenced: it is skipped and flagged in the status word.
#include "common.cuh"

namespace ic {
namespace {

constexpr int HEADS_PER_CTA = 4;
constexpr int KB = 16;          // keys per step
constexpr int MAXD = 576;       // largest d_qk / d_v
constexpr int PER_LANE = MAXD / 32;

template <typename T>
__global__ void __launch_bounds__(32 * HEADS_PER_CTA)
attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ kmat, int64_t ks,
                 const T* __restrict__ vmat, int64_t vs, const int32_t* __restrict__ idx, int k,
                 int Lq, int q_start, int T_keys, int Hq, int d_qk, int d_v, float scale,
                 T* __restrict__ out, uint32_t* status) {
    const int64_t row = blockIdx.x;
    const int b = (int)(row / Lq);
    const int i = (int)(row - (int64_t)b * Lq);
    const int t = q_start + i;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y * HEADS_PER_CTA + warp;
    const bool head_ok = h < Hq;

    extern __shared__ float sm[];
    float* k_s = sm;                   // [KB][d_qk]
    float* v_s = k_s + KB * d_qk;      // [KB][d_v]
    __shared__ int sel[KB];

    float qv[PER_LANE];
#pragma unroll
    for (int c = 0; c < PER_LANE; ++c) {
        const int d = lane + 32 * c;
        qv[c] = (head_ok && d < d_qk) ? load_as_float(q + (row * Hq + h) * d_qk + d) * scale : 0.f;
    }
    float o[PER_LANE];
#pragma unroll
    for (int c = 0; c < PER_LANE; ++c) o[c] = 0.f;
    float m = -INFINITY, l = 0.f;

    const int32_t* irow = idx + row * (int64_t)k;
    for (int base = 0; base < k; base += KB) {
        __syncthreads();  // previous step's tiles are consumed
        if (threadIdx.x < KB) {
            int j = base + threadIdx.x < k ? irow[base + threadIdx.x] : -1;
            if (j < -1 || j > t || j >= T_keys) {
                flag_status(status, IC_DEV_INDEX_RANGE);
                j = -1;
            }
            sel[threadIdx.x] = j;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < KB * d_qk; e += blockDim.x) {
            const int r = e / d_qk, c = e - r * d_qk;
            const int j = sel[r];
            k_s[e] = j >= 0 ? load_as_float(kmat + ((int64_t)b * T_keys + j) * ks + c) : 0.f;
        }
        for (int e = threadIdx.x; e < KB * d_v; e += blockDim.x) {
            const int r = e / d_v, c = e - r * d_v;
            const int j = sel[r];
            v_s[e] = j >= 0 ? load_as_float(vmat + ((int64_t)b * T_keys + j) * vs + c) : 0.f;
        }
        __syncthreads();
        if (!head_ok) continue;

        float logit[KB];
#pragma unroll
        for (int r = 0; r < KB; ++r) {
            float part = 0.f;
#pragma unroll
            for (int c = 0; c < PER_LANE; ++c) {
                const int d = lane + 32 * c;
                if (d < d_qk) part = fmaf(qv[c], k_s[r * d_qk + d], part);
            }
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
            logit[r] = sel[r] >= 0 ? part : -INFINITY;
        }
        float bm = m;
#pragma unroll
        for (int r = 0; r < KB; ++r) bm = fmaxf(bm, logit[r]);
        if (bm == -INFINITY) continue;  // no valid key yet
        const float corr = expf(m - bm);  // m = -inf on the first valid step -> 0
        l *= corr;
#pragma unroll
        for (int c = 0; c < PER_LANE; ++c) o[c] *= corr;
#pragma unroll
        for (int r = 0; r < KB; ++r) {
            const float p = expf(logit[r] - bm);
            l += p;
#pragma unroll
            for (int c = 0; c < PER_LANE; ++c) {
                const int d = lane + 32 * c;
                if (d < d_v) o[c] = fmaf(p, v_s[r * d_v + d], o[c]);
            }
        }
        m = bm;
    }
    if (!head_ok) return;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int c = 0; c < PER_LANE; ++c) {
        const int d = lane + 32 * c;
        if (d < d_v) store_from_float(out + (row * Hq + h) * d_v + d, o[c] * inv);
    }
}

template <typename T>
ic_status launch_typed(const void* q, const void* kmat, int64_t ks, const void* vmat, int64_t vs,
                       const int32_t* idx, int k, ic_rows r, int Hq, int d_qk, int d_v,
                       float scale, void* out, uint32_t* status, cudaStream_t s) {
    const size_t smem = sizeof(float) * (size_t)KB * (d_qk + d_v);
    auto kern = attn_simt_kernel<T>;
    // opt in to more than 48 KB whenever dynamic + static (sel[KB]) pass it
    if (smem + sizeof(int) * KB > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return cuda_error("attn_simt");
    }
    dim3 grid((unsigned)((int64_t)r.B * r.Lq), ceil_div(Hq, HEADS_PER_CTA));
    kern<<<grid, 32 * HEADS_PER_CTA, smem, s>>>(
        static_cast<const T*>(q), static_cast<const T*>(kmat), ks, static_cast<const T*>(vmat), vs,
        idx, k, r.Lq, r.q_start, r.T, Hq, d_qk, d_v, scale, static_cast<T*>(out), status);
    count_launch(IC_LK_ATTN);
    return last_launch_status();
}

}  // namespace

ic_status launch_attn_simt(const void* q, const void* kmat, int64_t ks, const void* vmat,
                           int64_t vs, const int32_t* idx, int k, ic_dtype dt, ic_rows r, int Hq,
                           int d_qk, int d_v, float scale, void* out, uint32_t* status,
                           cudaStream_t s) {
    if (d_qk > MAXD || d_v > MAXD) return IC_ERR_UNSUPPORTED;
    if (dt == IC_F32)
        return launch_typed<float>(q, kmat, ks, vmat, vs, idx, k, r, Hq, d_qk, d_v, scale, out,
                                   status, s);
    if (dt == IC_BF16)
        return launch_typed<__nv_bfloat16>(q, kmat, ks, vmat, vs, idx, k, r, Hq, d_qk, d_v, scale,
                                           out, status, s);
    return IC_ERR_UNSUPPORTED;
}

}  // namespace ic
