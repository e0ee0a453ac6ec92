// indexer_simt.cu -- lightning-indexer scores on the CUDA cores.
//
// Computes scores[b,i,s] = sum_h w[b,i,h] * max(0, q_I[b,i,h,:] . k_I[b,s,:])
// for s <= t = q_start + i (the indexer scores every preceding token of each
// query: IndexCache summary, es page, section 1 "El Problema").  This is the
// exact-float32 path (float32 operands have no exact tensor-core kind) and the
// path for shapes the tensor-core kernel does not cover.  The tensor-core
// kernel is in indexer_tc.cu.
//
// Work split: one CTA = one query row x 128 consecutive keys, one thread per
// key.  The row's q_I (H_I x d_I) and w sit in shared memory as float; the key
// tile is staged transposed (d-major) so thread s reads column s without bank
// conflicts while q_I is a broadcast.
#include "common.cuh"

namespace ic {
namespace {

constexpr int KT = 128;  // keys per CTA

template <typename T>
__global__ void __launch_bounds__(KT)
indexer_simt_kernel(const T* __restrict__ q_idx, const float* __restrict__ q_scale,
                    const float* __restrict__ w, const T* __restrict__ k_idx,
                    const float* __restrict__ k_scale, int Lq, int q_start, int T_keys, int H,
                    int d, float* __restrict__ scores, int64_t ld) {
    const int key_tile = blockIdx.y;
    const int b = blockIdx.x / Lq;
    const int i = blockIdx.x - b * Lq;
    const int t = q_start + i;
    const int s0 = key_tile * KT;
    if (s0 > t) return;  // whole tile is above the causal diagonal

    extern __shared__ float smem[];
    float* q_s = smem;              // [H][d]
    float* w_s = q_s + H * d;       // [H]
    float* k_s = w_s + H;           // [d][KT] (transposed)

    const int64_t qrow = (int64_t)b * Lq + i;
    const T* qp = q_idx + qrow * H * d;
    for (int e = threadIdx.x; e < H * d; e += KT) q_s[e] = load_as_float(qp + e);
    for (int h = threadIdx.x; h < H; h += KT) w_s[h] = w[qrow * H + h];

    const int n_keys = min(KT, t + 1 - s0);
    const T* kp = k_idx + ((int64_t)b * T_keys + s0) * d;
    for (int e = threadIdx.x; e < n_keys * d; e += KT) {
        const int s = e / d, c = e - s * d;
        k_s[c * KT + s] = load_as_float(kp + e);
    }
    __syncthreads();

    const int s = threadIdx.x;
    if (s >= n_keys) return;
    float acc = 0.f;
    for (int h = 0; h < H; ++h) {
        const float* qh = q_s + h * d;
        float dot = 0.f;
        for (int c = 0; c < d; ++c) dot = fmaf(qh[c], k_s[c * KT + s], dot);
        acc = fmaf(w_s[h], fmaxf(dot, 0.f), acc);
    }
    if (q_scale != nullptr) acc *= q_scale[qrow] * k_scale[(int64_t)b * T_keys + s0 + s];
    scores[qrow * ld + s0 + s] = acc;
}

template <typename T>
ic_status launch_typed(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                       const float* k_scale, ic_rows r, int H, int d, float* scores, int64_t ld,
                       cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)H * d + H + (size_t)d * KT);
    auto kern = indexer_simt_kernel<T>;
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return cuda_error("indexer_simt");
    }
    const int last_t = r.q_start + r.Lq - 1;
    if (ceil_div(last_t + 1, KT) > 65535) return IC_ERR_UNSUPPORTED;
    dim3 grid((unsigned)((int64_t)r.B * r.Lq), ceil_div(last_t + 1, KT));
    kern<<<grid, KT, smem, s>>>(static_cast<const T*>(q_idx), q_scale, w,
                                static_cast<const T*>(k_idx), k_scale, r.Lq, r.q_start, r.T, H, d,
                                scores, ld);
    count_launch(IC_LK_INDEXER);
    return last_launch_status();
}

}  // namespace

ic_status launch_indexer_simt(const void* q_idx, const float* q_scale, const float* w,
                              const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r,
                              int H_I, int d_I, float* scores, int64_t ld, cudaStream_t s) {
    // shared memory: q row + weights + transposed key tile must fit one CTA
    if ((size_t)H_I * d_I + H_I + (size_t)d_I * KT > 56 * 1024) return IC_ERR_UNSUPPORTED;
    switch (dt) {
        case IC_F32:
            return launch_typed<float>(q_idx, nullptr, w, k_idx, nullptr, r, H_I, d_I, scores, ld, s);
        case IC_BF16:
            return launch_typed<__nv_bfloat16>(q_idx, nullptr, w, k_idx, nullptr, r, H_I, d_I,
                                               scores, ld, s);
        case IC_FP8_E4M3:
            return launch_typed<__nv_fp8_e4m3>(q_idx, q_scale, w, k_idx, k_scale, r, H_I, d_I,
                                               scores, ld, s);
    }
    return IC_ERR_UNSUPPORTED;
}

}  // namespace ic
