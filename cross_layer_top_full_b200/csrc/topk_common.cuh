// topk_common.cuh -- shared pieces of the top-k kernels: the order-preserving
// key of a float score and a block-wide radix select of one row.
//
// Top-k rule (DSA keeps the k most relevant keys per query; IndexCache
// summary, es page, section 1): row t keeps the min(k, t+1) candidates s <= t
// with the largest score, equal scores going to the smaller position and -0.0
// counting as +0.0; the kept positions are written ascending, -1 padded.
#pragma once

#include "common.cuh"

namespace ic {

// Candidates of score row `row` (= b*Lq + i): t + 1 with t = q_start + i,
// or with per-sequence lengths (seq_lens != nullptr) t = seq_lens[b] - Lq + i;
// a length outside [Lq, T_max] gives 0 candidates (an all -1 row).
__device__ __forceinline__ int row_candidates(int64_t row, int Lq, int q_start,
                                              const int32_t* __restrict__ seq_lens, int T_max) {
    const int i = (int)(row % Lq);
    if (seq_lens == nullptr) return q_start + i + 1;
    const int Tb = __ldg(seq_lens + row / Lq);
    return (Tb >= Lq && Tb <= T_max) ? Tb - Lq + i + 1 : 0;
}

// Histogram update of one warp: +1 at hist[digit] for every live lane.  A
// warp whose lanes all carry the same digit (clustered scores) adds 32 from
// one lane; otherwise each live lane adds its own 1 (shared-memory atomics
// resolve the few collisions of scattered digits).  Every lane of the warp
// must call it; dead lanes pass a digit no live lane can have.
__device__ __forceinline__ void warp_hist_add(uint32_t* hist, uint32_t digit, bool live) {
    const uint32_t d0 = __shfl_sync(0xffffffffu, digit, 0);
    if (__all_sync(0xffffffffu, digit == d0)) {
        if ((threadIdx.x & 31) == 0 && live) atomicAdd(&hist[digit], 32u);
    } else if (live) {
        atomicAdd(&hist[digit], 1u);
    }
}

// Larger score -> larger key; -0.0 and +0.0 give the same key.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NWARPS>
struct SelectState {
    uint32_t hist[256];
    uint32_t warp_cnt[2][NWARPS];
    uint32_t prefix;      // digits chosen so far
    uint32_t need;        // elements equal to the final tau still to keep
};

// Pick the digit holding the need-th largest element: scan bins from 255
// down and append the digit (wbits wide, <= 8; bins above 2^wbits are empty)
// to st.prefix.  Executed by one warp; lane L owns bins 255-8L .. 248-8L.
template <int NWARPS>
__device__ __forceinline__ void choose_digit(SelectState<NWARPS>& st, int wbits = 8) {
    const int lane = threadIdx.x & 31;
    uint32_t c[8];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        c[j] = st.hist[255 - 8 * lane - j];
        sum += c[j];
    }
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
                st.prefix = (st.prefix << wbits) | (uint32_t)(255 - 8 * lane - j);
                st.need = need - before;
                break;
            }
            before += c[j];
        }
    }
}

// Block-wide top-k of one row of n scores (NT threads, all of the block).
// keys_s: shared memory for up to cache_keys keys (0 = re-read the row).
template <int NT>
__device__ void select_row(const float* __restrict__ src, int n, int k, int32_t* __restrict__ dst,
                           uint32_t* keys_s, int cache_keys, SelectState<NT / 32>& st) {
    constexpr int NW = NT / 32;
    if (n <= k) {  // every candidate is kept
        for (int j = threadIdx.x; j < k; j += NT) dst[j] = j < n ? j : -1;
        return;
    }
    const bool cached = n <= cache_keys;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    __syncthreads();  // st may be reused by the caller
    if (threadIdx.x == 0) { st.prefix = 0; st.need = (uint32_t)k; }

    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int j = threadIdx.x; j < 256; j += NT) st.hist[j] = 0;
        __syncthreads();
        const uint32_t prefix = st.prefix;
        // round the loop up to whole warps: every lane takes part in the warp update
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
            warp_hist_add(st.hist, digit, live);
        }
        __syncthreads();
        if (warp == 0) choose_digit(st);
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
        if (lane == 0) st.warp_cnt[buf][warp] = __popc(bg) | ((uint32_t)__popc(be) << 16);
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
        if (gt || (eq && eq_before < need_eq)) dst[gt_before + min(eq_before, need_eq)] = j;
        run_gt += tot_gt;
        run_eq += tot_eq;
        // warp_cnt is double-buffered, so one barrier per chunk suffices
    }
}

// Block-wide: the bin d holding the k-th largest key of the row histogram,
// and how many keys lie in higher bins.  hist in shared memory.
template <int NT>
__device__ void find_bin11(const uint32_t* hist, uint32_t k, uint32_t& d_out, uint32_t& above_out,
                           uint32_t* warp_sum) {
    constexpr int HBINS = 2048;
    constexpr int PER = HBINS / NT;  // bins per thread, highest bins first
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t c[PER];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        c[j] = hist[HBINS - 1 - PER * threadIdx.x - j];
        sum += c[j];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    uint32_t before_warp = 0;
    for (int w = 0; w < warp; ++w) before_warp += warp_sum[w];
    incl += before_warp;
    const uint32_t excl = incl - sum;
    if (excl < k && incl >= k) {  // exactly one thread
        uint32_t before = excl;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            if (before + c[j] >= k) {
                d_out = (uint32_t)(HBINS - 1 - PER * threadIdx.x - j);
                above_out = before;
                break;
            }
            before += c[j];
        }
    }
    __syncthreads();
}

// Block-wide radix select over m keys in shared memory: the need-th largest
// key (tau) and how many keys equal to tau fall inside the top `need`.
template <int NT>
__device__ void select_smem(const uint32_t* keys, int m, uint32_t need, SelectState<NT / 32>& st) {
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) { st.prefix = 0; st.need = need; }
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int j = threadIdx.x; j < 256; j += NT) st.hist[j] = 0;
        __syncthreads();
        const uint32_t prefix = st.prefix;
        const int m_round = (m + 31) & ~31;
        for (int j = threadIdx.x; j < m_round; j += NT) {
            bool live = j < m;
            uint32_t key = live ? keys[j] : 0u;
            live = live && (pass == 0 || (key >> (shift + 8)) == prefix);
            const uint32_t digit = live ? ((key >> shift) & 255u) : 256u;
            warp_hist_add(st.hist, digit, live);
        }
        __syncthreads();
        if (warp == 0) choose_digit(st);
        __syncthreads();
    }
}

// Block-wide radix select over m keys in shared memory whose top `pbits`
// bits all equal `pval`: the need-th largest key (-> st.prefix) and how many
// keys equal to it fall inside the top `need` (-> st.need).  Digits of up to
// 8 bits; plain shared atomics (the keys of one bin are spread out).
template <int NT>
__device__ void select_smem_known(const uint32_t* keys, int m, uint32_t need, uint32_t pval,
                                  int pbits, SelectState<NT / 32>& st) {
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) { st.prefix = pval; st.need = need; }
    for (int rem = 32 - pbits; rem > 0;) {
        const int wbits = rem < 8 ? rem : 8;
        const int shift = rem - wbits;
        for (int j = threadIdx.x; j < 256; j += NT) st.hist[j] = 0;
        __syncthreads();
        const uint32_t prefix = st.prefix;
        for (int j = threadIdx.x; j < m; j += NT) {
            const uint32_t key = keys[j];
            if ((uint64_t)key >> rem == (uint64_t)prefix)
                atomicAdd(&st.hist[(key >> shift) & ((1u << wbits) - 1u)], 1u);
        }
        __syncthreads();
        if (warp == 0) choose_digit(st, wbits);
        __syncthreads();
        rem -= wbits;
    }
}

}  // namespace ic
