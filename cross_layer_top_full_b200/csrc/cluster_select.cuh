// cluster_select.cuh -- the exact top-k of one row whose candidates are cached,
// as order-preserving keys, in the shared memory of the CTAs of one
// thread-block cluster (each CTA one contiguous segment, in position order
// by CTA rank).
//
// Top-k rule (DSA keeps the k most relevant keys per query; IndexCache
// summary, es page, section 1): the k largest scores, ties to the smaller
// position, -0.0 = +0.0; kept positions written ascending.
//
// The key of the k-th largest score, tau, is found digit by digit, most
// significant first (11, 11 and 10 bits):
//   1. every CTA histograms the digit of its keys that still match the
//      digits chosen so far (warp-aggregated shared-memory atomics);
//   2. cluster barrier; CTA c sums bins [c*W/CL, (c+1)*W/CL) of all CL
//      histograms through distributed shared memory, and their total;
//   3. cluster barrier; every CTA reads the CL slice totals, finds the slice
//      and then, in its owner's reduced bins, the bin that holds the
//      need-th largest remaining key, and appends that digit.
// Then each CTA counts its keys above tau and equal to tau; after one more
// cluster barrier every CTA knows, from all counts, where its kept positions
// go and how many of its equal-to-tau keys to keep (the smaller positions
// first, so segments of lower rank keep theirs first), and writes them in
// position order.  Every wait is a hardware cluster barrier that all CTAs of
// the cluster reach in the same sequence: no flag, no spin-wait, no global
// workspace.
#pragma once

#include "topk_common.cuh"

namespace ic {
namespace csel {

constexpr int HBINS = 2048;             // 11-bit digits

template <int NW>
struct __align__(16) ClusterSmem {
    uint32_t hist[HBINS];               // this CTA's histogram of the current digit
    uint32_t red[HBINS];                // reduced bins owned by this CTA (W / CL of them)
    uint32_t warp_cnt[2][NW];
    uint32_t slice_tot;                 // total of the reduced bins owned by this CTA
    uint32_t cnt_gt, cnt_eq;            // keys > tau and == tau in this CTA's segment
    uint32_t prefix, need;              // digits chosen so far; keys still to take at the prefix
};

__device__ __forceinline__ uint32_t ld_dsmem(uint32_t cluster_addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_ctas() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t map_rank(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(r)
                 : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"(rank));
    return r;
}

// Cluster-wide barrier of all threads.  A CTA barrier first brings every
// warp of the CTA to this point converged; the cluster barrier itself is the
// non-.aligned form, whose arrive and wait each thread may execute on its
// own, so its correctness does not rest on how the compiler reconverges a
// warp after divergent code.
__device__ __forceinline__ void cluster_barrier() {
    __syncthreads();
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// One warp: among the `m` counts c[0..m-1] (index 0 = the LOWEST bin of the
// range), find the highest-first position where the running count from the
// top reaches `need`.  Returns (index, count strictly above it).  Each lane
// holds ceil(m/32) consecutive counts from the top.
__device__ __forceinline__ void warp_find_from_top(const uint32_t* c, int m, uint32_t need,
                                                   bool remote, uint32_t remote_base,
                                                   uint32_t& idx_out, uint32_t& before_out) {
    const int lane = threadIdx.x & 31;
    const int per = (m + 31) / 32;
    uint32_t sum = 0;
    // lane L covers top-down positions L*per .. L*per + per - 1 (index m-1-pos)
    for (int j = 0; j < per; ++j) {
        const int pos = lane * per + j;
        if (pos < m) {
            const int idx = m - 1 - pos;
            sum += remote ? ld_dsmem(remote_base + 4u * idx) : c[idx];
        }
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, incl >= need);
    const int src = hit ? __ffs(hit) - 1 : 31;
    uint32_t idx = 0, before = 0;
    if (lane == src) {
        before = incl - sum;
        for (int j = 0; j < per; ++j) {
            const int pos = lane * per + j;
            if (pos >= m) break;
            const int i = m - 1 - pos;
            const uint32_t ci = remote ? ld_dsmem(remote_base + 4u * i) : c[i];
            if (before + ci >= need) { idx = (uint32_t)i; break; }
            before += ci;
        }
    }
    idx_out = __shfl_sync(0xffffffffu, idx, src);
    before_out = __shfl_sync(0xffffffffu, before, src);
}


// Exact top-k of one row of n > k candidates, the segment [s0, s0 + m) of
// which is cached in this CTA's shared memory as order keys `keys`; called
// by all NT threads of every CTA of the cluster (CL CTAs, this one `rank`),
// with the segments of increasing rank covering the row in order.  Writes
// this CTA's kept positions into dst[0..k).  Ends with a cluster barrier.
template <int NT>
__device__ void cluster_select(ClusterSmem<NT / 32>& S, const uint32_t* keys, int m, int s0, int k,
                               int32_t* __restrict__ dst, uint32_t CL, uint32_t rank) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        S.prefix = 0;
        S.need = (uint32_t)k;
    }
    __syncthreads();

    // ---------------------------------------------------------------- digits
    int done_bits = 0;
    for (int pass = 0; pass < 3; ++pass) {
        const int width = pass < 2 ? 11 : 10;
        const int W = 1 << width;
        const int shift = 32 - done_bits - width;
        for (int b = threadIdx.x; b < W; b += NT) S.hist[b] = 0;
        __syncthreads();
        const uint32_t prefix = S.prefix;
        const int m_round = (m + 31) & ~31;
        for (int j = threadIdx.x; j < m_round; j += NT) {
            bool live = j < m;
            uint32_t key = live ? keys[j] : 0u;
            if (done_bits > 0) live = live && (key >> (32 - done_bits)) == prefix;
            const uint32_t digit = live ? ((key >> shift) & (uint32_t)(W - 1)) : 0xffffffffu;
            const uint32_t peers = __match_any_sync(0xffffffffu, digit);
            if (live && lane == __ffs(peers) - 1) atomicAdd(&S.hist[digit], __popc(peers));
        }
        cluster_barrier();   // every CTA's histogram is complete
        // reduce my slice of the bins over the cluster
        const int per = W / (int)CL;
        uint32_t part = 0;
        for (int t = threadIdx.x; t < per; t += NT) {
            const int bin = (int)rank * per + t;
            uint32_t sum = 0;
            for (uint32_t c = 0; c < CL; ++c) sum += ld_dsmem(map_rank(&S.hist[bin], c));
            S.red[t] = sum;
            part += sum;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) S.warp_cnt[0][warp] = part;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t tot = 0;
            for (int w = 0; w < NW; ++w) tot += S.warp_cnt[0][w];
            S.slice_tot = tot;
        }
        cluster_barrier();   // every CTA's reduced slice and total are complete
        if (warp == 0) {
            const uint32_t need = S.need;
            // the slice (owner CTA) holding the need-th largest key, from the top
            uint32_t owner, above_slices;
            {
                uint32_t tot = lane < (int)CL ? ld_dsmem(map_rank(&S.slice_tot, (uint32_t)lane)) : 0u;
                // top-down: slice CL-1 holds the highest bins
                const int pos = lane;                       // top-down position
                const int sl = (int)CL - 1 - pos;
                // every lane takes part in the shuffle (a full-mask shuffle that
                // some lanes skip never completes); lanes past CL then drop it
                const uint32_t from_sl = __shfl_sync(0xffffffffu, tot, sl < 0 ? 0 : sl);
                const uint32_t mine = pos < (int)CL ? from_sl : 0u;
                uint32_t incl = mine;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += v;
                }
                const uint32_t hit = __ballot_sync(0xffffffffu, incl >= need && pos < (int)CL);
                const int p = hit ? __ffs(hit) - 1 : 0;
                owner = (uint32_t)((int)CL - 1 - p);
                above_slices = __shfl_sync(0xffffffffu, incl - mine, p);
            }
            uint32_t bin_in_slice, before;
            warp_find_from_top(nullptr, per, need - above_slices, true, map_rank(&S.red[0], owner),
                               bin_in_slice, before);
            if (lane == 0) {
                const uint32_t digit = owner * (uint32_t)per + bin_in_slice;
                S.prefix = (S.prefix << width) | digit;
                S.need = need - above_slices - before;
            }
        }
        __syncthreads();
        done_bits += width;
    }
    const uint32_t tau = S.prefix;
    const uint32_t need_eq = S.need;      // keys equal to tau to keep (smallest positions first)

    // ---------------------------------------------------------------- counts
    {
        uint32_t gt = 0, eq = 0;
        for (int j = threadIdx.x; j < m; j += NT) {
            const uint32_t key = keys[j];
            gt += key > tau ? 1u : 0u;
            eq += key == tau ? 1u : 0u;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gt += __shfl_xor_sync(0xffffffffu, gt, o);
            eq += __shfl_xor_sync(0xffffffffu, eq, o);
        }
        if (lane == 0) {
            S.warp_cnt[0][warp] = gt;
            S.warp_cnt[1][warp] = eq;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t a = 0, b = 0;
            for (int w = 0; w < NW; ++w) { a += S.warp_cnt[0][w]; b += S.warp_cnt[1][w]; }
            S.cnt_gt = a;
            S.cnt_eq = b;
        }
    }
    cluster_barrier();   // every CTA's counts are complete
    uint32_t out_off = 0, eq_keep = 0;
    {
        // lower ranks hold smaller positions: they write first and keep their
        // equal-to-tau keys first
        uint32_t eq_before = 0;
        for (uint32_t c = 0; c < rank; ++c) {
            const uint32_t g = ld_dsmem(map_rank(&S.cnt_gt, c));
            const uint32_t e = ld_dsmem(map_rank(&S.cnt_eq, c));
            const uint32_t keep = eq_before >= need_eq ? 0u : min(e, need_eq - eq_before);
            out_off += g + keep;
            eq_before += e;
        }
        eq_keep = eq_before >= need_eq ? 0u : min(S.cnt_eq, need_eq - eq_before);
    }
    __syncthreads();

    // ---------------------------------------------------------------- ordered write
    {
        uint32_t run_gt = 0, run_eq = 0;
        const uint32_t lt_mask = (1u << lane) - 1u;
        const int m_round = (m + NT - 1) / NT * NT;
        for (int base = 0; base < m_round; base += NT) {
            const int j = base + threadIdx.x;
            const uint32_t key = j < m ? keys[j] : 0u;
            const bool gt = j < m && key > tau;
            const bool eq = j < m && key == tau;
            const uint32_t bg = __ballot_sync(0xffffffffu, gt);
            const uint32_t be = __ballot_sync(0xffffffffu, eq);
            const int buf = (base / NT) & 1;
            if (lane == 0) S.warp_cnt[buf][warp] = __popc(bg) | ((uint32_t)__popc(be) << 16);
            __syncthreads();
            uint32_t pre_gt = 0, pre_eq = 0, tot_gt = 0, tot_eq = 0;
#pragma unroll
            for (int w2 = 0; w2 < NW; ++w2) {
                const uint32_t v = S.warp_cnt[buf][w2];
                if (w2 < warp) { pre_gt += v & 0xffffu; pre_eq += v >> 16; }
                tot_gt += v & 0xffffu;
                tot_eq += v >> 16;
            }
            const uint32_t gt_before = run_gt + pre_gt + __popc(bg & lt_mask);
            const uint32_t eq_before = run_eq + pre_eq + __popc(be & lt_mask);
            if (gt || (eq && eq_before < eq_keep))
                dst[out_off + gt_before + min(eq_before, eq_keep)] = s0 + j;
            run_gt += tot_gt;
            run_eq += tot_eq;
        }
    }
    cluster_barrier();   // no CTA leaves while another may still read its counts
}

}  // namespace csel
}  // namespace ic
