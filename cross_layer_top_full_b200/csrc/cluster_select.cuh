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
// significant first (11, 11 and 10 bits).  Each pass: every CTA histograms
// the digit of its keys that still match the digits chosen so far (shared-
// memory atomics); cluster barrier; every CTA obtains the sums of all CL
// histograms through distributed shared memory (the same sums in every CTA:
// for 4 or more CTAs each first sums its own slice of the bins, and after
// another cluster barrier every CTA reads all slices) and appends the digit
// holding the need-th largest remaining key.  As soon as the cluster
// holds at most CAND_CAP keys at the prefix (after 11 or 22 bits), every CTA
// compacts its keys there; after a cluster barrier every CTA gathers all of
// them and finds tau among them with a local radix select (the same
// deterministic result in every CTA), and from the gathered keys and the
// lower-ranked CTAs' counts above the prefix where its kept positions go.
// Only when a prefix of 22 bits still holds more (heavy ties) are all 32
// bits resolved and the per-CTA counts exchanged once more.  Each CTA then
// writes its kept positions in position order, keeping its keys equal to
// tau after those of lower-ranked CTAs (smaller positions first).  Every
// wait is a hardware cluster barrier that all CTAs of the cluster reach in
// the same sequence (the path taken is decided from values every CTA holds
// identically): no flag, no spin-wait, no global workspace.
#pragma once

#include <cstddef>

#include "topk_common.cuh"

namespace ic {
namespace csel {

constexpr int HBINS = 2048;             // 11-bit digits

constexpr int CAND_CAP = 2 * HBINS;   // keys of bin d0 the compaction path takes (cluster total)

template <int NW>
struct __align__(16) ClusterSmem {
    // this CTA's histogram of the current digit, in hist[0] and hist[1] by
    // turns (another CTA may still be reading the previous one); on the
    // compaction path the two together hold the gathered candidates of
    // every CTA (CAND_CAP keys)
    uint32_t hist[2][HBINS];
    uint32_t red[HBINS];                // the cluster's sums of the current digit (local)
    uint32_t slice[HBINS / 4];          // this CTA's slice of those sums (clusters of 4 or more)
    uint32_t cand[CAND_CAP];            // this CTA's keys of the chosen bin (compaction path)
    SelectState<NW> st;                 // local radix select over the gathered candidates
    uint32_t warp_cnt[2][NW];
    uint32_t cnt_gt, cnt_eq;            // keys > tau and == tau in this CTA's segment
    uint32_t prefix, need;              // digits chosen so far; keys still to take at the prefix
    uint32_t bin_total;                 // the cluster's keys at the prefix
    uint32_t n_cand, gt0;               // this CTA's keys at the prefix, and above it
    uint32_t cand_off[17];              // gathered candidates: CTA c's start (c <= CL)
    uint32_t gt_before;                 // keys above the prefix in the lower-ranked CTAs
};
static_assert(2 * HBINS >= CAND_CAP, "gathered candidates fit in the two histograms");

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


// One pass of shared-memory histogramming (warp_hist_add) over this CTA's
// keys: bin (key >> shift) & (W-1) of every key whose bits above the digit
// equal `prefix` (all keys when done_bits == 0).  All NT threads.
template <int NT>
__device__ __forceinline__ void digit_histogram(uint32_t* hist, const uint32_t* keys, int m,
                                                int done_bits, int width, uint32_t prefix) {
    const int W = 1 << width;
    const int shift = 32 - done_bits - width;
    for (int b = threadIdx.x; b < W; b += NT) hist[b] = 0;
    __syncthreads();
    const int m_round = (m + 31) & ~31;      // whole warps: every lane takes part in the update
    for (int j = threadIdx.x; j < m_round; j += NT) {
        bool live = j < m;
        const uint32_t key = live ? keys[j] : 0u;
        if (done_bits > 0) live = live && (key >> (32 - done_bits)) == prefix;
        const uint32_t digit = live ? ((key >> shift) & (uint32_t)(W - 1)) : 0xffffffffu;
        warp_hist_add(hist, digit, live);
    }
}

// Writes this CTA's kept positions (keys > tau, and the first eq_keep keys
// equal to tau) in position order from dst[out_off].  Every warp takes a
// contiguous range of the segment: it counts its kept keys, one block-wide
// scan of the counts gives it its offset, and it writes its keys in order
// with warp ballots (no block barrier per chunk).  All NT threads.
template <int NT>
__device__ __forceinline__ void ordered_write(uint32_t (&warp_cnt)[2][NT / 32], const uint32_t* keys,
                                              int m, int s0, uint32_t tau, uint32_t out_off,
                                              uint32_t eq_keep, int32_t* __restrict__ dst) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = ((m + NW - 1) / NW + 31) & ~31;          // keys per warp, whole 32-key steps
    const int b0 = min(m, warp * per), b1 = min(m, b0 + per);
    uint32_t ngt = 0, neq = 0;
    for (int j0 = b0; j0 < b1; j0 += 32) {                   // the same trip count in every lane
        const int j = j0 + lane;
        const uint32_t key = j < b1 ? keys[j] : 0u;
        ngt += __popc(__ballot_sync(0xffffffffu, j < b1 && key > tau));
        neq += __popc(__ballot_sync(0xffffffffu, j < b1 && key == tau));
    }
    __syncthreads();                                         // warp_cnt may still be read
    if (lane == 0) {
        warp_cnt[0][warp] = ngt;
        warp_cnt[1][warp] = neq;
    }
    __syncthreads();
    uint32_t run_gt = 0, run_eq = 0;                         // kept keys of the lower warps
    for (int w = 0; w < warp; ++w) {
        run_gt += warp_cnt[0][w];
        run_eq += warp_cnt[1][w];
    }
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int j0 = b0; j0 < b1; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t key = j < b1 ? keys[j] : 0u;
        const bool gt = j < b1 && key > tau;
        const bool eq = j < b1 && key == tau;
        const uint32_t bg = __ballot_sync(0xffffffffu, gt);
        const uint32_t be = __ballot_sync(0xffffffffu, eq);
        const uint32_t gt_before = run_gt + __popc(bg & lt_mask);
        const uint32_t eq_before = run_eq + __popc(be & lt_mask);
        if (gt || (eq && eq_before < eq_keep))
            dst[out_off + gt_before + min(eq_before, eq_keep)] = s0 + j;
        run_gt += __popc(bg);
        run_eq += __popc(be);
    }
}

// Block-wide sum of one value per thread; the result in every thread.
template <int NT>
__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* scratch /* NT/32 words */) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();                     // scratch may still be read by a previous use
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) t += scratch[w];
    return t;
}

// Exact top-k of one row of n > k candidates, the segment [s0, s0 + m) of
// which is cached in this CTA's shared memory as order keys `keys`; called
// by all NT threads of every CTA of the cluster (CL CTAs, this one `rank`),
// with the segments of increasing rank covering the row in order.  Writes
// this CTA's kept positions into dst[0..k).  Ends with a cluster barrier.
template <int NT>
__device__ void cluster_select(ClusterSmem<NT / 32>& S, const uint32_t* keys, int m, int s0, int k,
                               int32_t* __restrict__ dst, uint32_t CL, uint32_t rank) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // ------------------------------------------------ digits, most significant first
    // Each pass: histogram of the next digit of the keys at the prefix; every
    // CTA sums all CL histograms (the same sums everywhere) and extends the
    // prefix by the digit holding the need-th largest key.  As soon as the
    // cluster holds at most CAND_CAP keys at the prefix, they are compacted.
    uint32_t prefix = 0, need = (uint32_t)k;
    int done = 0;
    for (int pass = 0; pass < 3; ++pass) {
        const int width = pass < 2 ? 11 : 10;
        const int W = 1 << width;
        uint32_t* local = S.hist[pass & 1];
        digit_histogram<NT>(local, keys, m, done, width, prefix);
        cluster_barrier();   // every CTA's histogram is complete
        if (CL < 4) {
            // every CTA sums every bin over the CL histograms; the CL remote
            // loads of a bin are all in flight before they are added
            for (int b = threadIdx.x; b < W; b += NT) {
                uint32_t v[4];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (c < (int)CL) v[c] = ld_dsmem(map_rank(&local[b], (uint32_t)c));
                uint32_t sum = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (c < (int)CL) sum += v[c];
                S.red[b] = sum;
            }
        } else {
            // two steps, W (CL + 1) remote loads per CTA instead of W CL: CTA
            // `rank` sums its slice of the bins over the CL histograms, then
            // every CTA reads all CL slices
            const int per = W / (int)CL;
            for (int t = threadIdx.x; t < per; t += NT) {
                const int bin = (int)rank * per + t;
                uint32_t v[16];
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    if (c < (int)CL) v[c] = ld_dsmem(map_rank(&local[bin], (uint32_t)c));
                uint32_t sum = 0;
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    if (c < (int)CL) sum += v[c];
                S.slice[t] = sum;
            }
            cluster_barrier();   // every CTA's slice is complete
            for (int b0 = 0; b0 < W; b0 += 4 * NT) {
                uint32_t v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int b = b0 + u * NT + threadIdx.x;
                    v[u] = b < W ? ld_dsmem(map_rank(&S.slice[b % per], (uint32_t)(b / per))) : 0u;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int b = b0 + u * NT + threadIdx.x;
                    if (b < W) S.red[b] = v[u];
                }
            }
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t d, above;
            warp_find_from_top(S.red, W, need, false, 0u, d, above);
            if (lane == 0) {
                S.prefix = (prefix << width) | d;
                S.need = need - above;           // keys still to take at the new prefix
                S.bin_total = S.red[d];
            }
        }
        __syncthreads();
        prefix = S.prefix;
        need = S.need;
        done += width;
        if (done < 32 && S.bin_total <= (uint32_t)CAND_CAP) break;   // the same in every CTA
    }
    uint32_t tau, need_eq, out_off, eq_keep;
    if (done < 32) {
        // ----------------------------------------------- compaction path
        // this CTA's keys at the prefix (any order) and its count above it
        const int sh = 32 - done;
        if (threadIdx.x == 0) S.n_cand = 0;
        __syncthreads();
        uint32_t gt0 = 0;
        const int m_round = (m + 31) & ~31;      // whole warps: ballot and shuffle take every lane
        for (int j = threadIdx.x; j < m_round; j += NT) {
            const uint32_t key = j < m ? keys[j] : 0u;
            const uint32_t top = key >> sh;
            const bool cand = j < m && top == prefix;
            gt0 += (j < m && top > prefix) ? 1u : 0u;
            const uint32_t bal = __ballot_sync(0xffffffffu, cand);
            if (bal != 0u) {                     // the same in every lane
                const int src = __ffs(bal) - 1;
                uint32_t slot0 = 0;
                if (lane == src) slot0 = atomicAdd(&S.n_cand, __popc(bal));
                slot0 = __shfl_sync(0xffffffffu, slot0, src);
                if (cand) S.cand[slot0 + __popc(bal & ((1u << lane) - 1u))] = key;
            }
        }
        gt0 = block_sum<NT>(gt0, S.warp_cnt[0]);
        if (threadIdx.x == 0) S.gt0 = gt0;
        cluster_barrier();   // every CTA's candidates and counts are complete; no CTA
                             // reads another's histograms any more
        if (warp == 0) {
            const uint32_t nc = lane < (int)CL ? ld_dsmem(map_rank(&S.n_cand, (uint32_t)lane)) : 0u;
            const uint32_t g0 = lane < (int)CL ? ld_dsmem(map_rank(&S.gt0, (uint32_t)lane)) : 0u;
            uint32_t incl = nc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            uint32_t gb = lane < (int)rank ? g0 : 0u;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) gb += __shfl_xor_sync(0xffffffffu, gb, o);
            if (lane <= (int)CL) S.cand_off[lane] = incl - nc;   // lane CL: the total
            if (lane == 0) S.gt_before = gb;
        }
        __syncthreads();
        // every CTA's candidates, in rank order, into this CTA's two histograms
        uint32_t* gathered = &S.hist[0][0];
        const uint32_t total = S.cand_off[CL];
        for (uint32_t base = 0; base < total; base += 8u * NT) {
            uint32_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t i = base + (uint32_t)u * NT + threadIdx.x;
                v[u] = 0u;
                if (i < total) {
                    uint32_t c = 0;
                    while (c + 1 < CL && S.cand_off[c + 1] <= i) ++c;
                    v[u] = ld_dsmem(map_rank(&S.cand[i - S.cand_off[c]], c));
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t i = base + (uint32_t)u * NT + threadIdx.x;
                if (i < total) gathered[i] = v[u];
            }
        }
        __syncthreads();
        // tau among the gathered keys at the prefix (identical in every CTA)
        select_smem_known<NT>(gathered, (int)total, need, prefix, done, S.st);
        tau = S.st.prefix;
        need_eq = S.st.need;
        // keys above and equal to tau in the lower-ranked CTAs' candidates, and
        // this CTA's keys equal to tau
        const uint32_t lo = S.cand_off[rank], hi = S.cand_off[rank + 1];
        uint32_t before = 0, eq_me = 0;
        for (uint32_t i = threadIdx.x; i < hi; i += NT) {
            const uint32_t key = gathered[i];
            if (i < lo) before += (key > tau ? 1u : 0u) | (key == tau ? 0x10000u : 0u);
            else eq_me += key == tau ? 1u : 0u;
        }
        before = block_sum<NT>(before, S.warp_cnt[0]);
        eq_me = block_sum<NT>(eq_me, S.warp_cnt[0]);
        const uint32_t gt_p = before & 0xffffu, eq_p = before >> 16;
        out_off = S.gt_before + gt_p + min(eq_p, need_eq);
        eq_keep = need_eq > eq_p ? min(eq_me, need_eq - eq_p) : 0u;
    } else {
        // ----------------------------------------------- every bit resolved (heavy ties)
        tau = prefix;
        need_eq = need;        // keys equal to tau to keep (smallest positions first)
        uint32_t gt = 0, eq = 0;
        for (int j = threadIdx.x; j < m; j += NT) {
            const uint32_t key = keys[j];
            gt += key > tau ? 1u : 0u;
            eq += key == tau ? 1u : 0u;
        }
        gt = block_sum<NT>(gt, S.warp_cnt[0]);
        eq = block_sum<NT>(eq, S.warp_cnt[0]);
        if (threadIdx.x == 0) {
            S.cnt_gt = gt;
            S.cnt_eq = eq;
        }
        cluster_barrier();   // every CTA's counts are complete
        // lower ranks hold smaller positions: they write first and keep their
        // equal-to-tau keys first
        uint32_t off = 0, eq_before = 0;
        for (uint32_t c = 0; c < rank; ++c) {
            off += ld_dsmem(map_rank(&S.cnt_gt, c));
            eq_before += ld_dsmem(map_rank(&S.cnt_eq, c));
        }
        out_off = off + min(eq_before, need_eq);
        eq_keep = need_eq > eq_before ? min(eq, need_eq - eq_before) : 0u;
    }
    ordered_write<NT>(S.warp_cnt, keys, m, s0, tau, out_off, eq_keep, dst);
    cluster_barrier();   // no CTA leaves while another may still read its shared memory
}

}  // namespace csel
}  // namespace ic
