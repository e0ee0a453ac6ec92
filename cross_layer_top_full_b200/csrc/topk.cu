// topk.cu -- per-row top-k of the indexer scores, one CTA per row (the
// many-row path of prefill).  topk_cluster.cu and topk_multi.cu hold the
// paths for few, long rows (decode), which spread each row over many CTAs.
//
// DSA keeps the k most relevant keys per query (IndexCache summary, es page,
// section 1).  Row t keeps the min(k, t+1) candidates s <= t with the largest
// score; equal scores go to the smaller position and -0.0 counts as +0.0; the
// kept positions are written in ascending order and padded with -1.
//
// Method (rows of up to 65536 candidates): each float becomes an
// order-preserving 32-bit key (flip all bits of negatives, set the sign bit
// of non-negatives; -0.0 is first mapped to +0.0).  The row is read from
// memory ONCE: while it streams in, every key's top 16 bits are kept in
// shared memory and its top 11 bits are counted in a 2048-bin histogram
// (shared-memory atomics; a warp whose 32 keys share one digit adds 32 at
// once, so clustered digits do not serialise).  The bin d that holds the k-th largest key splits the row into
// keys that are surely kept (top 11 bits above d), surely dropped (below d)
// and the candidates (equal to d).  One pass over the shared-memory keys
// collects the candidates' positions; only their full scores are fetched
// again (from L2), and a radix select over them finds the exact key tau of
// the k-th largest score and, among keys equal to tau, the last position
// kept (smaller positions first).  The kept candidates are marked in a
// bitmap, and a final pass in position order writes every surely-kept or
// marked position with a block-wide prefix count, so the output is
// ascending without a sort.  Three passes over the row instead of one per
// radix digit.  Rows whose candidate bin overflows its shared-memory list
// (heavily tied or degenerate scores), and rows longer than 65536, take the
// plain radix select of topk_common.cuh (four 8-bit passes over the row).
#include "topk_common.cuh"

namespace ic {
namespace {

constexpr int NT = 256;
constexpr int NW = NT / 32;
constexpr int HBINS = 2048;
constexpr int N_MAX = 65536;         // candidates of a row kept in shared memory (16 bits each)
constexpr int CAND_CAP = 2048;       // candidates of the threshold bin resolved exactly

struct RowSmem {
    uint32_t hist[HBINS];
    uint32_t cand_key[CAND_CAP];
    uint32_t cand_pos[CAND_CAP];
    uint32_t warp_sum[NW];
    uint32_t warp_cnt[2][NW];
    uint32_t d, above, n_cand, n_eq;
    SelectState<NW> st;
};

__global__ void __launch_bounds__(NT)
topk_rows_kernel(const float* __restrict__ scores, int64_t ld, int Lq, int q_start, int k,
                 int32_t* __restrict__ idx, int n_max, const int32_t* __restrict__ seq_lens,
                 int T_max) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RowSmem& S = *reinterpret_cast<RowSmem*>(smem_raw);
    const int words = (n_max + 31) / 32;
    uint32_t* keep = reinterpret_cast<uint32_t*>(smem_raw + sizeof(RowSmem));        // [words]
    uint16_t* hi = reinterpret_cast<uint16_t*>(keep + ((words + 3) & ~3));            // [n_max]

    pdl_trigger();
    pdl_wait();
    const int64_t row = blockIdx.x;
    const int n = row_candidates(row, Lq, q_start, seq_lens, T_max);
    const float* src = scores + row * ld;
    int32_t* dst = idx + row * (int64_t)k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (n <= k) {  // every candidate is kept
        for (int j = threadIdx.x; j < k; j += NT) dst[j] = j < n ? j : -1;
        return;
    }
    for (int b = threadIdx.x; b < HBINS; b += NT) S.hist[b] = 0;
    for (int w = threadIdx.x; w < (n + 31) / 32; w += NT) keep[w] = 0;
    if (threadIdx.x == 0) { S.n_cand = 0; S.n_eq = 0; }
    __syncthreads();

    // ---- pass 1: read the row once; top 16 bits to shared memory, histogram
    // of the top 11 bits.  Four consecutive scores per thread and step (the
    // row starts on a 16-byte boundary); the loop runs in whole warps.
    const bool vec = (reinterpret_cast<uintptr_t>(src) & 15) == 0;
    for (int base = 0; base < n; base += 4 * NT) {
        const int j = base + 4 * threadIdx.x;
        float f[4];
        if (vec && j + 3 < n) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(src + j));
            f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) f[q] = j + q < n ? src[j + q] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const bool live = j + q < n;
            const uint32_t key = order_key(f[q]);
            if (live) hi[j + q] = (uint16_t)(key >> 16);
            const uint32_t digit = live ? (key >> 21) : 0xffffffffu;
            warp_hist_add(S.hist, digit, live);
        }
    }
    __syncthreads();
    find_bin11<NT>(S.hist, (uint32_t)k, S.d, S.above, S.warp_sum);   // ends with a barrier
    const uint32_t d = S.d;

    // ---- pass 2: positions of the candidates (keys in bin d), their full keys
    for (int base = 0; base < n; base += NT) {
        const int j = base + threadIdx.x;
        const bool cand = j < n && ((uint32_t)hi[j] >> 5) == d;
        const uint32_t bal = __ballot_sync(0xffffffffu, cand);
        if (bal) {
            uint32_t slot0 = 0;
            if (lane == __ffs(bal) - 1) slot0 = atomicAdd(&S.n_cand, __popc(bal));
            slot0 = __shfl_sync(0xffffffffu, slot0, __ffs(bal) - 1);
            const uint32_t slot = slot0 + __popc(bal & ((1u << lane) - 1u));
            if (cand && slot < CAND_CAP) {
                S.cand_pos[slot] = (uint32_t)j;
                S.cand_key[slot] = order_key(src[j]);
            }
        }
    }
    __syncthreads();
    const uint32_t m_all = S.n_cand;
    if (m_all > (uint32_t)CAND_CAP) {
        // degenerate row: plain radix select over the whole row
        select_row<NT>(src, n, k, dst, nullptr, 0, S.st);
        return;
    }
    const int m = (int)m_all;

    // ---- exact resolve among the candidates
    const uint32_t need1 = (uint32_t)k - S.above;          // keys still to take from bin d
    select_smem_known<NT>(S.cand_key, m, need1, d, 11, S.st);
    const uint32_t tau = S.st.prefix, need_eq = S.st.need;
    __syncthreads();
    uint32_t n_eq = 0;
    for (int j = threadIdx.x; j < m; j += NT) n_eq += S.cand_key[j] == tau ? 1u : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    if (lane == 0 && n_eq) atomicAdd(&S.n_eq, n_eq);
    __syncthreads();
    if (S.n_eq > need_eq) {
        // ties at tau: keys above tau are kept; among the keys equal to tau the
        // need_eq smallest positions are, i.e. the need_eq largest ~position
        for (int j = threadIdx.x; j < m; j += NT) {
            const uint32_t key = S.cand_key[j], pos = S.cand_pos[j];
            if (key > tau) atomicOr(&keep[pos >> 5], 1u << (pos & 31));
            S.cand_key[j] = key == tau ? ~pos : 0u;    // ~pos > 0 for every position
        }
        __syncthreads();
        select_smem<NT>(S.cand_key, m, need_eq, S.st);
        const uint32_t pos_cut = ~S.st.prefix;
        __syncthreads();
        for (int j = threadIdx.x; j < m; j += NT) {
            const uint32_t v = S.cand_key[j];
            if (v != 0u && ~v <= pos_cut) atomicOr(&keep[(~v) >> 5], 1u << ((~v) & 31));
        }
    } else {
        // every key equal to tau is kept
        for (int j = threadIdx.x; j < m; j += NT) {
            const uint32_t pos = S.cand_pos[j];
            if (S.cand_key[j] >= tau) atomicOr(&keep[pos >> 5], 1u << (pos & 31));
        }
    }
    __syncthreads();

    // ---- pass 3: write the kept positions in order.  Every warp takes a
    // contiguous range of the row: it counts its kept keys, one scan of the
    // counts gives its offset, then it writes them in order with ballots.
    const int per = ((n + NW - 1) / NW + 31) & ~31;          // keys per warp, whole 32-key steps
    const int b0 = min(n, warp * per), b1 = min(n, b0 + per);
    auto kept = [&](int j) -> bool {
        if (j >= b1) return false;
        const uint32_t dg = (uint32_t)hi[j] >> 5;
        return dg > d || (dg == d && ((keep[j >> 5] >> (j & 31)) & 1u));
    };
    uint32_t cnt = 0;
    for (int j0 = b0; j0 < b1; j0 += 32) cnt += __popc(__ballot_sync(0xffffffffu, kept(j0 + lane)));
    if (lane == 0) S.warp_cnt[0][warp] = cnt;
    __syncthreads();
    uint32_t run = 0;
#pragma unroll
    for (int w2 = 0; w2 < NW; ++w2)
        if (w2 < warp) run += S.warp_cnt[0][w2];
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int j0 = b0; j0 < b1; j0 += 32) {
        const int j = j0 + lane;
        const bool kp = kept(j);
        const uint32_t b = __ballot_sync(0xffffffffu, kp);
        if (kp) dst[run + __popc(b & lt_mask)] = j;
        run += __popc(b);
    }
}

// Rows longer than the shared-memory key cache: plain radix select, the
// row re-read on each of its passes.
constexpr int NT_LONG = 512;

__global__ void __launch_bounds__(NT_LONG)
topk_radix_kernel(const float* __restrict__ scores, int64_t ld, int Lq, int q_start, int k,
                  int32_t* __restrict__ idx, const int32_t* __restrict__ seq_lens, int T_max) {
    pdl_trigger();
    pdl_wait();
    const int64_t row = blockIdx.x;
    const int n = row_candidates(row, Lq, q_start, seq_lens, T_max);
    __shared__ SelectState<NT_LONG / 32> st;
    select_row<NT_LONG>(scores + row * ld, n, k, idx + row * (int64_t)k, nullptr, 0, st);
}

}  // namespace

ic_status launch_topk_rows(const float* scores, int64_t ld, ic_rows r, int k, int32_t* idx,
                           cudaStream_t s, const int32_t* seq_lens) {
    const int n_max = r.q_start + r.Lq;  // candidates of the last row
    const int64_t rows = (int64_t)r.B * r.Lq;
    if (n_max <= N_MAX) {
        const int words = (n_max + 31) / 32;
        const size_t smem = sizeof(RowSmem) + sizeof(uint32_t) * ((words + 3) & ~3) +
                            sizeof(uint16_t) * (size_t)((n_max + 7) & ~7);
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return cuda_error("topk");
        if (launch_ex(topk_rows_kernel, dim3((unsigned)rows), dim3(NT), smem, s, pdl_rows(rows), 0,
                      scores, ld, r.Lq, r.q_start, k, idx, n_max, seq_lens, r.T) != cudaSuccess)
            return cuda_error("topk");
    } else {
        if (launch_ex(topk_radix_kernel, dim3((unsigned)rows), dim3(NT_LONG), 0, s, pdl_rows(rows),
                      0, scores, ld, r.Lq, r.q_start, k, idx, seq_lens, r.T) != cudaSuccess)
            return cuda_error("topk");
    }
    count_launch(IC_LK_TOPK);
    return last_launch_status();
}

}  // namespace ic
