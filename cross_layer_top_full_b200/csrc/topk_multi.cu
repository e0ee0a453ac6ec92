// topk_multi.cu -- top-k of few, long rows (decode) spread over many CTAs.
//
// Same rule as topk.cu (keep the min(k, t+1) largest scores, ties to the
// smaller position, -0.0 = +0.0, ascending output padded with -1; DSA's
// per-query top-k, IndexCache summary, es page, section 1).  A decode step has
// only B rows of up to ~10^5..10^6 scores, so one CTA per row would leave
// most SMs idle; here every row is cut into chunks of CHUNK scores, one CTA
// per chunk, in three launches (no CTA ever waits for another):
//   K1  per-chunk histogram of the top 11 bits of the keys, added into a
//       per-row histogram in the workspace;
//   K2  every chunk finds, from the row histogram, the bin d holding the k-th
//       largest key; it counts its keys above d and appends its keys in bin d
//       (the candidates) with their positions to a per-row list.  The last
//       chunk of a row to finish (an atomic arrival counter) resolves the
//       candidates exactly: tau = the key of the k-th largest score, pos_cut =
//       the position of the last equal-to-tau key that is kept; it then turns
//       the per-chunk counts into output offsets;
//   K3  every chunk writes its kept positions (key > tau, or key == tau and
//       position <= pos_cut) at its offset in position order.
// If a row's candidate bin overflows the list (heavily tied or degenerate
// scores), the last chunk runs the whole row with the one-CTA radix select
// instead and marks it done.
#include <algorithm>

#include "topk_common.cuh"

namespace ic {
namespace {

constexpr int CHUNK = 8192;     // scores per CTA
constexpr int NT = 256;
constexpr int NW = NT / 32;
constexpr int HBITS = 11;
constexpr int HBINS = 1 << HBITS;
constexpr int CAPG = 8192;      // candidates per row kept for the exact resolve
constexpr int CAPS = 2048;      // candidates one chunk stages in shared memory
constexpr int MAX_CHUNKS = 4096;

// per-row control words
enum { RW_CAND_N = 0, RW_ARRIVE = 1, RW_TAU = 2, RW_POS_CUT = 3, RW_DONE = 4, RW_WORDS = 8 };

struct MultiWs {
    uint32_t* hist;      // [R][HBINS]    (zeroed per call)
    uint32_t* ctl;       // [R][RW_WORDS] (zeroed per call)
    uint32_t* chunk_gt;  // [R][nch]
    uint32_t* chunk_off; // [R][nch]
    uint32_t* cand_key;  // [R][CAPG]
    uint32_t* cand_pos;  // [R][CAPG]
    int nch;
};

__device__ __forceinline__ int row_n(int64_t row, int Lq, int q_start) {
    return q_start + (int)(row % Lq) + 1;
}

__device__ __forceinline__ uint32_t digit11(uint32_t key) { return key >> (32 - HBITS); }

// Load this thread's 32 scores of a chunk as 8 independent float4 loads
// (element s0 + 4*(threadIdx.x + NT*i) + q), so all loads are in flight at
// once; elements at or beyond s1 are marked invalid.
struct Chunk32 {
    uint32_t key[32];
    uint32_t valid;  // bit 4*i+q
};

__device__ __forceinline__ void load_chunk(const float* __restrict__ src, int s0, int s1, Chunk32& c) {
    float4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int j = s0 + 4 * ((int)threadIdx.x + NT * i);
        if (j + 3 < s1) {
            v[i] = __ldg(reinterpret_cast<const float4*>(src + j));
        } else {
            v[i].x = j < s1 ? src[j] : 0.f;
            v[i].y = j + 1 < s1 ? src[j + 1] : 0.f;
            v[i].z = j + 2 < s1 ? src[j + 2] : 0.f;
            v[i].w = j + 3 < s1 ? src[j + 3] : 0.f;
        }
    }
    c.valid = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int j = s0 + 4 * ((int)threadIdx.x + NT * i);
        const float f[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            c.key[4 * i + q] = order_key(f[q]);
            if (j + q < s1) c.valid |= 1u << (4 * i + q);
        }
    }
}

__device__ __forceinline__ int chunk_pos(int s0, int e) {  // e = 4*i+q
    return s0 + 4 * ((int)threadIdx.x + NT * (e >> 2)) + (e & 3);
}

// ------------------------------------------------------------------------ K1
__global__ void __launch_bounds__(NT)
topk_hist_kernel(const float* __restrict__ scores, int64_t ld, int Lq, int q_start, int k,
                 MultiWs ws) {
    const int64_t row = blockIdx.y;
    const int n = row_n(row, Lq, q_start);
    const int s0 = blockIdx.x * CHUNK;
    if (n <= k || s0 >= n) return;
    const int s1 = min(n, s0 + CHUNK);
    // one private histogram per warp (plain shared atomics: no cross-warp
    // contention), merged at the end
    extern __shared__ uint32_t hw[];   // [NW][HBINS]
    for (int b = threadIdx.x; b < NW * HBINS; b += NT) hw[b] = 0;
    __syncthreads();
    const float* src = scores + row * ld;
    uint32_t* mine = hw + (threadIdx.x >> 5) * HBINS;
    Chunk32 c;
    load_chunk(src, s0, s1, c);
#pragma unroll
    for (int e = 0; e < 32; ++e)
        if ((c.valid >> e) & 1u) atomicAdd(&mine[digit11(c.key[e])], 1u);
    __syncthreads();
    uint32_t* gh = ws.hist + row * HBINS;
    for (int b = threadIdx.x; b < HBINS; b += NT) {
        uint32_t sum = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) sum += hw[w * HBINS + b];
        if (sum) atomicAdd(&gh[b], sum);
    }
}

// ------------------------------------------------------------------------ K2
__global__ void __launch_bounds__(NT)
topk_cand_kernel(const float* __restrict__ scores, int64_t ld, int Lq, int q_start, int k,
                 int32_t* __restrict__ idx, MultiWs ws) {
    const int64_t row = blockIdx.y;
    const int n = row_n(row, Lq, q_start);
    const int s0 = blockIdx.x * CHUNK;
    if (n <= k || s0 >= n) return;
    const int s1 = min(n, s0 + CHUNK);
    const int nch = (n + CHUNK - 1) / CHUNK;
    const int lane = threadIdx.x & 31;

    extern __shared__ uint32_t dyn[];          // resolve: cand keys + positions, chunk counts
    __shared__ uint32_t h[HBINS];
    __shared__ uint32_t warp_sum[NW];
    __shared__ uint32_t sh_d, sh_above, sh_last, sh_cnt, sh_n, sh_base;
    __shared__ SelectState<NW> st;

    const uint32_t* gh = ws.hist + row * HBINS;
    for (int b = threadIdx.x; b < HBINS; b += NT) h[b] = __ldcg(gh + b);
    if (threadIdx.x == 0) { sh_cnt = 0; sh_n = 0; }
    __syncthreads();
    find_bin11<NT>(h, (uint32_t)k, sh_d, sh_above, warp_sum);
    const uint32_t d = sh_d;

    // my chunk: count keys above bin d, append the keys of bin d
    const float* src = scores + row * ld;
    uint32_t* ctl = ws.ctl + row * RW_WORDS;
    uint32_t* ckey = ws.cand_key + row * CAPG;
    uint32_t* cpos = ws.cand_pos + row * CAPG;
    // candidates are staged in shared memory first (one global reservation
    // per chunk instead of one contended atomic per warp step)
    uint32_t* stage_key = dyn;
    uint32_t* stage_pos = dyn + CAPS;
    uint32_t above = 0;
    Chunk32 c;
    load_chunk(src, s0, s1, c);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const bool live = (c.valid >> e) & 1u;
        const uint32_t key = c.key[e];
        const uint32_t dg = digit11(key);
        above += (live && dg > d) ? 1u : 0u;
        const bool cand = live && dg == d;
        const uint32_t bal = __ballot_sync(0xffffffffu, cand);
        if (bal) {
            uint32_t base = 0;
            if (lane == __ffs(bal) - 1) base = atomicAdd(&sh_n, __popc(bal));
            base = __shfl_sync(0xffffffffu, base, __ffs(bal) - 1);
            const uint32_t slot = base + __popc(bal & ((1u << lane) - 1u));
            if (cand && slot < CAPS) {
                stage_key[slot] = key;
                stage_pos[slot] = (uint32_t)chunk_pos(s0, e);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // a chunk with more candidates than it can stage forces the row onto
        // the one-CTA fallback (reserve past the row's capacity)
        const uint32_t n_c = sh_n;
        sh_base = atomicAdd(&ctl[RW_CAND_N], n_c <= (uint32_t)CAPS ? n_c : (uint32_t)CAPG + 1u);
    }
    __syncthreads();
    {
        const uint32_t n_c = min(sh_n, (uint32_t)CAPS);
        for (uint32_t j = threadIdx.x; j < n_c; j += NT) {
            const uint32_t slot = sh_base + j;
            if (slot < (uint32_t)CAPG) {
                ckey[slot] = stage_key[j];
                cpos[slot] = stage_pos[j];
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
    if (lane == 0) atomicAdd(&sh_cnt, above);
    __threadfence();   // this chunk's candidates are visible before it arrives
    __syncthreads();
    if (threadIdx.x == 0) {
        ws.chunk_gt[row * ws.nch + blockIdx.x] = sh_cnt;
        __threadfence();
        sh_last = atomicAdd(&ctl[RW_ARRIVE], 1u) == (uint32_t)(nch - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (!sh_last) return;

    // ---------------- the last chunk of the row resolves it
    __threadfence();
    const uint32_t m_all = __ldcg(&ctl[RW_CAND_N]);
    int32_t* dst = idx + row * (int64_t)k;
    if (m_all > (uint32_t)CAPG) {
        // the candidate bin overflowed: run the whole row here
        select_row<NT>(src, n, k, dst, nullptr, 0, st);
        if (threadIdx.x == 0) ctl[RW_DONE] = 1u;
        return;
    }
    const int m = (int)m_all;
    uint32_t* skey = dyn;                 // [CAPG]
    uint32_t* spos = dyn + CAPG;          // [CAPG]
    uint32_t* sel = dyn + 2 * CAPG;       // [nch] selected per chunk
    for (int j = threadIdx.x; j < m; j += NT) {
        skey[j] = __ldcg(ckey + j);
        spos[j] = __ldcg(cpos + j);
    }
    for (int c = threadIdx.x; c < nch; c += NT) sel[c] = __ldcg(ws.chunk_gt + row * ws.nch + c);
    __syncthreads();
    const uint32_t need1 = (uint32_t)k - sh_above;   // keys still to take from bin d
    select_smem_known<NT>(skey, m, need1, d, HBITS, st);
    const uint32_t tau = st.prefix, need_eq = st.need;
    __syncthreads();
    // ties at tau: keep the need_eq smallest positions among the equal keys
    uint32_t n_eq = 0;
    for (int j = threadIdx.x; j < m; j += NT) n_eq += skey[j] == tau ? 1u : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    if (threadIdx.x == 0) sh_cnt = 0;
    __syncthreads();
    if (lane == 0) atomicAdd(&sh_cnt, n_eq);
    __syncthreads();
    uint32_t pos_cut = 0xffffffffu;                 // every equal key is kept
    if (sh_cnt > need_eq) {
        for (int j = threadIdx.x; j < m; j += NT) spos[j] = skey[j] == tau ? ~spos[j] : 0u;
        __syncthreads();
        select_smem<NT>(spos, m, need_eq, st);
        pos_cut = ~st.prefix;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < m; j += NT) {
        const uint32_t key = skey[j];
        const uint32_t pos = __ldcg(cpos + j);
        if (key > tau || (key == tau && pos <= pos_cut)) atomicAdd(&sel[pos / CHUNK], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t run = 0;
        for (int c = 0; c < nch; ++c) {
            ws.chunk_off[row * ws.nch + c] = run;
            run += sel[c];
        }
        ctl[RW_TAU] = tau;
        ctl[RW_POS_CUT] = pos_cut;
    }
}

// ------------------------------------------------------------------------ K3
__global__ void __launch_bounds__(NT)
topk_write_kernel(const float* __restrict__ scores, int64_t ld, int Lq, int q_start, int k,
                  int32_t* __restrict__ idx, MultiWs ws) {
    const int64_t row = blockIdx.y;
    const int n = row_n(row, Lq, q_start);
    const int s0 = blockIdx.x * CHUNK;
    int32_t* dst = idx + row * (int64_t)k;
    if (n <= k) {
        if (blockIdx.x == 0)
            for (int j = threadIdx.x; j < k; j += NT) dst[j] = j < n ? j : -1;
        return;
    }
    if (s0 >= n) return;
    const uint32_t* ctl = ws.ctl + row * RW_WORDS;
    if (__ldcg(&ctl[RW_DONE])) return;
    const int s1 = min(n, s0 + CHUNK);
    const uint32_t tau = __ldcg(&ctl[RW_TAU]);
    const uint32_t pos_cut = __ldcg(&ctl[RW_POS_CUT]);
    const uint32_t off = __ldcg(ws.chunk_off + row * ws.nch + blockIdx.x);
    const float* src = scores + row * ld;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __shared__ uint32_t wcnt[NW];
    // each warp owns a contiguous segment of CHUNK/NW scores: 8 steps of 128,
    // lane l holding elements 4l..4l+3 of each step (all loads issued first)
    const int a = s0 + warp * (CHUNK / NW);
    float4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int j = a + 128 * i + 4 * lane;
        if (j + 3 < s1) {
            v[i] = __ldg(reinterpret_cast<const float4*>(src + j));
        } else {
            v[i].x = j < s1 ? src[j] : 0.f;
            v[i].y = j + 1 < s1 ? src[j + 1] : 0.f;
            v[i].z = j + 2 < s1 ? src[j + 2] : 0.f;
            v[i].w = j + 3 < s1 ? src[j + 3] : 0.f;
        }
    }
    uint32_t keep = 0;   // bit 4*i+q
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int j = a + 128 * i + 4 * lane;
        const float f[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t key = order_key(f[q]);
            const bool kp = j + q < s1 && (key > tau || (key == tau && (uint32_t)(j + q) <= pos_cut));
            keep |= (kp ? 1u : 0u) << (4 * i + q);
        }
    }
    uint32_t cnt = __popc(keep);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) wcnt[warp] = cnt;
    __syncthreads();
    uint32_t w_off = off;
    for (int w = 0; w < warp; ++w) w_off += wcnt[w];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t mine = (keep >> (4 * i)) & 15u;
        const uint32_t n_mine = __popc(mine);
        uint32_t incl = n_mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t2 = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t2;
        }
        uint32_t pos = w_off + incl - n_mine;
        const int j = a + 128 * i + 4 * lane;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if ((mine >> q) & 1u) dst[pos++] = j + q;
        w_off += __shfl_sync(0xffffffffu, incl, 31);
    }
}

MultiWs carve(void* scratch, int64_t rows, int nch) {
    MultiWs w;
    uint32_t* p = static_cast<uint32_t*>(scratch);
    w.hist = p;
    p += rows * HBINS;
    w.ctl = p;
    p += rows * RW_WORDS;
    w.chunk_gt = p;
    p += rows * nch;
    w.chunk_off = p;
    p += rows * nch;
    w.cand_key = p;
    p += rows * CAPG;
    w.cand_pos = p;
    w.nch = nch;
    return w;
}

}  // namespace

bool topk_multi_applies(ic_rows r, int k) {
    const int64_t rows = (int64_t)r.B * r.Lq;
    const int n_max = r.q_start + r.Lq;
    const int nch = (n_max + CHUNK - 1) / CHUNK;
    return rows <= 256 && n_max >= 2 * CHUNK && n_max > k && nch <= MAX_CHUNKS;
}

size_t topk_multi_scratch_bytes(ic_rows r, int k) {
    if (!topk_multi_applies(r, k)) return 0;
    const int64_t rows = (int64_t)r.B * r.Lq;
    const int nch = (r.q_start + r.Lq + CHUNK - 1) / CHUNK;
    return sizeof(uint32_t) * (size_t)rows * (HBINS + RW_WORDS + 2 * (size_t)nch + 2 * CAPG);
}

ic_status launch_topk_multi(const float* scores, int64_t ld, ic_rows r, int k, int32_t* idx,
                            void* scratch, cudaStream_t s) {
    const int64_t rows = (int64_t)r.B * r.Lq;
    const int nch = (r.q_start + r.Lq + CHUNK - 1) / CHUNK;
    MultiWs ws = carve(scratch, rows, nch);
    // per-call state that must start at zero: row histograms and control words
    if (cudaMemsetAsync(ws.hist, 0, sizeof(uint32_t) * rows * (HBINS + RW_WORDS), s) != cudaSuccess)
        return cuda_error("topk_multi");
    const size_t smem2 = sizeof(uint32_t) * std::max<size_t>(2 * CAPG + (size_t)nch, 2 * CAPS);
    if (cudaFuncSetAttribute(topk_cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem2) != cudaSuccess ||
        cudaFuncSetAttribute(topk_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(sizeof(uint32_t) * NW * HBINS)) != cudaSuccess)
        return cuda_error("topk_multi");
    dim3 grid(nch, (unsigned)rows);
    topk_hist_kernel<<<grid, NT, sizeof(uint32_t) * NW * HBINS, s>>>(scores, ld, r.Lq, r.q_start, k, ws);
    count_launch(IC_LK_TOPK);
    topk_cand_kernel<<<grid, NT, smem2, s>>>(scores, ld, r.Lq, r.q_start, k, idx, ws);
    count_launch(IC_LK_TOPK);
    topk_write_kernel<<<grid, NT, 0, s>>>(scores, ld, r.Lq, r.q_start, k, idx, ws);
    count_launch(IC_LK_TOPK);
    return last_launch_status();
}

}  // namespace ic
