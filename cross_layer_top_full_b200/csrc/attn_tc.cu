// attn_tc.cu -- sparse multi-query attention over a 576-wide latent KV cache
// on the tcgen05 tensor cores, with a split-k path for decode.
//
// For query row (b,i) at position t, head h in 0..127 and the selected key
// rows J (valid entries of idx[b,i,:]):
//   p = softmax_j(scale * q[b,i,h,0:576] . KV[b,j,0:576]),
//   out[b,i,h,0:512] = sum_j p_j KV[b,j,0:512]
// (core attention over the k selected keys, O(Lk): IndexCache summary, es
// page, section 1; the value is the first 512 columns of the latent row).
//
// Why two CTAs per query row: the accumulator O is 128 heads x 512 float32,
// which is all of one SM's tensor memory.  A cluster of two CTAs therefore
// splits the latent dimension evenly: CTA r gathers only its 288 columns of
// every selected row (value columns 256r..256r+255 and rope columns
// 512+32r..512+32r+31), computes the partial logits S_r = Q_r K_r^T on the
// tensor core, scales them to base-2 units and swaps them with its partner
// through distributed shared memory as float16 (both CTAs round their own
// half the same way and add the halves in the same order, so both run the
// very same online softmax).  Each then accumulates its own 256 value
// columns, O_r += P V_r, in TMEM.  No key byte is gathered twice and no flop
// is done twice.
//
// Per CTA (416 threads), persistent over work units (one unit = one query
// row, or one split of a row's indices in decode):
//   warps 0-3  gather: per unit, one pass over the unit's indices computes
//              the per-block validity masks and the block count; then
//              16-byte cp.async of the selected rows' columns into swizzled
//              tiles (3 stages of 64 keys); invalid rows are zero-filled;
//   warps 4-11 softmax, two warpgroups (thread = head = TMEM lane; warpgroup
//              w takes keys 32w..32w+31 of each 64-key block): partial S
//              from TMEM, rounded to float16 and sent straight into the
//              partner's tile with st.async (counted in bytes on the
//              partner's mbarrier, no fence or arrive on the sender), row
//              max over all 64 keys computed by both warpgroups, online
//              softmax in base
//              2 with lazy rescaling (O is rescaled only when the running max
//              grows by more than 2^8), P as bf16 written back into TMEM over
//              its S columns, final normalisation and store;
//   warp 12    TMEM allocation, TMA load of Q_r (the next unit's Q is loaded
//              while the current unit finishes), single-thread MMA issue:
//              S(j) = Q_r K_r(j)^T (K = 288), then O += P(j-1) V_r(j-1) with
//              P read from TMEM ("TS" form), software-pipelined so the tensor
//              core works on block j while block j-1 is in softmax.
// TMEM: O at columns 0..255, two S/P buffers at 256..319 and 320..383.
// Shared memory: Q_r 72 KB, 3 KV stages of 36 KB, 2 float16 logit tiles of
// 16 KB (written by the partner), per-unit masks, barriers (~219 KB).
//
// Decode (few query rows): each row's k indices are split over several CTA
// pairs, which write unnormalised (O, m, l) partials; a small combine kernel
// merges them by log-sum-exp.
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "sm100.cuh"

namespace ic {
namespace {

using namespace sm100;

constexpr int HQ = 128;
constexpr int KVW = 576;             // latent row width (K), first 512 = V
constexpr int DV = 512;
constexpr int NB = 64;               // keys per block
constexpr int Q_ATOM = HQ * 128;     // one 64-column slice of Q (128-byte rows)
constexpr int Q_ROPE = HQ * 64;      // the 32 rope columns of Q (64-byte rows)
constexpr int KV_ATOM = NB * 128;    // one 64-column slice of a key block
constexpr int KV_ROPE = NB * 64;     // the 32 rope columns of a key block
constexpr int KV_STAGE = 4 * KV_ATOM + KV_ROPE;     // 36 KB
constexpr int NSTAGE = 3;
constexpr int X_TILE = HQ * NB * 2;                 // 16 KB of float16 logits
constexpr int MAX_UNIT_BLOCKS = 64;                 // at most 4096 indices per unit
constexpr int OFF_Q = 0;
constexpr int OFF_KV = 4 * Q_ATOM + Q_ROPE;         // 72 KB
constexpr int OFF_X = OFF_KV + NSTAGE * KV_STAGE;   // partner's float16 logits
constexpr int OFF_MASK = OFF_X + 2 * X_TILE;
constexpr int OFF_BARS = OFF_MASK + 2 * MAX_UNIT_BLOCKS * 8;
constexpr int N_THREADS = 416;
constexpr int TMEM_COLS = 512;
constexpr uint32_t TM_O = 0;
constexpr uint32_t TM_S = 256;                      // S/P buffer s at TM_S + 64 s
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_THRESHOLD = 8.f;            // log2 units
constexpr float HALF_MAX = 65504.f;

struct __align__(8) AttnBars {
    uint64_t q_full, q_empty;
    uint64_t kv_full[NSTAGE], kv_empty[NSTAGE];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2];
    uint64_t x_full[2];
    uint64_t o_done, o_final, o_free;
    uint64_t info_full[2], info_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int n_blocks[2];
    int red[2][4];
    uint64_t scan_done[2];      // gather warps: per-unit reduction of the last valid index
    uint64_t l_ready[2];        // softmax warpgroups: per-unit row sums published
    float half_l[2][2][HQ];     // [unit parity][warpgroup][row] row sum at the end of a unit
};

constexpr size_t SMEM_BYTES = 1024 + OFF_BARS + sizeof(AttnBars);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

__device__ __forceinline__ bool idx_valid(int v, int t, int T) { return v >= 0 && v <= t && v < T; }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b, float& ra, float& rb) {
    __nv_bfloat16 x = __float2bfloat16_rn(a), y = __float2bfloat16_rn(b);
    ra = __bfloat162float(x);
    rb = __bfloat162float(y);
    return (uint32_t)__bfloat16_as_ushort(x) | ((uint32_t)__bfloat16_as_ushort(y) << 16);
}

// float16 pair of two base-2 logits (clamped to the float16 range), and the
// rounded values back as float
__device__ __forceinline__ uint32_t pack_half(float a, float b, float& ra, float& rb) {
    const __half x = __float2half_rn(fminf(fmaxf(a, -HALF_MAX), HALF_MAX));
    const __half y = __float2half_rn(fminf(fmaxf(b, -HALF_MAX), HALF_MAX));
    ra = __half2float(x);
    rb = __half2float(y);
    return (uint32_t)__half_as_ushort(x) | ((uint32_t)__half_as_ushort(y) << 16);
}

__device__ __forceinline__ void unpack_half(uint32_t w, float& a, float& b) {
    a = __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
    b = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
}

struct AttnArgs {
    const __nv_bfloat16* kv;
    const int32_t* idx;
    __nv_bfloat16* out;
    float* part_o;      // [units][128][512] (split-k only)
    float2* part_ml;    // [units][128]      (split-k only)
    uint32_t* status;
    int k, B, Lq, q_start, T;
    int splits, keys_per_split, n_units;
    float scale_log2;
};

struct Unit {
    int row, b, t, e0, e1, unit;
};

__device__ __forceinline__ Unit decode_unit(const AttnArgs& a, int seq) {
    Unit u;
    u.unit = a.n_units - 1 - seq;               // heaviest rows first in prefill
    u.row = u.unit / a.splits;
    const int split = u.unit - u.row * a.splits;
    u.b = u.row / a.Lq;
    u.t = a.q_start + (u.row - u.b * a.Lq);
    u.e0 = split * a.keys_per_split;
    u.e1 = min(a.k, u.e0 + a.keys_per_split);
    return u;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(N_THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_qr,
               const AttnArgs args) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    AttnBars* bars = reinterpret_cast<AttnBars*>(smem + OFF_BARS);
    uint32_t* masks = reinterpret_cast<uint32_t*>(smem + OFF_MASK);   // [2][2*MAX_UNIT_BLOCKS]
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t r = cluster_rank();
    const uint32_t peer = r ^ 1u;
    const int pair = (int)(blockIdx.x >> 1);
    const int n_pairs = (int)(gridDim.x >> 1);
    volatile int* abort = &bars->abort;
    uint32_t* status = args.status;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&bars->kv_full[s], 128);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->s_free[s], 1);
            mbar_init(&bars->p_full[s], 8);
            mbar_init(&bars->x_full[s], 1);
            mbar_init(&bars->info_full[s], 1);
            mbar_init(&bars->info_empty[s], 9);
        }
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->o_final, 1);
        mbar_init(&bars->o_free, 8);
        mbar_init(&bars->drain, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->scan_done[s], 4);
            mbar_init(&bars->l_ready[s], 8);
        }
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 12) tmem_alloc<TMEM_COLS>(&bars->tmem_base);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();  // the partner's barriers are initialised before any remote arrive
    const uint32_t tmem = bars->tmem_base;

    if (warp < 4) {
        // ------------------------------------------------------------ gather
        const int gt = threadIdx.x;
        const int krow = gt >> 1;                 // key row of the block this thread fills
        const int half = gt & 1;                  // which half of the row's 16-byte chunks
        uint32_t g = 0;
        int n = 0;
        for (int seq = pair; seq < args.n_units; seq += n_pairs, ++n) {
            const Unit u = decode_unit(args, seq);
            const int32_t* idx_row = args.idx + (int64_t)u.row * args.k;
            const int ip = n & 1;
            if (!warp_wait(&bars->info_empty[ip], ((n >> 1) & 1) ^ 1, status, abort)) break;
            // validity masks of the unit's blocks and its last valid index
            int last = -1;
            const int n_ent = u.e1 - u.e0;
            for (int base = 0; base < n_ent; base += 128) {
                const int e = u.e0 + base + gt;
                const int v = e < u.e1 ? idx_row[e] : -1;
                const bool ok = idx_valid(v, u.t, args.T);
                if (!ok && v != -1 && r == 0) flag_status(status, IC_DEV_INDEX_RANGE);
                if (ok) last = e;
                const uint32_t bal = __ballot_sync(0xffffffffu, ok);
                const int word = base / 32 + warp;
                if (lane == 0 && word < 2 * MAX_UNIT_BLOCKS) masks[ip * 2 * MAX_UNIT_BLOCKS + word] = bal;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
            if (lane == 0) bars->red[ip][warp] = last;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->scan_done[ip]);
            if (!warp_wait(&bars->scan_done[ip], (n >> 1) & 1, status, abort)) break;
            last = max(max(bars->red[ip][0], bars->red[ip][1]), max(bars->red[ip][2], bars->red[ip][3]));
            const int nb = last < 0 ? 0 : (last - u.e0) / NB + 1;
            if (gt == 0) {
                bars->n_blocks[ip] = nb;
                mbar_arrive(&bars->info_full[ip]);
            }
            const __nv_bfloat16* kv_b = args.kv + (int64_t)u.b * args.T * KVW;
            bool ok_all = true;
            for (int j = 0; j < nb; ++j, ++g) {
                const int s = g % NSTAGE;
                const int e = u.e0 + j * NB + krow;
                const int v = e < u.e1 ? idx_row[e] : -1;   // issued before the wait
                if (!warp_wait(&bars->kv_empty[s], ((g / NSTAGE) & 1) ^ 1, status, abort)) {
                    ok_all = false;
                    break;
                }
                const bool ok = idx_valid(v, u.t, args.T);
                const __nv_bfloat16* src = kv_b + (int64_t)(ok ? v : 0) * KVW;
                const uint32_t nbytes = ok ? 16u : 0u;
                const uint32_t stage = smem_base + OFF_KV + s * KV_STAGE;
#pragma unroll
                for (int c = 0; c < 16; ++c) {       // value columns: atoms 2*half, 2*half+1
                    const int a = 2 * half + (c >> 3), ch = c & 7;
                    cp_async16(stage + a * KV_ATOM + krow * 128 + ((ch ^ (krow & 7)) << 4),
                               src + r * 256 + a * 64 + ch * 8, nbytes);
                }
#pragma unroll
                for (int c = 2 * half; c < 2 * half + 2; ++c)   // rope columns (64-byte rows)
                    cp_async16(stage + 4 * KV_ATOM + krow * 64 + ((c ^ ((krow >> 1) & 3)) << 4),
                               src + 512 + r * 32 + c * 8, nbytes);
                cp_async_arrive_noinc(&bars->kv_full[s]);
            }
            if (!ok_all) break;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp < 12) {
        // ------------------------------------------------------------ softmax
        const int quad = warp & 3;                // TMEM lanes 32*quad .. +31
        const int wg = (warp - 4) >> 2;           // warpgroup: keys 32*wg .. 32*wg+31 of a block
        const int h = quad * 32 + lane;           // head of this thread
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const bool arm = warp == 4 && lane == 0;  // arms x_full with the expected bytes
        uint32_t g = 0, o_use = 0;
        int n = 0;
        bool ok = true;
        for (int seq = pair; seq < args.n_units && ok; seq += n_pairs, ++n) {
            const Unit u = decode_unit(args, seq);
            const int ip = n & 1;
            if (!warp_wait(&bars->info_full[ip], (n >> 1) & 1, status, abort)) { ok = false; break; }
            const int nb = bars->n_blocks[ip];
            float m_use = -INFINITY, l = 0.f;
            for (int j = 0; j < nb; ++j, ++g) {
                const int s = g & 1;
                const uint32_t ph = (g >> 1) & 1;
                if (arm) mbar_arrive_expect_tx(&bars->x_full[s], X_TILE);
                if (!warp_wait(&bars->s_full[s], ph, status, abort)) { ok = false; break; }
                tc_fence_after();
                // own partial logits of all 64 keys -> base-2 units -> float16;
                // this warpgroup sends its 32 to the partner
                float xo[NB];
                uint32_t hw[NB / 2];
                {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(t_lane + TM_S + 64 * s, r0);
                    tmem_ld32(t_lane + TM_S + 64 * s + 32, r1);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        hw[x] = pack_half(__uint_as_float(r0[2 * x]) * args.scale_log2,
                                          __uint_as_float(r0[2 * x + 1]) * args.scale_log2,
                                          xo[2 * x], xo[2 * x + 1]);
                        hw[16 + x] = pack_half(__uint_as_float(r1[2 * x]) * args.scale_log2,
                                               __uint_as_float(r1[2 * x + 1]) * args.scale_log2,
                                               xo[32 + 2 * x], xo[32 + 2 * x + 1]);
                    }
                }
                {
                    // my warpgroup's 32 values go straight into row h of the
                    // partner's tile s; each 16-byte st.async counts its bytes on
                    // the partner's x_full[s] (no fence or arrive on this side)
                    const uint32_t x_remote = map_to_rank(smem_base + OFF_X + s * X_TILE + h * 128, peer);
                    const uint32_t bar_remote = map_to_rank(smem_u32(&bars->x_full[s]), peer);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int c = 4 * wg + q;
                        const uint32_t w0 = wg ? hw[16 + 4 * q] : hw[4 * q];
                        const uint32_t w1 = wg ? hw[17 + 4 * q] : hw[4 * q + 1];
                        const uint32_t w2 = wg ? hw[18 + 4 * q] : hw[4 * q + 2];
                        const uint32_t w3 = wg ? hw[19 + 4 * q] : hw[4 * q + 3];
                        st_async_v4(x_remote + ((c ^ (h & 7)) << 4), w0, w1, w2, w3, bar_remote);
                    }
                }
                const uint32_t m_lo = masks[ip * 2 * MAX_UNIT_BLOCKS + 2 * j];
                const uint32_t m_hi = masks[ip * 2 * MAX_UNIT_BLOCKS + 2 * j + 1];
                if (!warp_wait_cluster(&bars->x_full[s], ph, status, abort)) { ok = false; break; }
                const uint4* xp = reinterpret_cast<const uint4*>(smem + OFF_X + s * X_TILE + h * 128);
                float xs[NB];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 w4 = xp[c ^ (h & 7)];
                    const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float p0, p1;
                        unpack_half(wv[e], p0, p1);
                        const int kk = 8 * c + 2 * e;
                        // canonical order: half 0 + half 1 on both CTAs
                        const float s0 = r == 0 ? xo[kk] + p0 : p0 + xo[kk];
                        const float s1 = r == 0 ? xo[kk + 1] + p1 : p1 + xo[kk + 1];
                        const uint32_t mw = kk < 32 ? m_lo : m_hi;
                        xs[kk] = ((mw >> (kk & 31)) & 1u) ? s0 : -INFINITY;
                        xs[kk + 1] = ((mw >> ((kk + 1) & 31)) & 1u) ? s1 : -INFINITY;
                    }
                }
                // row max over all 64 keys (both warpgroups compute it: no exchange)
                float mx[32];
#pragma unroll
                for (int x = 0; x < 32; ++x) mx[x] = fmaxf(xs[2 * x], xs[2 * x + 1]);
#pragma unroll
                for (int w = 16; w > 0; w >>= 1)
#pragma unroll
                    for (int x = 0; x < w; ++x) mx[x] = fmaxf(mx[x], mx[x + w]);
                const float mloc = mx[0];
                float alpha = 1.f;
                bool rescale = false;
                if (mloc > m_use + RESCALE_THRESHOLD || (m_use == -INFINITY && mloc > -INFINITY)) {
                    alpha = m_use == -INFINITY ? 0.f : ex2_approx(m_use - mloc);
                    m_use = mloc;
                    rescale = true;
                }
                uint32_t pw[16];
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const float a0 = wg ? xs[32 + 2 * x] : xs[2 * x];
                    const float a1 = wg ? xs[33 + 2 * x] : xs[2 * x + 1];
                    const float p0 = a0 == -INFINITY ? 0.f : ex2_approx(a0 - m_use);
                    const float p1 = a1 == -INFINITY ? 0.f : ex2_approx(a1 - m_use);
                    const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                    pw[x] = *reinterpret_cast<const uint32_t*>(&pb);
                    ps[x & 3] += __low2float(pb) + __high2float(pb);
                }
                l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
                if (rescale && j > 0) {
                    // O must hold P(j-1) V(j-1) before it is rescaled; each
                    // warpgroup rescales its 128 of the 256 value columns
                    if (!warp_wait(&bars->o_done, (g - 1) & 1, status, abort)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        const uint32_t col = TM_O + 128 * wg + 32 * c;
                        tmem_ld32(t_lane + col, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
                        tmem_st32(t_lane + col, o);
                    }
                }
                tmem_st16(t_lane + TM_S + 64 * s + 16 * wg, pw);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[s]);
            }
            if (!ok) break;
            // ---------------------------------------------------------- unit epilogue
            const bool split = args.splits > 1;
            bars->half_l[ip][wg][h] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->l_ready[ip]);
            if (!warp_wait(&bars->l_ready[ip], (n >> 1) & 1, status, abort)) { ok = false; break; }
            const float l_all = bars->half_l[ip][0][h] + bars->half_l[ip][1][h];
            if (nb > 0) {
                if (!warp_wait(&bars->o_final, o_use & 1, status, abort)) { ok = false; break; }
                tc_fence_after();
                const float inv = l_all > 0.f ? 1.f / l_all : 0.f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    const int ocol = 128 * wg + 32 * c;          // column of O in TMEM
                    tmem_ld32(t_lane + TM_O + ocol, o);
                    tmem_ld_wait();
                    const int col = (int)r * 256 + ocol;        // column of the output row
                    if (!split) {
                        uint4* dst = reinterpret_cast<uint4*>(args.out + ((int64_t)u.row * HQ + h) * DV + col);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            float d0, d1;
                            uint4 pk;
                            pk.x = pack_bf16(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv, d0, d1);
                            pk.y = pack_bf16(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv, d0, d1);
                            pk.z = pack_bf16(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv, d0, d1);
                            pk.w = pack_bf16(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv, d0, d1);
                            dst[v] = pk;
                        }
                    } else {
                        float4* dst = reinterpret_cast<float4*>(args.part_o + ((int64_t)u.unit * HQ + h) * DV + col);
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                                 __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->o_free);
                ++o_use;
            } else if (!split) {
                // no valid key: the output row is zero
                uint4* dst = reinterpret_cast<uint4*>(args.out + ((int64_t)u.row * HQ + h) * DV + r * 256 + 128 * wg);
                for (int v = 0; v < 16; ++v) dst[v] = make_uint4(0, 0, 0, 0);
            }
            if (split && r == 0 && wg == 0)
                args.part_ml[(int64_t)u.unit * HQ + h] = make_float2(m_use, nb > 0 ? l_all : 0.f);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->info_empty[ip]);
        }
    } else {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_f32acc(1, 1, HQ, NB);            // S = Q K^T
            constexpr uint32_t id_pv = idesc_f32acc(1, 1, HQ, 256, 0, 1);    // O += P V (V MN-major)
            const uint32_t q_addr = smem_base + OFF_Q;
            uint32_t g = 0, o_use = 0;
            bool issued = false, ok = true;
            int nb_next = -1;
            bool q_loaded_next = false;
            auto load_q = [&](int seq) {
                const Unit u = decode_unit(args, seq);
                mbar_arrive_expect_tx(&bars->q_full, 4 * Q_ATOM + Q_ROPE);
                for (int a = 0; a < 4; ++a)
                    tma_load_2d(smem + OFF_Q + a * Q_ATOM, &map_q, &bars->q_full, (int)r * 256 + a * 64,
                                u.row * HQ);
                tma_load_2d(smem + OFF_Q + 4 * Q_ATOM, &map_qr, &bars->q_full, 512 + (int)r * 32,
                            u.row * HQ);
            };
            auto pv = [&](uint32_t gg, bool first) -> bool {
                const int s = gg & 1;
                if (!mbar_wait(&bars->p_full[s], (gg >> 1) & 1, status, abort)) return false;
                if (first && o_use > 0 &&
                    !mbar_wait(&bars->o_free, (o_use - 1) & 1, status, abort))
                    return false;
                tc_fence_after();
                const uint32_t v_addr = smem_base + OFF_KV + (gg % NSTAGE) * KV_STAGE;
#pragma unroll
                for (int kk = 0; kk < NB / 16; ++kk) {
                    const uint64_t db = desc_sw128(v_addr + kk * 16 * 128, 8192, 1024);
                    mma_bf16_ts(tmem + TM_O, tmem + TM_S + 64 * s + kk * 8, db, id_pv,
                                (!first || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bars->kv_empty[gg % NSTAGE]);
                mma_commit(&bars->s_free[s]);
                mma_commit(&bars->o_done);
                return true;
            };
            int n = 0;
            for (int seq = pair; seq < args.n_units && ok; seq += n_pairs, ++n) {
                int nb;
                if (nb_next >= 0) {
                    nb = nb_next;
                    nb_next = -1;
                } else {
                    if (!mbar_wait(&bars->info_full[n & 1], (n >> 1) & 1, status, abort)) break;
                    nb = bars->n_blocks[n & 1];
                    mbar_arrive(&bars->info_empty[n & 1]);
                }
                if (nb == 0) continue;
                if (!q_loaded_next) {
                    if (o_use > 0 && !mbar_wait(&bars->q_empty, (o_use - 1) & 1, status, abort)) break;
                    load_q(seq);
                }
                q_loaded_next = false;
                if (!mbar_wait(&bars->q_full, o_use & 1, status, abort)) break;
                for (int j = 0; j < nb; ++j, ++g) {
                    const int s = g & 1;
                    const int ks = g % NSTAGE;
                    if (!mbar_wait(&bars->kv_full[ks], (g / NSTAGE) & 1, status, abort) ||
                        !mbar_wait(&bars->s_free[s], ((g >> 1) & 1) ^ 1, status, abort)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_smem();  // cp.async data -> tensor-core reads
                    tc_fence_after();
                    const uint32_t kv_addr = smem_base + OFF_KV + ks * KV_STAGE;
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t da = desc_sw128(q_addr + a * Q_ATOM + kk * 32, 16, 1024);
                            const uint64_t db = desc_sw128(kv_addr + a * KV_ATOM + kk * 32, 16, 1024);
                            mma_bf16(tmem + TM_S + 64 * s, da, db, id_s, (a | kk) != 0);
                        }
                    }
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const uint64_t da = desc_sw64(q_addr + 4 * Q_ATOM + kk * 32);
                        const uint64_t db = desc_sw64(kv_addr + 4 * KV_ATOM + kk * 32);
                        mma_bf16(tmem + TM_S + 64 * s, da, db, id_s, 1u);
                    }
                    issued = true;
                    mma_commit(&bars->s_full[s]);
                    if (j == nb - 1) {
                        // Q is free once these MMAs finish: fetch the next unit's Q now
                        mma_commit(&bars->q_empty);
                        if (seq + n_pairs < args.n_units) {
                            const int n1 = n + 1;
                            if (!mbar_wait(&bars->info_full[n1 & 1], (n1 >> 1) & 1, status, abort)) {
                                ok = false;
                                break;
                            }
                            nb_next = bars->n_blocks[n1 & 1];
                            mbar_arrive(&bars->info_empty[n1 & 1]);
                            if (nb_next > 0) {
                                if (!mbar_wait(&bars->q_empty, o_use & 1, status, abort)) {
                                    ok = false;
                                    break;
                                }
                                load_q(seq + n_pairs);
                                q_loaded_next = true;
                            }
                        }
                    }
                    if (j >= 1 && !pv(g - 1, j == 1)) { ok = false; break; }
                }
                if (!ok) break;
                if (!pv(g - 1, nb == 1)) break;
                mma_commit(&bars->o_final);
                ++o_use;
            }
            if (issued) {
                mma_commit(&bars->drain);   // every MMA of this CTA has finished
                mbar_wait(&bars->drain, 0, status, abort);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the partner no longer writes into this CTA's shared memory
    if (warp == 12) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem);
    }
}

// Merge split-k partials: out = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c.
__global__ void __launch_bounds__(128)
attn_combine_kernel(const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                    int splits, __nv_bfloat16* __restrict__ out) {
    const int64_t row = blockIdx.x;
    const int h = blockIdx.y;
    const int d = threadIdx.x * 4;
    float M = -INFINITY;
    for (int c = 0; c < splits; ++c) {
        const float2 ml = part_ml[(row * splits + c) * HQ + h];
        if (ml.y > 0.f) M = fmaxf(M, ml.x);
    }
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    if (M > -INFINITY) {
        for (int c = 0; c < splits; ++c) {
            const int64_t u = row * splits + c;
            const float2 ml = part_ml[u * HQ + h];
            if (!(ml.y > 0.f)) continue;
            const float wgt = exp2f(ml.x - M);
            den += wgt * ml.y;
            const float4 o = *reinterpret_cast<const float4*>(part_o + (u * HQ + h) * DV + d);
            num.x += wgt * o.x;
            num.y += wgt * o.y;
            num.z += wgt * o.z;
            num.w += wgt * o.w;
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    __nv_bfloat16* dst = out + (row * HQ + h) * DV + d;
    dst[0] = __float2bfloat16_rn(num.x * inv);
    dst[1] = __float2bfloat16_rn(num.y * inv);
    dst[2] = __float2bfloat16_rn(num.z * inv);
    dst[3] = __float2bfloat16_rn(num.w * inv);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

// Split-k plan: number of splits of the k indices per query row.  A unit
// (one split of one row) holds at most MAX_UNIT_BLOCKS blocks of indices.
void plan_splits(const ic_rows& r, int k, int& splits, int& keys_per_split) {
    const int64_t rows = (int64_t)r.B * r.Lq;
    const int pairs = std::max(1, sm_count() / 2);
    const int nblk = ceil_div(k, NB);
    const int min_splits = ceil_div(nblk, MAX_UNIT_BLOCKS);
    splits = min_splits;
    if (rows < pairs) {
        double best = 1e30;
        for (int s = min_splits; s <= std::max(min_splits, std::min(nblk, 32)); ++s) {
            const double waves = (double)ceil_div64(rows * s, pairs);
            const double cost = waves * (ceil_div(nblk, s) + 1.5);
            if (cost < best - 1e-9) {
                best = cost;
                splits = s;
            }
        }
    }
    keys_per_split = ceil_div(nblk, splits) * NB;
    splits = ceil_div(k, keys_per_split);
}

}  // namespace

bool attn_tc_supported(const void* kmat, const void* vmat, int64_t ks, int64_t vs, ic_dtype dt,
                       int Hq, int d_qk, int d_v) {
    return dt == IC_BF16 && Hq == HQ && d_qk == KVW && d_v == DV && kmat == vmat && ks == KVW &&
           vs == KVW;
}

size_t attn_tc_scratch_bytes(ic_rows r, int k) {
    int splits, kps;
    plan_splits(r, k, splits, kps);
    if (splits <= 1) return 0;
    const size_t units = (size_t)r.B * r.Lq * splits;
    return units * HQ * DV * sizeof(float) + 256 + units * HQ * sizeof(float2);
}

ic_status launch_attn_tc(const void* q, const void* kv, int64_t ks, const int32_t* idx, int k,
                         ic_rows r, float scale, void* out, uint32_t* status, void* scratch,
                         size_t scratch_bytes, cudaStream_t s) {
    (void)ks;
    if (((uintptr_t)q & 15) || ((uintptr_t)kv & 15) || ((uintptr_t)out & 15))
        return IC_ERR_INVALID_ARG;
    auto fn = encode_fn();
    if (fn == nullptr) return IC_ERR_CUDA;
    CUtensorMap map_q, map_qr;
    cuuint64_t dims[2] = {(cuuint64_t)KVW, (cuuint64_t)r.B * r.Lq * HQ};
    cuuint64_t strides[1] = {(cuuint64_t)KVW * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)HQ};
    cuuint32_t box_r[2] = {32, (cuuint32_t)HQ};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&map_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return IC_ERR_CUDA;
    if (fn(&map_qr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box_r,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return IC_ERR_CUDA;

    AttnArgs a;
    a.kv = static_cast<const __nv_bfloat16*>(kv);
    a.idx = idx;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.status = status;
    a.k = k;
    a.B = r.B;
    a.Lq = r.Lq;
    a.q_start = r.q_start;
    a.T = r.T;
    a.scale_log2 = scale * LOG2E;
    plan_splits(r, k, a.splits, a.keys_per_split);
    const int64_t units = (int64_t)r.B * r.Lq * a.splits;
    if (2 * units > 0x7fffffff) return IC_ERR_UNSUPPORTED;
    a.n_units = (int)units;
    a.part_o = nullptr;
    a.part_ml = nullptr;
    if (a.splits > 1) {
        if (scratch_bytes < attn_tc_scratch_bytes(r, k) || scratch == nullptr) return IC_ERR_WORKSPACE;
        a.part_o = static_cast<float*>(scratch);
        a.part_ml = reinterpret_cast<float2*>(static_cast<char*>(scratch) +
                                              (size_t)units * HQ * DV * sizeof(float) + 256 -
                                              (((size_t)units * HQ * DV * sizeof(float)) & 255));
    }
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES) != cudaSuccess)
        return IC_ERR_CUDA;
    const int64_t pairs = std::min<int64_t>(units, std::max(1, sm_count() / 2));
    attn_tc_kernel<<<(unsigned)(2 * pairs), N_THREADS, SMEM_BYTES, s>>>(map_q, map_qr, a);
    count_launch(IC_LK_ATTN_TC);
    ic_status st = last_launch_status();
    if (st != IC_OK || a.splits <= 1) return st;
    dim3 grid((unsigned)((int64_t)r.B * r.Lq), HQ);
    attn_combine_kernel<<<grid, 128, 0, s>>>(a.part_o, a.part_ml, a.splits,
                                             static_cast<__nv_bfloat16*>(out));
    count_launch(IC_LK_COMBINE);
    return last_launch_status();
}

}  // namespace ic
