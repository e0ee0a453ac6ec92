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
// splits the latent dimension: CTA r gathers only its part of every selected
// row (r = 0: columns 0..255 and the 64 rope columns 512..575; r = 1:
// columns 256..511), computes the partial logits S_r = Q_r K_r^T on the
// tensor core, and the pair swaps S_r through distributed shared memory.
// Both add the halves in the same order (S_0 + S_1), so both run the very
// same online softmax; each then accumulates its own 256 value columns,
// O_r += P V_r, in TMEM.  No key byte is gathered twice and no flop is done
// twice.
//
// Per CTA (288 threads):
//   warps 0-3  gather: 16-byte cp.async of the selected rows' columns into
//              128-byte-swizzled tiles (2 stages of 64 keys); rows with an
//              invalid index are zero-filled and masked;
//   warps 4-7  softmax (thread = head = TMEM lane): partial S from TMEM,
//              exchange, online softmax in base 2 with lazy rescaling (O is
//              rescaled only when the running max grows by more than 2^8),
//              P as bf16 written back into TMEM over its S columns, final
//              normalisation and store;
//   warp 8     TMEM allocation, TMA load of Q_r, single-thread MMA issue:
//              S(j) = Q_r K_r(j)^T (K = 320 or 256), then O += P(j-1) V_r(j-1)
//              with P read from TMEM (the "TS" form), software-pipelined so
//              the tensor core works on block j while block j-1 is in softmax.
// TMEM: O at columns 0..255, two S/P buffers at 256..319 and 320..383.
//
// Decode (few query rows): each row's k indices are split over several CTA
// pairs, which write unnormalised (O, m, l) partials; a small combine kernel
// merges them by log-sum-exp.
#include <cudaTypedefs.h>

#include <algorithm>

#include "sm100.cuh"

namespace ic {
namespace {

using namespace sm100;

constexpr int HQ = 128;
constexpr int KVW = 576;             // latent row width (K), first 512 = V
constexpr int DV = 512;
constexpr int NB = 64;               // keys per block
constexpr int Q_ATOM = HQ * 128;     // bytes of one 64-column slice of Q
constexpr int KV_ATOM = NB * 128;    // bytes of one 64-column slice of a key block
constexpr int MAX_ATOMS = 5;
constexpr int KV_STAGE = MAX_ATOMS * KV_ATOM;   // 40 KB
constexpr int X_TILE = HQ * NB * 4;             // 32 KB partial-logit tile
constexpr int OFF_Q = 0;
constexpr int OFF_KV = MAX_ATOMS * Q_ATOM;      // 80 KB
constexpr int OFF_X = OFF_KV + 2 * KV_STAGE;    // 160 KB
constexpr int OFF_BARS = OFF_X + 2 * X_TILE;    // 224 KB
constexpr int N_THREADS = 288;
constexpr int TMEM_COLS = 512;
constexpr uint32_t TM_O = 0;
constexpr uint32_t TM_S = 256;                  // S/P buffer s at TM_S + 64 s
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_THRESHOLD = 8.f;        // log2 units

struct __align__(8) AttnBars {
    uint64_t q_full;
    uint64_t kv_full[2], kv_empty[2];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2];
    uint64_t x_full[2];
    uint64_t o_done, o_final;
    uint32_t tmem_base;
    int abort;
    int n_blocks;
    int red[4];
};

constexpr size_t SMEM_BYTES = 1024 + OFF_BARS + sizeof(AttnBars);

__device__ __forceinline__ int atom_col0(int r, int a) { return a < 4 ? r * 256 + a * 64 : 512; }

__device__ __forceinline__ bool idx_valid(int v, int t, int T) { return v >= 0 && v <= t && v < T; }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b, float& ra, float& rb) {
    __nv_bfloat16 x = __float2bfloat16_rn(a), y = __float2bfloat16_rn(b);
    ra = __bfloat162float(x);
    rb = __bfloat162float(y);
    return (uint32_t)__bfloat16_as_ushort(x) | ((uint32_t)__bfloat16_as_ushort(y) << 16);
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(N_THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const AttnArgs args) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    AttnBars* bars = reinterpret_cast<AttnBars*>(smem + OFF_BARS);
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t r = cluster_rank();
    const uint32_t peer = r ^ 1u;
    const int n_atoms = r == 0 ? 5 : 4;
    volatile int* abort = &bars->abort;
    uint32_t* status = args.status;

    // work unit: heaviest rows first (later rows select more keys in prefill)
    const int unit = args.n_units - 1 - (int)(blockIdx.x >> 1);
    const int row = unit / args.splits;
    const int split = unit - row * args.splits;
    const int b = row / args.Lq;
    const int t = args.q_start + (row - b * args.Lq);
    const int e0 = split * args.keys_per_split;
    const int e1 = min(args.k, e0 + args.keys_per_split);
    const int32_t* idx_row = args.idx + (int64_t)row * args.k;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->kv_full[s], 128);
            mbar_init(&bars->kv_empty[s], 1);
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->s_free[s], 1);
            mbar_init(&bars->p_full[s], 128);
            mbar_init(&bars->x_full[s], 128);
        }
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->o_final, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    // number of 64-key blocks up to the last valid index of this unit's range
    if (warp < 4) {
        int last = -1;
        for (int e = e0 + (int)threadIdx.x; e < e1; e += 128) {
            const int v = idx_row[e];
            if (idx_valid(v, t, args.T)) last = e;
            else if (v != -1 && r == 0) flag_status(status, IC_DEV_INDEX_RANGE);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
        if (lane == 0) bars->red[warp] = last;
    }
    if (warp == 8) tmem_alloc<TMEM_COLS>(&bars->tmem_base);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) {
        const int last = max(max(bars->red[0], bars->red[1]), max(bars->red[2], bars->red[3]));
        bars->n_blocks = last < 0 ? 0 : (last - e0) / NB + 1;
    }
    cluster_sync();  // partner's barriers are initialised before any remote arrive
    const int n_blocks = bars->n_blocks;
    const uint32_t tmem = bars->tmem_base;

    if (warp < 4) {
        // ------------------------------------------------------------ gather
        const int gt = threadIdx.x;
        const int krow = gt >> 1;                 // key row of the block this thread fills
        const int half = gt & 1;                  // which half of the row's 16-byte chunks
        const int per_half = n_atoms * 4;         // chunks per half-row
        for (int j = 0; j < n_blocks; ++j) {
            const int s = j & 1;
            if (!mbar_wait(&bars->kv_empty[s], ((j >> 1) & 1) ^ 1, status, abort)) break;
            const int e = e0 + j * NB + krow;
            const int v = e < e1 ? idx_row[e] : -1;
            const bool ok = idx_valid(v, t, args.T);
            const __nv_bfloat16* src_row = args.kv + ((int64_t)b * args.T + (ok ? v : 0)) * KVW;
            const uint32_t dst_row = smem_base + OFF_KV + s * KV_STAGE + krow * 128;
#pragma unroll 4
            for (int c = half * per_half; c < (half + 1) * per_half; ++c) {
                const int a = c >> 3, ch = c & 7;
                const uint32_t dst = dst_row + a * KV_ATOM + ((ch ^ (krow & 7)) << 4);
                cp_async16(dst, src_row + atom_col0(r, a) + ch * 8, ok ? 16u : 0u);
            }
            cp_async_arrive_noinc(&bars->kv_full[s]);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax
        const int quad = warp - 4;                // TMEM lanes 32*quad .. +31
        const int h = quad * 32 + lane;           // head of this thread
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        float m_use = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_blocks && ok; ++j) {
            const int s = j & 1;
            const uint32_t ph = (j >> 1) & 1;
            // validity mask of the block's 64 keys (bit = key)
            const int eb = e0 + j * NB;
            const int v_lo = eb + lane < e1 ? idx_row[eb + lane] : -1;
            const int v_hi = eb + 32 + lane < e1 ? idx_row[eb + 32 + lane] : -1;
            const uint32_t m_lo = __ballot_sync(0xffffffffu, idx_valid(v_lo, t, args.T));
            const uint32_t m_hi = __ballot_sync(0xffffffffu, idx_valid(v_hi, t, args.T));

            if (!mbar_wait(&bars->s_full[s], ph, status, abort)) { ok = false; break; }
            tc_fence_after();
            float sp[NB];
            {
                uint32_t r0[32], r1[32];
                tmem_ld32(t_lane + TM_S + 64 * s, r0);
                tmem_ld32(t_lane + TM_S + 64 * s + 32, r1);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    sp[x] = __uint_as_float(r0[x]);
                    sp[32 + x] = __uint_as_float(r1[x]);
                }
            }
            // swap partial logits with the partner CTA (row h of its X tile s)
            const uint32_t x_local = smem_base + OFF_X + s * X_TILE + h * 256;
            const uint32_t x_remote = map_to_rank(x_local, peer);
#pragma unroll
            for (int c = 0; c < 16; ++c)
                st_cluster_v4(x_remote + ((c ^ (h & 15)) << 4), sp[4 * c], sp[4 * c + 1],
                              sp[4 * c + 2], sp[4 * c + 3]);
            mbar_arrive_remote(map_to_rank(smem_u32(&bars->x_full[s]), peer));
            if (!mbar_wait_cluster(&bars->x_full[s], ph, status, abort)) { ok = false; break; }
            const float4* xp = reinterpret_cast<const float4*>(smem + OFF_X + s * X_TILE + h * 256);
            float xs[NB];
            float mloc = -INFINITY;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float4 o = xp[c ^ (h & 15)];
                const float ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int kk = 4 * c + q;
                    // canonical order S_0 + S_1 on both CTAs
                    const float sfull = r == 0 ? sp[kk] + ov[q] : ov[q] + sp[kk];
                    const bool valid = ((kk < 32 ? m_lo >> kk : m_hi >> (kk - 32)) & 1u) != 0;
                    xs[kk] = valid ? sfull * args.scale_log2 : -INFINITY;
                    mloc = fmaxf(mloc, xs[kk]);
                }
            }
            float alpha = 1.f;
            bool rescale = false;
            if (mloc > m_use + RESCALE_THRESHOLD || (m_use == -INFINITY && mloc > -INFINITY)) {
                alpha = m_use == -INFINITY ? 0.f : exp2f(m_use - mloc);
                m_use = mloc;
                rescale = true;
            }
            uint32_t pw[32];
            float psum = 0.f;
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                const float p0 = xs[2 * x] == -INFINITY ? 0.f : exp2f(xs[2 * x] - m_use);
                const float p1 = xs[2 * x + 1] == -INFINITY ? 0.f : exp2f(xs[2 * x + 1] - m_use);
                float q0, q1;
                pw[x] = pack_bf16(p0, p1, q0, q1);
                psum += q0 + q1;
            }
            l = l * alpha + psum;
            if (rescale && j > 0) {
                // O must hold P(j-1) V(j-1) before it is rescaled
                if (!mbar_wait(&bars->o_done, (j - 1) & 1, status, abort)) { ok = false; break; }
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t o[32];
                    tmem_ld32(t_lane + TM_O + 32 * c, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
                    tmem_st32(t_lane + TM_O + 32 * c, o);
                }
                tmem_st_wait();
            }
            tmem_st32(t_lane + TM_S + 64 * s, pw);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars->p_full[s]);
        }
        // ---------------------------------------------------------- epilogue
        const bool split = args.splits > 1;
        if (n_blocks > 0 && ok) {
            if (mbar_wait(&bars->o_final, 0, status, abort)) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t o[32];
                    tmem_ld32(t_lane + TM_O + 32 * c, o);
                    tmem_ld_wait();
                    const int col = (int)r * 256 + 32 * c;
                    if (!split) {
                        uint4* dst = reinterpret_cast<uint4*>(
                            args.out + ((int64_t)row * HQ + h) * DV + col);
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
                        float4* dst = reinterpret_cast<float4*>(
                            args.part_o + ((int64_t)unit * HQ + h) * DV + col);
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                                 __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
                    }
                }
            }
        } else if (n_blocks == 0 && !split) {
            // no valid key: the output row is zero
            uint4* dst = reinterpret_cast<uint4*>(args.out + ((int64_t)row * HQ + h) * DV + r * 256);
            for (int v = 0; v < 32; ++v) dst[v] = make_uint4(0, 0, 0, 0);
        }
        if (split && r == 0) args.part_ml[(int64_t)unit * HQ + h] = make_float2(m_use, n_blocks > 0 ? l : 0.f);
    } else {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_blocks > 0) {
            mbar_arrive_expect_tx(&bars->q_full, n_atoms * Q_ATOM);
            for (int a = 0; a < n_atoms; ++a)
                tma_load_2d(smem + OFF_Q + a * Q_ATOM, &map_q, &bars->q_full, atom_col0(r, a),
                            row * HQ);
            constexpr uint32_t id_s = idesc_f32acc(1, 1, HQ, NB);            // S = Q K^T
            constexpr uint32_t id_pv = idesc_f32acc(1, 1, HQ, 256, 0, 1);    // O += P V (V MN-major)
            const uint32_t q_addr = smem_base + OFF_Q;
            bool ok = mbar_wait(&bars->q_full, 0, status, abort);
            auto pv = [&](int jj) -> bool {
                const int s = jj & 1;
                if (!mbar_wait(&bars->p_full[s], (jj >> 1) & 1, status, abort)) return false;
                tc_fence_after();
                const uint32_t v_addr = smem_base + OFF_KV + s * KV_STAGE;
#pragma unroll
                for (int kk = 0; kk < NB / 16; ++kk) {
                    const uint64_t db = desc_sw128(v_addr + kk * 16 * 128, 8192, 1024);
                    mma_bf16_ts(tmem + TM_O, tmem + TM_S + 64 * s + kk * 8, db, id_pv,
                                (jj > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bars->kv_empty[s]);
                mma_commit(&bars->s_free[s]);
                mma_commit(&bars->o_done);
                return true;
            };
            for (int j = 0; j < n_blocks && ok; ++j) {
                const int s = j & 1;
                const uint32_t ph = (j >> 1) & 1;
                if (!mbar_wait(&bars->kv_full[s], ph, status, abort) ||
                    !mbar_wait(&bars->s_free[s], ph ^ 1, status, abort)) {
                    ok = false;
                    break;
                }
                fence_proxy_async_smem();  // cp.async data -> tensor-core reads
                tc_fence_after();
                const uint32_t kv_addr = smem_base + OFF_KV + s * KV_STAGE;
                for (int a = 0; a < n_atoms; ++a) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t da = desc_sw128(q_addr + a * Q_ATOM + kk * 32, 16, 1024);
                        const uint64_t db = desc_sw128(kv_addr + a * KV_ATOM + kk * 32, 16, 1024);
                        mma_bf16(tmem + TM_S + 64 * s, da, db, id_s, (a | kk) != 0);
                    }
                }
                mma_commit(&bars->s_full[s]);
                if (j >= 1 && !pv(j - 1)) { ok = false; break; }
            }
            if (ok) ok = pv(n_blocks - 1);
            mma_commit(&bars->o_final);
            // all MMAs of this CTA have finished before TMEM is released
            mbar_wait(&bars->o_final, 0, status, abort);
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the partner no longer writes into this CTA's shared memory
    if (warp == 8) {
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

// Split-k plan: number of splits of the k indices per query row.
void plan_splits(const ic_rows& r, int k, int& splits, int& keys_per_split) {
    const int64_t rows = (int64_t)r.B * r.Lq;
    const int pairs = std::max(1, sm_count() / 2);
    const int nblk = ceil_div(k, NB);
    splits = 1;
    if (rows < pairs) {
        double best = 1e30;
        for (int s = 1; s <= std::min(nblk, 32); ++s) {
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
    CUtensorMap map_q;
    cuuint64_t dims[2] = {(cuuint64_t)KVW, (cuuint64_t)r.B * r.Lq * HQ};
    cuuint64_t strides[1] = {(cuuint64_t)KVW * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)HQ};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&map_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
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
    attn_tc_kernel<<<(unsigned)(2 * units), N_THREADS, SMEM_BYTES, s>>>(map_q, a);
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
