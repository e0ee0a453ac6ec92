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
// tensor core, scales them to base-2 units and sends them to its partner
// through distributed shared memory as 16-bit fixed point: per head and
// block, an offset m at or above the largest valid partial logit and a
// power-of-two step fitted to the block's range, each value sent as
// (m - x) / step.  A key can decide the softmax while its partial logit on
// one CTA lies far below that CTA's block maximum (the other half makes up
// for it), so the rounding must not grow with the distance from m as a
// float16 difference's does: here it is at most one step, range / 2^15, for
// every key, which keeps sharp logits of a hundred and more base-2 units
// inside the attention tolerance.  Each CTA adds its own half in float32,
// straight from TMEM, to the partner's rebuilt half; each then runs the
// online softmax and accumulates its own 256 value columns, O_r += P V_r, in
// TMEM, normalised by its own softmax sum.  No key byte is gathered twice
// and no flop is done twice.
//
// Per CTA (512 threads), persistent over work units (one unit = one query
// row, or one split of a row's indices in decode):
//   warps 0-3  gather: per unit, one batched pass over the unit's indices
//              computes the per-block validity masks and the block count;
//              then TMA four-row gathers (tile::gather4) of the selected
//              rows' columns into 128-byte-swizzled tiles (4 stages of 64
//              keys); an invalid index becomes an out-of-range row, which
//              TMA fills with zeros;
//   warps 4-7  exchange (thread = head = TMEM lane): at the start of a unit,
//              the unit's Q_r columns that the S MMA reads from TMEM (value
//              slice 3 and the 32 rope columns); per 64-key block, partial S
//              from TMEM -> base 2 -> (offset, step, 16-bit codes),
//              sent straight into the partner's inbox with st.async (counted
//              in bytes on the partner's mbarrier); they run ahead of the
//              softmax warps by up to the two inbox slots.  The encode, the
//              scaling of S and the softmax warps' rebuild use packed f32x2
//              arithmetic (two keys per instruction);
//   warps 8-11 softmax (thread = head): own half (float32, from TMEM) + the
//              partner's rebuilt half (relative to the running max, folded
//              into the rebuild), row max, online softmax in base 2 with lazy
//              rescaling (O is rescaled only when the running max grows by
//              more than 2^8), P as bf16 into TMEM over the S columns, the
//              row sum l of the same rounded P, final normalisation and store;
//   warp 12    TMEM allocation, TMA load of Q_r's value slices 0-2 (the next
//              unit's while the current unit finishes), and single-thread
//              issue of S(j) = Q_r K_r(j)^T (K = 288; A from shared memory for
//              slices 0-2, from TMEM for slice 3 and the rope columns) as
//              soon as block j is gathered;
//   warp 13    single-thread issue of O += P(j) V_r(j), P read from TMEM
//              ("TS" form), as soon as P(j) is ready.  Two issuing threads
//              keep a P V from waiting behind the gather of a later block.
//   warps 14-15 idle (they complete the MMA warps' warpgroup, so that the
//              gather and MMA warpgroups can hand registers to the exchange
//              and softmax warpgroups with setmaxnreg).
// TMEM: O at columns 0..255, three S/P buffers at 256..447, Q_r slice 3 and
// rope columns at 448..495.  Keeping that part of Q_r in TMEM frees the
// shared memory for a fourth KV stage.
// Shared memory: Q_r slices 0-2 48 KB, 4 KV stages of 36 KB, 2 inbox tiles of
// 16-bit fixed-point logits (16 KB) + 512 B of per-head offset/step words
// (written by the partner),
// per-unit masks, barriers (~227 KB).
//
// Every wait is bounded (sm100.cuh); a wait that runs out records its site
// in the second status word: 1-3 gather (info_empty, scan_done, kv_empty),
// 4-6 exchange (info_full, s_full, peer_free), 7-11 softmax (info_full,
// own_full, x_full, o_done, o_final), 12-20 S issuer (info_full, q_empty,
// q_full, q_tmem_full, kv_full, s_free, next info_full, next q_empty, drain),
// 21-24 P V issuer (info_full, p_full, o_free, drain).
//
// Decode (few query rows): each row's k indices are split over several CTA
// pairs, which write unnormalised partials (O as bf16; m, l as float32, per
// CTA half); a small combine kernel merges them by log-sum-exp.
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
constexpr int KV_ATOM = NB * 128;    // one 64-column slice of a key block
constexpr int KV_ROPE = NB * 64;     // the 32 rope columns of a key block
constexpr int KV_STAGE = 4 * KV_ATOM + KV_ROPE;     // 36 KB
constexpr int NSTAGE = 4;
constexpr int NSBUF = 3;                            // S/P buffers in TMEM
constexpr int X_TILE = HQ * NB * 2;                 // 16 KB of 16-bit fixed-point partial logits
constexpr int X_QUAD = X_TILE / 4;                  // the 32 rows of one TMEM lane quadrant
constexpr int X_OFF = HQ * 4;                       // per-head offset/step words of one inbox slot
constexpr int X_OFF_QUAD = X_OFF / 4;
constexpr int MAX_UNIT_BLOCKS = 32;                 // at most 2048 indices per unit
constexpr int Q_SMEM_ATOMS = 3;                     // value slices 0-2 of Q_r in shared memory;
                                                    // slice 3 and the rope columns live in TMEM
constexpr int OFF_Q = 0;
constexpr int OFF_KV = Q_SMEM_ATOMS * Q_ATOM;       // 48 KB
constexpr int OFF_X = OFF_KV + NSTAGE * KV_STAGE;   // partner's fixed-point partial logits
constexpr int OFF_XOFF = OFF_X + 2 * X_TILE;        // partner's per-head offset/step words
constexpr int OFF_MASK = OFF_XOFF + 2 * X_OFF;
constexpr int OFF_BARS = OFF_MASK + 2 * MAX_UNIT_BLOCKS * 8;
constexpr int GW = 4;                               // gather warps
constexpr int KPW = NB / GW;                        // key rows of a block per gather warp
constexpr int W_Y = GW + 4, W_S = GW + 8, W_PV = GW + 9;   // first warp of each role (exchange: GW)
constexpr int N_THREADS = 32 * (GW + 12);           // gather, 4 exchange, 4 softmax, 2 MMA, 2 idle warps
// Registers per thread after the warpgroups re-balance them (setmaxnreg):
// the gather and MMA warpgroups give theirs up to the exchange and softmax
// warpgroups.  Launched at 128 (16 warps x 32 x 128 = 65536), the shares
// add up to the same total: 4 x 32 x (72 + 184 + 184 + 72) = 65536.
constexpr int REGS_SMALL = 72, REGS_LARGE = 184;
static_assert(4 * 32 * (2 * REGS_SMALL + 2 * REGS_LARGE) == N_THREADS * 128, "register shares");
constexpr int KV_FULL_ARRIVALS = GW;                // one expect-tx arrival per gather warp
static_assert(W_PV + 3 == N_THREADS / 32, "warp roles");
constexpr int TMEM_COLS = 512;
constexpr uint32_t TM_O = 0;
constexpr uint32_t TM_S = 256;                      // S/P buffer b at TM_S + 64 b
constexpr uint32_t TM_QT = TM_S + 64 * NSBUF;       // Q_r slice 3 (32 cols) + rope (16 cols), bf16 pairs
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_THRESHOLD = 8.f;            // log2 units
static_assert(TM_QT + 48 <= TMEM_COLS, "tensor memory budget");

struct __align__(8) AttnBars {
    uint64_t q_full, q_empty, q_tmem_full;
    uint64_t kv_full[NSTAGE], kv_empty[NSTAGE];
    uint64_t s_full[NSBUF], s_free[NSBUF];
    uint64_t own_full[NSBUF][4];    // exchange warp q has read S of the buffer
    uint64_t p_full[NSBUF];         // softmax warps -> MMA: P in TMEM
    uint64_t x_full[2][4];          // [inbox slot][quad]: the partner's 32 rows (counted in bytes)
    uint64_t peer_free[2][4];       // the partner's softmax warp q has read its inbox slot
    uint64_t o_done[2];             // P V of block g finished (barrier g & 1)
    uint64_t o_final, o_free;
    uint64_t info_full[2], info_empty[2];
    uint64_t drain[2];
    uint64_t scan_done[2];          // gather warps: per-unit reduction of the last valid index
    uint32_t tmem_base;
    int abort;
    int n_blocks[2];
    int red[2][4];
};

// the dynamic shared memory base is at least 16-byte aligned, so rounding it
// up to the 1024-byte alignment of the swizzled tiles takes at most 1008 bytes
constexpr size_t SMEM_BYTES = 1008 + OFF_BARS + sizeof(AttnBars);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

__device__ __forceinline__ bool idx_valid(int v, int t, int T) { return v >= 0 && v <= t && v < T; }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&p);
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float min3(float a, float b, float c) {
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// The partner's half of a key block crosses as 16-bit fixed point, per head:
// x ~ m - u * step with u an unsigned 16-bit integer, m at or above the
// block's largest valid partial logit (a bfloat16, rounded up) and step the
// power of two that spreads the block's range over [0, 2^16).  So every valid
// value is rebuilt to within about one step, which shrinks with the block's
// range, not with the logit's magnitude as a float16 difference would.  The
// range is taken 2^-15 wide of its value, so no valid code can round to 2^16
// (no clamp); an invalid key (-inf) gives an infinite code whose low 16 bits
// are 0 and rebuilds to a finite value: it is -inf on the receiving side
// already.
struct XCode {
    float scale, ms;    // 1/step and m/step (both exact)
    uint32_t word;      // bfloat16 m in bits 0-15, the float32 exponent field of step in 16-23
};

__device__ __forceinline__ XCode x_encoder(float mb, float mn) {
    uint32_t mbits = __float_as_uint(mb);
    mbits = (mbits >> 31) ? (mbits & 0xffff0000u) : ((mbits + 0xffffu) & 0xffff0000u);
    const float m = __uint_as_float(mbits);
    const float range = (m - mn) * (1.f + 0x1p-15f);
    int k = 0;                                      // step = 2^-k
    if (range > 0.f && range < INFINITY)            // range in [2^e, 2^(e+1)): k = 15 - e
        k = min(30, max(-30, 142 - (int)((__float_as_uint(range) >> 23) & 0xffu)));
    XCode c;
    c.scale = __uint_as_float((uint32_t)(127 + k) << 23);
    c.ms = m * c.scale;
    c.word = (mbits >> 16) | ((uint32_t)(127 - k) << 16);
    return c;
}

// two values {lo = a, hi = b} as 16-bit codes (m - x) / step, rounded
// Two float32 values in one 64-bit register pair, for the packed (f32x2)
// FFMA / FADD / FMUL of sm_100: one instruction for two lanes' worth of
// the same arithmetic, rounded exactly as two scalar operations.
__device__ __forceinline__ uint64_t f2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 f2_split(uint64_t v) {
    float a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
    return make_float2(a, b);
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint32_t x_encode2(const XCode& c, float a, float b) {
    // 2^23 + u for both values (u in the low 16 bits of each)
    const float2 u = f2_split(fadd2(ffma2(f2(a, b), f2(-c.scale, -c.scale), f2(c.ms, c.ms)),
                                    f2(8388608.f, 8388608.f)));
    return __byte_perm(__float_as_uint(u.x), __float_as_uint(u.y), 0x5410);
}

// The partner's value of a code u, minus a constant z (the running max):
// m - u*step - z = cz - (2^23 + u)*step with cz = m - z + 2^23*step, the
// float (2^23 + u) made from the code's bits directly (the softmax warps'
// rebuild loop does two codes at a time with f32x2 FFMAs).

// acc + the two bf16 values of a packed pair (each added in float32)
__device__ __forceinline__ float add_bf16x2(uint32_t p, float acc) {
    float r;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
        "add.rn.f32.bf16 %0, lo, %2;\n\tadd.rn.f32.bf16 %0, hi, %0;\n\t}"
        : "=f"(r) : "r"(p), "f"(acc));
    return r;
}

// This thread's (head's) own partial logits of a 64-key S buffer in base-2
// units, the keys of invalid indices (mask bits 0) set to -inf.
__device__ __forceinline__ void own_logits(uint32_t taddr, float sl2, const uint32_t* mask2,
                                           float (&x)[NB]) {
    uint32_t r0[32], r1[32];
    tmem_ld32(taddr, r0);
    tmem_ld32(taddr + 32, r1);
    const uint32_t m_lo = mask2[0], m_hi = mask2[1];
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
        const float2 a = f2_split(fmul2(f2(__uint_as_float(r0[c]), __uint_as_float(r0[c + 1])), f2(sl2, sl2)));
        const float2 b = f2_split(fmul2(f2(__uint_as_float(r1[c]), __uint_as_float(r1[c + 1])), f2(sl2, sl2)));
        x[c] = a.x;
        x[c + 1] = a.y;
        x[32 + c] = b.x;
        x[32 + c + 1] = b.y;
    }
    if ((m_lo & m_hi) != 0xffffffffu) {
#pragma unroll
        for (int c = 0; c < NB; ++c)
            if (!(((c < 32 ? m_lo : m_hi) >> (c & 31)) & 1u)) x[c] = -INFINITY;
    }
}

// largest of 64 values
__device__ __forceinline__ float max64(const float (&v)[NB]) {
    float mx[21];
#pragma unroll
    for (int x = 0; x < 21; ++x) mx[x] = max3(v[3 * x], v[3 * x + 1], v[3 * x + 2]);
    float m = max3(mx[0], mx[1], v[63]);
#pragma unroll
    for (int x = 2; x + 1 < 21; x += 2) m = max3(m, mx[x], mx[x + 1]);
    return fmaxf(m, mx[20]);
}

// smallest of 64 values
__device__ __forceinline__ float min64(const float (&v)[NB]) {
    float mn[21];
#pragma unroll
    for (int x = 0; x < 21; ++x) mn[x] = min3(v[3 * x], v[3 * x + 1], v[3 * x + 2]);
    float m = min3(mn[0], mn[1], v[63]);
#pragma unroll
    for (int x = 2; x + 1 < 21; x += 2) m = min3(m, mn[x], mn[x + 1]);
    return fminf(m, mn[20]);
}

// smallest of the values above -inf (+inf if there is none)
__device__ __forceinline__ float min64_finite(const float (&v)[NB]) {
    float m = INFINITY;
#pragma unroll
    for (int c = 0; c < NB; ++c) m = fminf(m, v[c] > -INFINITY ? v[c] : INFINITY);
    return m;
}

struct AttnArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* kv;
    const int32_t* idx;
    __nv_bfloat16* out;
    __nv_bfloat16* part_o;  // [units][128][512] unnormalised O (split-k only)
    float2* part_ml;    // [units][2][128]     (split-k only; (m, l) of each CTA half)
    uint32_t* status;
    int k, B, Lq, q_start, T;
    int splits, keys_per_split, n_units;
    float scale_log2;
    // KV rows: dense (seq_lens == nullptr) at b*T + s; paged at
    // block_table[b*max_pages + s/page_size]*page_size + s%page_size, with
    // per-sequence lengths (queries at seq_lens[b] - Lq + i, T = the upper bound)
    const int32_t* seq_lens;
    const int32_t* block_table;
    int max_pages, page_size, num_pages;
    int kv_rows;        // rows of the KV tensor map; row kv_rows is the zero-filled stand-in
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
    const int i = u.row - u.b * a.Lq;
    if (a.seq_lens == nullptr) {
        u.t = a.q_start + i;
    } else {
        // a length outside [Lq, T] leaves the row without a valid index
        const int Tb = __ldg(a.seq_lens + u.b);
        u.t = (Tb >= a.Lq && Tb <= a.T) ? Tb - a.Lq + i : -1;
    }
    u.e0 = split * a.keys_per_split;
    u.e1 = min(a.k, u.e0 + a.keys_per_split);
    return u;
}

// KV tensor-map row of key position v of sequence b (v already checked to
// lie in [0, t]); a page outside [0, num_pages) gives the zero-filled row and
// the index-range status bit.
__device__ __forceinline__ int kv_row(const AttnArgs& a, int b, int v) {
    if (a.seq_lens == nullptr) return b * a.T + v;
    const int page = __ldg(a.block_table + (int64_t)b * a.max_pages + v / a.page_size);
    if (page < 0 || page >= a.num_pages) {
        flag_status(a.status, IC_DEV_INDEX_RANGE);
        return a.kv_rows;
    }
    return page * a.page_size + v % a.page_size;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(N_THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap map_q,
               const __grid_constant__ CUtensorMap map_kv, const __grid_constant__ CUtensorMap map_kvr,
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
        mbar_init(&bars->q_tmem_full, 4);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&bars->kv_full[s], KV_FULL_ARRIVALS);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int s = 0; s < NSBUF; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->s_free[s], 1);
            mbar_init(&bars->p_full[s], 4);
            for (int q = 0; q < 4; ++q) mbar_init(&bars->own_full[s][q], 1);
        }
        for (int s = 0; s < 2; ++s) {
            for (int q = 0; q < 4; ++q) {
                mbar_init(&bars->x_full[s][q], 1);
                mbar_init(&bars->peer_free[s][q], 1);
            }
            mbar_init(&bars->o_done[s], 1);
            mbar_init(&bars->info_full[s], 1);
            mbar_init(&bars->info_empty[s], 10);
            mbar_init(&bars->scan_done[s], GW);
        }
        mbar_init(&bars->o_final, 1);
        mbar_init(&bars->o_free, 4);
        mbar_init(&bars->drain[0], 1);
        mbar_init(&bars->drain[1], 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == W_S) tmem_alloc<TMEM_COLS>(&bars->tmem_base);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();  // the partner's barriers are initialised before any remote arrive
    const uint32_t tmem = bars->tmem_base;
    // everything above is on-chip; the indices, Q and the KV rows may come
    // from the kernel before this one on the stream
    pdl_trigger();
    pdl_wait();

    // Warpgroups 0 (gather) and 3 (the two MMA issuers and two idle warps)
    // shrink to REGS_SMALL, 1 (exchange) and 2 (softmax) grow to REGS_LARGE;
    // every warp of a warpgroup executes its group's instruction.
    if (warp < GW) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(REGS_SMALL) : "memory");
    else if (warp < W_S) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(REGS_LARGE) : "memory");
    else asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(REGS_SMALL) : "memory");
    if (warp < GW) {
        // ------------------------------------------------------------ gather
        const int gt = threadIdx.x;
        uint32_t g = 0;
        int n = 0;
        for (int seq = pair; seq < args.n_units; seq += n_pairs, ++n) {
            const Unit u = decode_unit(args, seq);
            const int32_t* idx_row = args.idx + (int64_t)u.row * args.k;
            const int ip = n & 1;
            if (!warp_wait(&bars->info_empty[ip], ((n >> 1) & 1) ^ 1, status, abort, 1)) break;
            // validity masks of the unit's blocks and its last valid index; the
            // loads go out SCAN_BATCH at a time so the scan costs a few memory
            // round trips, not one per 32*GW indices
            int last = -1;
            const int n_ent = u.e1 - u.e0;
            constexpr int SCAN_BATCH = 8;
            for (int base0 = 0; base0 < n_ent; base0 += SCAN_BATCH * 32 * GW) {
                int v[SCAN_BATCH];
#pragma unroll
                for (int q = 0; q < SCAN_BATCH; ++q) {
                    const int e = u.e0 + base0 + q * 32 * GW + gt;
                    v[q] = e < u.e1 ? idx_row[e] : -1;
                }
#pragma unroll
                for (int q = 0; q < SCAN_BATCH; ++q) {
                    const int base = base0 + q * 32 * GW;
                    if (base >= n_ent) break;
                    const int e = u.e0 + base + gt;
                    const bool ok = idx_valid(v[q], u.t, args.T);
                    if (!ok && v[q] != -1 && r == 0) flag_status(status, IC_DEV_INDEX_RANGE);
                    if (ok) last = e;
                    const uint32_t bal = __ballot_sync(0xffffffffu, ok);
                    const int word = base / 32 + warp;
                    if (lane == 0 && word < 2 * MAX_UNIT_BLOCKS) masks[ip * 2 * MAX_UNIT_BLOCKS + word] = bal;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
            if (lane == 0) bars->red[ip][warp] = last;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->scan_done[ip]);
            if (!warp_wait(&bars->scan_done[ip], (n >> 1) & 1, status, abort, 2)) break;
            last = bars->red[ip][0];
#pragma unroll
            for (int w = 1; w < GW; ++w) last = max(last, bars->red[ip][w]);
            const int nb = last < 0 ? 0 : (last - u.e0) / NB + 1;
            if (gt == 0) {
                bars->n_blocks[ip] = nb;
                mbar_arrive(&bars->info_full[ip]);
            }
            // warp w fills key rows KPW*w .. KPW*w + KPW-1 of each block; lane
            // L < KPW holds the row of key KPW*w + L (the indices of block j+1
            // are loaded while block j is issued).  An invalid index becomes
            // the out-of-range row B*T, which TMA fills with zeros.
            const int oob_row = args.kv_rows;
            bool ok_all = true;
            const int key = warp * KPW + lane;
            int v_next = (lane < KPW && u.e0 + key < u.e1) ? idx_row[u.e0 + key] : -1;
            for (int j = 0; j < nb; ++j, ++g) {
                const int s = g % NSTAGE;
                const int v_lane = v_next;
                if (j + 1 < nb) {
                    const int e1 = u.e0 + (j + 1) * NB + key;
                    v_next = (lane < KPW && e1 < u.e1) ? idx_row[e1] : -1;
                }
                const int row_lane = idx_valid(v_lane, u.t, args.T) ? kv_row(args, u.b, v_lane) : oob_row;
                if (!warp_wait(&bars->kv_empty[s], ((g / NSTAGE) & 1) ^ 1, status, abort, 3)) {
                    ok_all = false;
                    break;
                }
                const uint32_t stage = smem_base + OFF_KV + s * KV_STAGE;
                // (KPW/4) groups of 4 rows x (four 64-column value slices + the 32
                // rope columns) tile::gather4 copies; copy c (group c / 5, slice
                // c % 5) is issued by lane c % 32
                constexpr int OPS = KPW / 4 * 5;
                if (lane == 0) mbar_arrive_expect_tx(&bars->kv_full[s], KPW / 4 * (4 * 512 + 256));
                __syncwarp();
#pragma unroll
                for (int c0 = 0; c0 < OPS; c0 += 32) {
                    const int c = c0 + lane;
                    const int grp = (c < OPS ? c : 0) / 5, sl = c % 5;
                    const int r0 = __shfl_sync(0xffffffffu, row_lane, 4 * grp);
                    const int r1 = __shfl_sync(0xffffffffu, row_lane, 4 * grp + 1);
                    const int r2 = __shfl_sync(0xffffffffu, row_lane, 4 * grp + 2);
                    const int r3 = __shfl_sync(0xffffffffu, row_lane, 4 * grp + 3);
                    if (c < OPS) {
                        const int krow = KPW * warp + 4 * grp;
                        if (sl < 4)
                            tma_gather4(stage + sl * KV_ATOM + krow * 128, &map_kv, &bars->kv_full[s],
                                        (int)r * 256 + sl * 64, r0, r1, r2, r3);
                        else
                            tma_gather4(stage + 4 * KV_ATOM + krow * 64, &map_kvr, &bars->kv_full[s],
                                        512 + (int)r * 32, r0, r1, r2, r3);
                    }
                }
            }
            if (!ok_all) break;
        }
        // drain: every gather this warp issued has landed before the CTA may
        // exit (on the abort path some were never consumed by an S MMA); a
        // stage another warp never filled gives up after 50 ms
        if (lane == 0)
            for (uint32_t j = g > (uint32_t)NSTAGE ? g - NSTAGE : 0; j < g; ++j)
                mbar_wait_drain(&bars->kv_full[j % NSTAGE], (j / NSTAGE) & 1, 50000000ull);
        __syncwarp();
    } else if (warp < W_Y) {
        // ------------------------------------------------------------ exchange
        const int quad = warp & 3;                // TMEM lanes 32*quad .. +31
        const int h = quad * 32 + lane;           // head of this thread
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t x_remote = map_to_rank(smem_base + OFF_X + h * 128, peer);
        const uint32_t xoff_remote = map_to_rank(smem_base + OFF_XOFF + h * 4, peer);
        const float sl2 = args.scale_log2;
        uint32_t g = 0;
        int n = 0;
        bool ok = true;
        for (int seq = pair; seq < args.n_units && ok; seq += n_pairs, ++n) {
            const int ip = n & 1;
            if (!warp_wait(&bars->info_full[ip], (n >> 1) & 1, status, abort, 4)) break;
            const int nb = bars->n_blocks[ip];
            __syncwarp();
            if (nb > 0) {
                // Q_r columns the S MMA reads from TMEM (value slice 3 and the rope
                // columns), row h, packed as bf16 pairs.  Every S MMA of the previous
                // unit has finished: this warp has seen the S of its last block.
                const Unit u = decode_unit(args, seq);
                const __nv_bfloat16* qrow = args.q + ((int64_t)u.row * HQ + h) * KVW;
                uint32_t qa[32], qb[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 v = *reinterpret_cast<const uint4*>(qrow + (int)r * 256 + 192 + 8 * i);
                    qa[4 * i] = v.x; qa[4 * i + 1] = v.y; qa[4 * i + 2] = v.z; qa[4 * i + 3] = v.w;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 v = *reinterpret_cast<const uint4*>(qrow + 512 + (int)r * 32 + 8 * i);
                    qb[4 * i] = v.x; qb[4 * i + 1] = v.y; qb[4 * i + 2] = v.z; qb[4 * i + 3] = v.w;
                }
                tmem_st32(t_lane + TM_QT, qa);
                tmem_st16(t_lane + TM_QT + 32, qb);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->q_tmem_full);
            }
            // Per block: this CTA's half of the logits to the partner.  The
            // softmax warp of the quadrant combines the two halves; this warp
            // runs ahead of it by up to the two inbox slots.
            for (int j = 0; j < nb; ++j) {
                const uint32_t gs = g + j;
                const int sb = gs % NSBUF;
                const int slot = gs & 1;
                if (!warp_wait(&bars->s_full[sb], (gs / NSBUF) & 1, status, abort, 5)) { ok = false; break; }
                tc_fence_after();
                float x[NB];
                own_logits(t_lane + TM_S + 64 * sb, sl2, masks + ip * 2 * MAX_UNIT_BLOCKS + 2 * j, x);
                // S(gs) has been read: the softmax warp may read it too and then
                // overwrite it with P
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->own_full[sb][quad]);
                // the encoding's offset and step come from the block's largest and
                // smallest VALID partial logits (invalid keys are -inf from here on)
                const float mb = max64(x);
                float mn = min64(x);
                if (mn == -INFINITY) mn = min64_finite(x);      // a block with invalid keys
                const XCode xc = x_encoder(mb, mn);
                // the partner's softmax warp q must have finished this inbox slot
                // (block gs-2)
                if (!warp_wait_cluster(&bars->peer_free[slot][quad], ((gs >> 1) & 1) ^ 1, status, abort, 6)) {
                    ok = false;
                    break;
                }
                // row h of the partner's inbox, 16 bytes (8 keys) at a time, and
                // the head's offset/step word; each st.async counts its bytes on the
                // partner's x_full (no fence or arrive on this side)
                const uint32_t xr = x_remote + slot * X_TILE;
                const uint32_t br = map_to_rank(smem_u32(&bars->x_full[slot][quad]), peer);
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_async_v4(xr + ((c ^ (h & 7)) << 4),
                                x_encode2(xc, x[8 * c + 0], x[8 * c + 1]),
                                x_encode2(xc, x[8 * c + 2], x[8 * c + 3]),
                                x_encode2(xc, x[8 * c + 4], x[8 * c + 5]),
                                x_encode2(xc, x[8 * c + 6], x[8 * c + 7]), br);
                st_async_b32(xoff_remote + slot * X_OFF, xc.word, br);
            }
            g += nb;
            // the unit's masks have been read: the gather warps may refill them
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->info_empty[ip]);
        }
    } else if (warp < W_S) {
        // ------------------------------------------------------------ softmax
        const int quad = warp & 3;
        const int h = quad * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t free_remote0 = map_to_rank(smem_u32(&bars->peer_free[0][quad]), peer);
        const uint32_t free_remote1 = map_to_rank(smem_u32(&bars->peer_free[1][quad]), peer);
        const float sl2 = args.scale_log2;
        uint32_t g = 0, o_use = 0;
        int n = 0;
        bool ok = true;
        for (int seq = pair; seq < args.n_units && ok; seq += n_pairs, ++n) {
            const Unit u = decode_unit(args, seq);
            const int ip = n & 1;
            if (!warp_wait(&bars->info_full[ip], (n >> 1) & 1, status, abort, 7)) { ok = false; break; }
            const int nb = bars->n_blocks[ip];
            float m_use = 0.f;      // running max (log2 units); meaningful once m_set
            bool m_set = false;
            float l = 0.f;          // running sum of the bf16-rounded P
            for (int j = 0; j < nb; ++j, ++g) {
                const int sb = g % NSBUF;
                const int slot = g & 1;
                // arm this CTA's inbox slot for the partner's half of block g
                if (lane == 0) mbar_arrive_expect_tx(&bars->x_full[slot][quad], X_QUAD + X_OFF_QUAD);
                const uint32_t m_lo = masks[ip * 2 * MAX_UNIT_BLOCKS + 2 * j];
                const uint32_t m_hi = masks[ip * 2 * MAX_UNIT_BLOCKS + 2 * j + 1];
                // S(g) is final in TMEM and the exchange warp has read it
                if (!warp_wait(&bars->own_full[sb][quad], (g / NSBUF) & 1, status, abort, 8)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t s0[32], s1[32];
                tmem_ld32(t_lane + TM_S + 64 * sb, s0);
                tmem_ld32(t_lane + TM_S + 64 * sb + 32, s1);
                // the partner's half of block g
                if (!warp_wait_cluster(&bars->x_full[slot][quad], (g >> 1) & 1, status, abort, 9)) {
                    tmem_ld_wait();          // no TMEM load outlives the loop
                    ok = false;
                    break;
                }
                const uint32_t ow = reinterpret_cast<const uint32_t*>(smem + OFF_XOFF + slot * X_OFF)[h];
                const float pm = __uint_as_float(ow << 16);
                const float pstep = __uint_as_float(((ow >> 16) & 0xffu) << 23);
                // the running max is folded into the rebuild: values relative to m_use
                const float cz = fmaf(8388608.f, pstep, pm - m_use);
                const uint4* xp = reinterpret_cast<const uint4*>(smem + OFF_X + slot * X_TILE + h * 128);
                tmem_ld_wait();
                // full logits of the 64 keys in base 2, minus m_use: own half (float32)
                // plus the partner's half rebuilt from its codes; invalid keys -inf
                float sv[NB];
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const uint4 w4 = xp[cc ^ (h & 7)];                 // keys 8cc .. 8cc+7
                    const uint32_t pw4[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        // two keys at once: the codes' floats (2^23 + u), then
                        // cz - f*step and raw*sl2 + that, each as one f32x2 FFMA
                        const int key = 8 * cc + e;
                        const uint32_t w = pw4[e >> 1];
                        const uint64_t f = f2(__uint_as_float((w & 0xffffu) | 0x4b000000u),
                                              __uint_as_float(__byte_perm(w, 0x4b000000u, 0x7632)));
                        const uint64_t part = ffma2(f, f2(-pstep, -pstep), f2(cz, cz));
                        const uint64_t raw = key < 32 ? f2(__uint_as_float(s0[key]), __uint_as_float(s0[key + 1]))
                                                      : f2(__uint_as_float(s1[key - 32]), __uint_as_float(s1[key - 31]));
                        const float2 v = f2_split(ffma2(raw, f2(sl2, sl2), part));
                        sv[key] = v.x;
                        sv[key + 1] = v.y;
                    }
                }
                if ((m_lo & m_hi) != 0xffffffffu) {
#pragma unroll
                    for (int kk = 0; kk < NB; ++kk) {
                        const uint32_t mw = kk < 32 ? m_lo : m_hi;
                        if (!((mw >> (kk & 31)) & 1u)) sv[kk] = -INFINITY;
                    }
                }
                const float mrel = max64(sv);            // block max - m_use
                // every inbox value of this slot has been consumed (mrel depends on
                // all of them): hand the slot back to the partner's exchange warp
                __syncwarp();
                if (lane == 0) mbar_arrive_remote_relaxed(slot ? free_remote1 : free_remote0);
                bool rescale = false;
                float alpha = 1.f;
                if (mrel > -INFINITY && (!m_set || mrel > RESCALE_THRESHOLD)) {
                    rescale = m_set;             // O and l hold earlier blocks only if m was set
                    alpha = m_set ? ex2_approx(-mrel) : 0.f;
                    m_use += mrel;               // the block max
                    m_set = true;
#pragma unroll
                    for (int c = 0; c < NB; ++c) sv[c] -= mrel;
                }
                uint32_t pw[NB / 2];
                float ps[2] = {0.f, 0.f};
#pragma unroll
                for (int x = 0; x < NB / 2; ++x) {
                    pw[x] = pack_bf16(ex2_approx(sv[2 * x]), ex2_approx(sv[2 * x + 1]));
                    ps[x & 1] = add_bf16x2(pw[x], ps[x & 1]);
                }
                l = (rescale ? l * alpha : l) + (ps[0] + ps[1]);
                // The decision is per head (lane), but the O rescale below is
                // warp-collective (the wait shuffles over the whole warp and the
                // TMEM loads and stores are .aligned): the warp takes it when any
                // of its heads needs it, and the other heads scale by 1.
                if (__any_sync(0xffffffffu, rescale)) {
                    const float a = rescale ? alpha : 1.f;
                    // O and l must hold P V of block g-1 before they are rescaled
                    if (!warp_wait(&bars->o_done[(g - 1) & 1], ((g - 1) >> 1) & 1, status, abort, 10)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 8; ++c) {
                        uint32_t o[32];
                        tmem_ld32(t_lane + TM_O + 32 * c, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * a);
                        tmem_st32(t_lane + TM_O + 32 * c, o);
                    }
                }
                tmem_st32(t_lane + TM_S + 64 * sb, pw);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[sb]);
            }
            if (!ok) break;
            // ---------------------------------------------------------- unit epilogue
            const bool split = args.splits > 1;
            float l_all = 0.f;
            if (nb > 0) {
                if (!warp_wait(&bars->o_final, o_use & 1, status, abort, 11)) { ok = false; break; }
                tc_fence_after();
                l_all = m_set ? l : 0.f;
                const float inv = l_all > 0.f ? 1.f / l_all : 0.f;
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t o[32];
                    tmem_ld32(t_lane + TM_O + 32 * c, o);
                    tmem_ld_wait();
                    const int col = (int)r * 256 + 32 * c;     // column of the output row
                    if (!split) {
                        uint4* dst = reinterpret_cast<uint4*>(args.out + ((int64_t)u.row * HQ + h) * DV + col);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint4 pk;
                            pk.x = pack_bf16(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                            pk.y = pack_bf16(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                            pk.z = pack_bf16(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                            pk.w = pack_bf16(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
                            dst[v] = pk;
                        }
                    } else {
                        // unnormalised partial O as bf16 (the combine scales and normalises)
                        uint4* dst = reinterpret_cast<uint4*>(args.part_o + ((int64_t)u.unit * HQ + h) * DV + col);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint4 pk;
                            pk.x = pack_bf16(__uint_as_float(o[8 * v + 0]), __uint_as_float(o[8 * v + 1]));
                            pk.y = pack_bf16(__uint_as_float(o[8 * v + 2]), __uint_as_float(o[8 * v + 3]));
                            pk.z = pack_bf16(__uint_as_float(o[8 * v + 4]), __uint_as_float(o[8 * v + 5]));
                            pk.w = pack_bf16(__uint_as_float(o[8 * v + 6]), __uint_as_float(o[8 * v + 7]));
                            dst[v] = pk;
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->o_free);
                ++o_use;
            } else if (!split) {
                // no valid key: the output row is zero
                uint4* dst = reinterpret_cast<uint4*>(args.out + ((int64_t)u.row * HQ + h) * DV + r * 256);
                for (int v = 0; v < 32; ++v) dst[v] = make_uint4(0, 0, 0, 0);
            }
            // each CTA half keeps its own (m, l): the two CTAs' logits differ by
            // rounding, so their running maxima and sums may differ slightly
            if (split) args.part_ml[((int64_t)u.unit * 2 + r) * HQ + h] = make_float2(m_use, l_all);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->info_empty[ip]);
        }
    } else if (warp == W_S) {
        // ------------------------------------------------------------ S = Q K^T issuer
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_f32acc(1, 1, HQ, NB);            // S = Q K^T
            const uint32_t q_addr = smem_base + OFF_Q;
            uint32_t g = 0, o_use = 0;
            bool issued = false, ok = true;
            int nb_next = -1;
            bool q_loaded_next = false;
            auto load_q = [&](int seq) {
                const Unit u = decode_unit(args, seq);
                mbar_arrive_expect_tx(&bars->q_full, Q_SMEM_ATOMS * Q_ATOM);
                for (int a = 0; a < Q_SMEM_ATOMS; ++a)
                    tma_load_2d(smem + OFF_Q + a * Q_ATOM, &map_q, &bars->q_full, (int)r * 256 + a * 64,
                                u.row * HQ);
            };
            int n = 0;
            for (int seq = pair; seq < args.n_units && ok; seq += n_pairs, ++n) {
                int nb;
                if (nb_next >= 0) {
                    nb = nb_next;
                    nb_next = -1;
                } else {
                    if (!mbar_wait(&bars->info_full[n & 1], (n >> 1) & 1, status, abort, 12)) break;
                    nb = bars->n_blocks[n & 1];
                    mbar_arrive(&bars->info_empty[n & 1]);
                }
                if (nb == 0) continue;
                if (!q_loaded_next) {
                    if (o_use > 0 && !mbar_wait(&bars->q_empty, (o_use - 1) & 1, status, abort, 13)) break;
                    load_q(seq);
                }
                q_loaded_next = false;
                if (!mbar_wait(&bars->q_full, o_use & 1, status, abort, 14) ||
                    !mbar_wait(&bars->q_tmem_full, o_use & 1, status, abort, 15))
                    break;
                for (int j = 0; j < nb; ++j, ++g) {
                    const int sb = g % NSBUF;
                    const int ks = g % NSTAGE;
                    if (!mbar_wait(&bars->kv_full[ks], (g / NSTAGE) & 1, status, abort, 16) ||
                        !mbar_wait(&bars->s_free[sb], ((g / NSBUF) & 1) ^ 1, status, abort, 17)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t kv_addr = smem_base + OFF_KV + ks * KV_STAGE;
                    const uint32_t s_tm = tmem + TM_S + 64 * sb;
#pragma unroll
                    for (int a = 0; a < Q_SMEM_ATOMS; ++a) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t da = desc_sw128(q_addr + a * Q_ATOM + kk * 32, 16, 1024);
                            const uint64_t db = desc_sw128(kv_addr + a * KV_ATOM + kk * 32, 16, 1024);
                            mma_bf16(s_tm, da, db, id_s, (a | kk) != 0);
                        }
                    }
                    // value slice 3 and the rope columns: A (Q_r) from TMEM
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t db = desc_sw128(kv_addr + 3 * KV_ATOM + kk * 32, 16, 1024);
                        mma_bf16_ts(s_tm, tmem + TM_QT + kk * 8, db, id_s, 1u);
                    }
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const uint64_t db = desc_sw64(kv_addr + 4 * KV_ATOM + kk * 32);
                        mma_bf16_ts(s_tm, tmem + TM_QT + 32 + kk * 8, db, id_s, 1u);
                    }
                    issued = true;
                    mma_commit(&bars->s_full[sb]);
                }
                if (!ok) break;
                // Q is free once these MMAs finish: fetch the next unit's Q now
                mma_commit(&bars->q_empty);
                if (seq + n_pairs < args.n_units) {
                    const int n1 = n + 1;
                    if (!mbar_wait(&bars->info_full[n1 & 1], (n1 >> 1) & 1, status, abort, 18)) break;
                    nb_next = bars->n_blocks[n1 & 1];
                    mbar_arrive(&bars->info_empty[n1 & 1]);
                    if (nb_next > 0) {
                        if (!mbar_wait(&bars->q_empty, o_use & 1, status, abort, 19)) break;
                        load_q(seq + n_pairs);
                        q_loaded_next = true;
                    }
                }
                ++o_use;
            }
            if (issued) {
                mma_commit(&bars->drain[0]);   // every MMA this thread issued has finished
                mbar_wait(&bars->drain[0], 0, status, abort, 20);
            }
        }
    } else if (warp == W_PV) {
        // ------------------------------------------------------------ O += P V, l += P 1 issuer
        if (lane == 0) {
            constexpr uint32_t id_pv = idesc_f32acc(1, 1, HQ, 256, 0, 1);    // O += P V (V MN-major)
            uint32_t g = 0, o_use = 0;
            bool issued = false, ok = true;
            int n = 0;
            for (int seq = pair; seq < args.n_units && ok; seq += n_pairs, ++n) {
                if (!mbar_wait(&bars->info_full[n & 1], (n >> 1) & 1, status, abort, 21)) break;
                const int nb = bars->n_blocks[n & 1];
                mbar_arrive(&bars->info_empty[n & 1]);
                if (nb == 0) continue;
                for (int j = 0; j < nb; ++j, ++g) {
                    const int sb = g % NSBUF;
                    if (!mbar_wait(&bars->p_full[sb], (g / NSBUF) & 1, status, abort, 22) ||
                        (j == 0 && o_use > 0 && !mbar_wait(&bars->o_free, (o_use - 1) & 1, status, abort, 23))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t v_addr = smem_base + OFF_KV + (g % NSTAGE) * KV_STAGE;
                    const uint32_t p_tm = tmem + TM_S + 64 * sb;
#pragma unroll
                    for (int kk = 0; kk < NB / 16; ++kk) {
                        const uint64_t db = desc_sw128(v_addr + kk * 16 * 128, 8192, 1024);
                        mma_bf16_ts(tmem + TM_O, p_tm + kk * 8, db, id_pv, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    issued = true;
                    mma_commit(&bars->kv_empty[g % NSTAGE]);
                    mma_commit(&bars->s_free[sb]);
                    mma_commit(&bars->o_done[g & 1]);
                }
                if (!ok) break;
                mma_commit(&bars->o_final);
                ++o_use;
            }
            if (issued) {
                mma_commit(&bars->drain[1]);
                mbar_wait(&bars->drain[1], 0, status, abort, 24);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the partner no longer writes into this CTA's shared memory
    if (warp == W_S) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem);
    }
}

// Merge split-k partials: out = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c,
// with (m_c, l_c) of the CTA half that produced the columns (O_c in bf16:
// 2^-9 relative, inside the attention tolerance).
// Each thread merges 8 adjacent columns of one head (one 16-byte load per
// split), a CTA 4 heads: grid (rows, HQ / 4) x 256 threads.  Splits are read
// CH at a time with every load of a chunk in flight before the first is used
// (one memory round trip per chunk, not per split); the running maximum M
// rescales what earlier chunks added.  CH follows the split count, so that
// few splits keep few registers and the whole grid fits on the GPU at once.
constexpr int COMBINE_THREADS = 256;
constexpr int COMBINE_HEADS = COMBINE_THREADS / (DV / 8);     // 4 heads per CTA
template <int CH>
__global__ void __launch_bounds__(COMBINE_THREADS)
attn_combine_kernel(const __nv_bfloat16* __restrict__ part_o, const float2* __restrict__ part_ml,
                    int splits, __nv_bfloat16* __restrict__ out) {
    pdl_trigger();
    pdl_wait();
    const int64_t row = blockIdx.x;
    const int h = blockIdx.y * COMBINE_HEADS + (int)(threadIdx.x / (DV / 8));
    const int d = (int)(threadIdx.x % (DV / 8)) * 8;
    const int half = d / 256;
    float M = -INFINITY;
    float num[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float den = 0.f;
    for (int c0 = 0; c0 < splits; c0 += CH) {
        float2 ml[CH];
        uint4 o[CH];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int64_t u = row * splits + c0 + c;
            ml[c] = c0 + c < splits ? part_ml[(u * 2 + half) * HQ + h] : make_float2(-INFINITY, 0.f);
            o[c] = c0 + c < splits ? *reinterpret_cast<const uint4*>(part_o + (u * HQ + h) * DV + d)
                                   : make_uint4(0u, 0u, 0u, 0u);
        }
        float Mc = M;
#pragma unroll
        for (int c = 0; c < CH; ++c)
            if (ml[c].y > 0.f) Mc = fmaxf(Mc, ml[c].x);
        if (Mc == -INFINITY) continue;                   // nothing valid so far
        if (Mc > M) {
            const float a = M == -INFINITY ? 0.f : exp2f(M - Mc);
#pragma unroll
            for (int j = 0; j < 8; ++j) num[j] *= a;
            den *= a;
            M = Mc;
        }
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            if (!(ml[c].y > 0.f)) continue;
            const float wgt = exp2f(ml[c].x - M);
            den += wgt * ml[c].y;
            const uint32_t w4[4] = {o[c].x, o[c].y, o[c].z, o[c].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                num[2 * j] += wgt * __uint_as_float(w4[j] << 16);
                num[2 * j + 1] += wgt * __uint_as_float(w4[j] & 0xffff0000u);
            }
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint4 pk;
    pk.x = pack_bf16(num[0] * inv, num[1] * inv);
    pk.y = pack_bf16(num[2] * inv, num[3] * inv);
    pk.z = pack_bf16(num[4] * inv, num[5] * inv);
    pk.w = pack_bf16(num[6] * inv, num[7] * inv);
    *reinterpret_cast<uint4*>(out + (row * HQ + h) * DV + d) = pk;
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
// The split count minimises (waves of CTA pairs) x (blocks per split + a
// fixed cost per unit) among the counts whose units (rows x splits) do not
// pass max_units; the smallest admissible count is always kept, so the
// caller checks rows x splits against its own limit.
void plan_splits(const ic_rows& r, int k, int& splits, int& keys_per_split, int64_t max_units) {
    const int64_t rows = (int64_t)r.B * r.Lq;
    const int pairs = std::max(1, sm_count() / 2);
    const int nblk = ceil_div(k, NB);
    const int min_splits = ceil_div(nblk, MAX_UNIT_BLOCKS);
    splits = min_splits;
    if (rows < pairs) {
        double best = 1e30;
        for (int s = min_splits; s <= std::max(min_splits, std::min(nblk, 32)); ++s) {
            if (s > min_splits && rows * s > max_units) break;
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

int64_t attn_tc_units(ic_rows r, int k, int64_t max_units) {
    int splits, kps;
    plan_splits(r, k, splits, kps, max_units);
    return (int64_t)r.B * r.Lq * splits;
}

size_t attn_tc_scratch_bytes(ic_rows r, int k, int64_t max_units) {
    int splits, kps;
    plan_splits(r, k, splits, kps, max_units);
    if (splits <= 1) return 0;
    const size_t units = (size_t)r.B * r.Lq * splits;
    return units * HQ * DV * sizeof(__nv_bfloat16) + 256 + units * 2 * HQ * sizeof(float2);
}

namespace {

// r: planning rows (dense: the call's rows; paged: every sequence T_max long).
ic_status attn_tc_core(const void* q, const void* kv, const int32_t* idx, int k, ic_rows r,
                       float scale, void* out, uint32_t* status, void* scratch,
                       size_t scratch_bytes, cudaStream_t s, int64_t max_units,
                       const ic_paged_rows* pr) {
    if (((uintptr_t)q & 15) || ((uintptr_t)kv & 15) || ((uintptr_t)out & 15))
        return IC_ERR_INVALID_ARG;
    auto fn = encode_fn();
    if (fn == nullptr) return cuda_error("attn_tc");
    CUtensorMap map_q;
    cuuint64_t dims[2] = {(cuuint64_t)KVW, (cuuint64_t)r.B * r.Lq * HQ};
    cuuint64_t strides[1] = {(cuuint64_t)KVW * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)HQ};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&map_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cuda_error("attn_tc");

    // KV rows for the gathers: one box row of 64 value columns (128-byte
    // swizzle) or of the 32 rope columns (64-byte swizzle)
    const int64_t kv_rows = pr ? (int64_t)pr->num_pages * pr->page_size : (int64_t)r.B * r.T;
    if (kv_rows >= 0x7fffffff) return IC_ERR_UNSUPPORTED;
    CUtensorMap map_kv, map_kvr;
    cuuint64_t kdims[2] = {(cuuint64_t)KVW, (cuuint64_t)kv_rows};
    cuuint32_t kbox[2] = {64, 1};
    cuuint32_t kbox_r[2] = {32, 1};
    if (fn(&map_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kv), kdims, strides, kbox,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cuda_error("attn_tc");
    if (fn(&map_kvr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kv), kdims, strides, kbox_r,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cuda_error("attn_tc");

    AttnArgs a;
    a.q = static_cast<const __nv_bfloat16*>(q);
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
    a.seq_lens = pr ? pr->seq_lens : nullptr;
    a.block_table = pr ? pr->block_table : nullptr;
    a.max_pages = pr ? pr->max_pages : 0;
    a.page_size = pr ? pr->page_size : 1;
    a.num_pages = pr ? pr->num_pages : 0;
    a.kv_rows = (int)kv_rows;
    plan_splits(r, k, a.splits, a.keys_per_split, max_units);
    const int64_t units = (int64_t)r.B * r.Lq * a.splits;
    if (2 * units > 0x7fffffff) return IC_ERR_UNSUPPORTED;
    a.n_units = (int)units;
    a.part_o = nullptr;
    a.part_ml = nullptr;
    if (a.splits > 1) {
        if (scratch_bytes < attn_tc_scratch_bytes(r, k, max_units) || scratch == nullptr)
            return IC_ERR_WORKSPACE;
        const size_t o_bytes = (size_t)units * HQ * DV * sizeof(__nv_bfloat16);
        a.part_o = static_cast<__nv_bfloat16*>(scratch);
        a.part_ml = reinterpret_cast<float2*>(static_cast<char*>(scratch) + o_bytes + 256 -
                                              (o_bytes & 255));
    }
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES) != cudaSuccess)
        return cuda_error("attn_tc");
    const int64_t pairs = std::min<int64_t>(units, std::max(1, sm_count() / 2));
    const bool pdl = pdl_rows((int64_t)r.B * r.Lq);
    if (launch_ex(attn_tc_kernel, dim3((unsigned)(2 * pairs)), dim3(N_THREADS), SMEM_BYTES, s, pdl,
                  0, map_q, map_kv, map_kvr, a) != cudaSuccess)
        return cuda_error("attn_tc");
    count_launch(IC_LK_ATTN_TC);
    ic_status st = last_launch_status();
    if (st != IC_OK || a.splits <= 1) return st;
    static_assert(HQ % COMBINE_HEADS == 0, "combine grid");
    const dim3 grid((unsigned)((int64_t)r.B * r.Lq), HQ / COMBINE_HEADS);
    auto kern = a.splits <= 2 ? attn_combine_kernel<2>
              : a.splits <= 4 ? attn_combine_kernel<4>
              : a.splits <= 8 ? attn_combine_kernel<8>
                              : attn_combine_kernel<16>;
    if (launch_ex(kern, grid, dim3(COMBINE_THREADS), 0, s, pdl, 0, a.part_o, a.part_ml, a.splits,
                  static_cast<__nv_bfloat16*>(out)) != cudaSuccess)
        return cuda_error("attn_combine");
    count_launch(IC_LK_COMBINE);
    return last_launch_status();
}

}  // namespace

ic_status launch_attn_tc(const void* q, const void* kv, int64_t ks, const int32_t* idx, int k,
                         ic_rows r, float scale, void* out, uint32_t* status, void* scratch,
                         size_t scratch_bytes, cudaStream_t s, int64_t max_units) {
    (void)ks;
    return attn_tc_core(q, kv, idx, k, r, scale, out, status, scratch, scratch_bytes, s, max_units,
                        nullptr);
}

ic_status launch_attn_tc_paged(const void* q, const void* kv_pages, const int32_t* idx, int k,
                               const ic_paged_rows& pr, float scale, void* out, uint32_t* status,
                               void* scratch, size_t scratch_bytes, cudaStream_t s) {
    const ic_rows r = {pr.B, pr.Lq, pr.T_max - pr.Lq, pr.T_max};
    return attn_tc_core(q, kv_pages, idx, k, r, scale, out, status, scratch, scratch_bytes, s,
                        kNoUnitLimit, &pr);
}

}  // namespace ic
