// indexer_pipeline.cuh -- the lightning-indexer score pipeline on the
// 5th-generation tensor cores (tcgen05 + TMEM, operands staged by TMA), as a
// device function shared by the stand-alone indexer kernel (indexer_tc.cu:
// scores to global memory) and the fused decode indexer + top-k kernel
// (select_fused.cu: scores kept in shared memory as order keys).
//
// scores[b,i,s] = sum_h w[b,i,h] * max(0, q_I[b,i,h,:] . k_I[b,s,:])  for s <= t
// (the indexer scores every preceding token of each query, O(L^2) per layer:
// IndexCache summary, es page, section 1 "El Problema"; pt page, section 1
// "O Gargalo do Indexador").  With E4M3 operands the per-token scales
// multiply the finished head-sum (ReLU is positively homogeneous).
//
// GEMM orientation: M = 128 keys of one tile (TMEM lane = key), N = NTOK
// query tokens x H heads (TMEM column = token*H + head), K = d_I = 128.  The
// head-sum is then thread-local in the epilogue (no shuffles) and every warp
// handles 32 consecutive keys of a score row.
//
// Warp roles (one CTA):
//   warp 0      TMA producer: q_I block of a work item once, then a ring of
//               k_I tiles (STAGES deep);
//   warp 1      TMEM allocator + single-thread MMA issuer: per key tile
//               8 (bf16, K=16) or 4 (e4m3, K=32) MMAs into one of the TMEM
//               accumulators;
//   warps 2..9  epilogue: TMEM -> registers, release the accumulator, then
//               ReLU, weighted head-sum, causal mask, and the score to the sink.
#pragma once

#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace ic {
namespace idx {

using namespace sm100;

constexpr int BM = 128;          // keys per tile (MMA M)
constexpr int D_I = 128;         // indexer width handled here
constexpr int N_EPI_WARPS = 8;
constexpr int N_THREADS = 32 * (2 + N_EPI_WARPS);
constexpr int SMEM_BUDGET = 200 * 1024;

// BUDGET: shared memory for the key-tile ring and the query block.
template <int H, int NTOK, bool FP8, int BUDGET = SMEM_BUDGET>
struct Cfg {
    static constexpr int N = H * NTOK;                       // MMA N
    static constexpr int ESZ = FP8 ? 1 : 2;                  // bytes per element
    static constexpr int ATOMS = D_I * ESZ / 128;            // 128-byte K chunks per row
    static constexpr int A_BYTES = BM * D_I * ESZ;           // one key tile
    static constexpr int B_BYTES = N * D_I * ESZ;            // one query block
    static constexpr int STAGES_RAW = (BUDGET - B_BYTES) / A_BYTES;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    // One token per accumulator (decode): four accumulators and the two
    // epilogue warpgroups take alternate key tiles.  Several tokens (prefill):
    // two accumulators and each warpgroup takes half of every tile's tokens.
    static constexpr bool ALT_TILES = NTOK == 1;
    static constexpr int NACC = ALT_TILES ? 4 : 2;
    static constexpr int TMEM_COLS = (NACC * N) < 32 ? 32 : NACC * N;
    static constexpr int K_STEP_BYTES = 32;                  // K per MMA: 16 bf16 / 32 e4m3
    static constexpr int EPI_GROUPS = 2;
    static constexpr int TOK_PER_GROUP = ALT_TILES ? 1 : NTOK / 2;
    static constexpr int ACC_EMPTY_ARRIVALS = ALT_TILES ? 4 : 8;
    static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N");
    static_assert(STAGES >= 2, "pipeline depth");
    static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM allocation is a power of two");
};

struct Work {
    int n_groups, n_chunks, chunk_tiles, n_items;
};

// Where the keys of sequence b live.  Dense: rows b*T .. b*T + T-1 of k_I,
// every sequence T keys, queries from q_start.  Paged: sequence b has
// seq_lens[b] keys, its queries start at seq_lens[b] - Lq, and key position
// s is row block_table[b*max_pages + s/page_size]*page_size + s%page_size
// (page_size a multiple of the 128-key tile, so a tile never straddles pages).
struct Paging {
    const int32_t* seq_lens;      // nullptr: dense
    const int32_t* block_table;
    int max_pages, page_size, T_max;
    int64_t key_rows;             // rows of k_I (and of k_scale)
};

// This sequence's first query position and key count; false (and the
// index-range status bit) for a length outside [Lq, T_max].
__device__ __forceinline__ bool seq_extent(const Paging& pg, int b, int Lq, int q_start, int T,
                                           int& qs, int& Tb) {
    if (pg.seq_lens == nullptr) {
        qs = q_start;
        Tb = T;
        return true;
    }
    Tb = __ldg(pg.seq_lens + b);
    qs = Tb - Lq;
    return Tb >= Lq && Tb <= pg.T_max;
}

// First k_I row of the 128-key tile starting at logical key position s0.  A
// block-table entry outside the cache gives key_rows: the tile then lies
// past the end of the tensor map, which TMA fills with zeros, and its keys
// are dropped from the score row.
__device__ __forceinline__ int64_t key_row(const Paging& pg, int b, int T, int s0) {
    if (pg.seq_lens == nullptr) return (int64_t)b * T + s0;
    const int page = __ldg(pg.block_table + (int64_t)b * pg.max_pages + s0 / pg.page_size);
    if (page < 0 || (int64_t)page * pg.page_size >= pg.key_rows) return pg.key_rows;
    return (int64_t)page * pg.page_size + s0 % pg.page_size;
}

struct __align__(8) Bars {
    uint64_t a_full[8], a_empty[8];
    uint64_t b_full, b_empty;
    uint64_t acc_full[4], acc_empty[4];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool decode_item(int id, const Work& wk, int B, int Lq, int q_start,
                                            int T, const Paging& pg, int ntok, int& b, int& i0,
                                            int& kt0, int& kt1, int& qs, int& Tb) {
    const int per_group = B * wk.n_chunks;
    const int g = wk.n_groups - 1 - id / per_group;   // heaviest (latest) group first
    const int rem = id - (wk.n_groups - 1 - g) * per_group;
    b = rem / wk.n_chunks;
    const int c = rem - b * wk.n_chunks;
    i0 = g * ntok;
    if (!seq_extent(pg, b, Lq, q_start, T, qs, Tb)) return false;
    const int i_last = min(i0 + ntok, Lq) - 1;
    const int tiles = (qs + i_last + 1 + BM - 1) / BM;
    kt0 = c * wk.chunk_tiles;
    kt1 = min(kt0 + wk.chunk_tiles, tiles);
    return kt0 < kt1;
}

// A run of key tiles of one work item: sequence b, query rows i0.. (NTOK of
// them), key tiles kt0..kt1-1; qs / Tb are the sequence's first query
// position and key count.
struct Item {
    int b, i0, kt0, kt1, qs, Tb;
};

// The persistent schedule: items strided over the CTAs of the grid.
struct PersistentSched {
    Work wk;
    int B, Lq, q_start, T, ntok;
    Paging pg;
    int id;
    __device__ PersistentSched(const Work& w, int B_, int Lq_, int qs_, int T_, const Paging& p,
                               int nt)
        : wk(w), B(B_), Lq(Lq_), q_start(qs_), T(T_), ntok(nt), pg(p), id((int)blockIdx.x) {}
    // next item; `status` (may be null) receives the index-range bit for a
    // paged sequence whose length is out of range
    __device__ bool next(Item& it, uint32_t* status) {
        while (id < wk.n_items) {
            const int cur = id;
            id += (int)gridDim.x;
            if (decode_item(cur, wk, B, Lq, q_start, T, pg, ntok, it.b, it.i0, it.kt0, it.kt1, it.qs,
                            it.Tb))
                return true;
            if (status != nullptr && pg.seq_lens != nullptr && !(it.Tb >= Lq && it.Tb <= pg.T_max))
                flag_status(status, IC_DEV_INDEX_RANGE);
        }
        return false;
    }
};

// One fixed item per CTA (or none).
struct SingleSched {
    Item item;
    bool has;
    __device__ bool next(Item& it, uint32_t*) {
        if (!has) return false;
        has = false;
        it = item;
        return true;
    }
};

// Score sinks: where a finished score of (sequence b, query row i, key s) goes.
struct GlobalSink {
    float* scores;
    int64_t ld;
    int Lq;
    __device__ __forceinline__ void put(int b, int i, int s, float v) const {
        scores[((int64_t)b * Lq + i) * ld + s] = v;
    }
};


// Shared memory the pipeline of configuration C uses (from a 1024-byte
// aligned base).
template <class C, int H>
__host__ __device__ constexpr size_t pipeline_smem_bytes() {
    return (size_t)C::STAGES * C::A_BYTES + C::B_BYTES +
           sizeof(float) * (N_EPI_WARPS * C::TOK_PER_GROUP * (H + 1) + 4) + sizeof(Bars);
}

// The indexer pipeline of one CTA (all N_THREADS threads call it): TMA
// producer, single-thread MMA issuer and 8 epilogue warps over the items
// that `sched` hands out, each finished score (causal keys only) passed to
// sink.put.  smem: pipeline_smem_bytes<C, H>() bytes, 1024-byte aligned.
// Allocates and frees its TMEM; ends with a CTA barrier.
template <int H, int NTOK, bool FP8, class C, bool EARLY_TRIGGER = true, class Sched, class Sink>
__device__ __forceinline__ void indexer_pipeline(
    const CUtensorMap* map_k_p, const CUtensorMap* map_q_p, uint8_t* smem,
    const float* __restrict__ w, const float* __restrict__ q_scale,
    const float* __restrict__ k_scale, int Lq, int T, const Paging& pg, Sched sched0,
    const Sink& sink, uint32_t* status) {
    const CUtensorMap& map_k = *map_k_p;
    const CUtensorMap& map_q = *map_q_p;
    uint8_t* a_smem = smem;                                  // [STAGES][ATOMS][BM][128B]
    uint8_t* b_smem = a_smem + C::STAGES * C::A_BYTES;       // [ATOMS][N][128B]
    // per epilogue warp: its tokens' head weights and query scales
    float* w_smem = reinterpret_cast<float*>(b_smem + C::B_BYTES);   // [8][TOK_PER_GROUP][H]
    float* qs_smem = w_smem + N_EPI_WARPS * C::TOK_PER_GROUP * H;    // [8][TOK_PER_GROUP]
    Bars* bars = reinterpret_cast<Bars*>(
        (reinterpret_cast<uintptr_t>(qs_smem + N_EPI_WARPS * C::TOK_PER_GROUP) + 15) & ~uintptr_t(15));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int* abort = &bars->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&bars->a_full[s], 1);
            mbar_init(&bars->a_empty[s], 1);
        }
        mbar_init(&bars->b_full, 1);
        mbar_init(&bars->b_empty, 1);
        for (int s = 0; s < C::NACC; ++s) {
            mbar_init(&bars->acc_full[s], 1);
            mbar_init(&bars->acc_empty[s], C::ACC_EMPTY_ARRIVALS);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc<C::TMEM_COLS>(&bars->tmem_base);
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_q);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    // the keys, queries and weights may come from the stream's previous kernel
    if (EARLY_TRIGGER) pdl_trigger();
    pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t a_it = 0, b_it = 0;
            auto load_q = [&](int b, int i0, uint32_t& it) -> bool {
                if (!mbar_wait(&bars->b_empty, (it & 1) ^ 1, status, abort)) return false;
                mbar_arrive_expect_tx(&bars->b_full, C::B_BYTES);
                const int qrow = (b * Lq + i0) * H;
                for (int a = 0; a < C::ATOMS; ++a)
                    tma_load_2d(b_smem + a * (C::N * 128), &map_q, &bars->b_full, a * (128 / C::ESZ),
                                qrow);
                ++it;
                return true;
            };
            Sched sched = sched0;
            Item it;
            // (a paged sequence whose length is out of range has no keys: the
            // producer's schedule flags it)
            while (sched.next(it, status)) {
                const int b = it.b, i0 = it.i0, kt0 = it.kt0, kt1 = it.kt1;
                // The first key tiles of the item go out before the query block:
                // they only need free ring slots, which the previous item's MMAs
                // release, so they overlap its tail.
                const int pre = min(C::STAGES, kt1 - kt0);
                bool ok = true;
                for (int kt = kt0; kt < kt1; ++kt, ++a_it) {
                    if (kt == kt0 + pre) {
                        if (!load_q(b, i0, b_it)) { ok = false; break; }
                    }
                    const int s = a_it % C::STAGES;
                    const uint32_t ph = (a_it / C::STAGES) & 1;
                    if (!mbar_wait(&bars->a_empty[s], ph ^ 1, status, abort)) { ok = false; break; }
                    mbar_arrive_expect_tx(&bars->a_full[s], C::A_BYTES);
                    uint8_t* dst = a_smem + s * C::A_BYTES;
                    const int krow = (int)key_row(pg, b, T, kt * BM);
                    for (int a = 0; a < C::ATOMS; ++a)
                        tma_load_2d(dst + a * (BM * 128), &map_k, &bars->a_full[s],
                                    a * (128 / C::ESZ), krow);
                }
                if (ok && pre == kt1 - kt0 && !load_q(b, i0, b_it)) ok = false;
                if (!ok) break;
            }
            // drain: every issued load has landed before the CTA may exit
            for (uint32_t j = a_it > (uint32_t)C::STAGES ? a_it - C::STAGES : 0; j < a_it; ++j)
                mbar_wait(&bars->a_full[j % C::STAGES], (j / C::STAGES) & 1, status, abort);
            if (b_it) mbar_wait(&bars->b_full, (b_it - 1) & 1, status, abort);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f32acc(FP8 ? 0u : 1u, FP8 ? 0u : 1u, BM, C::N);
            uint32_t a_it = 0, b_it = 0, acc_it = 0;
            const uint32_t a_base = smem_u32(a_smem), b_base = smem_u32(b_smem);
            bool issued = false;
            Sched sched = sched0;
            Item it;
            while (sched.next(it, nullptr)) {
                const int kt0 = it.kt0, kt1 = it.kt1;
                if (!mbar_wait(&bars->b_full, b_it & 1, status, abort)) break;
                bool ok = true;
                for (int kt = kt0; kt < kt1; ++kt, ++a_it, ++acc_it) {
                    const int s = a_it % C::STAGES;
                    const int acc = acc_it % C::NACC;
                    if (!mbar_wait(&bars->a_full[s], (a_it / C::STAGES) & 1, status, abort) ||
                        !mbar_wait(&bars->acc_empty[acc], ((acc_it / C::NACC) & 1) ^ 1, status, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + acc * C::N;
                    const uint32_t a_stage = a_base + s * C::A_BYTES;
#pragma unroll
                    for (int a = 0; a < C::ATOMS; ++a) {
#pragma unroll
                        for (int kk = 0; kk < 128 / C::K_STEP_BYTES; ++kk) {
                            const uint64_t da = desc_sw128(a_stage + a * (BM * 128) + kk * C::K_STEP_BYTES, 16, 1024);
                            const uint64_t db = desc_sw128(b_base + a * (C::N * 128) + kk * C::K_STEP_BYTES, 16, 1024);
                            if (FP8) mma_f8(d_tmem, da, db, idesc, (a | kk) != 0);
                            else mma_bf16(d_tmem, da, db, idesc, (a | kk) != 0);
                        }
                    }
                    issued = true;
                    mma_commit(&bars->a_empty[s]);      // k tile may be overwritten
                    mma_commit(&bars->acc_full[acc]);   // accumulator ready
                }
                if (!ok) break;
                mma_commit(&bars->b_empty);             // q block may be overwritten
                ++b_it;
            }
            if (issued) {
                mma_commit(&bars->drain);               // all MMAs of this CTA finished
                mbar_wait(&bars->drain, 0, status, abort);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;                     // 0..7
        const int group = ew >> 2;                   // which half of the tokens
        const int quad = warp & 3;                   // TMEM lanes 32*quad .. +31
        if (group < C::EPI_GROUPS) {
            uint32_t acc_it = 0;
            Sched sched = sched0;
            Item it;
            while (sched.next(it, nullptr)) {
                const int b = it.b, i0 = it.i0, kt0 = it.kt0, kt1 = it.kt1, qs = it.qs, Tb = it.Tb;
                // stage this item's head weights (and query scales) of my tokens
                // in this warp's own buffer: only the warp itself reads it
                float* w_w = w_smem + ew * C::TOK_PER_GROUP * H;
                float* qs_w = qs_smem + ew * C::TOK_PER_GROUP;
                __syncwarp();
                const int tok0 = C::ALT_TILES ? 0 : group * C::TOK_PER_GROUP;   // my first token
                for (int e = lane; e < C::TOK_PER_GROUP * H; e += 32) {
                    const int i = i0 + tok0 + e / H;
                    w_w[e] = i < Lq ? w[((int64_t)b * Lq + i) * H + e % H] : 0.f;
                }
                if (FP8 && lane < C::TOK_PER_GROUP) {
                    const int i = i0 + tok0 + lane;
                    qs_w[lane] = i < Lq ? q_scale[(int64_t)b * Lq + i] : 0.f;
                }
                __syncwarp();
                // Where a tile's keys live (a block-table load when paged) and this
                // lane's key scale (FP8) are global loads that do not depend on the
                // accumulator.  With one token per accumulator (decode) the tile
                // epilogue is short and that latency would follow each tile's
                // accumulator: they are issued one of this warp's tiles ahead.
                struct TileMeta {
                    int64_t krow0;
                    float ks;
                };
                auto tile_meta = [&](int kt) -> TileMeta {
                    TileMeta m;
                    m.krow0 = key_row(pg, b, T, kt * BM);
                    m.ks = 1.f;
                    if (FP8 && kt * BM + quad * 32 + lane < Tb && m.krow0 < pg.key_rows)
                        m.ks = k_scale[m.krow0 + quad * 32 + lane];
                    return m;
                };
                constexpr bool AHEAD = C::ALT_TILES;               // this warp's tiles: every other one
                const int kt_mine = ((int)(acc_it & 1) != group) ? kt0 + 1 : kt0;
                TileMeta meta_next{};
                if (AHEAD) meta_next = tile_meta(kt_mine < kt1 ? kt_mine : kt0);
                bool ok = true;
                for (int kt = kt0; kt < kt1; ++kt, ++acc_it) {
                    if (C::ALT_TILES && (int)(acc_it & 1) != group) continue;   // the other warpgroup's tile
                    TileMeta meta = meta_next;
                    if (AHEAD && kt + 2 < kt1) meta_next = tile_meta(kt + 2);
                    const int acc = acc_it % C::NACC;
                    if (!warp_wait(&bars->acc_full[acc], (acc_it / C::NACC) & 1, status, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    float d[C::TOK_PER_GROUP][H];
                    const uint32_t t_row = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * C::N;
#pragma unroll
                    for (int jj = 0; jj < C::TOK_PER_GROUP; ++jj) {
                        const int j = tok0 + jj;
                        if constexpr (H >= 32) {
#pragma unroll
                            for (int h0 = 0; h0 < H; h0 += 32) {
                                uint32_t r[32];
                                tmem_ld32(t_row + j * H + h0, r);
#pragma unroll
                                for (int x = 0; x < 32; ++x) d[jj][h0 + x] = __uint_as_float(r[x]);
                            }
                        } else {
                            uint32_t r[16];
                            tmem_ld16(t_row + j * H, r);
#pragma unroll
                            for (int x = 0; x < 16; ++x) d[jj][x] = __uint_as_float(r[x]);
                        }
                    }
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->acc_empty[acc]);   // TMEM free again

                    if (!AHEAD) meta = tile_meta(kt);
                    const int s = kt * BM + quad * 32 + lane;
                    const bool key_ok = meta.krow0 < pg.key_rows;
                    if (!key_ok && lane == 0 && quad == 0) flag_status(status, IC_DEV_INDEX_RANGE);
                    const float ks = meta.ks;
#pragma unroll
                    for (int jj = 0; jj < C::TOK_PER_GROUP; ++jj) {
                        const int j = tok0 + jj;
                        const int i = i0 + j;
                        const float4* wv = reinterpret_cast<const float4*>(w_w + jj * H);
                        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                        for (int h = 0; h < H; h += 4) {
                            const float4 ww = wv[h / 4];
                            acc0 = fmaf(ww.x, fmaxf(d[jj][h + 0], 0.f), acc0);
                            acc1 = fmaf(ww.y, fmaxf(d[jj][h + 1], 0.f), acc1);
                            acc0 = fmaf(ww.z, fmaxf(d[jj][h + 2], 0.f), acc0);
                            acc1 = fmaf(ww.w, fmaxf(d[jj][h + 3], 0.f), acc1);
                        }
                        float sc = acc0 + acc1;
                        if (FP8) sc *= qs_w[jj] * ks;
                        if (i < Lq && s <= qs + i) sink.put(b, i, s, key_ok ? sc : -INFINITY);
                    }
                }
                if (!ok) break;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<C::TMEM_COLS>(tmem_base);
    }
}

}  // namespace idx
}  // namespace ic
