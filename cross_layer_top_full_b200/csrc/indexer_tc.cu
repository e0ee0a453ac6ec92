// indexer_tc.cu -- lightning-indexer scores on the 5th-generation tensor
// cores (tcgen05 + TMEM, operands staged by TMA).
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
// stores 32 consecutive keys of a score row (coalesced).
//
// Warp roles (persistent CTA, one per SM):
//   warp 0      TMA producer: q_I block of the work item once, then a ring of
//               k_I tiles (STAGES deep);
//   warp 1      TMEM allocator + single-thread MMA issuer: per key tile
//               8 (bf16, K=16) or 4 (e4m3, K=32) MMAs into one of two TMEM
//               accumulators;
//   warps 2..9  epilogue: TMEM -> registers, release the accumulator, then
//               ReLU, weighted head-sum, causal mask, float32 stores.
// Work item = (sequence b, group of NTOK query rows, chunk of key tiles);
// items are ordered heaviest group first and strided over the CTAs.  Key
// tiles above a group's last causal key are never loaded.
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace ic {
namespace {

using namespace sm100;

constexpr int BM = 128;          // keys per tile (MMA M)
constexpr int D_I = 128;         // indexer width handled here
constexpr int N_EPI_WARPS = 8;
constexpr int N_THREADS = 32 * (2 + N_EPI_WARPS);
constexpr int SMEM_BUDGET = 200 * 1024;

template <int H, int NTOK, bool FP8>
struct Cfg {
    static constexpr int N = H * NTOK;                       // MMA N
    static constexpr int ESZ = FP8 ? 1 : 2;                  // bytes per element
    static constexpr int ATOMS = D_I * ESZ / 128;            // 128-byte K chunks per row
    static constexpr int A_BYTES = BM * D_I * ESZ;           // one key tile
    static constexpr int B_BYTES = N * D_I * ESZ;            // one query block
    static constexpr int STAGES_RAW = (SMEM_BUDGET - B_BYTES) / A_BYTES;
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

template <int H, int NTOK, bool FP8>
__global__ void __launch_bounds__(N_THREADS, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                  const float* __restrict__ w, const float* __restrict__ q_scale,
                  const float* __restrict__ k_scale, float* __restrict__ scores, int64_t ld, int B,
                  int Lq, int q_start, int T, Work wk, Paging pg, uint32_t* status) {
    using C = Cfg<H, NTOK, FP8>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
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
            for (int id = blockIdx.x; id < wk.n_items; id += gridDim.x) {
                int b, i0, kt0, kt1, qs, Tb;
                if (!decode_item(id, wk, B, Lq, q_start, T, pg, NTOK, b, i0, kt0, kt1, qs, Tb)) {
                    // a paged sequence whose length is out of range has no keys
                    if (pg.seq_lens != nullptr && !(Tb >= Lq && Tb <= pg.T_max))
                        flag_status(status, IC_DEV_INDEX_RANGE);
                    continue;
                }
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
            for (int id = blockIdx.x; id < wk.n_items; id += gridDim.x) {
                int b, i0, kt0, kt1, qs, Tb;
                if (!decode_item(id, wk, B, Lq, q_start, T, pg, NTOK, b, i0, kt0, kt1, qs, Tb)) continue;
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
            for (int id = blockIdx.x; id < wk.n_items; id += gridDim.x) {
                int b, i0, kt0, kt1, qs, Tb;
                if (!decode_item(id, wk, B, Lq, q_start, T, pg, NTOK, b, i0, kt0, kt1, qs, Tb)) continue;
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
                bool ok = true;
                for (int kt = kt0; kt < kt1; ++kt, ++acc_it) {
                    if (C::ALT_TILES && (int)(acc_it & 1) != group) continue;   // the other warpgroup's tile
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

                    const int s = kt * BM + quad * 32 + lane;
                    const int64_t krow0 = key_row(pg, b, T, kt * BM);
                    const bool key_ok = krow0 < pg.key_rows;
                    if (!key_ok && lane == 0 && quad == 0) flag_status(status, IC_DEV_INDEX_RANGE);
                    float ks = 1.f;
                    if (FP8 && s < Tb && key_ok) ks = k_scale[krow0 + quad * 32 + lane];
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
                        if (i < Lq && s <= qs + i)
                            scores[((int64_t)b * Lq + i) * ld + s] = key_ok ? sc : -INFINITY;
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

// 2D map over a [rows, 128-element] row-major matrix, box = 128 bytes x box_rows,
// 128-byte swizzle (the UMMA K-major canonical layout).
bool make_map(CUtensorMap* map, const void* base, int64_t rows, bool fp8, int box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const int esz = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)D_I, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D_I * esz};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int H, int NTOK, bool FP8>
ic_status launch_cfg(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                     const float* k_scale, ic_rows r, float* scores, int64_t ld, uint32_t* status,
                     cudaStream_t s, const Paging& pg, int64_t key_rows) {
    using C = Cfg<H, NTOK, FP8>;
    CUtensorMap map_k, map_q;
    if (!make_map(&map_k, k_idx, key_rows, FP8, BM)) return cuda_error("indexer_tc");
    if (!make_map(&map_q, q_idx, (int64_t)r.B * r.Lq * H, FP8, C::N)) return cuda_error("indexer_tc");
    Work wk;
    wk.n_groups = ceil_div(r.Lq, NTOK);
    // dense: the last row's candidates; paged: the longest possible sequence
    const int max_tiles = ceil_div(r.q_start + r.Lq, BM);
    const int base_items = r.B * wk.n_groups;
    const int sms = num_sms();
    int split = 1;
    if (base_items < 2 * sms) split = ceil_div(2 * sms, base_items);
    wk.chunk_tiles = ceil_div(max_tiles, split);
    wk.n_chunks = ceil_div(max_tiles, wk.chunk_tiles);
    const int64_t items = (int64_t)base_items * wk.n_chunks;
    if (items > 0x7fffffff) return IC_ERR_UNSUPPORTED;
    wk.n_items = (int)items;
    const size_t smem = 1024 + (size_t)C::STAGES * C::A_BYTES + C::B_BYTES +
                        sizeof(float) * (N_EPI_WARPS * C::TOK_PER_GROUP * (H + 1) + 4) + sizeof(Bars);
    auto kern = indexer_tc_kernel<H, NTOK, FP8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return cuda_error("indexer_tc");
    const int grid = (int)std::min<int64_t>(items, sms);
    kern<<<grid, N_THREADS, smem, s>>>(map_k, map_q, w, q_scale, k_scale, scores, ld, r.B, r.Lq,
                                       r.q_start, r.T, wk, pg, status);
    count_launch(IC_LK_INDEXER_TC);
    return last_launch_status();
}

template <int H, bool FP8>
ic_status launch_h(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                   const float* k_scale, ic_rows r, float* scores, int64_t ld, uint32_t* status,
                   cudaStream_t s, const Paging& pg, int64_t key_rows) {
    constexpr int NT_WIDE = 256 / H;
    if (r.Lq <= 2)  // decode: one token per accumulator, the scan is HBM-bound
        return launch_cfg<H, 1, FP8>(q_idx, q_scale, w, k_idx, k_scale, r, scores, ld, status, s,
                                     pg, key_rows);
    return launch_cfg<H, NT_WIDE, FP8>(q_idx, q_scale, w, k_idx, k_scale, r, scores, ld, status,
                                       s, pg, key_rows);
}

ic_status launch_any(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                     const float* k_scale, ic_dtype dt, ic_rows r, int H_I, float* scores,
                     int64_t ld, uint32_t* status, cudaStream_t s, const Paging& pg,
                     int64_t key_rows) {
    const bool fp8 = dt == IC_FP8_E4M3;
#define IC_IDX_CASE(HH)                                                                         \
    case HH:                                                                                    \
        return fp8 ? launch_h<HH, true>(q_idx, q_scale, w, k_idx, k_scale, r, scores, ld,      \
                                        status, s, pg, key_rows)                                \
                   : launch_h<HH, false>(q_idx, q_scale, w, k_idx, k_scale, r, scores, ld,     \
                                         status, s, pg, key_rows);
    switch (H_I) {
        IC_IDX_CASE(16)
        IC_IDX_CASE(32)
        IC_IDX_CASE(64)
        IC_IDX_CASE(128)
    }
#undef IC_IDX_CASE
    return IC_ERR_UNSUPPORTED;
}

}  // namespace

bool indexer_tc_supported(ic_dtype dt, int H_I, int d_I) {
    return (dt == IC_BF16 || dt == IC_FP8_E4M3) && d_I == D_I &&
           (H_I == 16 || H_I == 32 || H_I == 64 || H_I == 128);
}

ic_status launch_indexer_tc(const void* q_idx, const float* q_scale, const float* w,
                            const void* k_idx, const float* k_scale, ic_dtype dt, ic_rows r,
                            int H_I, int d_I, float* scores, int64_t ld, uint32_t* status,
                            cudaStream_t s) {
    if (!indexer_tc_supported(dt, H_I, d_I)) return IC_ERR_UNSUPPORTED;
    if (((uintptr_t)q_idx & 15) || ((uintptr_t)k_idx & 15)) return IC_ERR_INVALID_ARG;
    const Paging dense = {nullptr, nullptr, 0, 0, 0, (int64_t)r.B * r.T};
    return launch_any(q_idx, q_scale, w, k_idx, k_scale, dt, r, H_I, scores, ld, status, s, dense,
                      (int64_t)r.B * r.T);
}

ic_status launch_indexer_tc_paged(const void* q_idx, const float* q_scale, const float* w,
                                  const void* k_pages, const float* k_scale_pages, ic_dtype dt,
                                  const ic_paged_rows& pr, int H_I, int d_I, float* scores,
                                  int64_t ld, uint32_t* status, cudaStream_t s) {
    if (!indexer_tc_supported(dt, H_I, d_I)) return IC_ERR_UNSUPPORTED;
    if (((uintptr_t)q_idx & 15) || ((uintptr_t)k_pages & 15)) return IC_ERR_INVALID_ARG;
    const Paging pg = {pr.seq_lens, pr.block_table, pr.max_pages, pr.page_size, pr.T_max,
                       (int64_t)pr.num_pages * pr.page_size};
    // planning rows: every sequence as long as T_max
    const ic_rows r = {pr.B, pr.Lq, pr.T_max - pr.Lq, pr.T_max};
    return launch_any(q_idx, q_scale, w, k_pages, k_scale_pages, dt, r, H_I, scores, ld, status, s,
                      pg, (int64_t)pr.num_pages * pr.page_size);
}

}  // namespace ic
