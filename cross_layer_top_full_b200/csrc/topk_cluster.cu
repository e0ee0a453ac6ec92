// topk_cluster.cu -- top-k of few, long rows (decode) in ONE launch: one
// thread-block cluster per row, the row's scores read from memory once.
//
// Same rule as topk.cu (keep the min(k, t+1) largest scores, ties to the
// smaller position, -0.0 = +0.0, ascending output padded with -1; DSA's
// per-query top-k, IndexCache summary, es page, section 1).
//
// A row of n candidates is cut into CL contiguous segments (CL = the cluster
// size, 1..8), one per CTA, each read from memory once and cached in shared
// memory as order-preserving 32-bit keys; cluster_select.cuh then finds the
// exact top-k with three radix digits reduced over distributed shared memory
// and cluster barriers only (no flag, no spin-wait, no global workspace).
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "cluster_select.cuh"

namespace ic {
namespace {

using csel::ClusterSmem;

constexpr int NT = 512;
constexpr int CL_MAX = 16;              // non-portable cluster size (B200: up to 16)
constexpr int SEG_MAX = 40960;          // keys of one CTA cached in shared memory (160 KB)

__global__ void __launch_bounds__(NT, 1)
topk_cluster_kernel(const float* __restrict__ scores, int64_t ld, int Lq, int q_start, int k,
                    int32_t* __restrict__ idx, const int32_t* __restrict__ seq_lens, int T_max) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    ClusterSmem<NT / 32>& S = *reinterpret_cast<ClusterSmem<NT / 32>*>(smem_raw);
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(ClusterSmem<NT / 32>));

    pdl_trigger();
    pdl_wait();
    const uint32_t CL = csel::cluster_ctas();
    const uint32_t rank = csel::cta_rank();
    const int64_t row = blockIdx.x / CL;
    const int n = row_candidates(row, Lq, q_start, seq_lens, T_max);
    int32_t* dst = idx + row * (int64_t)k;

    if (n <= k) {  // every candidate is kept (the same decision in every CTA of the cluster)
        if (rank == 0)
            for (int j = threadIdx.x; j < k; j += NT) dst[j] = j < n ? j : -1;
        return;
    }
    // this CTA's segment [s0, s1): CL pieces of a multiple of 4 keys
    const int seg = ((n + (int)CL - 1) / (int)CL + 3) & ~3;
    const int s0 = min(n, (int)rank * seg);
    const int s1 = min(n, s0 + seg);
    const int m = s1 - s0;
    const float* src = scores + row * ld + s0;
    // scores -> order keys in shared memory (16-byte loads: s0 and the row
    // start are multiples of 4 floats), four loads in flight per thread
    for (int j0 = 4 * threadIdx.x; j0 < m; j0 += 16 * NT) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + 4 * NT * u;
            if (j + 3 < m) v[u] = __ldg(reinterpret_cast<const float4*>(src + j));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + 4 * NT * u;
            if (j + 3 < m) {
                *reinterpret_cast<uint4*>(keys + j) =
                    make_uint4(order_key(v[u].x), order_key(v[u].y), order_key(v[u].z), order_key(v[u].w));
            } else {
                for (int q = j; q < m; ++q) keys[q] = order_key(src[q]);
            }
        }
    }
    __syncthreads();
    csel::cluster_select<NT>(S, keys, m, s0, k, dst, CL, rank);
}


size_t cluster_smem(int seg) { return sizeof(ClusterSmem<NT / 32>) + (size_t)seg * sizeof(uint32_t); }

int segment(int n_max, int cl) { return ((n_max + cl - 1) / cl + 3) & ~3; }

// Co-resident clusters of size cl with `smem` bytes per CTA (0 if none fits).
int active_clusters(int cl, size_t smem) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cl, 1, 1);
    cfg.blockDim = dim3(NT, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

bool kernel_attributes_set() {
    static int done = -1;
    if (done < 0)
        done = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)cluster_smem(SEG_MAX)) == cudaSuccess &&
               cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                    1) == cudaSuccess;
    if (!done) cudaGetLastError();
    return done;
}

}  // namespace

// Cluster size for `rows` rows of up to n_max candidates: among the sizes
// whose segment fits in shared memory, the one that minimises (waves of
// co-resident clusters) x (keys per CTA), i.e. the most CTAs per row that
// still keep the rows in as few waves as possible.  0 if none fits.
int topk_cluster_size(ic_rows r, int k) {
    const int64_t rows = (int64_t)r.B * r.Lq;
    const int n_max = r.q_start + r.Lq;
    if (rows <= 0 || n_max <= k || !kernel_attributes_set()) return 0;
    // the occupancy queries cost host time: one answer per (device, rows, n_max)
    int dev = 0;
    cudaGetDevice(&dev);
    static std::mutex mu;
    static std::map<std::tuple<int, int64_t, int>, int> cache;
    const auto key = std::make_tuple(dev, rows, n_max);
    {
        std::lock_guard<std::mutex> lock(mu);
        const auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    int best = 0;
    double best_cost = 1e300;
    for (int cl = 1; cl <= CL_MAX; cl *= 2) {
        const int seg = segment(n_max, cl);
        if (seg > SEG_MAX) continue;
        const int act = active_clusters(cl, cluster_smem(seg));
        if (act <= 0) continue;
        const double cost = (double)((rows + act - 1) / act) * (double)seg;
        if (cost < best_cost * 0.999) {
            best_cost = cost;
            best = cl;
        }
    }
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = best;
    return best;
}

bool topk_cluster_applies(ic_rows r, int k) {
    const int64_t rows = (int64_t)r.B * r.Lq;
    // few rows (decode); long enough that a row needs more than one CTA
    return rows <= 256 && r.q_start + r.Lq > 4096 && topk_cluster_size(r, k) > 0;
}

ic_status launch_topk_cluster(const float* scores, int64_t ld, ic_rows r, int k, int32_t* idx,
                              cudaStream_t s, const int32_t* seq_lens) {
    const int cl = topk_cluster_size(r, k);
    if (cl == 0) return IC_ERR_UNSUPPORTED;
    const int64_t rows = (int64_t)r.B * r.Lq;
    const int n_max = r.q_start + r.Lq;
    const size_t smem = cluster_smem(segment(n_max, cl));
    if (launch_ex(topk_cluster_kernel, dim3((unsigned)(rows * cl)), dim3(NT), smem, s,
                  pdl_rows(rows), (unsigned)cl, scores, ld, r.Lq, r.q_start, k, idx, seq_lens,
                  r.T) != cudaSuccess)
        return cuda_error("topk_cluster");
    count_launch(IC_LK_TOPK);
    return last_launch_status();
}

}  // namespace ic
