// attn_noalloc.cu -- a workspace-free variant of the latent sparse attention.
//
// Some callers cannot allocate device memory at the point where they run
// attention: an inference engine whose memory pool hands out all of the GPU
// at start-up and forbids allocation in its serving loop, a plugin that is
// only given input and output buffers by its host framework, or a latency-
// critical step in which a cudaMalloc (which may synchronise the device) is
// not acceptable.  ic_sparse_attn needs a caller-provided workspace for the
// split-k partials of decode; this variant keeps them instead in a
// file-scope device array of fixed size, so the caller passes only inputs and
// outputs.
//
// The array (IC_NOALLOC_SCRATCH_BYTES) is part of the library's device image:
// every GPU that loads the library holds it until the process exits.  All
// calls share it and it keeps the previous call's contents; the status word
// at its start is cleared at the beginning of every call, and the partials
// are always written before they are read.  Two calls whose kernels overlap on
// the GPU (different streams, or different host threads) race on the array.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace ic {
namespace {

constexpr size_t kStatusBytes = 256;
// split-k units (query rows x splits) whose partials fit in the array
constexpr int64_t kMaxUnits = 64;

// status word (first 256 bytes) followed by the split-k partials
static __device__ __align__(256) unsigned char g_noalloc_scratch[IC_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
struct ScratchAddr {
    void* ctx;    // the CUDA context the address was looked up in
    void* addr;   // device address of g_noalloc_scratch in that context
};
ScratchAddr g_scratch_addr[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Device address of the scratch array in the current device's current
// context.  Looked up with cudaGetSymbolAddress on the first call on each
// device, with that device current, and again whenever that device's
// context has changed since (for example after a cudaDeviceReset, which
// frees the old address).  Returns nullptr on failure.
void* scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    CtxGetCurrentFn get = ctx_get_current();
    if (get == nullptr) return nullptr;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    ScratchAddr& e = g_scratch_addr[dev];
    if (ctx == nullptr || e.addr == nullptr || e.ctx != (void*)ctx) {
        // binds the device's primary context first when none is current yet
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return nullptr;
        e.ctx = (void*)ctx;
        e.addr = p;
    }
    return e.addr;
}

}  // namespace
}  // namespace ic

using namespace ic;

extern "C" ic_status ic_sparse_attn_noalloc(const void* q, const void* kv, const int32_t* idx,
                                             int k, ic_rows r, float scale, void* out,
                                             int32_t* device_status, void* stream) {
    if (r.B < 0 || r.Lq < 0 || r.q_start < 0 || r.T < 0 || (int64_t)r.q_start + r.Lq > r.T)
        return IC_ERR_INVALID_ARG;
    if (k < 1 || k > 16384) return IC_ERR_INVALID_ARG;
    if (r.B == 0 || r.Lq == 0) return IC_OK;
    if (!q || !kv || !idx || !out) return IC_ERR_INVALID_ARG;
    // rows that split their keys need partials in the array: plan at most
    // kMaxUnits units (rows x splits); only when even the fewest splits a row
    // can have (ceil(k / 2048)) leave more units is the call refused
    const size_t need = attn_tc_scratch_bytes(r, k, kMaxUnits);
    if (need > 0 && attn_tc_units(r, k, kMaxUnits) > kMaxUnits) return IC_ERR_WORKSPACE;
    if (need > IC_NOALLOC_SCRATCH_BYTES - kStatusBytes) return IC_ERR_WORKSPACE;
    char* base = static_cast<char*>(scratch_address());
    if (base == nullptr) return cuda_error("attn_noalloc");
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t* status = reinterpret_cast<uint32_t*>(base);
    if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return cuda_error("attn_noalloc");
    ic_status st = launch_attn_tc(q, kv, 576, idx, k, r, scale, out, status, base + kStatusBytes,
                                  IC_NOALLOC_SCRATCH_BYTES - kStatusBytes, s, kMaxUnits);
    if (st != IC_OK) return st;
    if (device_status != nullptr &&
        cudaMemcpyAsync(device_status, status, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
        return cuda_error("attn_noalloc");
    return IC_OK;
}
