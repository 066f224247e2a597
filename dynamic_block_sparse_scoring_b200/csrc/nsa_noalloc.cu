// nsa_sparse_attn_fwd_noalloc: the gated sparse-attention forward with its
// block selection, for callers that cannot allocate device memory.
//
// Who needs it: plugin hosts whose execute call must not allocate (the host
// framework owns every device buffer and only hands over inputs and outputs),
// and latency-critical callers for which cudaMalloc/cudaFree are off limits
// because they can synchronise the whole device.  nsa_sparse_attn_fwd needs a
// caller-provided workspace when it selects the blocks itself; this variant
// uses a fixed array that lives in this library instead.
//
// The scratch array below is a file-scope __device__ array, so every GPU that
// loads the library holds NOALLOC_SCRATCH_BYTES of device memory until the
// process exits.  Its host-side name is only a stand-in for the symbol: the
// device address is looked up with cudaGetSymbolAddress, once per device, on
// the first call made with that device current, and cached.
//
// All calls share the one array and it keeps the last call's contents.  The
// array holds the selected block ids, which the selection kernel overwrites
// completely (every slot, -1 padding included) before the attention reads
// them, so nothing in it has to start at zero.  Calls whose work overlaps on
// the GPU (different streams, or different host threads without ordering)
// race on the array: order them, e.g. by issuing them on one stream.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(32) << 20;   // 32 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[MAX_DEVICES] = {nullptr};

// Device address of g_noalloc_scratch on the current device.
nsa_status scratch_address(void** addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return NSA_ERR_CUDA;
    if (dev < 0 || dev >= MAX_DEVICES) return NSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NSA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return NSA_OK;
}

}  // namespace

extern "C" nsa_status nsa_sparse_attn_fwd_noalloc(const nsa_config* cfg, const void* q,
                                                  const void* k, const void* v, const float* kbar,
                                                  const void* kcmp, const void* vcmp,
                                                  const float* gates, void* out, void* stream) {
    size_t need = 0;
    nsa_status st = nsa_workspace_size_min(cfg, &need);
    if (st != NSA_OK) return st;
    if (need > NOALLOC_SCRATCH_BYTES) return NSA_ERR_WORKSPACE;
    void* scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != NSA_OK) return st;
    return nsa_sparse_attn_fwd(cfg, q, k, v, kbar, kcmp, vcmp, gates, nullptr, out, scratch,
                               NOALLOC_SCRATCH_BYTES, stream);
}
