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
// device address is looked up with cudaGetSymbolAddress on every call, with
// the caller's device current (a host-side lookup; nothing is cached, so a
// cudaDeviceReset or another context on the same device cannot leave a stale
// address behind).
//
// All calls share the one array and it keeps the last call's contents.  It is
// handed to nsa_sparse_attn_fwd as a workspace of NOALLOC_SCRATCH_BYTES bytes,
// so it holds whatever scratch the plan for that size uses: the selected block
// ids always, and the plan's index lists and partial results when the
// problem's full workspace fits.  Every plan writes or clears what it reads
// before reading it, so nothing in the array has to start at zero.  Calls
// whose work overlaps on the GPU (different streams, or different host
// threads without ordering) race on the array: order them, e.g. by issuing
// them on one stream.
#include "common.cuh"

namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(32) << 20;   // 32 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current context.
nsa_status scratch_address(void** addr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NSA_ERR_CUDA;
    *addr = p;
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
