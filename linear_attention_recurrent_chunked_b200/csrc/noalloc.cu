// gdn_chunk_fwd_noalloc: the chunked forward with its scratch memory built into
// the library, for callers that cannot allocate device memory themselves.
//
// Who needs it: code running under a memory manager that has already reserved
// the GPU's memory (so a cudaMalloc would fail or fragment the pool), plugins
// whose host application owns all device allocations, and latency-critical
// paths that must not pay cudaMalloc / cudaFree's implicit synchronisation.
// They still pass their own inputs and outputs; only the workspace that
// gdn_chunk_fwd normally receives from the caller comes from here.
//
// The scratch is a file-scope __device__ array, so every GPU that loads the
// library holds kNoallocScratchBytes of it until the process exits. When a
// call's preferred workspace (gdn_chunk_fwd_workspace_size) is larger than the
// array, the forward runs with the coarser time segmentation that fits. In host
// code the array's name is only a host-side stand-in, never a device address:
// every call looks up the array's device address in the context that is current
// on the calling thread, with cudaGetSymbolAddress (a host-side table lookup;
// the first lookup in a context may load the library's module, so make the first
// call on a device before any stream capture). The address is deliberately not
// cached: after a cudaDeviceReset, or with another context made current, a cached
// address would belong to a context that no longer exists or is not current.
// All calls on a device share the one array; it keeps whatever the last call
// left in it, and the forward path rewrites everything it reads (the error word
// included) before use. Calls that overlap on the GPU (different streams, or
// threads racing on one stream) race on the array and must be serialised by the
// caller.
#include "common.cuh"

namespace gdn {
gdn_status record_error(gdn_status s, const char *msg);
}

namespace {

constexpr size_t kNoallocScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr size_t kMinWorkspaceBytes = 256;                   // gdn_chunk_fwd's minimum (the error word)

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of the scratch array in the current context (looked up on every call).
cudaError_t scratch_for_current_context(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" size_t gdn_chunk_fwd_workspace_size(int N, int T_tot, int H, int dk, int dv, gdn_dtype dtype);
extern "C" gdn_status gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                                    const float *S0, const int32_t *cu_seqlens, int N, int T_tot, int H, int dk,
                                    int dv, gdn_dtype dtype, void *o, float *S_T, void *workspace, size_t ws_bytes,
                                    void *stream);

extern "C" gdn_status gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                                            const float *beta, const float *S0, const int32_t *cu_seqlens, int N,
                                            int T_tot, int H, int dk, int dv, gdn_dtype dtype, void *o, float *S_T,
                                            void *stream) {
    // gdn_chunk_fwd needs at least its 256-byte error word and uses whatever
    // more it gets to split long sequences into segments; the built-in array
    // must at least hold that minimum.
    if (kNoallocScratchBytes < kMinWorkspaceBytes)
        return gdn::record_error(GDN_ERR_WORKSPACE,
                                 "the built-in scratch is smaller than the minimum workspace; use gdn_chunk_fwd "
                                 "with a caller-provided workspace");
    void *ws = nullptr;
    const cudaError_t e = scratch_for_current_context(&ws);
    if (e != cudaSuccess) return gdn::record_error(GDN_ERR_CUDA, cudaGetErrorString(e));
    return gdn_chunk_fwd(q, k, v, g, beta, S0, cu_seqlens, N, T_tot, H, dk, dv, dtype, o, S_T, ws,
                         kNoallocScratchBytes, stream);
}
