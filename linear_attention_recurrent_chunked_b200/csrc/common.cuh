// Device helpers shared by the library's kernels (not by the oracle).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

// Device error word layout (first 4 bytes of the chunk workspace).
enum : uint32_t { ERRBIT_SEQLENS = 1u, ERRBIT_TIMEOUT = 2u, ERRBIT_INTERNAL = 4u, ERRBIT_BOUNDS = 8u };

// Index checks of the GDN_DEBUG_CHECKS build: an index into a workspace region or an output,
// checked against the region's size. Out of range, the error word gets ERRBIT_BOUNDS and the
// access goes to index 0 instead (in range), so that the kernel finishes without touching memory
// outside the region and the host reads the error. In the normal build the index passes unchanged
// and no code is generated.
#ifdef GDN_DEBUG_CHECKS
__device__ __noinline__ inline void debug_out_of_bounds(uint32_t *err) { atomicOr(err, ERRBIT_BOUNDS); }
template <typename I>
__device__ __forceinline__ I checked(I idx, I lim, uint32_t *err) {
    if (idx < lim) return idx;
    debug_out_of_bounds(err);
    return I(0);
}
#else
template <typename I>
__device__ __forceinline__ I checked(I idx, I, uint32_t *) {
    return idx;
}
#endif

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float *p) { return *p; }
    static __device__ __forceinline__ void store(float *p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

// Four consecutive elements as fp32 (8-byte load for bf16, 16-byte load for fp32).
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    uint2 raw = *reinterpret_cast<const uint2 *>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// Input preparation of the raw-input entry points (the layer's own gates and normalisation):
// the decay exponent g = -softplus(a) (alpha = exp(g)) of a raw gate logit a, with
// softplus(a) = max(a, 0) + log(1 + exp(-|a|)); the write strength beta = sigmoid(b); and the
// factor 1 / max(||x||, 1e-12) that normalises a vector whose squared norm is ss.
__device__ __forceinline__ float neg_softplus(float a) { return -(fmaxf(a, 0.f) + log1pf(expf(-fabsf(a)))); }
__device__ __forceinline__ float sigmoid_f(float b) { return 1.f / (1.f + expf(-b)); }
__device__ __forceinline__ float inv_norm(float ss) { return rsqrtf(fmaxf(ss, 1e-24f)); }

// Sequence bounds from cu_seqlens (device) or equal split, clamped to [0, T_tot].
__device__ __forceinline__ void seq_bounds(const int32_t *cu, int n, int N, int T_tot, int &t0, int &t1) {
    if (cu) {
        t0 = cu[n];
        t1 = cu[n + 1];
    } else {
        const int L = T_tot / N;
        t0 = n * L;
        t1 = t0 + L;
    }
    t0 = min(max(t0, 0), T_tot);
    t1 = min(max(t1, t0), T_tot);
}

}  // namespace gdn
