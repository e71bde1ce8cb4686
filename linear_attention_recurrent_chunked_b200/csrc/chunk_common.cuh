// Helpers shared by the two tensor-core chunk paths (chunk_tc.cu, chunk_ws.cu):
// small shared-memory / cp.async wrappers, the segment lookup and the TMA
// descriptor of a token-major [T][H][128] bf16 tensor.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace gdn {
namespace chunk {

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Wait until at most one committed cp.async group of this thread is still pending.
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
// Eight fp32 values as one 16-byte bf16 run.
__device__ __forceinline__ void st_run8(uint32_t addr, const float *x) {
    st_shared_v4(addr, tc::pack_bf16x2(x[0], x[1]), tc::pack_bf16x2(x[2], x[3]), tc::pack_bf16x2(x[4], x[5]),
                 tc::pack_bf16x2(x[6], x[7]));
}
// 2^x on the MUFU unit (inputs here are <= 0; results below 2^-126 flush to zero).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Segment of global index gseg: sequence n, index s within it, count ns, token range [a, b).
struct Segment {
    int n, s, ns, a, b, seq_end;
};
__device__ __forceinline__ bool find_segment(const int32_t *seg_off, const int32_t *cu, int N, int T_tot, int gseg,
                                             int seg_tokens, Segment &sg) {
    if (!seg_off) {  // one segment per sequence
        sg.n = gseg;
        sg.s = 0;
        sg.ns = 1;
    } else {
        if (gseg >= seg_off[N]) return false;
        int lo = 0, hi = N - 1;
        while (lo < hi) {  // largest n with seg_off[n] <= gseg
            const int mid = (lo + hi + 1) >> 1;
            if (seg_off[mid] <= gseg) lo = mid; else hi = mid - 1;
        }
        sg.n = lo;
        sg.s = gseg - seg_off[lo];
        sg.ns = seg_off[lo + 1] - seg_off[lo];
    }
    int t0, t1;
    seq_bounds(cu, sg.n, N, T_tot, t0, t1);
    sg.seq_end = t1;
    if (sg.ns == 1) {
        sg.a = t0;
        sg.b = t1;
    } else {
        sg.a = min(t1, t0 + sg.s * seg_tokens);
        sg.b = min(t1, sg.a + seg_tokens);
    }
    return true;
}

// TMA descriptor of a token-major bf16 tensor [T][H][128]: boxes of 64
// columns (128 bytes) x 1 head x 64 tokens, written to shared memory with the
// 128-byte swizzle, out-of-range tokens reading as zero; or (whole_rows) boxes
// of whole 256-byte rows x 64 tokens without swizzle, for the output store.
inline cudaError_t make_row_map(CUtensorMap *map, const __nv_bfloat16 *base, int H, int T, bool whole_rows = false) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!encode) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {128u, (cuuint64_t)H, (cuuint64_t)std::max(T, 1)};
    const cuuint64_t strides[2] = {256u, (cuuint64_t)H * 256u};
    const cuuint32_t box[3] = {whole_rows ? 128u : 64u, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16 *>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              whole_rows ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace chunk
}  // namespace gdn
