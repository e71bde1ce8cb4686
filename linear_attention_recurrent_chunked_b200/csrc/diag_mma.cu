// Diagnostic: one tensor-core tile, D = A * B^T, through the same
// descriptor / TMEM helpers the chunked kernel uses. It exists so that the
// tests can pin the operand layouts (K-major and MN-major views of the
// no-swizzle core-matrix tiles, two stride conventions) and the TMEM
// accumulator layout against a CPU matmul, independently of the full path.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace gdn {
namespace {

// Stage a row-major [rows][cols] bf16 matrix (logical operand rows = MN, cols = K)
// into a core-matrix tile. mn_major: the tile's X axis is K and its 16-byte
// runs go along MN; otherwise X = MN and runs go along K. variant 0 puts
// X-neighbouring core matrices next to each other (sx = 128), variant 1 puts
// Y-neighbours next to each other (sy = 128).
__device__ void stage(uint8_t *dst, const __nv_bfloat16 *src, int rows, int cols, int mn_major, int variant,
                      uint32_t &sx, uint32_t &sy) {
    const int nx = mn_major ? cols : rows, ny = mn_major ? rows : cols;
    if (variant == 0) { sx = 128; sy = (uint32_t)nx * 16; } else { sy = 128; sx = (uint32_t)ny * 16; }
    for (int idx = threadIdx.x; idx < rows * cols; idx += blockDim.x) {
        const int r = idx / cols, c = idx % cols;
        const int x = mn_major ? c : r, y = mn_major ? r : c;
        *reinterpret_cast<__nv_bfloat16 *>(dst + tc::tile_off(x, y, sx, sy)) = src[idx];
    }
}

// 128-byte-swizzled staging (variant 2): K-major tiles have rows = MN and
// 128-byte rows along K; MN-major tiles have rows = K and 128-byte rows along MN.
__device__ void stage_sw128(uint8_t *dst, const __nv_bfloat16 *src, int rows, int cols, int mn_major) {
    const int R = mn_major ? cols : rows;  // tile rows
    for (int idx = threadIdx.x; idx < rows * cols; idx += blockDim.x) {
        const int r = idx / cols, c = idx % cols;
        const int tr = mn_major ? c : r, tc_ = mn_major ? r : c;
        *reinterpret_cast<__nv_bfloat16 *>(dst + tc::sw128_off(tr, tc_, R)) = src[idx];
    }
}

__global__ void __launch_bounds__(128) k_diag_mma(const __nv_bfloat16 *A, const __nv_bfloat16 *B, float *D, int M,
                                                  int N, int K, int a_mn, int b_mn, int variant) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tslot;
    uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);  // 1024-byte aligned base
    uint8_t *sA = smem, *sB = smem + 65536;
    uint32_t axs = 0, ays = 0, bxs = 0, bys = 0;
    if (variant == 2) {
        stage_sw128(sA, A, M, K, a_mn);
        stage_sw128(sB, B, N, K, b_mn);
    } else {
        stage(sA, A, M, K, a_mn, variant, axs, ays);
        stage(sB, B, N, K, b_mn, variant, bxs, bys);
    }
    tc::fence_smem_to_async();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) tc::tmem_alloc(&tslot, 256);
    if (threadIdx.x == 0) {
        tc::mbar_init(&mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tslot;
    if (threadIdx.x == 0) {
        const uint32_t idesc = tc::make_idesc_bf16(M, N, a_mn, b_mn);
        if (variant == 2) {
            // K-major: rows = MN, SBO = 1024 (8-row groups); a K=16 step moves 32 bytes inside
            // the 128-byte row, and K >= 64 continues in the second column half (R x 128 bytes on).
            // MN-major: rows = K, SBO = 1024 (8-row K groups), LBO = K x 128 (next 64-wide MN half);
            // a K=16 step is 16 rows = 2048 bytes.
            for (int kk = 0; kk < K / 16; ++kk) {
                const uint32_t a_off = a_mn ? kk * 2048u : (uint32_t)((kk >> 2) * M * 128 + (kk & 3) * 32);
                const uint32_t b_off = b_mn ? kk * 2048u : (uint32_t)((kk >> 2) * N * 128 + (kk & 3) * 32);
                const uint64_t ad = tc::make_desc_sw128(tc::smem_u32(sA) + a_off, a_mn ? (uint32_t)K * 128 : 16, 1024);
                const uint64_t bd = tc::make_desc_sw128(tc::smem_u32(sB) + b_off, b_mn ? (uint32_t)K * 128 : 16, 1024);
                tc::mma_bf16(tmem, ad, bd, idesc, kk > 0);
            }
        } else {
            // K-major: SBO = X stride (MN), LBO = Y stride (K); one K=16 step = 2 core matrices along Y.
            // MN-major: SBO = Y stride (MN), LBO = X stride (K); one K=16 step = 2 core matrices along X.
            const uint32_t a_sbo = a_mn ? ays : axs, a_lbo = a_mn ? axs : ays, a_step = 2 * (a_mn ? axs : ays);
            const uint32_t b_sbo = b_mn ? bys : bxs, b_lbo = b_mn ? bxs : bys, b_step = 2 * (b_mn ? bxs : bys);
            for (int kk = 0; kk < K / 16; ++kk) {
                const uint64_t ad = tc::make_desc(tc::smem_u32(sA) + kk * a_step, a_lbo, a_sbo);
                const uint64_t bd = tc::make_desc(tc::smem_u32(sB) + kk * b_step, b_lbo, b_sbo);
                tc::mma_bf16(tmem, ad, bd, idesc, kk > 0);
            }
        }
        tc::mma_commit(&mbar);
    }
    const bool done = tc::mbar_wait(&mbar, 0);
    tc::fence_after_sync();
    // Dump every TMEM lane (128) x N columns, so an M=64 layout is visible too.
    for (int c0 = 0; c0 < N; c0 += 16) {
        float r[16];
        tc::tmem_ld16(tc::taddr(tmem, 32 * warp, c0), r);
        for (int i = 0; i < 16 && c0 + i < N; ++i)
            D[(size_t)(32 * warp + lane) * N + c0 + i] = done ? r[i] : __int_as_float(0x7fc00000);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_diag_mma_tile(const void *A, const void *B, float *D, int M, int N, int K, int a_mn,
                                        int b_mn, int variant, void *stream) {
    if (!A || !B || !D) return GDN_ERR_NULL;
    const bool n_ok = (M == 128) ? (N % 16 == 0) : (N % 8 == 0);
    if ((M != 64 && M != 128) || N < 16 || N > 256 || !n_ok || K < 16 || K > 128 || K % 16 || variant < 0 ||
        variant > 2 || (a_mn & ~1) || (b_mn & ~1))
        return GDN_ERR_SHAPE;
    if (variant == 2 && (N > 128 || (a_mn && K < 64 && M > 64) || (b_mn && K < 64 && N > 64)))
        return GDN_ERR_SHAPE;  // swizzled tiles: N <= 128; an MN-major tile wider than 64 needs K >= 64 rows per half
    const int smem = 1024 + 65536 + 65536;
    cudaError_t e = cudaFuncSetAttribute(gdn::k_diag_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    gdn::k_diag_mma<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(A), static_cast<const __nv_bfloat16 *>(B), D, M, N, K, a_mn, b_mn, variant);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" gdn_status gdn_diag_ut_solve(const float *A, float *T, void *stream) {
    if (!A || !T) return GDN_ERR_NULL;
    return gdn::launch_diag_ut_solve(A, T, static_cast<cudaStream_t>(stream)) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
