// The UT/WY triangular solve of one chunk: T = (I + A)^{-1} for a strictly
// lower-triangular 64 x 64 fp32 matrix A (the forward-substitution step of the
// chunked rewrite; page 2, "Resumen Tecnico", Metodologia, recurrent-layer
// item, names it as the kernel whose inefficiency first made the chunked form
// lose, and the narrative's second finding attributes that to repeated work
// and stop-start waiting). Here it is one block-wide routine with no per-row
// launches and a fixed, short dependency chain:
//
//   1. the four 16 x 16 diagonal blocks, T_ii = (I + A_ii)^{-1}, by exact fp32
//      forward substitution (one warp per block, one lane per column);
//   2. 16 -> 32: for the blocks (1,0) and (3,2), T_ij = -T_ii (A_ij T_jj);
//   3. 32 -> 64: T[32:64, 0:32] = -T[32:64, 32:64] (A[32:64, 0:32] T[0:32, 0:32]).
//
// Steps 2 and 3 are 16-row-granular products, below the M = 64 minimum of
// tcgen05.mma, so they use warp-level mma.sync m16n8k8 with tf32 operands and
// fp32 accumulation. The fp32 values go in as they are, with no rounding
// instruction: the tensor cores take them at tf32 precision (relative error at
// most 2^-10, that of truncation), under the bf16 rounding the solve's result
// receives when it becomes an MMA operand.
#pragma once

#include <stdint.h>

namespace gdn {
namespace ut {

constexpr int AP = 68;   // pitch of A and T: rows 16-byte aligned; 8 consecutive rows' 16-byte chunks and the
                         // mma fragment patterns (4 g + t) hit distinct banks
constexpr int XP = 40;   // pitch of the product scratch

__device__ __forceinline__ uint32_t tf32(float x) { return __float_as_uint(x); }

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// One warp: d (a 16 x 8 tile, mma accumulator layout) = X[16 x K] * Y[K x 8],
// X row-major with pitch px, Y row-major with pitch py (fp32 in shared memory).
__device__ __forceinline__ void warp_mm(float (&d)[4], const float *X, int px, const float *Y, int py, int K) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    d[0] = d[1] = d[2] = d[3] = 0.f;
    for (int k = 0; k < K; k += 8) {
        const uint32_t a[4] = {tf32(X[g * px + k + t]), tf32(X[(g + 8) * px + k + t]), tf32(X[g * px + k + t + 4]),
                               tf32(X[(g + 8) * px + k + t + 4])};
        const uint32_t b[2] = {tf32(Y[(k + t) * py + g]), tf32(Y[(k + t + 4) * py + g])};
        mma_tf32(d, a, b);
    }
}

// Store a warp tile (16 x 8) to row-major fp32 with pitch p, times `scale`.
__device__ __forceinline__ void warp_store(float *Z, int p, const float (&d)[4], float scale) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    Z[g * p + 2 * t] = scale * d[0];
    Z[g * p + 2 * t + 1] = scale * d[1];
    Z[(g + 8) * p + 2 * t] = scale * d[2];
    Z[(g + 8) * p + 2 * t + 1] = scale * d[3];
}

// Block-wide solve; requires blockDim.x == 256. A, T: [64][AP] fp32 in shared
// memory, 16-byte aligned (A zero on and above the diagonal). X: scratch of 32 * XP floats.
// T may be the same buffer as A: every block of A is read (and the reads
// synchronised) before the block of T at its place is written, and T's blocks
// above the diagonal are then A's zeros already. Ends with a __syncthreads.
__device__ __forceinline__ void solve64(const float *A, float *T, float *X) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // ---- 1. diagonal blocks (warps 0-3) and the zero upper blocks (warps 4-7)
    if (warp < 4) {
        if (lane < 16) {
            const int j = lane, o = 16 * warp;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                // row i of the block in 16-byte broadcast loads (rows are 16-byte aligned: AP % 4 == 0);
                // four partial sums, so that the dependent chain of a row is a quarter as long
                const float *arow = A + (o + i) * AP + o;
                float acc[4] = {(i == j) ? 1.f : 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int s4 = 0; s4 < i; s4 += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(arow + s4);
                    acc[0] = fmaf(-a4.x, x[s4], acc[0]);
                    if (s4 + 1 < i) acc[1] = fmaf(-a4.y, x[s4 + 1], acc[1]);
                    if (s4 + 2 < i) acc[2] = fmaf(-a4.z, x[s4 + 2], acc[2]);
                    if (s4 + 3 < i) acc[3] = fmaf(-a4.w, x[s4 + 3], acc[3]);
                }
                x[i] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            }
            __syncwarp(0x0000ffffu);  // every lane has read its block of A before T overwrites it (A may be T)
#pragma unroll
            for (int i = 0; i < 16; ++i) T[(o + i) * AP + o + j] = x[i];
        }
    } else if (A != T) {
        for (int e = tid - 128; e < 6 * 256; e += 128) {
            const int b = e >> 8, ri = (e >> 4) & 15, cj = e & 15;
            const int bi = (b < 3) ? 0 : (b < 5 ? 1 : 2);
            const int bj = (b < 3) ? b + 1 : (b < 5 ? b - 1 : 3);
            T[(16 * bi + ri) * AP + 16 * bj + cj] = 0.f;
        }
    }
    __syncthreads();
    // ---- 2. blocks (1,0) and (3,2): X_b = A_ij T_jj, then T_ij = -T_ii X_b (warps 0-3: block b = w/2, n-tile w%2).
    // A warp's second product reads back only its own 16 x 8 tile of X_b; the two warps of a block
    // meet (named barrier 2 + b, 64 threads) so that both have read A_ij before T_ij overwrites it.
    if (warp < 4) {
        const int b = warp >> 1, nt = warp & 1, i = 1 + 2 * b, j = i - 1;
        float d[4];
        warp_mm(d, A + (16 * i) * AP + 16 * j, AP, T + (16 * j) * AP + 16 * j + 8 * nt, AP, 16);
        warp_store(X + b * 16 * XP + 8 * nt, XP, d, 1.f);
        if (b == 0)
            asm volatile("bar.sync 2, 64;" ::: "memory");
        else
            asm volatile("bar.sync 3, 64;" ::: "memory");
        warp_mm(d, T + (16 * i) * AP + 16 * i, AP, X + b * 16 * XP + 8 * nt, XP, 16);
        warp_store(T + (16 * i) * AP + 16 * j + 8 * nt, AP, d, -1.f);
    }
    __syncthreads();
    // ---- 3. X = A[32:64, 0:32] T[0:32, 0:32]; T[32:64, 0:32] = -T[32:64, 32:64] X (warp: m-tile w/4, n-tile w%4)
    {
        const int mt = warp >> 2, nt = warp & 3;
        float d[4];
        warp_mm(d, A + (32 + 16 * mt) * AP, AP, T + 8 * nt, AP, 32);
        warp_store(X + 16 * mt * XP + 8 * nt, XP, d, 1.f);
    }
    __syncthreads();
    {
        const int mt = warp >> 2, nt = warp & 3;
        float d[4];
        warp_mm(d, T + (32 + 16 * mt) * AP + 32, AP, X + 8 * nt, XP, 32);
        warp_store(T + (32 + 16 * mt) * AP + 8 * nt, AP, d, -1.f);
    }
    __syncthreads();
}

}  // namespace ut
}  // namespace gdn
