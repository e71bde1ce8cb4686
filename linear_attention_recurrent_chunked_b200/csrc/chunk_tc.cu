// Chunked gated delta rule on the sm_100a tensor cores (bf16 inputs, d = 128,
// chunk C = 64): tcgen05.mma with bf16 operands staged in shared memory and
// fp32 accumulators in TMEM; the fp32 state lives in TMEM while a CTA walks
// its chunks.
//
// The pages give the shape of the method only: the token-by-token scan of
// the recurrent layers becomes a chunk-wise delta-rule form with an
// intra-chunk part, an inter-chunk part and a forward-substitution step,
// whose one slow kernel had to be fixed before the chunked form won (page 1,
// abstract, result (i); page 2, "Resumen Tecnico", Metodologia,
// recurrent-layer item, and the narrative's second finding). Per chunk of
// one (sequence, head), with S the d_v x d_k state entering the chunk,
// G_r = sum_{s<=r} g_s, gamma_r = exp(G_r), e_s = exp(G_C - G_s):
//
//   X1 = [K;Q] K^T                  A_rs = beta_r exp(G_r-G_s) (KK^T)_rs, s<r
//                                   P_rs = exp(G_r-G_s) (QK^T)_rs,      s<=r
//   T  = (I + A)^{-1}               (ut_solve.cuh)
//   W^T = K^T (T diag(beta gamma))^T,   U^T = V^T (T diag(beta))^T
//   O1 = S Q^T,   Dl = U^T - S W^T  (= Delta^T),   Dt = Delta^T diag(e)
//   O^T = O1 diag(gamma) + Dl P^T   (written to o)
//   S  <- gamma_C S + Dt K          (the state entering the next chunk)
//
// Every product is one M = 128 tcgen05.mma group (D = A B^T): accumulator row
// m sits in TMEM lane m. A CTA has 8 warps; warp w reads TMEM lanes
// 32*(w%4)..+31 and the two warpgroups split the columns, so each thread owns
// half of one accumulator row and writes it back in whichever shared-memory
// orientation the next MMA wants. No operand is transposed through shared
// memory: a tile written with 16-byte runs along one axis is read either
// K-major or MN-major (see tc.cuh). Outputs are staged through shared memory
// so that the stores to o are whole 256-byte rows.
//
// Parallelism over time. A sequence's chunks may be split into segments that
// run concurrently (the host picks the segment length so that the CTAs fill
// the GPU when there are few (sequence, head) pairs). Per chunk the state
// map is affine, S -> S M_c + N_c, so over a segment S_end = S_start Phi +
// S_loc. Pass A (k_chunk_tc_trans) runs every segment but the last of each
// sequence from S = 0 (giving S_loc) and, on a second set of 128 rows, from
// X = I with the V-term dropped (giving Phi = X_end); it writes both to the
// workspace. Pass B (k_chunk_tc) first folds the earlier segments,
// S <- S Phi_j + S_loc_j starting from S0, then runs its own chunks with
// outputs; the last segment writes S_T. Without segmentation pass B alone
// runs, one CTA per (sequence, head).
//
// Chunk c+1's K, Q, V, g, beta are fetched with cp.async while chunk c
// computes. Partial chunks are zero-filled (k = q = v = 0, g = 0, beta = 0),
// which zeroes their rows of A, W, U, Delta and keeps G flat.
#include <algorithm>

#include "chunk_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "ut_solve.cuh"

namespace gdn {
namespace {

using namespace chunk;
using bf16 = __nv_bfloat16;
constexpr int C = 64;     // chunk length
constexpr int D = 128;    // head size (dk = dv)
constexpr int NT = 256;   // threads per CTA (two threads per TMEM lane)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int AP = ut::AP;

// ---- shared memory maps (bytes). Tiles use 8x16-byte core matrices with
// X-neighbouring core matrices adjacent (sx = 128) and sy = 16 * rows.
// Output pass: K and Q share one buffer ([K;Q] is one 128-row operand per column half).
namespace smo {
__device__ __forceinline__ constexpr uint32_t KQ(int b) { return b ? 32768u : 0u; }
__device__ __forceinline__ constexpr uint32_t V(int b) { return b ? 81920u : 65536u; }   // [V_lo | V_hi], 128-byte swizzled
__device__ __forceinline__ constexpr uint32_t GB(int b) { return b ? 98816u : 98304u; }  // raw g[64], beta[64]
constexpr uint32_t KQ_HALF = 16384;  // [K_lo | Q_lo | K_hi | Q_hi], 8 KB each, 128-byte swizzled
constexpr uint32_t T1 = 99328;                  // 64 r x 64 s, sy = 1024   (T diag(beta gamma))
constexpr uint32_t T2 = 107520;                 // 64 r x 64 s               (T diag(beta))
constexpr uint32_t OST = T1;                    // output staging o[r][v] bf16 (64 x 256 B), over T1+T2
constexpr uint32_t P = 115712;                  // 64 r x 64 s
constexpr uint32_t W = 123904;                  // 128 k x 64 r, sy = 2048 (runs along r)
constexpr uint32_t S = 140288;                  // 128 v x 128 k, sy = 2048 (bf16 copy of the state)
constexpr uint32_t UNI = 173056;                // union: {Dl, Dt} bf16  |  {A, T} fp32 [64][AP]
constexpr uint32_t DL = UNI, DT = UNI + 16384;  // 128 v x 64 s, sy = 2048
constexpr uint32_t AF = UNI, TF = UNI + 64 * ut::AP * 4;
constexpr uint32_t VEC = UNI + 2 * 64 * ut::AP * 4;  // G (log2 units), gamma, e, beta: 4 x 64 fp32
constexpr uint32_t BAR = VEC + 1024;            // mbarriers + TMEM slot (see tmem_setup)
constexpr uint32_t TOTAL = BAR + 128;
constexpr uint32_t SCR = W;                     // fp32 scratch of the solve (W is free then)
// segment fold (before the chunk loop): two buffers of {Phi_hi, Phi_lo} bf16 tiles; S_hi is the S tile, S_lo sits in UNI
constexpr uint32_t FOLD_PHI0 = 0, FOLD_PHI1 = 65536, FOLD_SLO = UNI;
}  // namespace smo
// Transition pass: no Q; a second state (X) tile.
namespace smt {
__device__ __forceinline__ constexpr uint32_t K(int b) { return b ? 16384u : 0u; }
__device__ __forceinline__ constexpr uint32_t V(int b) { return b ? 49152u : 32768u; }
__device__ __forceinline__ constexpr uint32_t GB(int b) { return b ? 66048u : 65536u; }
constexpr uint32_t K_HALF = 8192;    // [K_lo | K_hi], 128-byte swizzled
constexpr uint32_t T1 = 67584;
constexpr uint32_t T2 = 75776;
constexpr uint32_t W = 83968;
constexpr uint32_t S = 100352;                  // bf16 copy of S_loc
constexpr uint32_t X = 133120;                  // bf16 copy of X
constexpr uint32_t UNI = 165888;                // {Dt_S, Dt_X} bf16 | {A, T} fp32
constexpr uint32_t DTS = UNI, DTX = UNI + 16384;
constexpr uint32_t AF = UNI, TF = UNI + 64 * ut::AP * 4;
constexpr uint32_t VEC = UNI + 2 * 64 * ut::AP * 4;
constexpr uint32_t BAR = VEC + 1024;
constexpr uint32_t TOTAL = BAR + 128;
constexpr uint32_t SCR = W;
}  // namespace smt

// TMEM columns (512 allocated per CTA).
// Output pass: fp32 state S, state update, X1 then W^T, U^T, Delta-part then O2, O1.
constexpr uint32_t TM_S = 0, TM_SU = 128, TM_XW = 256, TM_U = 320, TM_DD = 384, TM_O1 = 448;
// Transition pass: S_loc, X (both updated in place), X1 then W^T, U^T, S W^T, X W^T.
constexpr uint32_t TT_S = 0, TT_X = 128, TT_XW = 256, TT_U = 320, TT_DS = 384, TT_DX = 448;

// Fetch chunk [cs, cs + L) of head h into one buffer. K, Q (if with_q) and V
// arrive by TMA as 128-byte-swizzled tiles (SWIZZLE_128B boxes of 64 tokens x
// 64 columns), two column halves per matrix: K halves at kq and kq + k_half,
// Q halves 8 KB after each K half (so that [K; Q] forms one 128-row operand
// per column half), V halves at vt and vt + 8192. Thread 32 issues them and
// arms the buffer's mbarrier with the byte count. Rows past the end of the
// tensor are zero-filled by TMA; rows past the end of the sequence (the next
// sequence's tokens in a packed batch) do arrive, and are neutralised by
// their zero g and beta (below): they only reach rows and columns of A, P,
// W, U and Delta that are multiplied by beta = 0 or never written out.
// g and beta come by cp.async (4-byte copies), zero-filled past L.
__device__ __forceinline__ void load_chunk(uint32_t kq, uint32_t k_half, bool with_q, uint32_t vt, uint32_t gb,
                                           uint64_t *lbar, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                           const CUtensorMap *tm_v, const float *g, const float *beta, int cs,
                                           int L, int H, int h) {
    const int tid = threadIdx.x;
    if (tid == 32) {
        tc::mbar_arrive_expect_tx(lbar, (with_q ? 6u : 4u) * 8192u);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tc::tma_load_3d(kq + hf * k_half, tm_k, lbar, 64 * hf, h, cs);
            if (with_q) tc::tma_load_3d(kq + hf * k_half + 8192, tm_q, lbar, 64 * hf, h, cs);
            tc::tma_load_3d(vt + hf * 8192, tm_v, lbar, 64 * hf, h, cs);
        }
    }
    if (tid < 2 * C) {
        const int r = tid & 63;
        const bool ok = r < L;
        const size_t off = (size_t)(cs + (ok ? r : 0)) * H + h;
        if (tid < C)
            cp_async4(gb + 4 * r, g + off, ok ? 4u : 0u);
        else
            cp_async4(gb + 256 + 4 * r, beta + off, ok ? 4u : 0u);
    }
    cp_async_commit();
}

// All threads agree whether the wait succeeded (bounded wait on the MMA barrier).
__device__ __forceinline__ bool wait_all_ok(uint64_t *bar, uint32_t parity) {
    const bool ok = tc::mbar_wait(bar, parity);
    tc::fence_after_sync();
    return __syncthreads_and(ok) != 0;
}

// G = cumsum(g) in log2 units (warp 0, two positions per lane), then gamma,
// e = exp(G_C - G) and beta into the vector area. Ends with a barrier between
// the cumsum and the derived vectors; the caller's next barrier publishes them.
__device__ __forceinline__ void chunk_scalars(const float *graw, float *Gl, float *gam, float *dte, float *bet) {
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid < 32) {
        const float a = graw[2 * lane] * kLog2e, b2 = a + graw[2 * lane + 1] * kLog2e;
        float sc = b2;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, sc, off);
            if (lane >= off) sc += y;
        }
        Gl[2 * lane] = sc - b2 + a;
        Gl[2 * lane + 1] = sc;
    }
    __syncthreads();
    if (tid < C) {
        gam[tid] = ex2(Gl[tid]);
        dte[tid] = ex2(Gl[C - 1] - Gl[tid]);
        bet[tid] = graw[64 + tid];
    }
}

// X1 epilogue: accumulator rows 0..63 -> A (fp32, pitch AP), rows 64..127 ->
// P (bf16 tile at p_tile, if p_tile != 0); this thread's columns [32 half, +32).
__device__ __forceinline__ void x1_epilogue(float *A, uint32_t p_tile, uint32_t tl_x1, const float *Gl,
                                            const float *bet, int row, int half) {
    const int r = row & 63, s0 = 32 * half;
    const bool is_a = row < 64;
    if (!is_a && !p_tile) return;
    if (r < s0) {  // the whole column range lies above the diagonal (warp-uniform)
        if (is_a) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4 *>(A + r * AP + s0 + i) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 32; i += 8) st_run8(p_tile + tc::tile_off(r, s0 + i, 128, 1024), z);
        }
        return;
    }
    float x[32];
    tc::tmem_ld16(tl_x1 + s0, *reinterpret_cast<float(*)[16]>(x));
    tc::tmem_ld16(tl_x1 + s0 + 16, *reinterpret_cast<float(*)[16]>(x + 16));
    const float Gr = Gl[r];
    if (is_a) {
        const float br = bet[r];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            float4 a;
            a.x = (s0 + i < r) ? br * ex2(Gr - Gl[s0 + i]) * x[i] : 0.f;
            a.y = (s0 + i + 1 < r) ? br * ex2(Gr - Gl[s0 + i + 1]) * x[i + 1] : 0.f;
            a.z = (s0 + i + 2 < r) ? br * ex2(Gr - Gl[s0 + i + 2]) * x[i + 2] : 0.f;
            a.w = (s0 + i + 3 < r) ? br * ex2(Gr - Gl[s0 + i + 3]) * x[i + 3] : 0.f;
            *reinterpret_cast<float4 *>(A + r * AP + s0 + i) = a;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int s = s0 + i;
            x[i] = (s <= r) ? ex2(Gr - Gl[s]) * x[i] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 32; i += 8) st_run8(p_tile + tc::tile_off(r, s0 + i, 128, 1024), x + i);
    }
}

// T = (I + A)^{-1}, then T1 = T diag(beta gamma) and T2 = T diag(beta) as bf16 tiles.
__device__ __forceinline__ void solve_and_scale(const float *A, float *T, float *scratch, uint32_t t1, uint32_t t2,
                                                const float *gam, const float *bet, int half) {
    ut::solve64(A, T, scratch);
    const int task = threadIdx.x & 127, r = task & 63, s0 = 32 * half;
    const bool first = task < 64;
    const uint32_t dst = first ? t1 : t2;
#pragma unroll
    for (int i0 = 0; i0 < 32; i0 += 8) {
        const float4 t0 = *reinterpret_cast<const float4 *>(T + r * AP + s0 + i0);
        const float4 t1 = *reinterpret_cast<const float4 *>(T + r * AP + s0 + i0 + 4);
        float x[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int s = s0 + i0 + i;
            x[i] *= bet[s] * (first ? gam[s] : 1.f);
        }
        st_run8(dst + tc::tile_off(r, s0 + i0, 128, 1024), x);
    }
}

// W epilogue: thread (k, half) writes W[32 half .. +32][k] into row k of the W tile (runs along r).
__device__ __forceinline__ void w_epilogue(uint32_t w_tile, uint32_t tl_w, int row, int half) {
#pragma unroll
    for (int c0 = 32 * half; c0 < 32 * half + 32; c0 += 16) {
        float x[16];
        tc::tmem_ld16(tl_w + c0, x);
        st_run8(w_tile + tc::tile_off(row, c0, 128, 2048), x);
        st_run8(w_tile + tc::tile_off(row, c0 + 8, 128, 2048), x + 8);
    }
}

// Generic-proxy smem writes and TMEM accesses done; make them visible to the tensor core and sync.
__device__ __forceinline__ void handoff_to_mma() {
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
}

// bars[0..3]: MMA completion per chunk; the TMEM slot at byte 32 (bars[4]);
// bars[5..6]: TMA loads; bars[7]: segment-fold MMAs; bars[8..9]: fold inputs.
__device__ __forceinline__ void tmem_setup(uint32_t *tslot, uint64_t *bars) {
    if ((threadIdx.x >> 5) == 0) tc::tmem_alloc(tslot, 512);
    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) tc::mbar_init(&bars[i], 1);
        for (int i = 5; i < 10; ++i) tc::mbar_init(&bars[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
}

// Split a row run into bf16 hi / lo parts (x = hi + lo + O(2^-16 |x|)) and store both.
__device__ __forceinline__ void st_run8_split(uint32_t hi_addr, uint32_t lo_addr, const float *x) {
    float hi[8], lo[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        hi[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
        lo[i] = x[i] - hi[i];
    }
    st_run8(hi_addr, hi);
    st_run8(lo_addr, lo);
}

// Segment fold on the tensor cores: S <- S Phi_j + S_loc_j for the sequence's
// segments j = 0..count-1, starting from S0 (or zero). S and each Phi are
// split into bf16 hi + lo parts and S Phi = S_hi Phi_hi + S_hi Phi_lo +
// S_lo Phi_hi (fp32 accumulation in TMEM; the dropped S_lo Phi_lo term is
// ~2^-16 relative). Phi_hi / Phi_lo arrive as ready-made operand tiles
// (written by the transition pass) by bulk copy, double-buffered. The
// result lands as the fp32 state in TMEM (TM_S) and its bf16 copy in the S tile.
// Returns false (all threads agreeing) if a bounded wait gave up; the error bit is then set in err.
__device__ bool segment_fold(uint32_t sb, uint32_t tm, uint32_t tl, uint64_t *bars, uint32_t *err,
                             const float *S0row, const float *slots, size_t slot0, size_t slot_step, int count,
                             int row, int half) {
    const int tid = threadIdx.x;
    const uint32_t shi = sb + smo::S, slo = sb + smo::FOLD_SLO;
    const uint32_t phbuf[2] = {sb + smo::FOLD_PHI0, sb + smo::FOLD_PHI1};
    const uint32_t id_km128 = tc::make_idesc_bf16(128, 128, 0, 1);
    // S_hi / S_lo from S0 (thread (v, half): columns [64 half, +64) of row v)
#pragma unroll 1
    for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 8) {
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = S0row ? S0row[c0 + i] : 0.f;
        st_run8_split(shi + tc::tile_off(row, c0, 128, 2048), slo + tc::tile_off(row, c0, 128, 2048), x);
    }
    if (tid == 32) {
        tc::mbar_arrive_expect_tx(&bars[8], 65536u);
        tc::bulk_load(phbuf[0], slots + slot0 + D * D, 65536u, &bars[8]);
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    for (int j = 0; j < count; ++j) {
        const int b = j & 1;
        if (tid == 32 && j + 1 < count) {  // prefetch the next transition's tiles
            tc::mbar_arrive_expect_tx(&bars[8 + (b ^ 1)], 65536u);
            tc::bulk_load(phbuf[b ^ 1], slots + slot0 + (j + 1) * slot_step + D * D, 65536u, &bars[8 + (b ^ 1)]);
        }
        if (tid == 0) {
            tc::fence_after_sync();
            if (!tc::mbar_wait(&bars[8 + b], (uint32_t)((j >> 1) & 1))) atomicOr(err, ERRBIT_TIMEOUT);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t ah = tc::make_desc(shi + kk * 4096, 2048, 128);
                const uint64_t al = tc::make_desc(slo + kk * 4096, 2048, 128);
                const uint64_t bh = tc::make_desc(phbuf[b] + kk * 256, 128, 2048);
                const uint64_t bl = tc::make_desc(phbuf[b] + 32768 + kk * 256, 128, 2048);
                tc::mma_bf16(tm + TM_SU, ah, bh, id_km128, kk > 0);
                tc::mma_bf16(tm + TM_SU, ah, bl, id_km128, 1);
                tc::mma_bf16(tm + TM_SU, al, bh, id_km128, 1);
            }
            tc::mma_commit(&bars[7]);
        }
        // this thread's half row of S_loc, fetched while the MMAs run
        float4 sl[16];
        {
            const float4 *Sloc = reinterpret_cast<const float4 *>(slots + slot0 + j * slot_step + (size_t)row * D +
                                                                  64 * half);
#pragma unroll
            for (int i = 0; i < 16; ++i) sl[i] = Sloc[i];
        }
        if (!wait_all_ok(&bars[7], (uint32_t)(j & 1))) {
            if (tid == 0) atomicOr(err, ERRBIT_TIMEOUT);
            return false;
        }
        const bool last = j + 1 == count;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            const int c0 = 64 * half + 16 * blk;
            float d[16];
            tc::tmem_ld16(tl + TM_SU + c0, d);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                d[4 * i] += sl[4 * blk + i].x; d[4 * i + 1] += sl[4 * blk + i].y;
                d[4 * i + 2] += sl[4 * blk + i].z; d[4 * i + 3] += sl[4 * blk + i].w;
            }
            if (last) {
                tc::tmem_st16(tl + TM_S + c0, d);
                st_run8(shi + tc::tile_off(row, c0, 128, 2048), d);
                st_run8(shi + tc::tile_off(row, c0 + 8, 128, 2048), d + 8);
            } else {
                st_run8_split(shi + tc::tile_off(row, c0, 128, 2048), slo + tc::tile_off(row, c0, 128, 2048), d);
                st_run8_split(shi + tc::tile_off(row, c0 + 8, 128, 2048), slo + tc::tile_off(row, c0 + 8, 128, 2048),
                              d + 8);
            }
        }
        tc::tmem_st_wait();
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
    }
    return true;
}

// ============================================================================ output pass
__global__ void __launch_bounds__(NT, 1)
    k_chunk_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const float *__restrict__ g, const float *__restrict__ beta, const float *S0,
               const int32_t *__restrict__ cu, int N, int T_tot, int H, bf16 *__restrict__ o, float *S_T,
               uint32_t *__restrict__ err, const int32_t *__restrict__ seg_off, int seg_tokens,
               const float *__restrict__ slots) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if (*err & ERRBIT_SEQLENS) return;  // malformed cu_seqlens: write nothing
    Segment sg;
    const int h = blockIdx.x;
    if (!find_segment(seg_off, cu, N, T_tot, blockIdx.y, seg_tokens, sg)) return;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127;   // the TMEM lane (accumulator row) this thread reads
    const int half = tid >> 7;   // which half of the columns it handles
    const uint32_t sb = tc::smem_u32(smem);
    if (sb & 1023u) {  // swizzled tiles need a 1024-byte aligned shared-memory base
        if (threadIdx.x == 0) atomicOr(err, ERRBIT_INTERNAL);
        return;
    }
    float *Gl = reinterpret_cast<float *>(smem + smo::VEC);  // G * log2(e)
    float *gam = Gl + 64, *dte = Gl + 128, *bet = Gl + 192;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + smo::BAR);
    uint64_t *lbar = bars + 5;  // one TMA barrier per input buffer
    tmem_setup(reinterpret_cast<uint32_t *>(smem + smo::BAR + 32), bars);
    const uint32_t tm = *reinterpret_cast<uint32_t *>(smem + smo::BAR + 32);
    const uint32_t tl = tm + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's TMEM lane quarter
    const size_t sidx = ((size_t)sg.n * H + h) * D * D;

    // ---- initial state of this segment: S0 (first segment) or the fold of the earlier segments
    bool ok = true;
    if (sg.s > 0) {
        // slots are laid out [gseg][h][S_loc fp32, Phi_hi tile, Phi_lo tile]; segment j of this sequence is gseg = seg_off[n] + j
        ok = segment_fold(sb, tm, tl, bars, err, S0 ? S0 + sidx + (size_t)row * D : nullptr, slots,
                          ((size_t)seg_off[sg.n] * H + h) * 2 * D * D, (size_t)H * 2 * D * D, sg.s, row, half);
    } else {
        // thread (v, half) owns columns [64 half, 64 half + 64) of row v
        const float *src = S0 ? S0 + sidx + (size_t)row * D : nullptr;
#pragma unroll 1
        for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
            float r[16];
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                const float4 x = src ? *reinterpret_cast<const float4 *>(src + c0 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                r[i] = x.x; r[i + 1] = x.y; r[i + 2] = x.z; r[i + 3] = x.w;
            }
            tc::tmem_st16(tl + TM_S + c0, r);
            st_run8(sb + smo::S + tc::tile_off(row, c0, 128, 2048), r);
            st_run8(sb + smo::S + tc::tile_off(row, c0 + 8, 128, 2048), r + 8);
        }
        tc::tmem_st_wait();
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
    }
    const int nchunks = (sg.b - sg.a + C - 1) / C;
    if (ok && nchunks > 0)
        load_chunk(sb + smo::KQ(0), smo::KQ_HALF, true, sb + smo::V(0), sb + smo::GB(0), &lbar[0], &tm_q, &tm_k,
                   &tm_v, g, beta, sg.a, min(C, sg.b - sg.a), H, h);

    const uint32_t id_kk64 = tc::make_idesc_bf16(128, 64, 0, 0);
    const uint32_t id_mk64 = tc::make_idesc_bf16(128, 64, 1, 0);
    const uint32_t id_km64 = tc::make_idesc_bf16(128, 64, 0, 1);
    const uint32_t id_km128 = tc::make_idesc_bf16(128, 128, 0, 1);

    for (int c = 0; ok && c < nchunks; ++c) {
        const int cs = sg.a + c * C, L = min(C, sg.b - cs), b = c & 1;
        const uint32_t par = (uint32_t)(c & 1);
        const uint32_t kq = sb + smo::KQ(b), vt = sb + smo::V(b);
        if (tid == 64) tc::bulk_wait_read();  // the previous chunk's output store has left the staging rows
        cp_async_wait_all();
        tc::fence_smem_to_async();
        __syncthreads();
        chunk_scalars(reinterpret_cast<const float *>(smem + smo::GB(b)), Gl, gam, dte, bet);
        // ---- MMA group 1: X1 = [K;Q] K^T and O1 = S Q^T (after this buffer's TMA bytes landed)
        if (tid == 0) {
            tc::fence_after_sync();
            if (!tc::mbar_wait(&lbar[b], (uint32_t)((c >> 1) & 1))) atomicOr(err, ERRBIT_TIMEOUT);
            // swizzled K-major: a K=16 step is 32 bytes within the 128-byte row; columns 64.. in the next half
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * smo::KQ_HALF + (kk & 3) * 32;
                const uint64_t a = tc::make_desc_sw128(kq + off, 16, 1024);
                tc::mma_bf16(tm + TM_XW, a, a, id_kk64, kk > 0);  // B = first 64 rows of the same operand (K)
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t a = tc::make_desc(sb + smo::S + kk * 4096, 2048, 128);
                const uint64_t bq =
                    tc::make_desc_sw128(kq + (kk >> 2) * smo::KQ_HALF + (kk & 3) * 32 + 8192, 16, 1024);
                tc::mma_bf16(tm + TM_O1, a, bq, id_kk64, kk > 0);
            }
            tc::mma_commit(&bars[0]);
        }
        if (c + 1 < nchunks)
            load_chunk(sb + smo::KQ(b ^ 1), smo::KQ_HALF, true, sb + smo::V(b ^ 1), sb + smo::GB(b ^ 1), &lbar[b ^ 1],
                       &tm_q, &tm_k, &tm_v, g, beta, cs + C, min(C, sg.b - cs - C), H, h);
        if (!(ok = wait_all_ok(&bars[0], par))) break;
        x1_epilogue(reinterpret_cast<float *>(smem + smo::AF), sb + smo::P, tl + TM_XW, Gl, bet, row, half);
        tc::fence_before_sync();
        __syncthreads();
        solve_and_scale(reinterpret_cast<const float *>(smem + smo::AF), reinterpret_cast<float *>(smem + smo::TF),
                        reinterpret_cast<float *>(smem + smo::SCR), sb + smo::T1, sb + smo::T2, gam, bet, half);
        handoff_to_mma();
        // ---- MMA group 2: W^T = K^T T1^T, U^T = V^T T2^T (A operands: MN-major views)
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                // swizzled MN-major views: 16 token rows = 2048 bytes; LBO = distance of the column halves
                tc::mma_bf16(tm + TM_XW, tc::make_desc_sw128(kq + kk * 2048, smo::KQ_HALF, 1024),
                             tc::make_desc(sb + smo::T1 + kk * 2048, 1024, 128), id_mk64, kk > 0);
                tc::mma_bf16(tm + TM_U, tc::make_desc_sw128(vt + kk * 2048, 8192, 1024),
                             tc::make_desc(sb + smo::T2 + kk * 2048, 1024, 128), id_mk64, kk > 0);
            }
            tc::mma_commit(&bars[1]);
        }
        if (!(ok = wait_all_ok(&bars[1], par))) break;
        w_epilogue(sb + smo::W, tl + TM_XW, row, half);
        handoff_to_mma();
        // ---- MMA group 3: S W^T (B operand: MN-major view of the W tile)
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                tc::mma_bf16(tm + TM_DD, tc::make_desc(sb + smo::S + kk * 4096, 2048, 128),
                             tc::make_desc(sb + smo::W + kk * 256, 128, 2048), id_km64, kk > 0);
            tc::mma_commit(&bars[2]);
        }
        if (!(ok = wait_all_ok(&bars[2], par))) break;
        // ---- Delta epilogue: Delta^T[v][s] = U^T[v][s] - (S W^T)[v][s]; Dl = Delta^T, Dt = Delta^T diag(e)
#pragma unroll
        for (int c0 = 32 * half; c0 < 32 * half + 32; c0 += 16) {
            float u[16], d[16];
            tc::tmem_ld16(tl + TM_U + c0, u);
            tc::tmem_ld16(tl + TM_DD + c0, d);
#pragma unroll
            for (int i = 0; i < 16; ++i) u[i] -= d[i];
            st_run8(sb + smo::DL + tc::tile_off(row, c0, 128, 2048), u);
            st_run8(sb + smo::DL + tc::tile_off(row, c0 + 8, 128, 2048), u + 8);
#pragma unroll
            for (int i = 0; i < 16; ++i) u[i] *= dte[c0 + i];
            st_run8(sb + smo::DT + tc::tile_off(row, c0, 128, 2048), u);
            st_run8(sb + smo::DT + tc::tile_off(row, c0 + 8, 128, 2048), u + 8);
        }
        handoff_to_mma();
        // ---- MMA group 4: O2 = Dl P^T (into the Delta-part columns), SU = Dt K (B: MN-major view of K)
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                tc::mma_bf16(tm + TM_DD, tc::make_desc(sb + smo::DL + kk * 4096, 2048, 128),
                             tc::make_desc(sb + smo::P + kk * 2048, 1024, 128), id_kk64, kk > 0);
                tc::mma_bf16(tm + TM_SU, tc::make_desc(sb + smo::DT + kk * 4096, 2048, 128),
                             tc::make_desc_sw128(kq + kk * 2048, smo::KQ_HALF, 1024), id_km128, kk > 0);
            }
            tc::mma_commit(&bars[3]);
        }
        if (!(ok = wait_all_ok(&bars[3], par))) break;
        // ---- outputs: o[cs + r][h][v] = gamma_r O1[v][r] + O2[v][r], staged as rows o[r][.] in shared memory
        {
            uint8_t *ost = smem + smo::OST;
#pragma unroll
            for (int c0 = 32 * half; c0 < 32 * half + 32; c0 += 16) {
                float a[16], d[16];
                tc::tmem_ld16(tl + TM_O1 + c0, a);
                tc::tmem_ld16(tl + TM_DD + c0, d);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    *reinterpret_cast<bf16 *>(ost + (c0 + i) * 256 + 2 * row) =
                        __float2bfloat16_rn(fmaf(gam[c0 + i], a[i], d[i]));
            }
        }
        // A whole chunk, or a partial one that ends the tensor (TMA clips the rows past it), goes out
        // as one bulk tensor store; a partial chunk followed by another sequence's tokens is copied
        // row by row so that those tokens' outputs are not overwritten.
        if (L == C || cs + L >= T_tot) {
            tc::fence_smem_to_async();
            __syncthreads();
            if (tid == 64) tc::tma_store_3d(&tm_o, sb + smo::OST, 0, h, cs);
        } else {
            __syncthreads();
            const uint8_t *ost = smem + smo::OST;
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int idx = it * NT + tid, r = idx >> 4, j = idx & 15;
                if (r < L) {
                    const uint4 val = *reinterpret_cast<const uint4 *>(ost + r * 256 + j * 16);
                    *reinterpret_cast<uint4 *>(o + ((size_t)(cs + r) * H + h) * D + 8 * j) = val;
                }
            }
        }
        // ---- state: S <- gamma_C S + SU (fp32 in TMEM), bf16 copy to the S tile
        {
            const float gC = gam[C - 1];
#pragma unroll 1
            for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
                float s[16], u[16];
                tc::tmem_ld16(tl + TM_S + c0, s);
                tc::tmem_ld16(tl + TM_SU + c0, u);
#pragma unroll
                for (int i = 0; i < 16; ++i) s[i] = fmaf(gC, s[i], u[i]);
                tc::tmem_st16(tl + TM_S + c0, s);
                st_run8(sb + smo::S + tc::tile_off(row, c0, 128, 2048), s);
                st_run8(sb + smo::S + tc::tile_off(row, c0 + 8, 128, 2048), s + 8);
            }
            tc::tmem_st_wait();
        }
        handoff_to_mma();
    }
    cp_async_wait_all();
    if (tid == 64) tc::bulk_wait_all();
    if (!ok) {
        if (tid == 0) atomicOr(err, ERRBIT_TIMEOUT);
    } else if (sg.s == sg.ns - 1) {
        // ---- final state (last segment of the sequence)
        float *dst = S_T + sidx + (size_t)row * D;
#pragma unroll 1
        for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
            float r[16];
            tc::tmem_ld16(tl + TM_S + c0, r);
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4 *>(dst + c0 + i) = make_float4(r[i], r[i + 1], r[i + 2], r[i + 3]);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, 512);
}

// ============================================================================ transition pass
// For every segment except the last of its sequence: S_loc (from S = 0, with
// the V-term) and Phi (from X = I, without it), written to the workspace slot
// [gseg][h] as two fp32 128 x 128 matrices.
__global__ void __launch_bounds__(NT, 1)
    k_chunk_tc_trans(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const float *__restrict__ g, const float *__restrict__ beta, const int32_t *__restrict__ cu,
                     int N, int T_tot, int H,
                     uint32_t *__restrict__ err, const int32_t *__restrict__ seg_off, int seg_tokens,
                     float *__restrict__ slots) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if (*err & ERRBIT_SEQLENS) return;
    Segment sg;
    const int h = blockIdx.x;
    if (!find_segment(seg_off, cu, N, T_tot, blockIdx.y, seg_tokens, sg)) return;
    if (sg.s == sg.ns - 1) return;  // the last segment's transition is never needed
    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, half = tid >> 7;
    const uint32_t sb = tc::smem_u32(smem);
    if (sb & 1023u) {
        if (threadIdx.x == 0) atomicOr(err, ERRBIT_INTERNAL);
        return;
    }
    float *Gl = reinterpret_cast<float *>(smem + smt::VEC);
    float *gam = Gl + 64, *dte = Gl + 128, *bet = Gl + 192;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + smt::BAR);
    uint64_t *lbar = bars + 5;
    tmem_setup(reinterpret_cast<uint32_t *>(smem + smt::BAR + 32), bars);
    const uint32_t tm = *reinterpret_cast<uint32_t *>(smem + smt::BAR + 32);
    const uint32_t tl = tm + ((uint32_t)((warp & 3) * 32) << 16);

    // ---- S_loc = 0, X = I (fp32 in TMEM, bf16 copies in the S / X tiles)
#pragma unroll 1
    for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
        float z[16], x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            z[i] = 0.f;
            x[i] = (c0 + i == row) ? 1.f : 0.f;
        }
        tc::tmem_st16(tl + TT_S + c0, z);
        tc::tmem_st16(tl + TT_X + c0, x);
        st_run8(sb + smt::S + tc::tile_off(row, c0, 128, 2048), z);
        st_run8(sb + smt::S + tc::tile_off(row, c0 + 8, 128, 2048), z + 8);
        st_run8(sb + smt::X + tc::tile_off(row, c0, 128, 2048), x);
        st_run8(sb + smt::X + tc::tile_off(row, c0 + 8, 128, 2048), x + 8);
    }
    tc::tmem_st_wait();
    const int nchunks = (sg.b - sg.a + C - 1) / C;
    if (nchunks > 0)
        load_chunk(sb + smt::K(0), smt::K_HALF, false, sb + smt::V(0), sb + smt::GB(0), &lbar[0], nullptr, &tm_k,
                   &tm_v, g, beta, sg.a, min(C, sg.b - sg.a), H, h);

    // X1's A operand covers 128 rows; rows 64..127 read unrelated shared memory
    // (no Q here) and land in accumulator rows this pass never reads.
    const uint32_t id_kk64 = tc::make_idesc_bf16(128, 64, 0, 0);
    const uint32_t id_mk64 = tc::make_idesc_bf16(128, 64, 1, 0);
    const uint32_t id_km64 = tc::make_idesc_bf16(128, 64, 0, 1);
    const uint32_t id_km128 = tc::make_idesc_bf16(128, 128, 0, 1);
    bool ok = true;

    for (int c = 0; c < nchunks; ++c) {
        const int cs = sg.a + c * C, b = c & 1;
        const uint32_t par = (uint32_t)(c & 1);
        const uint32_t kt = sb + smt::K(b), vt = sb + smt::V(b);
        cp_async_wait_all();
        tc::fence_smem_to_async();
        __syncthreads();
        chunk_scalars(reinterpret_cast<const float *>(smem + smt::GB(b)), Gl, gam, dte, bet);
        if (tid == 0) {
            tc::fence_after_sync();
            if (!tc::mbar_wait(&lbar[b], (uint32_t)((c >> 1) & 1))) atomicOr(err, ERRBIT_TIMEOUT);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t a = tc::make_desc_sw128(kt + (kk >> 2) * smt::K_HALF + (kk & 3) * 32, 16, 1024);
                tc::mma_bf16(tm + TT_XW, a, a, id_kk64, kk > 0);
            }
            tc::mma_commit(&bars[0]);
        }
        if (c + 1 < nchunks)
            load_chunk(sb + smt::K(b ^ 1), smt::K_HALF, false, sb + smt::V(b ^ 1), sb + smt::GB(b ^ 1), &lbar[b ^ 1],
                       nullptr, &tm_k, &tm_v, g, beta, cs + C, min(C, sg.b - cs - C), H, h);
        if (!(ok = wait_all_ok(&bars[0], par))) break;
        x1_epilogue(reinterpret_cast<float *>(smem + smt::AF), 0, tl + TT_XW, Gl, bet, row, half);
        tc::fence_before_sync();
        __syncthreads();
        solve_and_scale(reinterpret_cast<const float *>(smem + smt::AF), reinterpret_cast<float *>(smem + smt::TF),
                        reinterpret_cast<float *>(smem + smt::SCR), sb + smt::T1, sb + smt::T2, gam, bet, half);
        handoff_to_mma();
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                tc::mma_bf16(tm + TT_XW, tc::make_desc_sw128(kt + kk * 2048, smt::K_HALF, 1024),
                             tc::make_desc(sb + smt::T1 + kk * 2048, 1024, 128), id_mk64, kk > 0);
                tc::mma_bf16(tm + TT_U, tc::make_desc_sw128(vt + kk * 2048, 8192, 1024),
                             tc::make_desc(sb + smt::T2 + kk * 2048, 1024, 128), id_mk64, kk > 0);
            }
            tc::mma_commit(&bars[1]);
        }
        if (!(ok = wait_all_ok(&bars[1], par))) break;
        w_epilogue(sb + smt::W, tl + TT_XW, row, half);
        handoff_to_mma();
        // ---- S W^T and X W^T
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t bw = tc::make_desc(sb + smt::W + kk * 256, 128, 2048);
                tc::mma_bf16(tm + TT_DS, tc::make_desc(sb + smt::S + kk * 4096, 2048, 128), bw, id_km64, kk > 0);
                tc::mma_bf16(tm + TT_DX, tc::make_desc(sb + smt::X + kk * 4096, 2048, 128), bw, id_km64, kk > 0);
            }
            tc::mma_commit(&bars[2]);
        }
        if (!(ok = wait_all_ok(&bars[2], par))) break;
        // ---- Dt_S = (U^T - S W^T) diag(e), Dt_X = -(X W^T) diag(e); states scaled by gamma_C in place
#pragma unroll
        for (int c0 = 32 * half; c0 < 32 * half + 32; c0 += 16) {
            float u[16], d[16];
            tc::tmem_ld16(tl + TT_U + c0, u);
            tc::tmem_ld16(tl + TT_DS + c0, d);
#pragma unroll
            for (int i = 0; i < 16; ++i) u[i] = (u[i] - d[i]) * dte[c0 + i];
            st_run8(sb + smt::DTS + tc::tile_off(row, c0, 128, 2048), u);
            st_run8(sb + smt::DTS + tc::tile_off(row, c0 + 8, 128, 2048), u + 8);
            tc::tmem_ld16(tl + TT_DX + c0, d);
#pragma unroll
            for (int i = 0; i < 16; ++i) d[i] = -d[i] * dte[c0 + i];
            st_run8(sb + smt::DTX + tc::tile_off(row, c0, 128, 2048), d);
            st_run8(sb + smt::DTX + tc::tile_off(row, c0 + 8, 128, 2048), d + 8);
        }
        {
            const float gC = gam[C - 1];
#pragma unroll 1
            for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
                float s[16], x[16];
                tc::tmem_ld16(tl + TT_S + c0, s);
                tc::tmem_ld16(tl + TT_X + c0, x);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    s[i] *= gC;
                    x[i] *= gC;
                }
                tc::tmem_st16(tl + TT_S + c0, s);
                tc::tmem_st16(tl + TT_X + c0, x);
            }
            tc::tmem_st_wait();
        }
        handoff_to_mma();
        // ---- S += Dt_S K, X += Dt_X K (accumulating into the scaled states)
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                const uint64_t bk = tc::make_desc_sw128(kt + kk * 2048, smt::K_HALF, 1024);
                tc::mma_bf16(tm + TT_S, tc::make_desc(sb + smt::DTS + kk * 4096, 2048, 128), bk, id_km128, 1);
                tc::mma_bf16(tm + TT_X, tc::make_desc(sb + smt::DTX + kk * 4096, 2048, 128), bk, id_km128, 1);
            }
            tc::mma_commit(&bars[3]);
        }
        if (!(ok = wait_all_ok(&bars[3], par))) break;
#pragma unroll 1
        for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
            float s[16], x[16];
            tc::tmem_ld16(tl + TT_S + c0, s);
            tc::tmem_ld16(tl + TT_X + c0, x);
            st_run8(sb + smt::S + tc::tile_off(row, c0, 128, 2048), s);
            st_run8(sb + smt::S + tc::tile_off(row, c0 + 8, 128, 2048), s + 8);
            st_run8(sb + smt::X + tc::tile_off(row, c0, 128, 2048), x);
            st_run8(sb + smt::X + tc::tile_off(row, c0 + 8, 128, 2048), x + 8);
        }
        handoff_to_mma();
    }
    cp_async_wait_all();
    if (!ok) {
        if (tid == 0) atomicOr(err, ERRBIT_TIMEOUT);
    } else {
        // slot: S_loc (fp32 row-major), then Phi as bf16 hi and lo operand tiles
        // (rows k, 16-byte runs along k', sx = 128, sy = 2048), byte for byte the
        // shared-memory layout the output pass's fold reads them in.
        float *slot = slots + ((size_t)blockIdx.y * H + h) * 2 * D * D;
        uint8_t *phi_hi = reinterpret_cast<uint8_t *>(slot + D * D), *phi_lo = phi_hi + 32768;
#pragma unroll 1
        for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
            float s[16], x[16];
            tc::tmem_ld16(tl + TT_S + c0, s);
            tc::tmem_ld16(tl + TT_X + c0, x);
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4 *>(slot + (size_t)row * D + c0 + i) = make_float4(s[i], s[i + 1], s[i + 2], s[i + 3]);
#pragma unroll
            for (int r8 = 0; r8 < 16; r8 += 8) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float h0 = __bfloat162float(__float2bfloat16_rn(x[r8 + i]));
                    const float h1 = __bfloat162float(__float2bfloat16_rn(x[r8 + i + 1]));
                    hi[i / 2] = tc::pack_bf16x2(h0, h1);
                    lo[i / 2] = tc::pack_bf16x2(x[r8 + i] - h0, x[r8 + i + 1] - h1);
                }
                const uint32_t off = tc::tile_off(row, c0 + r8, 128, 2048);
                *reinterpret_cast<uint4 *>(phi_hi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(phi_lo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, 512);
}

// Segment plan: validates cu_seqlens (error word) and writes seg_off[0..N],
// the exclusive prefix of max(1, ceil(ceil(L_n / C) / seg_chunks)).
__global__ void __launch_bounds__(256) k_plan(const int32_t *__restrict__ cu, int N, int T_tot, int seg_chunks,
                                              uint32_t *__restrict__ err, int32_t *__restrict__ seg_off) {
    __shared__ int part[256];
    __shared__ int bad;
    const int tid = threadIdx.x;
    if (tid == 0) bad = 0;
    __syncthreads();
    const int per = (N + 255) / 256;
    const int n0 = min(N, tid * per), n1 = min(N, n0 + per);
    auto nseg = [&](int n) {
        int L = cu ? cu[n + 1] - cu[n] : T_tot / N;
        L = max(L, 0);
        const int nc = (L + C - 1) / C;
        return max(1, (nc + seg_chunks - 1) / seg_chunks);
    };
    int sum = 0;
    bool b = false;
    for (int n = n0; n < n1; ++n) {
        if (cu) b |= cu[n + 1] < cu[n];
        sum += nseg(n);
    }
    if (tid == 0 && cu) b |= (cu[0] != 0) || (cu[N] != T_tot);
    if (b) atomicOr(&bad, 1);
    part[tid] = sum;
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int i = 0; i < 256; ++i) {
            const int x = part[i];
            part[i] = acc;
            acc += x;
        }
        seg_off[N] = acc;
        *err = bad ? ERRBIT_SEQLENS : 0u;
    }
    __syncthreads();
    int acc = part[tid];
    for (int n = n0; n < n1; ++n) {
        seg_off[n] = acc;
        acc += nseg(n);
    }
}

// Diagnostic wrapper of the solve: one 64 x 64 strictly lower fp32 matrix.
__global__ void __launch_bounds__(NT) k_diag_ut_solve(const float *__restrict__ Ag, float *__restrict__ Tg) {
    __shared__ __align__(16) float A[64 * AP], T[64 * AP], X[32 * ut::XP];
    for (int e = threadIdx.x; e < 64 * 64; e += NT) A[(e >> 6) * AP + (e & 63)] = Ag[e];
    __syncthreads();
    ut::solve64(A, T, X);
    for (int e = threadIdx.x; e < 64 * 64; e += NT) Tg[e] = T[(e >> 6) * AP + (e & 63)];
}

}  // namespace

// ---- host side
int chunk_tc_seg_chunks(int N, int T_tot, int H) {
    const long pairs = (long)N * H;
    const long nc_avg = ((long)T_tot / N + C - 1) / C;
    if (pairs >= 96 || nc_avg < 8) return 0;
    const long segs = 144 / pairs;
    if (segs < 2) return 0;
    return (int)std::max<long>(2, (nc_avg + segs - 1) / segs);
}

// Upper bound of sum_n max(1, ceil(ceil(L_n / C) / seg)) over any lengths with
// sum L_n = T_tot: each term is at most ceil(L_n / C) / seg + 1, and
// sum ceil(L_n / C) <= (T_tot + (C - 1) N) / C.
size_t chunk_tc_seg_slots(int N, int T_tot, int seg_chunks) {
    const long nc_bound = ((long)T_tot + (long)(C - 1) * N) / C;
    return (size_t)(nc_bound / seg_chunks + N);
}

size_t chunk_tc_workspace(int N, int T_tot, int H, int seg_chunks) {
    if (seg_chunks <= 0) return 256;
    const size_t off = 256 + ((size_t)(N + 1) * 4 + 255) / 256 * 256;
    return off + chunk_tc_seg_slots(N, T_tot, seg_chunks) * H * 2 * D * D * sizeof(float);
}

using chunk::make_row_map;

cudaError_t launch_chunk_tc(const bf16 *q, const bf16 *k, const bf16 *v, const float *g, const float *beta,
                            const float *S0, const int32_t *cu, int N, int T_tot, int H, bf16 *o, float *S_T,
                            void *workspace, size_t ws_bytes, cudaStream_t st, const char **stage) {
    uint32_t *err = static_cast<uint32_t *>(workspace);
    CUtensorMap tm_q, tm_k, tm_v, tm_o;
    cudaError_t e;
    *stage = "TMA descriptor encoding";
    if ((e = make_row_map(&tm_o, o, H, T_tot, true)) != cudaSuccess) return e;
    if ((e = make_row_map(&tm_q, q, H, T_tot)) != cudaSuccess) return e;
    if ((e = make_row_map(&tm_k, k, H, T_tot)) != cudaSuccess) return e;
    if ((e = make_row_map(&tm_v, v, H, T_tot)) != cudaSuccess) return e;
    // Largest segmentation that fits the workspace (none at all needs only the error word).
    int seg_chunks = chunk_tc_seg_chunks(N, T_tot, H);
    while (seg_chunks > 0 && chunk_tc_workspace(N, T_tot, H, seg_chunks) > ws_bytes) {
        const long nc_avg = ((long)T_tot / N + C - 1) / C;
        seg_chunks = (seg_chunks * 2 >= nc_avg) ? 0 : seg_chunks * 2;
    }
    if (seg_chunks == 0) {
        *stage = "validate_seqlens";
        void *pv = prof_start("validate_seqlens", st);
        e = launch_validate_seqlens(cu, N, T_tot, err, st);
        prof_stop(pv);
        if (e != cudaSuccess) return e;
        *stage = "chunk_tc";
        e = cudaFuncSetAttribute(k_chunk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smo::TOTAL);
        if (e != cudaSuccess) return e;
        void *pr = prof_start("chunk_tc", st);
        k_chunk_tc<<<dim3(H, N), NT, smo::TOTAL, st>>>(tm_q, tm_k, tm_v, tm_o, g, beta, S0, cu, N, T_tot, H, o, S_T, err,
                                                         nullptr, 0, nullptr);
        prof_stop(pr);
        return cudaGetLastError();
    }
    int32_t *seg_off = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) + 256);
    float *slots = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + 256 +
                                             ((size_t)(N + 1) * 4 + 255) / 256 * 256);
    const int nslots = (int)chunk_tc_seg_slots(N, T_tot, seg_chunks);
    const int seg_tokens = seg_chunks * C;
    *stage = "plan";
    void *pr = prof_start("plan", st);
    k_plan<<<1, 256, 0, st>>>(cu, N, T_tot, seg_chunks, err, seg_off);
    prof_stop(pr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    *stage = "chunk_tc_trans";
    e = cudaFuncSetAttribute(k_chunk_tc_trans, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smt::TOTAL);
    if (e != cudaSuccess) return e;
    pr = prof_start("chunk_tc_trans", st);
    k_chunk_tc_trans<<<dim3(H, nslots), NT, smt::TOTAL, st>>>(tm_k, tm_v, g, beta, cu, N, T_tot, H, err, seg_off,
                                                               seg_tokens, slots);
    prof_stop(pr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    *stage = "chunk_tc";
    e = cudaFuncSetAttribute(k_chunk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smo::TOTAL);
    if (e != cudaSuccess) return e;
    pr = prof_start("chunk_tc", st);
    k_chunk_tc<<<dim3(H, nslots), NT, smo::TOTAL, st>>>(tm_q, tm_k, tm_v, tm_o, g, beta, S0, cu, N, T_tot, H, o, S_T, err,
                                                         seg_off, seg_tokens, slots);
    prof_stop(pr);
    return cudaGetLastError();
}

cudaError_t launch_diag_ut_solve(const float *A, float *T, cudaStream_t st) {
    k_diag_ut_solve<<<1, NT, 0, st>>>(A, T);
    return cudaGetLastError();
}

}  // namespace gdn
