// Causal attention of the hybrid backbone's attention layers, on the sm_100a tensor cores.
//
// The pages' backbone interleaves the recurrent layers with causal attention layers whose
// O(N^2) attention kernel collapsed prefill at long context until it was rewritten as per-head
// GEMMs writing the scores into the existing buffer (page 1, abstract: 17x faster prefill at
// 10k; page 2, "Resumen Tecnico", the attention rewrite). On B200 the scores are never written
// out at all: per (query tile, head) the score tile S = Q K_j^T lives in tensor memory, the
// softmax turns it into bf16 probabilities in place, and O += P V_j accumulates in tensor
// memory, key tile by key tile (the on-chip form of the same two per-head products):
//
//     s_tj = (q_t . k_j) * scale   (j <= t, same sequence),   o_t = sum_j softmax_j(s_tj) v_j
//
// One CTA per (query tile of 128 positions, head, sequence), the largest tiles dispatched
// first; roles:
//   loader   (1 thread)  TMA: the Q tile once, K and V tiles of 128 keys into 2-deep rings
//   MMA      (1 warp)    S_j = Q K_j^T (M=128, N=128, K=128) into one of three TMEM score buffers,
//                        two tiles ahead; O += P_j V_j (A = P_j in TMEM) once the softmax is done.
//                        A product writing a buffer is issued only after the O += P V that read
//                        the buffer's previous P has completed: a later tcgen05.mma is not ordered
//                        after an earlier one's tensor-memory operand reads.
//   softmax  (4 warps)   one query row per thread: scores * scale in log2 units, causal mask,
//                        row max and sum, P = 2^(s - m) as bf16 pairs written over the score
//                        buffer; O is rescaled (read, scaled, written back in TMEM) only when a
//                        row's maximum grows by more than 8 (so P <= 256 in between); at the end
//                        o_t = O_t / l_t goes out as a bf16 row.
// Every wait is bounded in time; a timeout sets the error word and all roles leave their loops.
#include "chunk_common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

using bf16 = __nv_bfloat16;
constexpr int TQ = 128, TK = 128, D = 128;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;  // log2 units: rescale O only when the row maximum grows by more than this
constexpr uint32_t TILE = TQ * D * 2;  // 32 KB: two 64-column halves of 128 rows x 128 bytes (128-byte swizzle)
constexpr uint32_t OFF_Q = 0, OFF_K = TILE, OFF_V = 3 * TILE, OFF_BAR = 5 * TILE;
enum {
    QFULL = 0,
    KFULL = 1,    // [2]
    VFULL = 3,    // [2]
    KEMPTY = 5,   // [2] S_j has read K_j (commit)
    VEMPTY = 7,   // [2] PV_j has read V_j (commit)
    SFULL = 9,    // [3] S_j complete (commit), per score buffer
    PREADY = 12,  // [3] P_j written over its score buffer, O rescaled (128 softmax threads)
    PVD = 15,     // [3] O += P_j V_j has read the buffer's P (commit)
    OV = 18,      // O += P_j V_j complete (commit; one phase per key tile)
    FIN = 19,     // every MMA of the CTA done
    NBAR = 20
};
constexpr uint32_t OFF_CTL = OFF_BAR + 8 * NBAR;
constexpr uint32_t SMEM_TOTAL = OFF_CTL + 16 + 1024;
constexpr int NTHREADS = 192;  // loader warp, MMA warp, 4 softmax warps
constexpr int W_LOAD = 0, W_MMA = 1;
// TMEM columns: score buffers S0, S1, S2 (tile j in buffer j % 3; P_j overwrites the first 64
// columns of its buffer), O
constexpr uint32_t TM_S = 0, TM_O = 384;

struct Ctl {
    uint32_t tmem, abort;
};

// The timeout branch of wait_bar: sets the error word and aborts the CTA.
__device__ __noinline__ void wait_bar_timed_out(Ctl *ctl, uint32_t *err) {
    if (err) atomicOr(err, ERRBIT_TIMEOUT);
    *reinterpret_cast<volatile uint32_t *>(&ctl->abort) = 1u;
}
// Bounded wait for the phase `parity` of an mbarrier; gives up when another role has aborted, or
// after kWaitNs. The first test is inlined, the polling loop is a call (as a call the whole wait cost
// some 400 cycles even for a completed phase).
__device__ __noinline__ bool wait_bar_poll(uint64_t *bar, uint32_t parity, Ctl *ctl, uint32_t *err) {
    const uint64_t t0 = tc::globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((i & 15u) == 0) {
            if (*reinterpret_cast<volatile uint32_t *>(&ctl->abort)) return false;
            if (tc::globaltimer() - t0 > kWaitNs) {
                wait_bar_timed_out(ctl, err);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Ctl *ctl, uint32_t *err) {
    return tc::mbar_try_wait(bar, parity) || wait_bar_poll(bar, parity, ctl, err);
}
// wait_bar for a warp that issues MMAs as a whole (tc::*_w): every lane waits (converged), so that
// the warp stays converged for the elected issue.
__device__ __forceinline__ bool wait_bar_w(uint64_t *bar, uint32_t parity, Ctl *ctl, uint32_t *err) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, ctl, err));
}
__device__ __noinline__ void drain_bar(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = tc::globaltimer();
    while (!tc::mbar_try_wait(bar, parity))
        if (tc::globaltimer() - t0 > kWaitNs) return;
}

// TMEM <-> registers, 64 consecutive columns of this warp's lane quarter.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&r)[64]) {
    float a[32], b[32];
    tc::tmem_ld32(taddr, a);
    tc::tmem_ld32(taddr + 32, b);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        r[i] = a[i];
        r[32 + i] = b[i];
    }
}

// Work item of a CTA: blocks are numbered so that the query tiles with the most key tiles come
// first (block b: rank b / (H N) from the largest query-tile index, then head, then sequence).
__device__ __forceinline__ void item_of(int b, int H, int N, int max_qt, int &qi, int &h, int &n) {
    const int r = b / (H * N), rem = b - r * H * N;
    qi = max_qt - 1 - r;
    h = rem / N;
    n = rem - h * N;
}

__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const int32_t *__restrict__ cu, int N, int T_tot, int H,
               int max_qt, float scale, bf16 *__restrict__ o, uint32_t *__restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = tc::smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);
    const uint32_t sb = tc::smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (err && (*err & ERRBIT_SEQLENS)) return;
    int qi, h, n;
    item_of(blockIdx.x, H, N, max_qt, qi, h, n);
    int t0, t1;
    seq_bounds(cu, n, N, T_tot, t0, t1);
    const int L = t1 - t0, q0 = t0 + qi * TQ;
    if (qi * TQ >= L) return;  // this sequence has fewer query tiles
    const int nk = qi + 1;     // key tiles 0 .. qi (causal, tiles aligned to the sequence start)
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + OFF_CTL);
    if (warp == 0) tc::tmem_alloc(&ctl->tmem, 512);
    if (tid == 32) {
        for (int i = 0; i < NBAR; ++i) tc::mbar_init(&bar[i], (i >= PREADY && i < PREADY + 3) ? 128u : 1u);
        ctl->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = ctl->tmem;

    if (warp == W_LOAD) {
        if (lane == 0) {
            // a 128-row tile is four boxes of 64 columns x 64 rows: half (64 columns) at +16 KB, rows 64.. at +8 KB
            auto load_tile = [&](uint32_t dst, const CUtensorMap *map, uint64_t *b, int row0) {
                tc::mbar_arrive_expect_tx(b, TILE);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr)
                        tc::tma_load_3d(dst + hf * 16384 + rr * 8192, map, b, 64 * hf, h, row0 + 64 * rr);
            };
            load_tile(sb + OFF_Q, &tm_q, &bar[QFULL], q0);
            int issued_k = 0, issued_v = 0;
            bool ok = true;
            for (int j = 0; ok && j < nk; ++j) {
                const int b = j & 1;
                if (j >= 2 && !(ok = wait_bar(&bar[KEMPTY + b], (uint32_t)(((j >> 1) - 1) & 1), ctl, err))) break;
                load_tile(sb + OFF_K + b * TILE, &tm_k, &bar[KFULL + b], t0 + j * TK);
                issued_k = j + 1;
                if (j >= 2 && !(ok = wait_bar(&bar[VEMPTY + b], (uint32_t)(((j >> 1) - 1) & 1), ctl, err))) break;
                load_tile(sb + OFF_V + b * TILE, &tm_v, &bar[VFULL + b], t0 + j * TK);
                issued_v = j + 1;
            }
            drain_bar(&bar[QFULL], 0);
            for (int j = issued_k > 2 ? issued_k - 2 : 0; j < issued_k; ++j) drain_bar(&bar[KFULL + (j & 1)], (j >> 1) & 1);
            for (int j = issued_v > 2 ? issued_v - 2 : 0; j < issued_v; ++j) drain_bar(&bar[VFULL + (j & 1)], (j >> 1) & 1);
        }
    } else if (warp == W_MMA) {
        {  // the whole warp, lane 0 issuing
            const uint32_t id_s = tc::make_idesc_bf16(TQ, TK, 0, 0);  // Q K^T: both K-major
            const uint32_t id_o = tc::make_idesc_bf16(TQ, D, 0, 1);   // P V: V MN-major
            const tc::Desc dq = tc::split_desc(tc::make_desc_sw128(sb + OFF_Q, 16, 1024));
            const tc::Desc dk = tc::split_desc(tc::make_desc_sw128(sb + OFF_K, 16, 1024));
            const tc::Desc dv = tc::split_desc(tc::make_desc_sw128(sb + OFF_V, 16384, 1024));
            auto issue_s = [&](int j) {
                const uint32_t kb = (uint32_t)(j & 1) * TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    tc::mma_bf16_off_w(tm + TM_S + (j % 3) * 128, dq, off, dk, kb + off, id_s, kk > 0);
                }
                tc::mma_commit_w(&bar[SFULL + j % 3]);
                tc::mma_commit_w(&bar[KEMPTY + (j & 1)]);
            };
            bool ok = wait_bar_w(&bar[QFULL], 0, ctl, err);
            for (int j = 0; ok && j < 2 && j < nk; ++j) {
                if (!(ok = wait_bar_w(&bar[KFULL + j], 0, ctl, err))) break;
                tc::fence_after_sync();
                issue_s(j);
            }
            for (int j = 0; ok && j < nk; ++j) {
                const int b = j & 1, b3 = j % 3;
                if (!(ok = wait_bar_w(&bar[PREADY + b3], (uint32_t)((j / 3) & 1), ctl, err) &&
                           wait_bar_w(&bar[VFULL + b], (uint32_t)((j >> 1) & 1), ctl, err)))
                    break;
                tc::fence_after_sync();
                // O += P_j V_j: A = P_j (bf16 pairs in the score buffer's first 64 columns), B = V_j (MN-major)
#pragma unroll
                for (int kk = 0; kk < TK / 16; ++kk)
                    tc::mma_bf16_ts_off_w(tm + TM_O, tm + TM_S + b3 * 128 + 8 * kk, dv,
                                        b * TILE + kk * 2048, id_o, (j > 0 || kk > 0) ? 1u : 0u);
                tc::mma_commit_w(&bar[OV]);
                tc::mma_commit_w(&bar[VEMPTY + b]);
                tc::mma_commit_w(&bar[PVD + b3]);
                if (j + 2 < nk) {
                    // S_{j+2} goes to buffer (j + 2) % 3, whose last P (tile j - 1) must have been read
                    if (!(ok = wait_bar_w(&bar[KFULL + b], (uint32_t)(((j + 2) >> 1) & 1), ctl, err) &&
                               (j == 0 || wait_bar_w(&bar[PVD + (j + 2) % 3], (uint32_t)(((j - 1) / 3) & 1), ctl, err))))
                        break;
                    tc::fence_after_sync();
                    issue_s(j + 2);
                }
            }
            tc::mma_commit_w(&bar[FIN]);
            if (lane == 0) drain_bar(&bar[FIN], 0);
            __syncwarp();
        }
    } else {
        // ---------------------------------------------------------------- softmax (one query row per thread)
        const int r = (warp & 3) * 32 + lane;
        const uint32_t tl = tm + ((uint32_t)((warp & 3) * 32) << 16);
        const int qpos = qi * TQ + r;  // position within the sequence
        const float sc = scale * kLog2e;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; ok && j < nk; ++j) {
            const int b = j % 3;
            if (!(ok = __all_sync(0xffffffffu, wait_bar(&bar[SFULL + b], (uint32_t)((j / 3) & 1), ctl, err))))
                break;
            tc::fence_after_sync();
            float s[128];
            {
                float a[64], c[64];
                tmem_ld64(tl + TM_S + b * 128, a);
                tmem_ld64(tl + TM_S + b * 128 + 64, c);
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    s[i] = a[i];
                    s[64 + i] = c[i];
                }
            }
            // row maximum of the raw scores (the causal mask only cuts the diagonal key tile), in eight
            // independent partial maxima so that the reduction is not one 128-long dependent chain
            float pm[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) pm[u] = -INFINITY;
            if (j == qi) {
                const int lim = qpos - j * TK;  // key columns beyond this row's position are masked
#pragma unroll
                for (int i = 0; i < 128; ++i) {
                    s[i] = (i <= lim) ? s[i] : -INFINITY;
                    pm[i & 7] = fmaxf(pm[i & 7], s[i]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 128; ++i) pm[i & 7] = fmaxf(pm[i & 7], s[i]);
            }
            const float mt = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                   fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7]))) * sc;
            // lazy rescale: a new reference maximum only when this tile's exceeds it by more than kRescale
            float alpha = 1.f;
            const bool grow = mt > m_ref + kRescale;
            if (grow) {
                alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mt);
                m_ref = mt;
                l *= alpha;
            }
            if (j > 0 && __any_sync(0xffffffffu, grow)) {
                // O *= alpha for this warp's rows once O += P_{j-1} V_{j-1} is complete
                if (!(ok = __all_sync(0xffffffffu, wait_bar(&bar[OV], (uint32_t)((j - 1) & 1), ctl, err)))) break;
                tc::fence_after_sync();
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t u[32];
                    tc::tmem_ld32_nowait(tl + TM_O + c0, u);
                    tc::tmem_wait_ld(u);
#pragma unroll
                    for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
                    tc::tmem_st32(tl + TM_O + c0, u);
                }
            }
            // P = 2^(s sc - m_ref) (one FFMA and one MUFU.EX2 per score; masked scores give 0) as bf16 pairs
            // over the first 64 columns of the score buffer; the row sum in eight partial sums
            float ps[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) ps[u] = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 64) {
                uint32_t u[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float p0 = chunk::ex2(fmaf(s[c0 + 2 * i], sc, -m_ref));
                    const float p1 = chunk::ex2(fmaf(s[c0 + 2 * i + 1], sc, -m_ref));
                    ps[i & 7] += p0 + p1;
                    u[i] = tc::pack_bf16x2(p0, p1);
                }
                tc::tmem_st32(tl + TM_S + b * 128 + c0 / 2, u);
            }
            l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
            tc::tmem_st_wait();
            tc::fence_before_sync();
            tc::mbar_arrive(&bar[PREADY + b]);
        }
        // o = O / l once the last O += P V is complete
        if (ok) ok = __all_sync(0xffffffffu, wait_bar(&bar[OV], (uint32_t)((nk - 1) & 1), ctl, err));
        if (ok) {
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const bool valid = qpos < L;
            bf16 *dst = o + ((size_t)(t0 + qpos) * H + h) * D;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                float x[32];
                tc::tmem_ld32(tl + TM_O + c0, x);
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8)
                        *reinterpret_cast<uint4 *>(dst + c0 + i) = make_uint4(
                            tc::pack_bf16x2(x[i] * inv, x[i + 1] * inv), tc::pack_bf16x2(x[i + 2] * inv, x[i + 3] * inv),
                            tc::pack_bf16x2(x[i + 4] * inv, x[i + 5] * inv), tc::pack_bf16x2(x[i + 6] * inv, x[i + 7] * inv));
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, 512);
}

}  // namespace

cudaError_t launch_attn_fwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                            const int32_t *cu, int N, int T_tot, int H, int max_len, float scale, __nv_bfloat16 *o,
                            uint32_t *err, cudaStream_t st, const char **stage) {
    cudaError_t e;
    *stage = "error word";
    if (cu) {
        if ((e = launch_validate_seqlens(cu, N, T_tot, err, st)) != cudaSuccess) return e;
    } else if ((e = cudaMemsetAsync(err, 0, sizeof(uint32_t), st)) != cudaSuccess) {
        return e;
    }
    if (T_tot == 0 || max_len == 0) return cudaSuccess;
    CUtensorMap tm_q, tm_k, tm_v;
    *stage = "TMA descriptor encoding";
    if ((e = chunk::make_row_map(&tm_q, q, H, T_tot)) != cudaSuccess) return e;
    if ((e = chunk::make_row_map(&tm_k, k, H, T_tot)) != cudaSuccess) return e;
    if ((e = chunk::make_row_map(&tm_v, v, H, T_tot)) != cudaSuccess) return e;
    *stage = "attn_fwd";
    e = cudaFuncSetAttribute(k_attn_fwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_TOTAL);
    if (e != cudaSuccess) return e;
    const int max_qt = (max_len + TQ - 1) / TQ;
    void *pr = prof_start("attn_fwd", st);
    k_attn_fwd<<<max_qt * H * N, NTHREADS, SMEM_TOTAL, st>>>(tm_q, tm_k, tm_v, cu, N, T_tot, H, max_qt, scale, o, err);
    prof_stop(pr);
    return cudaGetLastError();
}

}  // namespace gdn
