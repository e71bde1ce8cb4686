// Input projection of the recurrent layer with int8 weights, on the sm_100a tensor cores.
//
// The pages' system keeps the language model's weights as 8-bit codes that are dequantised for
// the projections (page 1, abstract: int8 weights dequantised once; page 2, "Resumen Tecnico",
// the GEMM item). For the recurrent layer the projection turns hidden states x [T][D] into the
// layer's raw inputs: q, k, v (H heads of dk, dk, dv values, bf16) and the gate logits a, b
// (one per head, fp32), with one weight matrix of N = H (2 dk + dv) + 2 H output channels stored
// as int8 codes w[n][j] and one fp32 scale per channel:
//
//     y[t][n] = scale[n] * sum_j x[t][j] w[n][j]
//
// Columns in the order q, k, v, a, b (head-major inside each), written straight into the
// layouts gdn_chunk_fwd_raw / gdn_decode_step_raw read. The int8 codes are exact in bf16, so the
// product runs on bf16 operands with fp32 accumulation and the scale is applied to the fp32
// result: the dequantisation is exact and the weights cross HBM as int8 (half the bytes of bf16).
//
// One persistent CTA per SM walks output tiles of MT x 128 tokens x BN channels, K steps of 64:
// at prefill sizes MT = 2, BN = 128 (each converted weight tile serves two token tiles, halving the
// conversion per product), else MT = 1 and BN = 256, or 128 / 64 when there are too few tiles to
// fill the GPU (as for one decode step):
//   loaders   (2 threads)  TMA: x tiles (bf16, 128-byte swizzle) and int8 weight tiles, two 4-deep
//                          rings, freed by the MMAs and by the converters respectively
//   convert   (8 warps)    int8 tile -> bf16 K-major 128-byte-swizzled operand tile, 3-deep ring
//                          (exact, on integer and fp32 pipes: codes_to_bf16x4)
//   MMA       (1 warp)     4 tcgen05.mma (M=128, N=BN, K=16) per K step and token tile into a TMEM
//                          accumulator (two sets of MT x BN columns: one tile's epilogue overlaps the next)
//   epilogue  (4 warps)    TMEM -> fp32 registers -> * scale -> bf16 / fp32 rows in global memory
// Every wait is bounded in time; a timeout sets the error word and all roles leave their loops.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace gdn {
namespace {

using bf16_t = __nv_bfloat16;
constexpr int BM = 128, BK = 64;
constexpr int NBSLOT = 3;
// ring depth of the x and int8 stages: deeper for the narrow tiles of small T, where each CTA's
// K loop is a chain of load latencies rather than of products
template <int BN, int MT>
constexpr int nstage() { return MT > 1 ? 4 : BN >= 256 ? 4 : BN >= 128 ? 6 : 8; }
constexpr int NSTAGE_MAX = 8;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr int NCONV = 256;                       // converter threads (8 warps)
constexpr int NTHREADS = 96 + NCONV + 128;       // x loader, MMA, w8 loader, converters, epilogue (15 warps)
constexpr int W_LOAD = 0, W_MMA = 1, W_LOADW = 2, W_CONV0 = 3, W_EPI0 = 3 + NCONV / 32;
enum {
    FULL = 0,                        // [stages] x tile of a stage landed (x loader arrive + bytes)
    EMPTY = FULL + NSTAGE_MAX,       // [stages] x stage free (MMA commit)
    WFULL = EMPTY + NSTAGE_MAX,      // [stages] int8 weight tile landed (w8 loader arrive + bytes)
    WEMPTY = WFULL + NSTAGE_MAX,     // [stages] int8 stage free (every converter)
    BFULL = WEMPTY + NSTAGE_MAX,     // [NBSLOT] bf16 weight tile written (every converter)
    BEMPTY = BFULL + NBSLOT,     // [NBSLOT] bf16 weight tile read by the MMAs (commit)
    AFULL = BEMPTY + NBSLOT,     // [2] accumulator complete (commit)
    AEMPTY = AFULL + 2,          // [2] accumulator read out (128 epilogue threads)
    FIN = AEMPTY + 2,            // every MMA of the CTA done (drained before TMEM is freed)
    NBAR = FIN + 1
};
__host__ __device__ constexpr uint32_t bar_count(int i) {
    return (i >= WEMPTY && i < WEMPTY + NSTAGE_MAX) ? (uint32_t)NCONV : (i >= BFULL && i < BFULL + NBSLOT) ? (uint32_t)NCONV
           : (i >= AEMPTY && i < AEMPTY + 2) ? 128u : 1u;
}

// Shared-memory layout for a tile of MT x 128 tokens and BN channels (x: MT x 128 x 64 bf16; w8: BN x 64
// int8; bf16 weight tile BN x 64).
template <int BN, int MT>
struct Lay {
    static constexpr int NSTAGE = nstage<BN, MT>();
    static constexpr uint32_t A_BYTES = MT * BM * BK * 2, W8_BYTES = BN * BK, B_BYTES = BN * BK * 2;
    static constexpr uint32_t OFF_A = 0, OFF_W8 = OFF_A + NSTAGE * A_BYTES, OFF_B = OFF_W8 + NSTAGE * W8_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_B + NBSLOT * B_BYTES, OFF_CTL = OFF_BAR + 8 * NBAR;
    static constexpr uint32_t TOTAL = OFF_CTL + 16 + 1024;  // + slack for the 1024-byte alignment
};
static_assert(Lay<256, 1>::TOTAL <= 232448 && Lay<128, 1>::TOTAL <= 232448 && Lay<64, 1>::TOTAL <= 232448 &&
                  Lay<128, 2>::TOTAL <= 232448,
              "shared memory");

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

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, uint64_t *mbar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(tc::smem_u32(mbar))
        : "memory");
}

// Four int8 codes (one 32-bit word) as two bf16 pairs, exactly and on full-rate pipes: with
// u = code + 128 (the word XOR 0x80808080), the fp32 with bit pattern 0x4B000000 | u is 2^23 + u,
// and subtracting 2^23 + 128 leaves the code exactly. A code needs at most 8 significant bits, so
// its bf16 is exactly the upper 16 bits of that fp32: a byte permute packs two of them.
__device__ __forceinline__ void codes_to_bf16x4(uint32_t word, uint32_t &lo, uint32_t &hi) {
    const uint32_t u = word ^ 0x80808080u;
    const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)) - 8388736.0f;
    const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651)) - 8388736.0f;
    const float f2 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)) - 8388736.0f;
    const float f3 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653)) - 8388736.0f;
    lo = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
    hi = __byte_perm(__float_as_uint(f2), __float_as_uint(f3), 0x7632);
}

// Where output column n goes: region 0..4 = q, k, v (bf16 [T][width]), a, b (fp32 [T][H]).
struct Route {
    int Hdk, Hdv, H, N;
};

template <int BN, int MT>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_proj_w8(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
              const float *__restrict__ scale, int T, int D, Route rt, bf16_t *__restrict__ q, bf16_t *__restrict__ k,
              bf16_t *__restrict__ v, float *__restrict__ ga, float *__restrict__ gb, uint32_t *__restrict__ err) {
    using L = Lay<BN, MT>;
    constexpr uint32_t TMEM_COLS = 2 * MT * BN < 32 ? 32 : 2 * MT * BN;
    constexpr int NSTAGE = L::NSTAGE;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = tc::smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);  // 1024-byte aligned for the swizzle
    const uint32_t sb = tc::smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + L::OFF_CTL);
    if (warp == 0) tc::tmem_alloc(&ctl->tmem, TMEM_COLS);
    if (tid == 32) {
        for (int i = 0; i < NBAR; ++i) tc::mbar_init(&bar[i], bar_count(i));
        ctl->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = ctl->tmem;
    const int mt = (T + MT * BM - 1) / (MT * BM), nt = (rt.N + BN - 1) / BN, ksteps = D / BK;
    const int ntiles = mt * nt;

    if (warp == W_LOAD || warp == W_LOADW) {
        // two loader threads: the x ring is freed by the MMAs, the int8 ring by the converters, so the
        // weight tiles (and their conversion) can run ahead of the products
        if (lane == 0) {
            const bool wl = warp == W_LOADW;
            uint64_t *full = &bar[wl ? WFULL : FULL], *empty = &bar[wl ? WEMPTY : EMPTY];
            int it = 0, issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
                const int m0 = (tile / nt) * MT * BM, n0 = (tile % nt) * BN;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % NSTAGE;
                    if (it >= NSTAGE && !(ok = wait_bar(&empty[s], (uint32_t)(((it / NSTAGE) - 1) & 1), ctl, err)))
                        break;
                    if (wl) {
                        tc::mbar_arrive_expect_tx(&full[s], L::W8_BYTES);
                        tma_load_2d(sb + L::OFF_W8 + s * L::W8_BYTES, &tm_w, &full[s], ks * BK, n0);
                    } else {
                        tc::mbar_arrive_expect_tx(&full[s], L::A_BYTES);
                        tma_load_2d(sb + L::OFF_A + s * L::A_BYTES, &tm_x, &full[s], ks * BK, m0);
                    }
                    issued = it + 1;
                }
            }
            for (int j = issued > NSTAGE ? issued - NSTAGE : 0; j < issued; ++j)
                drain_bar(&full[j % NSTAGE], (uint32_t)((j / NSTAGE) & 1));
        }
    } else if (warp == W_MMA) {
        {  // the whole warp, lane 0 issuing
            const uint32_t idesc = tc::make_idesc_bf16(BM, BN, 0, 0);
            const tc::Desc da = tc::split_desc(tc::make_desc_sw128(sb + L::OFF_A, 16, 1024));
            const tc::Desc db = tc::split_desc(tc::make_desc_sw128(sb + L::OFF_B, 16, 1024));
            int it = 0, ti = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++ti) {
                const int acc = ti & 1;
                if (ti >= 2 && !(ok = wait_bar_w(&bar[AEMPTY + acc], (uint32_t)(((ti >> 1) - 1) & 1), ctl, err))) break;
                tc::fence_after_sync();
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % NSTAGE, bs = it % NBSLOT;
                    if (!(ok = wait_bar_w(&bar[FULL + s], (uint32_t)((it / NSTAGE) & 1), ctl, err) &&
                               wait_bar_w(&bar[BFULL + bs], (uint32_t)((it / NBSLOT) & 1), ctl, err)))
                        break;
                    tc::fence_after_sync();
#pragma unroll
                    for (int m = 0; m < MT; ++m)
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            tc::mma_bf16_off_w(tm + (acc * MT + m) * BN, da, s * L::A_BYTES + m * BM * 128 + kk * 32, db,
                                               bs * L::B_BYTES + kk * 32, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit_w(&bar[EMPTY + s]);
                    tc::mma_commit_w(&bar[BEMPTY + bs]);
                }
                if (ok) tc::mma_commit_w(&bar[AFULL + acc]);
            }
            tc::mma_commit_w(&bar[FIN]);
            if (lane == 0) drain_bar(&bar[FIN], 0);
            __syncwarp();
        }
    } else if (warp < W_EPI0) {
        // ---------------------------------------------------------------- convert (NCONV threads)
        const int t = tid - 32 * W_CONV0;
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
            for (int ks = 0; ks < ksteps; ++ks, ++it) {
                const int s = it % NSTAGE, bs = it % NBSLOT;
                ok = wait_bar(&bar[WFULL + s], (uint32_t)((it / NSTAGE) & 1), ctl, err) &&
                     (it < NBSLOT || wait_bar(&bar[BEMPTY + bs], (uint32_t)(((it / NBSLOT) - 1) & 1), ctl, err));
                if (!(ok = __all_sync(0xffffffffu, ok))) break;
                tc::fence_after_sync();
                const uint8_t *w8 = smem + L::OFF_W8 + s * L::W8_BYTES;
                uint8_t *bt = smem + L::OFF_B + bs * L::B_BYTES;
                // 16-byte chunk c of the int8 tile (row c / 4, codes 16 (c % 4) ..): consecutive threads read
                // consecutive chunks; each becomes two 16-byte bf16 chunks of the row's swizzled 128 bytes
#pragma unroll
                for (int c = t; c < BN * BK / 16; c += NCONV) {
                    const int row = c >> 2, q4 = c & 3;
                    const uint4 raw = *reinterpret_cast<const uint4 *>(w8 + 16 * c);
                    uint32_t o[8];
                    codes_to_bf16x4(raw.x, o[0], o[1]);
                    codes_to_bf16x4(raw.y, o[2], o[3]);
                    codes_to_bf16x4(raw.z, o[4], o[5]);
                    codes_to_bf16x4(raw.w, o[6], o[7]);
                    const uint32_t rbase = (uint32_t)row * 128u, sw = (uint32_t)(row & 7);
                    *reinterpret_cast<uint4 *>(bt + rbase + (((2u * q4) ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4 *>(bt + rbase + (((2u * q4 + 1u) ^ sw) << 4)) =
                        make_uint4(o[4], o[5], o[6], o[7]);
                }
                tc::fence_smem_to_async();
                tc::mbar_arrive(&bar[BFULL + bs]);
                tc::mbar_arrive(&bar[WEMPTY + s]);  // this thread's reads of the int8 stage are done
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue (128 threads)
        const int row = (warp & 3) * 32 + lane;  // this thread's TMEM lane = token row of each token tile
        const uint32_t tl = tm + ((uint32_t)((warp & 3) * 32) << 16);
        int ti = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++ti) {
            const int acc = ti & 1;
            const int m0 = (tile / nt) * MT * BM, n0 = (tile % nt) * BN;
            if (!(ok = __all_sync(0xffffffffu, wait_bar(&bar[AFULL + acc], (uint32_t)((ti >> 1) & 1), ctl, err))))
                break;
            tc::fence_after_sync();
#pragma unroll 1
            for (int cm = 0; cm < MT * BN; cm += 32) {
                const int m = cm / BN, c0 = cm % BN;
                const int t = m0 + m * BM + row;
                float x[32];
                tc::tmem_ld32(tl + acc * MT * BN + cm, x);
                const int n = n0 + c0;
                if (t >= T || n >= rt.N) continue;
                if (n + 32 <= rt.N) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 s4 = __ldg(reinterpret_cast<const float4 *>(scale + n + i));
                        x[i] *= s4.x; x[i + 1] *= s4.y; x[i + 2] *= s4.z; x[i + 3] *= s4.w;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] *= (n + i < rt.N) ? __ldg(scale + n + i) : 0.f;
                }
                // 32 columns inside one bf16 region: four 16-byte stores; otherwise column by column
                const int r0 = n < rt.Hdk ? 0 : n < 2 * rt.Hdk ? 1 : n < 2 * rt.Hdk + rt.Hdv ? 2 : 3;
                const int base = r0 == 0 ? 0 : r0 == 1 ? rt.Hdk : 2 * rt.Hdk;
                const int width = r0 == 2 ? rt.Hdv : rt.Hdk;
                if (r0 < 3 && n + 32 <= base + width) {
                    bf16_t *dst = (r0 == 0 ? q : r0 == 1 ? k : v) + (size_t)t * width + (n - base);
#pragma unroll
                    for (int i = 0; i < 32; i += 8)
                        *reinterpret_cast<uint4 *>(dst + i) =
                            make_uint4(tc::pack_bf16x2(x[i], x[i + 1]), tc::pack_bf16x2(x[i + 2], x[i + 3]),
                                       tc::pack_bf16x2(x[i + 4], x[i + 5]), tc::pack_bf16x2(x[i + 6], x[i + 7]));
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int c = n + i;
                        if (c >= rt.N) break;
                        if (c < rt.Hdk) q[(size_t)t * rt.Hdk + c] = __float2bfloat16_rn(x[i]);
                        else if (c < 2 * rt.Hdk) k[(size_t)t * rt.Hdk + c - rt.Hdk] = __float2bfloat16_rn(x[i]);
                        else if (c < 2 * rt.Hdk + rt.Hdv) v[(size_t)t * rt.Hdv + c - 2 * rt.Hdk] = __float2bfloat16_rn(x[i]);
                        else if (c < 2 * rt.Hdk + rt.Hdv + rt.H) ga[(size_t)t * rt.H + c - 2 * rt.Hdk - rt.Hdv] = x[i];
                        else gb[(size_t)t * rt.H + c - 2 * rt.Hdk - rt.Hdv - rt.H] = x[i];
                    }
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&bar[AEMPTY + acc]);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, TMEM_COLS);
}

}  // namespace
}  // namespace gdn

namespace gdn {
namespace {

cudaError_t encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
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
    const cuuint64_t dims[2] = {inner, std::max<uint64_t>(outer, 1)};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int sm_count() {
    static int n = 0;
    static std::once_flag once;
    std::call_once(once, [] {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
    });
    return n;
}

}  // namespace

cudaError_t launch_proj_w8(const __nv_bfloat16 *x, const int8_t *w, const float *scale, int T, int D, int H, int dk,
                           int dv, __nv_bfloat16 *q, __nv_bfloat16 *k, __nv_bfloat16 *v, float *a, float *b,
                           uint32_t *err, cudaStream_t st, const char **stage) {
    cudaError_t e;
    *stage = "error word reset";
    if ((e = cudaMemsetAsync(err, 0, sizeof(uint32_t), st)) != cudaSuccess) return e;
    const int N = H * (2 * dk + dv) + 2 * H;
    if (T == 0) return cudaSuccess;
    *stage = "proj_w8";
    // Tiles: at prefill sizes two token tiles of 128 per tile with 128 channels, when that still
    // gives every SM a tile; otherwise one token tile and the widest channel tile of 256 / 128 / 64
    // that does (small T, e.g. one decode step, is bound by reading the weights and needs many CTAs
    // to do so).
    const long mt1 = (T + BM - 1) / BM, mt2 = (T + 2 * BM - 1) / (2 * BM);
    auto launch = [&](auto kernel, int BNv, int MTv, uint32_t smem_bytes) -> cudaError_t {
        cudaError_t ea = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes);
        if (ea != cudaSuccess) return ea;
        CUtensorMap tm_x, tm_w2;
        ea = encode_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)D, (uint64_t)T, (uint64_t)D * 2, BK,
                       BM * MTv, CU_TENSOR_MAP_SWIZZLE_128B);
        if (ea != cudaSuccess) return ea;
        ea = encode_2d(&tm_w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, (uint64_t)D, (uint64_t)N, (uint64_t)D, BK, BNv,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
        if (ea != cudaSuccess) return ea;
        const long tiles = (MTv > 1 ? mt2 : mt1) * ((N + BNv - 1) / BNv);
        const int grid = (int)std::min<long>(tiles, sm_count());
        void *pr = prof_start("proj_w8", st);
        kernel<<<grid, NTHREADS, smem_bytes, st>>>(tm_x, tm_w2, scale, T, D, Route{H * dk, H * dv, H, N}, q, k, v,
                                                    a, b, err);
        prof_stop(pr);
        return cudaSuccess;
    };
    if (mt2 * ((N + 127) / 128) >= sm_count()) {
        e = launch(k_proj_w8<128, 2>, 128, 2, Lay<128, 2>::TOTAL);
    } else {
        int bn = 64;
        for (int cand : {256, 128})
            if (mt1 * ((N + cand - 1) / cand) >= sm_count()) {
                bn = cand;
                break;
            }
        if (bn == 256) e = launch(k_proj_w8<256, 1>, 256, 1, Lay<256, 1>::TOTAL);
        else if (bn == 128) e = launch(k_proj_w8<128, 1>, 128, 1, Lay<128, 1>::TOTAL);
        else e = launch(k_proj_w8<64, 1>, 64, 1, Lay<64, 1>::TOTAL);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn
