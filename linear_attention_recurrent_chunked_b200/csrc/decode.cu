// Decode step and sequential scan: the token-at-a-time form of the gated delta
// rule (page 2, "Resumen Tecnico", Metodologia, recurrent-layer item: the scan
// that the chunked form replaces).
//
// Row update, for every row i of the d_v x d_k state S of one (sequence, head):
//     a_i = S_i . k,  b_i = S_i . q,  delta_i = beta (v_i - alpha a_i)
//     S_i <- alpha S_i + delta_i k,   o_i = alpha b_i + delta_i (k . q)
// which is S_new = alpha S (I - beta k k^T) + beta v k^T and o = S_new q with
// S read once and written once.
//
// Thread mapping (both kernels): a CTA of 128 threads owns 64 rows of one
// (sequence, head) state. Warp w owns rows [16w, 16w+16); inside a warp, lane
// = 8*sub + part: `sub` picks one row of a group of four, `part` one 16-byte
// column slot. A warp-wide load therefore reads four full 128-byte row
// segments (coalesced float4), and a row's dot products reduce over the 8
// `part` lanes with three xor-shuffles. Each thread holds 4 rows x D/8 columns
// of S in registers (64 fp32 at D = 128).
#include "common.cuh"
#include "kernels.h"

namespace gdn {

namespace {

constexpr int kRowsPerCta = 64;
constexpr int kThreads = 128;

__device__ __forceinline__ float red8(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    return x;
}

template <typename T, int D>
struct RowBlock {
    static constexpr int J = D / 32;  // float4 column slots per thread
    float s[4][J][4];
    int row0, sub, part;

    __device__ __forceinline__ void init_mapping(int rb) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        sub = lane >> 3;
        part = lane & 7;
        row0 = rb * kRowsPerCta + warp * 16;
    }
    __device__ __forceinline__ int row(int i) const { return row0 + 4 * i + sub; }
    __device__ __forceinline__ int col(int j) const { return part * 4 + 32 * j; }

    __device__ __forceinline__ void load(const float *Sh) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < J; ++j) {
                float4 x = *reinterpret_cast<const float4 *>(Sh + (size_t)row(i) * D + col(j));
                s[i][j][0] = x.x; s[i][j][1] = x.y; s[i][j][2] = x.z; s[i][j][3] = x.w;
            }
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < J; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) s[i][j][c] = 0.f;
    }
    __device__ __forceinline__ void store(float *Sh) const {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < J; ++j)
                *reinterpret_cast<float4 *>(Sh + (size_t)row(i) * D + col(j)) =
                    make_float4(s[i][j][0], s[i][j][1], s[i][j][2], s[i][j][3]);
    }
    // One token: updates the rows and returns o for row(i) in out[i] (valid in every lane).
    __device__ __forceinline__ void step(const float (&kc)[J][4], const float (&qc)[J][4], const float (&vr)[4],
                                         float alpha, float beta, float (&out)[4]) {
        float kq = 0.f;
#pragma unroll
        for (int j = 0; j < J; ++j)
#pragma unroll
            for (int c = 0; c < 4; ++c) kq = fmaf(kc[j][c], qc[j][c], kq);
        kq = red8(kq);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float a = 0.f, b = 0.f;
#pragma unroll
            for (int j = 0; j < J; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    a = fmaf(s[i][j][c], kc[j][c], a);
                    b = fmaf(s[i][j][c], qc[j][c], b);
                }
            a = red8(a);
            b = red8(b);
            const float delta = beta * (vr[i] - alpha * a);
#pragma unroll
            for (int j = 0; j < J; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) s[i][j][c] = fmaf(alpha, s[i][j][c], delta * kc[j][c]);
            out[i] = fmaf(alpha, b, delta * kq);
        }
    }
};

template <typename T, int D>
__device__ __forceinline__ void load_token(const T *qt, const T *kt, const T *vt, const RowBlock<T, D> &rb,
                                           float (&kc)[D / 32][4], float (&qc)[D / 32][4], float (&vr)[4]) {
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
        float4 a = load4(kt + rb.col(j));
        float4 b = load4(qt + rb.col(j));
        kc[j][0] = a.x; kc[j][1] = a.y; kc[j][2] = a.z; kc[j][3] = a.w;
        qc[j][0] = b.x; qc[j][1] = b.y; qc[j][2] = b.z; qc[j][3] = b.w;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) vr[i] = Elem<T>::load(vt + rb.row(i));
}

// grid.x = B*H*(D/64): one CTA per 64 rows of one (b, h) state. RAW: q, k arrive unnormalised
// and g, beta hold the gate logits a, b: q and k are L2-normalised here (their squared norms
// reduce over the same 8 lanes as the row dot products), alpha = exp(-softplus(a)) and
// beta = sigmoid(b).
template <typename T, int D, bool RAW>
__global__ void __launch_bounds__(kThreads) k_decode_step(const T *__restrict__ q, const T *__restrict__ k,
                                                          const T *__restrict__ v, const float *__restrict__ g,
                                                          const float *__restrict__ beta, float *__restrict__ S,
                                                          T *__restrict__ o) {
    constexpr int CPH = D / kRowsPerCta;
    const int bh = blockIdx.x / CPH;
    RowBlock<T, D> rb;
    rb.init_mapping(blockIdx.x % CPH);
    float *Sh = S + (size_t)bh * D * D;
    rb.load(Sh);
    float kc[D / 32][4], qc[D / 32][4], vr[4], out[4];
    load_token<T, D>(q + (size_t)bh * D, k + (size_t)bh * D, v + (size_t)bh * D, rb, kc, qc, vr);
    float alpha, b;
    if (RAW) {
        float kk = 0.f, qq = 0.f;
#pragma unroll
        for (int j = 0; j < D / 32; ++j)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                kk = fmaf(kc[j][c], kc[j][c], kk);
                qq = fmaf(qc[j][c], qc[j][c], qq);
            }
        const float sk = inv_norm(red8(kk)), sq = inv_norm(red8(qq));
#pragma unroll
        for (int j = 0; j < D / 32; ++j)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                kc[j][c] *= sk;
                qc[j][c] *= sq;
            }
        alpha = expf(neg_softplus(g[bh]));
        b = sigmoid_f(beta[bh]);
    } else {
        alpha = expf(g[bh]);
        b = beta[bh];
    }
    rb.step(kc, qc, vr, alpha, b, out);
    rb.store(Sh);
    if (rb.part == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) Elem<T>::store(o + (size_t)bh * D + rb.row(i), out[i]);
    }
}

// grid = (D/64, H, N): the rows of one (n, h) state stay in registers for the
// whole sequence; the next token's q, k, v are fetched while the current one
// is applied.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) k_seq_scan(const T *__restrict__ q, const T *__restrict__ k,
                                                       const T *__restrict__ v, const float *__restrict__ g,
                                                       const float *__restrict__ beta, const float *S0,
                                                       const int32_t *__restrict__ cu, int N, int T_tot, int H,
                                                       T *__restrict__ o, float *S_T) {
    const int h = blockIdx.y, n = blockIdx.z;
    RowBlock<T, D> rb;
    rb.init_mapping(blockIdx.x);
    int t0, t1;
    seq_bounds(cu, n, N, T_tot, t0, t1);
    const size_t sh = ((size_t)n * H + h) * D * D;
    if (S0) rb.load(S0 + sh); else rb.zero();
    float kc[D / 32][4], qc[D / 32][4], vr[4], out[4];
    float kn[D / 32][4], qn[D / 32][4], vn[4];
    if (t0 < t1) load_token<T, D>(q + ((size_t)t0 * H + h) * D, k + ((size_t)t0 * H + h) * D,
                                  v + ((size_t)t0 * H + h) * D, rb, kc, qc, vr);
    for (int t = t0; t < t1; ++t) {
        const size_t th = (size_t)t * H + h;
        const float alpha = expf(g[th]), b = beta[th];
        if (t + 1 < t1) {
            const size_t nh = th + H;
            load_token<T, D>(q + nh * D, k + nh * D, v + nh * D, rb, kn, qn, vn);
        }
        rb.step(kc, qc, vr, alpha, b, out);
        if (rb.part == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) Elem<T>::store(o + th * D + rb.row(i), out[i]);
        }
#pragma unroll
        for (int j = 0; j < D / 32; ++j)
#pragma unroll
            for (int c = 0; c < 4; ++c) { kc[j][c] = kn[j][c]; qc[j][c] = qn[j][c]; }
#pragma unroll
        for (int i = 0; i < 4; ++i) vr[i] = vn[i];
    }
    rb.store(S_T + sh);
}

}  // namespace

template <typename T, int D>
cudaError_t launch_decode_step(const T *q, const T *k, const T *v, const float *g, const float *beta, float *S,
                               int B, int H, T *o, cudaStream_t st, bool raw) {
    const int grid = B * H * (D / kRowsPerCta);
    if (raw)
        k_decode_step<T, D, true><<<grid, kThreads, 0, st>>>(q, k, v, g, beta, S, o);
    else
        k_decode_step<T, D, false><<<grid, kThreads, 0, st>>>(q, k, v, g, beta, S, o);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_seq_scan(const T *q, const T *k, const T *v, const float *g, const float *beta, const float *S0,
                            const int32_t *cu, int N, int T_tot, int H, T *o, float *S_T, cudaStream_t st) {
    dim3 grid(D / kRowsPerCta, H, N);
    k_seq_scan<T, D><<<grid, kThreads, 0, st>>>(q, k, v, g, beta, S0, cu, N, T_tot, H, o, S_T);
    return cudaGetLastError();
}

#define GDN_INST(T, D)                                                                                         \
    template cudaError_t launch_decode_step<T, D>(const T *, const T *, const T *, const float *, const float *, \
                                                  float *, int, int, T *, cudaStream_t, bool);               \
    template cudaError_t launch_seq_scan<T, D>(const T *, const T *, const T *, const float *, const float *,    \
                                               const float *, const int32_t *, int, int, int, T *, float *,   \
                                               cudaStream_t);
GDN_INST(float, 64)
GDN_INST(float, 128)
GDN_INST(__nv_bfloat16, 64)
GDN_INST(__nv_bfloat16, 128)
#undef GDN_INST

}  // namespace gdn
