// Chunked gated delta rule on CUDA cores in fp32 (the path for fp32 inputs).
//
// The pages give only the shape of the rewrite: the token-by-token scan of
// the recurrent layers becomes a chunk-wise delta-rule form with an
// intra-chunk part, an inter-chunk part and a forward-substitution kernel
// (page 1, abstract, result (i); page 2, "Resumen Tecnico", Metodologia,
// recurrent-layer item). The algebra is derived from the rule. For one chunk
// of C positions r, s (S_0 = state entering the chunk, G_r = sum_{s<=r} g_s,
// gamma_r = exp(G_r), Gamma_rs = exp(G_r - G_s) <= 1 for s <= r):
//
//   A_rs  = beta_r Gamma_rs (k_r . k_s)  (s < r)     P_rs = Gamma_rs (q_r . k_s)  (s <= r)
//   T     = (I + A)^{-1}                 (forward substitution)
//   W     = T diag(beta gamma) K,        U = T diag(beta) V
//   Delta = U - W S_0^T
//   O     = diag(gamma) Q S_0^T + P Delta
//   S_C   = gamma_C S_0 + Delta^T diag(exp(G_C - G_s)) K
//
// Every exponent is <= 0: decays are never split as exp(G_r) * exp(-G_s).
// Positions past the end of a sequence are padded with k = q = v = 0,
// g = 0 and beta = 0, which makes their rows of A, W, U and Delta zero and
// leaves G constant, so a partial last chunk needs no other masking.
//
// One CTA (256 threads) per (sequence, head) walks the chunks of its
// sequence; all intermediates live in shared memory in fp32. This path is
// built for exactness (fp32 inputs are checked to 1e-4 of max|o|), not speed.
#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int kSimtThreads = 256;

template <int D, int C>
struct SimtSmem {
    static constexpr int DP = D + 1;  // row pitch of the C x D tiles (odd: spreads banks)
    static constexpr int CP = C + 1;
    float K[C * DP], Q[C * DP], V[C * DP], W[C * DP], U[C * DP];
    float A[C * CP], T[C * CP], P[C * CP];
    float S[D * DP];
    float G[C], gam[C], dte[C], beta[C];
};

template <typename T, int D, int C>
__global__ void __launch_bounds__(kSimtThreads) k_chunk_simt(const T *__restrict__ q, const T *__restrict__ k,
                                                             const T *__restrict__ v, const float *__restrict__ g,
                                                             const float *__restrict__ beta, const float *S0,
                                                             const int32_t *__restrict__ cu, int N, int T_tot, int H,
                                                             T *__restrict__ o, float *S_T,
                                                             const uint32_t *__restrict__ err, int raw) {
    using Sm = SimtSmem<D, C>;
    constexpr int DP = Sm::DP, CP = Sm::CP;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Sm &sm = *reinterpret_cast<Sm *>(smem_raw);
    if (err && *err) return;  // malformed cu_seqlens: write nothing

    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
    int t0, t1;
    seq_bounds(cu, n, N, T_tot, t0, t1);
    const size_t sh = ((size_t)n * H + h) * D * D;
    for (int idx = tid; idx < D * D; idx += kSimtThreads)
        sm.S[(idx / D) * DP + idx % D] = S0 ? S0[sh + idx] : 0.f;
    __syncthreads();

    for (int c0 = t0; c0 < t1; c0 += C) {
        const int L = min(C, t1 - c0);
        // ---- load the chunk (zero padded past L)
        for (int idx = tid; idx < C * D; idx += kSimtThreads) {
            const int r = idx / D, j = idx % D;
            const bool ok = r < L;
            const size_t off = ((size_t)(c0 + r) * H + h) * D + j;
            sm.K[r * DP + j] = ok ? Elem<T>::load(k + off) : 0.f;
            sm.Q[r * DP + j] = ok ? Elem<T>::load(q + off) : 0.f;
            sm.V[r * DP + j] = ok ? Elem<T>::load(v + off) : 0.f;
        }
        if (tid < C) {
            // raw inputs: g and beta hold the gate logits a, b; g = -softplus(a), beta = sigmoid(b)
            const bool ok = tid < L;
            const float gv = ok ? g[(size_t)(c0 + tid) * H + h] : 0.f;
            const float bv = ok ? beta[(size_t)(c0 + tid) * H + h] : 0.f;
            sm.G[tid] = (raw && ok) ? neg_softplus(gv) : gv;
            sm.beta[tid] = (raw && ok) ? sigmoid_f(bv) : bv;
        }
        __syncthreads();
        if (raw) {  // raw inputs: L2-normalise the rows of K and Q (one warp per row)
            const int warp = tid >> 5, lane = tid & 31;
            for (int rr = warp; rr < 2 * L; rr += kSimtThreads / 32) {
                float *row = (rr < L ? sm.K : sm.Q) + (rr < L ? rr : rr - L) * DP;
                float ss = 0.f;
                for (int j = lane; j < D; j += 32) ss = fmaf(row[j], row[j], ss);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float sc = inv_norm(ss);
                for (int j = lane; j < D; j += 32) row[j] *= sc;
            }
            __syncthreads();
        }
        // ---- G = cumsum(g), gamma, decay to chunk end
        if (tid == 0) {
            float acc = 0.f;
            for (int r = 0; r < C; ++r) { acc += sm.G[r]; sm.G[r] = acc; }
        }
        __syncthreads();
        if (tid < C) {
            sm.gam[tid] = expf(sm.G[tid]);
            sm.dte[tid] = expf(sm.G[C - 1] - sm.G[tid]);
        }
        // ---- intra-chunk: A (strictly lower) and P (lower incl. diagonal)
        for (int idx = tid; idx < C * C; idx += kSimtThreads) {
            const int r = idx / C, s = idx % C;
            float a = 0.f, p = 0.f;
            if (s <= r) {
                float dk = 0.f, dq = 0.f;
                for (int j = 0; j < D; ++j) {
                    dk = fmaf(sm.K[r * DP + j], sm.K[s * DP + j], dk);
                    dq = fmaf(sm.Q[r * DP + j], sm.K[s * DP + j], dq);
                }
                const float e = expf(sm.G[r] - sm.G[s]);
                p = e * dq;
                if (s < r) a = sm.beta[r] * e * dk;
            }
            sm.A[r * CP + s] = a;
            sm.P[r * CP + s] = p;
        }
        __syncthreads();
        // ---- T = (I + A)^{-1}: forward substitution, one thread per column
        if (tid < C) {
            const int j = tid;
            for (int r = 0; r < C; ++r) {
                float acc = (r == j) ? 1.f : 0.f;
                for (int s = j; s < r; ++s) acc = fmaf(-sm.A[r * CP + s], sm.T[s * CP + j], acc);
                sm.T[r * CP + j] = (r < j) ? 0.f : acc;
            }
        }
        __syncthreads();
        // ---- W = T diag(beta gamma) K, U = T diag(beta) V
        for (int idx = tid; idx < C * D; idx += kSimtThreads) {
            const int r = idx / D, c = idx % D;
            float w = 0.f, u = 0.f;
            for (int s = 0; s <= r; ++s) {
                const float t = sm.T[r * CP + s] * sm.beta[s];
                w = fmaf(t * sm.gam[s], sm.K[s * DP + c], w);
                u = fmaf(t, sm.V[s * DP + c], u);
            }
            sm.W[r * DP + c] = w;
            sm.U[r * DP + c] = u;
        }
        __syncthreads();
        // ---- Delta = U - W S_0^T (in place over U)
        for (int idx = tid; idx < C * D; idx += kSimtThreads) {
            const int r = idx / D, i = idx % D;
            float acc = sm.U[r * DP + i];
            for (int j = 0; j < D; ++j) acc = fmaf(-sm.W[r * DP + j], sm.S[i * DP + j], acc);
            sm.U[r * DP + i] = acc;
        }
        __syncthreads();
        // ---- O = diag(gamma) Q S_0^T + P Delta
        for (int idx = tid; idx < L * D; idx += kSimtThreads) {
            const int r = idx / D, i = idx % D;
            float qs = 0.f, pd = 0.f;
            for (int j = 0; j < D; ++j) qs = fmaf(sm.Q[r * DP + j], sm.S[i * DP + j], qs);
            for (int s = 0; s <= r; ++s) pd = fmaf(sm.P[r * CP + s], sm.U[s * DP + i], pd);
            Elem<T>::store(o + ((size_t)(c0 + r) * H + h) * D + i, fmaf(sm.gam[r], qs, pd));
        }
        __syncthreads();
        // ---- S_C = gamma_C S_0 + Delta^T diag(exp(G_C - G_s)) K
        const float gC = sm.gam[C - 1];
        for (int idx = tid; idx < D * D; idx += kSimtThreads) {
            const int i = idx / D, j = idx % D;
            float acc = gC * sm.S[i * DP + j];
            for (int s = 0; s < L; ++s) acc = fmaf(sm.U[s * DP + i] * sm.dte[s], sm.K[s * DP + j], acc);
            sm.S[i * DP + j] = acc;
        }
        __syncthreads();
    }
    for (int idx = tid; idx < D * D; idx += kSimtThreads) S_T[sh + idx] = sm.S[(idx / D) * DP + idx % D];
}

}  // namespace

template <typename T, int D>
cudaError_t launch_chunk_simt(const T *q, const T *k, const T *v, const float *g, const float *beta, const float *S0,
                              const int32_t *cu, int N, int T_tot, int H, T *o, float *S_T, const uint32_t *err,
                              cudaStream_t st, bool raw) {
    constexpr int C = (D <= 64) ? 64 : 32;
    const size_t smem = sizeof(SimtSmem<D, C>);
    cudaError_t e = cudaFuncSetAttribute(k_chunk_simt<T, D, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(H, N);
    k_chunk_simt<T, D, C><<<grid, kSimtThreads, smem, st>>>(q, k, v, g, beta, S0, cu, N, T_tot, H, o, S_T, err,
                                                            raw ? 1 : 0);
    return cudaGetLastError();
}

#define GDN_INST(T, D)                                                                                        \
    template cudaError_t launch_chunk_simt<T, D>(const T *, const T *, const T *, const float *, const float *, \
                                                 const float *, const int32_t *, int, int, int, T *, float *,  \
                                                 const uint32_t *, cudaStream_t, bool);
GDN_INST(float, 64)
GDN_INST(float, 128)
GDN_INST(__nv_bfloat16, 64)
GDN_INST(__nv_bfloat16, 128)
#undef GDN_INST

}  // namespace gdn
