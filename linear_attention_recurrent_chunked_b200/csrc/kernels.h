// Internal launchers of the library's kernels (host side). Not part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

template <typename T, int D>
cudaError_t launch_decode_step(const T *q, const T *k, const T *v, const float *g, const float *beta, float *S,
                               int B, int H, T *o, cudaStream_t st, bool raw = false);

template <typename T, int D>
cudaError_t launch_seq_scan(const T *q, const T *k, const T *v, const float *g, const float *beta, const float *S0,
                            const int32_t *cu, int N, int T_tot, int H, T *o, float *S_T, cudaStream_t st);

template <typename T, int D>
cudaError_t launch_chunk_simt(const T *q, const T *k, const T *v, const float *g, const float *beta, const float *S0,
                              const int32_t *cu, int N, int T_tot, int H, T *o, float *S_T, const uint32_t *err,
                              cudaStream_t st, bool raw = false);

// Tensor-core chunked forward, bf16 inputs, dk = dv = 128. Launches the
// validation / plan, the optional transition pass and the output pass;
// *stage names the launch that failed when an error is returned. The
// workspace holds the error word, the segment offsets and the per-segment
// transition slots (chunk_tc_workspace bytes for the preferred plan; a
// smaller workspace selects a coarser segmentation or none).
cudaError_t launch_chunk_tc(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v, const float *g,
                            const float *beta, const float *S0, const int32_t *cu, int N, int T_tot, int H,
                            __nv_bfloat16 *o, float *S_T, void *workspace, size_t ws_bytes, cudaStream_t st,
                            const char **stage);
int chunk_tc_seg_chunks(int N, int T_tot, int H);
size_t chunk_tc_workspace(int N, int T_tot, int H, int seg_chunks);

// Pipelined tensor-core chunked forward (same contract as launch_chunk_tc):
// plan, the parallel prep pass (decay scalars and UT solve of every chunk),
// the transition pass with its links (seg_chunks > 0 only) and the output
// pass. Needs chunk_ws_workspace(N, T_tot, H, seg_chunks) bytes of workspace.
// raw: q, k are unnormalised and g, beta hold the gate logits a, b (g = -softplus(a),
// beta = sigmoid(b)); the normalisation and gates are applied inside the passes.
cudaError_t launch_chunk_ws(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v, const float *g,
                            const float *beta, const float *S0, const int32_t *cu, int N, int T_tot, int H,
                            __nv_bfloat16 *o, float *S_T, void *workspace, int seg_chunks, cudaStream_t st,
                            const char **stage, bool raw = false);
int chunk_ws_seg_chunks(int N, int T_tot, int H, bool varlen);  // varlen: cu_seqlens given
size_t chunk_ws_workspace(int N, int T_tot, int H, int seg_chunks);

// Input projection with int8 weights (W8A16 on the tensor cores): y = x (diag(scale) w)^T split
// into q, k, v (bf16) and the gate logits a, b (fp32). x [T][D] bf16 (D % 64 == 0), w [N][D] int8,
// N = H (2 dk + dv) + 2 H; err is the error word (reset here).
cudaError_t launch_proj_w8(const __nv_bfloat16 *x, const int8_t *w, const float *scale, int T, int D, int H, int dk,
                           int dv, __nv_bfloat16 *q, __nv_bfloat16 *k, __nv_bfloat16 *v, float *a, float *b,
                           uint32_t *err, cudaStream_t st, const char **stage);

// Causal attention (bf16, d = 128) over packed sequences: o_t = softmax_j<=t(scale q_t . k_j) v_j per
// head; q, k, v, o [T_tot][H][128]; cu (device, N+1 offsets) or NULL (N equal sequences);
// max_len = the longest sequence's length (bounds the grid); err = error word.
cudaError_t launch_attn_fwd(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                            const int32_t *cu, int N, int T_tot, int H, int max_len, float scale, __nv_bfloat16 *o,
                            uint32_t *err, cudaStream_t st, const char **stage);

// Failure injection for tests (set by gdn_debug_inject; off by default): the pipelined path's
// first segment of head 0 withholds its end-state flag, and waits for flags give up after
// flag_wait_ns (0 = the normal bound) instead of hanging.
struct Inject {
    bool withhold_first_link;
    uint64_t flag_wait_ns;
};
Inject inject_settings();

// Kernel timing hooks (no-ops unless gdn_profile_enable(1)): an event pair
// around the launches between prof_start and prof_stop, recorded on st.
void *prof_start(const char *name, cudaStream_t st);
void prof_stop(void *handle);
// Diagnostic: T = (I + A)^{-1} for one strictly lower 64 x 64 fp32 matrix (row-major, device).
cudaError_t launch_diag_ut_solve(const float *A, float *T, cudaStream_t st);

// Writes the workspace error word: ERRBIT_SEQLENS if cu_seqlens (device, N+1
// entries) is not 0 = c0 <= ... <= cN = T_tot, else 0. With cu == NULL it
// just clears the word.
cudaError_t launch_validate_seqlens(const int32_t *cu, int N, int T_tot, uint32_t *err, cudaStream_t st);

}  // namespace gdn
