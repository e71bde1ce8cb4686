/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated-delta-rule forward library
 *          (libgdn_b200.so).
 *
 * What is computed. Per sequence n and head h, the gated delta rule
 *
 *     alpha_t = exp(g_t)
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,    o_t = S_t q_t
 *
 * with S a d_v x d_k fp32 matrix (row = value index). This is the recurrent
 * layer of the hybrid gated delta network backbone in "A Modern Multimodal
 * Assistant on a 6 GB 2011 GPU" (page 1, abstract, result (i)), which runs
 * it in two forms: chunk by chunk (prefill) and one token at a time (the
 * sequential scan; decode). The update rule is that of the Gated Delta
 * Networks paper listed among page 3's references. The pages print no
 * interface; this one is the library's own.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, contiguous, owned by the
 *     caller, and 16-byte aligned (g and beta: 4-byte aligned). The library allocates no memory, never synchronises
 *     the stream (except gdn_chunk_fwd_check, which exists to do so), and
 *     launches everything on `stream` (a cudaStream_t passed as void*; NULL =
 *     the legacy default stream).
 *   - Layouts are token-major and row-major:
 *       q, k : [T][H][dk]   v, o : [T][H][dv]   (dtype gdn_dtype: fp32 or bf16)
 *       g, beta : [T][H] fp32   (g = natural-log decay, finite, g <= 0 expected;
 *                                beta in [0,1] expected)
 *       S, S0, S_T : [N][H][dv][dk] fp32
 *     q and k are expected L2-normalised by the caller; no normalisation,
 *     gating or scaling happens inside (o_t = S_t q_t, no query scale).
 *   - Supported head sizes: dk = dv in {64, 128}.
 *   - o is written in the input dtype (bf16: rounded to nearest even from the
 *     fp32 accumulator). States are fp32.
 *   - NaN/Inf inputs are undefined behaviour; they are not checked on the hot
 *     path. Decays below ~1e-38 may be flushed to zero.
 *   - Errors are returned as gdn_status, never thrown or trapped;
 *     gdn_last_error() gives a message for the calling thread's last non-OK
 *     status. Launch failures map to GDN_ERR_CUDA with the CUDA error text.
 */
#ifndef GDN_B200_H
#define GDN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_NULL = 1,      /* a required pointer is NULL */
    GDN_ERR_SHAPE = 2,     /* unsupported or inconsistent sizes */
    GDN_ERR_DTYPE = 3,     /* unknown dtype code */
    GDN_ERR_ALIGN = 4,     /* a pointer is not 16-byte aligned */
    GDN_ERR_SEQLENS = 5,   /* cu_seqlens not 0 = c0 <= c1 <= ... <= cN = T_tot */
    GDN_ERR_WORKSPACE = 6, /* workspace missing or smaller than required */
    GDN_ERR_CUDA = 7,      /* a CUDA launch or runtime call failed */
    GDN_ERR_TIMEOUT = 8,   /* a bounded device-side wait gave up */
    GDN_ERR_BOUNDS = 9     /* a device-side index check failed (library built with GDN_DEBUG_CHECKS) */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Library version, major*10000 + minor*100 + patch. */
int gdn_version(void);

/* Message for the calling thread's last non-OK status ("" if none). The
 * string is owned by the library and valid until the thread's next call. */
const char *gdn_last_error(void);

/*
 * Workspace bytes with which gdn_chunk_fwd runs its fastest plan for these
 * sizes (always >= 256). Any workspace of at least 256 bytes (the device
 * error word) is accepted. The bf16 path keeps a 9 KB record per (chunk,
 * head) (the chunk's solved triangular factor and decay vectors); when there
 * are few (sequence, head) pairs it also splits each sequence into segments
 * that run in parallel and keeps, per (segment, head), the segment's end
 * state and its affine map (together 192 KB, three d x d fp32 matrices' worth);
 * a smaller workspace selects fewer segments, down to none, then a path
 * without records. The workspace is
 * scratch owned by the caller: its contents on entry are ignored and on exit
 * are meaningless except for the error word read by gdn_chunk_fwd_check.
 * Two calls that overlap on the GPU must not share a workspace.
 */
size_t gdn_chunk_fwd_workspace_size(int N, int T_tot, int H, int dk, int dv, gdn_dtype dtype);

/*
 * Prefill: the chunked form of the rule over N packed sequences (page 1,
 * abstract, result (i): the recurrent layers rewritten chunk-wise; page 2,
 * "Resumen Tecnico", Metodologia, recurrent-layer item: an intra-chunk part,
 * an inter-chunk part and a forward-substitution step).
 *
 *   q, k      [T_tot][H][dk]  dtype      v [T_tot][H][dv] dtype
 *   g, beta   [T_tot][H]      fp32
 *   S0        [N][H][dv][dk]  fp32, or NULL for a zero initial state.
 *             May alias S_T (in-place state update).
 *   cu_seqlens [N+1] int32 on the device: sequence n is tokens
 *             [cu_seqlens[n], cu_seqlens[n+1]). NULL means N equal sequences
 *             of T_tot/N tokens (T_tot % N must be 0). Chunks restart at every
 *             sequence start; the last chunk of a sequence may be partial;
 *             an empty sequence gives S_T = S0 (or 0).
 *   o         [T_tot][H][dv] dtype  (output; must not alias any input)
 *   S_T       [N][H][dv][dk] fp32   (output: state after each sequence)
 *   workspace, ws_bytes: device memory, 256-byte aligned, ws_bytes >= 256
 *             (gdn_chunk_fwd_workspace_size(...) bytes for the fastest plan).
 *
 * A device-side cu_seqlens is validated on the device (the host cannot read
 * it without a synchronisation): if it is malformed, the kernels write
 * nothing to o / S_T and record GDN_ERR_SEQLENS in the workspace's error
 * word; gdn_chunk_fwd itself returns GDN_OK and gdn_chunk_fwd_check reports
 * the error. Which kernels run: bf16 inputs with dk = dv = 128 take the
 * tensor-core path (bf16 operands, fp32 accumulation and state); fp32 inputs
 * (either head size) and bf16 inputs with dk = dv = 64 take the fp32
 * CUDA-core chunked path, which has no tensor-core variant (same results up to
 * rounding, far slower).
 */
gdn_status gdn_chunk_fwd(const void *q, const void *k, const void *v,
                         const float *g, const float *beta, const float *S0,
                         const int32_t *cu_seqlens, int N, int T_tot, int H, int dk, int dv,
                         gdn_dtype dtype, void *o, float *S_T,
                         void *workspace, size_t ws_bytes, void *stream);

/*
 * Prefill from the layer's raw inputs: gdn_chunk_fwd with the input
 * preparation done inside the kernels instead of by the caller. The recurrent
 * layer of a gated delta network (page 1, abstract, result (i)) normalises its
 * queries and keys and derives its decay and write strength from gate logits;
 * the pages name the layer but print none of these steps, so this is the
 * plain reading of the layer's input contract:
 *     q_t = q_raw_t / max(||q_raw_t||_2, 1e-12),   k_t likewise (per token, head)
 *     g_t = -softplus(a_t)  (alpha_t = exp(g_t) = 1 / (1 + exp(a_t)))
 *     beta_t = sigmoid(b_t) = 1 / (1 + exp(-b_t))
 * and then the rule exactly as gdn_chunk_fwd. Arguments are gdn_chunk_fwd's
 * with q_raw, k_raw [T_tot][H][dk] (dtype, any norm) in place of q, k and the
 * fp32 gate logits a, b [T_tot][H] in place of g, beta. The normalisation and
 * gates are folded into the passes that read q, k, g and beta anyway: there is
 * no separate pass over the inputs. bf16 inputs with dk = dv = 128 run only
 * on the pipelined tensor-core path, whose workspace holds a record per
 * (chunk, head): gdn_chunk_fwd_workspace_size gives the size of the fastest
 * plan, a smaller workspace that still holds the records runs without time
 * segments, and one that does not gives GDN_ERR_WORKSPACE. fp32 inputs and
 * d = 64 take the fp32 CUDA-core path as in gdn_chunk_fwd.
 */
gdn_status gdn_chunk_fwd_raw(const void *q_raw, const void *k_raw, const void *v,
                             const float *a, const float *b, const float *S0,
                             const int32_t *cu_seqlens, int N, int T_tot, int H, int dk, int dv,
                             gdn_dtype dtype, void *o, float *S_T,
                             void *workspace, size_t ws_bytes, void *stream);

/*
 * gdn_chunk_fwd without a caller-provided workspace, for callers that cannot
 * allocate device memory: code running under a memory manager that has
 * already reserved the GPU's memory, plugins whose host application owns
 * every device allocation, and latency-critical paths that must not pay
 * cudaMalloc's implicit synchronisation. The paper has no counterpart of
 * this entry point; it is a property of this library only.
 *
 * Arguments, results and dtype dispatch are those of gdn_chunk_fwd; the
 * workspace comes from an 8 MiB array built into the library, which every
 * GPU that loads the library holds until the process exits. When the sizes'
 * preferred workspace (gdn_chunk_fwd_workspace_size) exceeds 8 MiB, the
 * forward runs with the coarser time segmentation that fits in it (the
 * results are the same up to rounding); GDN_ERR_WORKSPACE is returned only
 * if the array could not hold gdn_chunk_fwd's 256-byte minimum. The call
 * allocates nothing. Every call looks up the array's device address in the
 * context current on the calling thread (the first lookup in a context may
 * load the library's module: make the first call on a device before any
 * stream capture). All calls on a device share the array: calls that overlap
 * on the GPU race and must be serialised by the caller. The array's error word
 * is not readable through this entry point, so two device-side failures go
 * unreported here: a malformed device cu_seqlens (the kernels then write
 * nothing) and a bounded inter-block wait that gave up (GDN_ERR_TIMEOUT in
 * gdn_chunk_fwd_check; o and S_T are then incomplete). Callers that need
 * either reported use gdn_chunk_fwd + gdn_chunk_fwd_check.
 */
gdn_status gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                 const float *g, const float *beta, const float *S0,
                                 const int32_t *cu_seqlens, int N, int T_tot, int H, int dk, int dv,
                                 gdn_dtype dtype, void *o, float *S_T, void *stream);

/*
 * Synchronises `stream` and reads the device error word that the last
 * gdn_chunk_fwd on this workspace wrote: GDN_OK, GDN_ERR_SEQLENS,
 * GDN_ERR_TIMEOUT (a bounded inter-block wait gave up; outputs are then
 * incomplete) or, from a library built with GDN_DEBUG_CHECKS (the
 * libgdn_b200_debug.so variant, whose kernels check their indices into the
 * workspace and the outputs), GDN_ERR_BOUNDS (an index was out of range; the
 * access went to index 0 of its region instead). The word is reset by every
 * gdn_chunk_fwd call. On a timeout
 * of the pipelined path, gdn_last_error() names the first wait that gave up
 * (the mbarrier's shared-memory address and awaited parity, or the flag's
 * word offset in the workspace, with the block and thread), a diagnostic for
 * whoever changes the kernels.
 */
gdn_status gdn_chunk_fwd_check(const void *workspace, size_t ws_bytes, void *stream);

/*
 * Decode: one single-token step of the rule for B independent sequences
 * (the token-at-a-time form of page 2, "Resumen Tecnico", Metodologia,
 * recurrent-layer item). For every (b, h) and every row i of S:
 *     a = S_i . k,  b_i = S_i . q,  S_i <- alpha S_i + beta (v_i - alpha a) k,
 *     o_i = alpha b_i + beta (v_i - alpha a) (k . q)       (= (S_new q)_i)
 *   q, k [B][H][dk] dtype; v [B][H][dv] dtype; g, beta [B][H] fp32;
 *   S [B][H][dv][dk] fp32, updated in place; o [B][H][dv] dtype (output).
 * S is read once and written once per call.
 */
gdn_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const float *g, const float *beta, float *S,
                           int B, int H, int dk, int dv, gdn_dtype dtype, void *o, void *stream);

/*
 * Decode from raw inputs: gdn_decode_step with the input preparation of
 * gdn_chunk_fwd_raw done in the same kernel (q, k normalised, alpha =
 * exp(-softplus(a)), beta = sigmoid(b)). q_raw, k_raw [B][H][dk] dtype;
 * a, b [B][H] fp32 gate logits; everything else as gdn_decode_step.
 */
gdn_status gdn_decode_step_raw(const void *q_raw, const void *k_raw, const void *v,
                               const float *a, const float *b, float *S,
                               int B, int H, int dk, int dv, gdn_dtype dtype, void *o, void *stream);

/*
 * Input projection of the recurrent layer with int8 weights. The pages' system
 * keeps its language-model weights as 8-bit codes dequantised for the
 * projections (page 1, abstract; page 2, "Resumen Tecnico", the GEMM item);
 * this is that projection for the recurrent layer, producing exactly the raw
 * inputs gdn_chunk_fwd_raw / gdn_decode_step_raw take:
 *     y[t][n] = scale[n] * sum_j x[t][j] w[n][j]        (fp32 accumulation)
 * with output channels in the order q (H dk), k (H dk), v (H dv), a (H), b (H),
 * head-major inside each, N = H (2 dk + dv) + 2 H. The int8 codes are exact in
 * bf16: the product runs on the tensor cores with bf16 operands and the scale
 * is applied to the fp32 result, so the weights cross HBM as int8 and the
 * dequantisation is exact. The pages do not fix a quantisation scheme; this one
 * is symmetric with one scale per output channel.
 *   x [T][D] bf16 (D a positive multiple of 64); w [N][D] int8; scale [N] fp32;
 *   q_raw, k_raw [T][H][dk] bf16; v [T][H][dv] bf16; a, b [T][H] fp32
 *   (outputs, rounded to nearest even for bf16); H dk and H dv multiples of 8.
 *   workspace, ws_bytes: >= 256 bytes of device memory for the error word
 *   (gdn_chunk_fwd_check reads it: GDN_ERR_TIMEOUT if a bounded wait gave up).
 * Pointers 16-byte aligned (a, b: 4). Runs one persistent kernel on `stream`.
 */
gdn_status gdn_proj_w8(const void *x, const int8_t *w, const float *scale, int T, int D, int H, int dk,
                       int dv, void *q_raw, void *k_raw, void *v, float *a, float *b,
                       void *workspace, size_t ws_bytes, void *stream);

/*
 * Causal attention of the hybrid backbone's attention layers. The pages' backbone
 * interleaves the recurrent layers with causal attention layers, whose O(N^2)
 * kernel made long-context prefill collapse until it was rewritten as per-head
 * GEMMs (page 1, abstract: 17x faster prefill at 10k tokens; page 2, "Resumen
 * Tecnico", the attention rewrite). Per sequence, head h and position t:
 *     o_t = sum_{j <= t} softmax_j(scale * q_t . k_j) v_j
 * over the keys of the same sequence (standard scaled dot-product attention with
 * a causal mask; the pages do not write it out). The scores never leave the
 * chip: per query tile they live in tensor memory (see the implementation).
 *   q, k, v, o [T_tot][H][d] bf16, d = 128 (o: output, bf16 rounded to nearest)
 *   cu_seqlens [N+1] int32 on the device, or NULL for N equal sequences;
 *     max_len bounds the sequences' lengths (ignored when cu_seqlens is NULL)
 *   scale > 0, or <= 0 for 1 / sqrt(d)
 *   workspace, ws_bytes: >= 256 bytes of device memory for the error word
 *     (gdn_chunk_fwd_check reads it: GDN_ERR_SEQLENS for a malformed device
 *     cu_seqlens, then nothing is written; GDN_ERR_TIMEOUT for a bounded wait
 *     that gave up).
 * Pointers 16-byte aligned. dtype must be GDN_BF16 (GDN_ERR_DTYPE otherwise).
 */
gdn_status gdn_attn_fwd(const void *q, const void *k, const void *v, const int32_t *cu_seqlens, int N,
                        int T_tot, int H, int d, int max_len, float scale, gdn_dtype dtype, void *o,
                        void *workspace, size_t ws_bytes, void *stream);

/*
 * The sequential (token-by-token) scan on the GPU: the same result as
 * gdn_chunk_fwd, computed one token at a time with the decode step's row
 * update. It is the comparator for the chunked path's speed-up (page 1,
 * abstract, result (i) reports the chunked form 2.8 times faster than the
 * scan on a Fermi C2075), not a production path. Arguments as gdn_chunk_fwd, without a workspace. A
 * malformed device cu_seqlens is clamped into [0, T_tot] per sequence (no
 * access leaves the buffers) and gives meaningless results: validate it
 * with gdn_chunk_fwd + gdn_chunk_fwd_check.
 */
gdn_status gdn_seq_scan(const void *q, const void *k, const void *v,
                        const float *g, const float *beta, const float *S0,
                        const int32_t *cu_seqlens, int N, int T_tot, int H, int dk, int dv,
                        gdn_dtype dtype, void *o, float *S_T, void *stream);

/*
 * Diagnostic (used by the tests, not by the forward path): one tensor-core
 * tile D = A * B^T computed with the same shared-memory descriptors, TMEM
 * allocation and tcgen05.mma / tcgen05.ld helpers as the chunked kernel.
 *   A [M][K] bf16 row-major, B [N][K] bf16 row-major (device);
 *   D [128][N] fp32 (device): every TMEM lane is dumped, so for M = 64 the
 *     rows the hardware leaves unused are visible as well.
 *   a_mn / b_mn: 1 = stage that operand as an MN-major tile, 0 = K-major.
 *   variant: 0 or 1, the two no-swizzle core-matrix stride conventions of
 *     the kernels; 2, the 128-byte-swizzled tiles that TMA writes.
 * Limits: M in {64, 128}; 16 <= N <= 256 (multiple of 16 for M = 128, of 8
 * for M = 64; N <= 128 for variant 2); 16 <= K <= 128, multiple of 16.
 * Launches one CTA on `stream`.
 */
gdn_status gdn_diag_mma_tile(const void *A, const void *B, float *D, int M, int N, int K,
                             int a_mn, int b_mn, int variant, void *stream);

/*
 * Diagnostic (used by the tests): the chunked path's UT/WY solve on one
 * matrix, T = (I + A)^{-1}, with A a 64 x 64 fp32 row-major device matrix
 * that is zero on and above the diagonal and T its 64 x 64 fp32 result
 * (page 2, "Resumen Tecnico", Metodologia, recurrent-layer item: the
 * forward-substitution step of the chunked form). One CTA on `stream`.
 */
gdn_status gdn_diag_ut_solve(const float *A, float *T, void *stream);

/*
 * Failure injection, for tests of the failure path (off by default; process
 * wide, set it while no call is in flight). The pages describe no such thing;
 * it exists to show that a device-side wait that cannot complete ends with an
 * error status instead of hanging the GPU.
 *   GDN_INJECT_NONE: normal operation (wait_us ignored).
 *   GDN_INJECT_WITHHOLD_LINK: in every later gdn_chunk_fwd call that runs the
 *     pipelined bf16 tensor-core path (a workspace of at least
 *     gdn_chunk_fwd_workspace_size bytes) with a sequence split into parallel
 *     segments, the
 *     transition block of the first segment of head 0 computes as usual but
 *     never publishes its end state. The blocks that wait for it give up after
 *     wait_us microseconds (1 .. 1000000; instead of the normal 1 s bound),
 *     mark their own results failed so that blocks waiting on them give up
 *     too, record GDN_ERR_TIMEOUT in the workspace's error word and return.
 *     Outputs of the affected (sequence, head) pairs are then incomplete;
 *     other heads are unaffected. gdn_chunk_fwd_check reports the timeout.
 * Returns GDN_ERR_SHAPE for an unknown kind or an out-of-range wait_us.
 */
typedef enum { GDN_INJECT_NONE = 0, GDN_INJECT_WITHHOLD_LINK = 1 } gdn_inject_kind;
gdn_status gdn_debug_inject(int kind, unsigned wait_us);

/*
 * Kernel timing (measurement support, off by default). While enabled, every
 * entry point records a CUDA event pair on its stream around each kernel it
 * launches. gdn_profile_read waits for those events, writes per kernel name
 * the summed milliseconds (ms[i]) and launch count (counts[i]), the names
 * newline-separated into `names` (truncated to names_len), clears the record
 * and returns the number of kernel names (at most max_kernels). ms / counts /
 * names may be NULL. Not for use while a CUDA graph is being captured.
 */
void gdn_profile_enable(int on);
int gdn_profile_read(char *names, size_t names_len, float *ms, int *counts, int max_kernels);

#ifdef __cplusplus
}
#endif
#endif /* GDN_B200_H */
