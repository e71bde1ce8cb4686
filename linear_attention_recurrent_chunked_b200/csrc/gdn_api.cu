// C ABI of the library (declared in include/gdn.h): argument validation,
// error reporting and dispatch to the kernels. Host code only, apart from the
// small cu_seqlens validation kernel.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

namespace {

thread_local char g_msg[512] = "";

gdn_status fail(gdn_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

gdn_status ok() {
    g_msg[0] = '\0';
    return GDN_OK;
}

gdn_status cuda_fail(cudaError_t e, const char *what) {
    return fail(GDN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool misaligned(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

constexpr size_t kErrWordBytes = 256;  // error word, padded to keep later regions 256-byte aligned

// ---- optional per-kernel timing (gdn_profile_*): CUDA events recorded on the
// launching stream around each kernel the entry points launch.
struct ProfRec {
    const char *name;
    cudaEvent_t start, stop;
};
struct Prof {
    std::mutex mu;
    bool on = false;
    std::vector<ProfRec> recs;
    std::vector<cudaEvent_t> pool;
} g_prof;

cudaEvent_t prof_event() {
    if (!g_prof.pool.empty()) {
        cudaEvent_t e = g_prof.pool.back();
        g_prof.pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// RAII: records a start event now and a stop event (plus the record) at scope exit.
struct ProfScope {
    const char *name;
    cudaStream_t st;
    cudaEvent_t start = nullptr;
    ProfScope(const char *n, cudaStream_t s) : name(n), st(s) {
        std::lock_guard<std::mutex> lk(g_prof.mu);
        if (g_prof.on) {
            start = prof_event();
            cudaEventRecord(start, st);
        }
    }
    ~ProfScope() {
        if (!start) return;
        std::lock_guard<std::mutex> lk(g_prof.mu);
        cudaEvent_t stop = prof_event();
        cudaEventRecord(stop, st);
        g_prof.recs.push_back({name, start, stop});
    }
};

gdn_status check_common(const void *q, const void *k, const void *v, const float *g, const float *beta,
                        const void *o, int T_tot, int H, int dk, int dv, int dtype) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return fail(GDN_ERR_DTYPE, "dtype %d is not GDN_F32 or GDN_BF16", dtype);
    if (H < 1 || T_tot < 0) return fail(GDN_ERR_SHAPE, "H=%d T=%d out of range", H, T_tot);
    if (dk != dv || (dk != 64 && dk != 128))
        return fail(GDN_ERR_SHAPE, "head sizes dk=%d dv=%d unsupported (need dk == dv in {64, 128})", dk, dv);
    if (T_tot > 0 && (!q || !k || !v || !g || !beta || !o)) return fail(GDN_ERR_NULL, "q, k, v, g, beta and o are required");
    const void *ptrs[] = {q, k, v, o};
    for (const void *p : ptrs)
        if (misaligned(p)) return fail(GDN_ERR_ALIGN, "tensor pointer %p is not 16-byte aligned", p);
    if ((reinterpret_cast<uintptr_t>(g) | reinterpret_cast<uintptr_t>(beta)) & 3u)
        return fail(GDN_ERR_ALIGN, "g and beta must be 4-byte aligned");
    if ((double)T_tot * H * dk >= 9.0e18) return fail(GDN_ERR_SHAPE, "sizes overflow");
    return GDN_OK;
}

}  // namespace

namespace gdn {

__global__ void k_validate_seqlens(const int32_t *__restrict__ cu, int N, int T_tot, uint32_t *__restrict__ err) {
    // One warp: err = ERRBIT_SEQLENS unless cu[0] == 0, cu non-decreasing, cu[N] == T_tot.
    bool bad = false;
    if (cu) {
        for (int n = threadIdx.x; n < N; n += 32) bad |= cu[n + 1] < cu[n];
        if (threadIdx.x == 0) bad |= (cu[0] != 0) || (cu[N] != T_tot);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (threadIdx.x == 0) *err = bad ? ERRBIT_SEQLENS : 0u;
}

cudaError_t launch_validate_seqlens(const int32_t *cu, int N, int T_tot, uint32_t *err, cudaStream_t st) {
    k_validate_seqlens<<<1, 32, 0, st>>>(cu, N, T_tot, err);
    return cudaGetLastError();
}

struct ProfHandle {
    const char *name;
    cudaStream_t st;
    cudaEvent_t start;
};

// Every launch site brackets its kernel with these: an NVTX range named after the kernel (seen by
// Nsight tools when one is attached; a few nanoseconds otherwise) and, while profiling is enabled,
// a pair of CUDA events on the launch stream.
void *prof_start(const char *name, cudaStream_t st) {
    nvtxRangePushA(name);
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (!g_prof.on) return nullptr;
    ProfHandle *hd = new ProfHandle{name, st, prof_event()};
    cudaEventRecord(hd->start, st);
    return hd;
}

void prof_stop(void *handle) {
    nvtxRangePop();
    if (!handle) return;
    ProfHandle *hd = static_cast<ProfHandle *>(handle);
    std::lock_guard<std::mutex> lk(g_prof.mu);
    cudaEvent_t stop = prof_event();
    cudaEventRecord(stop, hd->st);
    g_prof.recs.push_back({hd->name, hd->start, stop});
    delete hd;
}

std::atomic<int> g_inject_kind{0};
std::atomic<unsigned long long> g_inject_wait_ns{0};

Inject inject_settings() {
    const int kind = g_inject_kind.load(std::memory_order_relaxed);
    return Inject{kind == GDN_INJECT_WITHHOLD_LINK, kind ? (uint64_t)g_inject_wait_ns.load() : 0ull};
}

// Sets the calling thread's last-error message (for entry points defined in other files).
gdn_status record_error(gdn_status s, const char *msg) { return fail(s, "%s", msg); }

}  // namespace gdn

extern "C" {

int gdn_version(void) { return 100; }

const char *gdn_last_error(void) { return g_msg; }

size_t gdn_chunk_fwd_workspace_size(int N, int T_tot, int H, int dk, int dv, gdn_dtype dtype) {
    if (dtype == GDN_BF16 && dk == 128 && dv == 128 && N >= 1 && H >= 1 && T_tot >= 0)
        // (the plan differs with and without cu_seqlens; the larger workspace covers both)
        return std::max({kErrWordBytes, gdn::chunk_ws_workspace(N, T_tot, H, gdn::chunk_ws_seg_chunks(N, T_tot, H, false)),
                         gdn::chunk_ws_workspace(N, T_tot, H, gdn::chunk_ws_seg_chunks(N, T_tot, H, true))});
    return kErrWordBytes;
}

static gdn_status chunk_fwd_impl(const void *q, const void *k, const void *v, const float *g, const float *beta,
                                 const float *S0, const int32_t *cu_seqlens, int N, int T_tot, int H, int dk, int dv,
                                 gdn_dtype dtype, void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream,
                                 bool raw) {
    gdn_status s = check_common(q, k, v, g, beta, o, T_tot, H, dk, dv, dtype);
    if (s != GDN_OK) return s;
    if (N < 1) return fail(GDN_ERR_SHAPE, "N=%d must be >= 1", N);
    if (!S_T) return fail(GDN_ERR_NULL, "S_T is required");
    if (misaligned(S0) || misaligned(S_T) || misaligned(cu_seqlens))
        return fail(GDN_ERR_ALIGN, "S0, S_T and cu_seqlens must be 16-byte aligned");
    if (!cu_seqlens && T_tot % N != 0)
        return fail(GDN_ERR_SEQLENS, "cu_seqlens is NULL and T_tot=%d is not a multiple of N=%d", T_tot, N);
    if (!workspace || ws_bytes < kErrWordBytes)
        return fail(GDN_ERR_WORKSPACE, "workspace of %zu bytes given, at least %zu needed", workspace ? ws_bytes : 0,
                    kErrWordBytes);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(GDN_ERR_ALIGN, "workspace must be 256-byte aligned");

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t *err = static_cast<uint32_t *>(workspace);
    cudaError_t e;
    if (dtype == GDN_BF16 && dk == 128) {
        const char *stage = "";
        // The pipelined path needs room for one prep record per (chunk, head) (and, split into
        // segments, the published segment states); with less workspace the single-kernel path runs.
        const int seg = gdn::chunk_ws_seg_chunks(N, T_tot, H, cu_seqlens != nullptr);
        const int use_seg = ws_bytes >= gdn::chunk_ws_workspace(N, T_tot, H, seg) ? seg : 0;
        if (ws_bytes >= gdn::chunk_ws_workspace(N, T_tot, H, use_seg)) {
            e = gdn::launch_chunk_ws(static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
                                     static_cast<const __nv_bfloat16 *>(v), g, beta, S0, cu_seqlens, N, T_tot, H,
                                     static_cast<__nv_bfloat16 *>(o), S_T, workspace, use_seg, st, &stage, raw);
            if (e != cudaSuccess) return cuda_fail(e, stage);
            return ok();
        }
        if (raw)
            return fail(GDN_ERR_WORKSPACE,
                        "raw inputs need the pipelined path: workspace of %zu bytes given, at least %zu needed",
                        ws_bytes, gdn::chunk_ws_workspace(N, T_tot, H, 0));
        e = gdn::launch_chunk_tc(static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
                                 static_cast<const __nv_bfloat16 *>(v), g, beta, S0, cu_seqlens, N, T_tot, H,
                                 static_cast<__nv_bfloat16 *>(o), S_T, workspace, ws_bytes, st, &stage);
        if (e != cudaSuccess) return cuda_fail(e, stage);
        return ok();
    }
    {
        ProfScope ps("validate_seqlens", st);
        e = gdn::launch_validate_seqlens(cu_seqlens, N, T_tot, err, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "cu_seqlens validation launch");
    ProfScope ps("chunk_simt", st);
    if (dtype == GDN_F32) {
        const float *qf = static_cast<const float *>(q), *kf = static_cast<const float *>(k),
                    *vf = static_cast<const float *>(v);
        float *of = static_cast<float *>(o);
        e = (dk == 64) ? gdn::launch_chunk_simt<float, 64>(qf, kf, vf, g, beta, S0, cu_seqlens, N, T_tot, H, of, S_T, err, st, raw)
                       : gdn::launch_chunk_simt<float, 128>(qf, kf, vf, g, beta, S0, cu_seqlens, N, T_tot, H, of, S_T, err, st, raw);
    } else {
        const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(q), *kb = static_cast<const __nv_bfloat16 *>(k),
                            *vb = static_cast<const __nv_bfloat16 *>(v);
        __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o);
        e = (dk == 64)
                ? gdn::launch_chunk_simt<__nv_bfloat16, 64>(qb, kb, vb, g, beta, S0, cu_seqlens, N, T_tot, H, ob, S_T, err, st, raw)
                : gdn::launch_chunk_simt<__nv_bfloat16, 128>(qb, kb, vb, g, beta, S0, cu_seqlens, N, T_tot, H, ob, S_T, err, st, raw);
    }
    if (e != cudaSuccess) return cuda_fail(e, "chunked forward launch");
    return ok();
}

gdn_status gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                         const float *S0, const int32_t *cu_seqlens, int N, int T_tot, int H, int dk, int dv,
                         gdn_dtype dtype, void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream) {
    return chunk_fwd_impl(q, k, v, g, beta, S0, cu_seqlens, N, T_tot, H, dk, dv, dtype, o, S_T, workspace, ws_bytes,
                          stream, false);
}

gdn_status gdn_chunk_fwd_raw(const void *q_raw, const void *k_raw, const void *v, const float *a, const float *b,
                             const float *S0, const int32_t *cu_seqlens, int N, int T_tot, int H, int dk, int dv,
                             gdn_dtype dtype, void *o, float *S_T, void *workspace, size_t ws_bytes, void *stream) {
    return chunk_fwd_impl(q_raw, k_raw, v, a, b, S0, cu_seqlens, N, T_tot, H, dk, dv, dtype, o, S_T, workspace,
                          ws_bytes, stream, true);
}

gdn_status gdn_chunk_fwd_check(const void *workspace, size_t ws_bytes, void *stream) {
    if (!workspace || ws_bytes < sizeof(uint32_t)) return fail(GDN_ERR_WORKSPACE, "workspace missing");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the error word, then (pipelined path) where the first timed-out wait was: the barrier's
    // shared-memory address + 1 or bit 30 + a flag's word offset, the block, the thread and parity
    uint32_t w[4] = {0, 0, 0, 0};
    const size_t n = ws_bytes >= sizeof(w) ? sizeof(w) : sizeof(uint32_t);
    cudaError_t e = cudaMemcpyAsync(w, workspace, n, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    const uint32_t word = w[0];
    if (word & gdn::ERRBIT_SEQLENS) return fail(GDN_ERR_SEQLENS, "cu_seqlens is not 0 = c0 <= c1 <= ... <= cN = T_tot");
    if (word & gdn::ERRBIT_TIMEOUT) {
        if (w[1] & (1u << 30))
            return fail(GDN_ERR_TIMEOUT, "a bounded device-side wait gave up (first: flag word %u, block (%u, %u), thread %u)",
                        w[1] & 0x3FFFFFFFu, w[2] & 0xFFFFu, w[2] >> 16, w[3] & 0xFFFFu);
        if (w[1])
            return fail(GDN_ERR_TIMEOUT,
                        "a bounded device-side wait gave up (first: mbarrier at shared address %u, parity %u, block "
                        "(%u, %u), thread %u)",
                        w[1] - 1u, w[3] >> 16, w[2] & 0xFFFFu, w[2] >> 16, w[3] & 0xFFFFu);
        return fail(GDN_ERR_TIMEOUT, "a bounded device-side wait gave up");
    }
    if (word & gdn::ERRBIT_INTERNAL) return fail(GDN_ERR_CUDA, "internal: misaligned shared-memory base, nothing written");
    if (word & gdn::ERRBIT_BOUNDS)
        return fail(GDN_ERR_BOUNDS, "a device-side index check failed (GDN_DEBUG_CHECKS build): an index into the "
                                    "workspace or an output was out of range and was redirected to 0");
    return ok();
}

static gdn_status decode_step_impl(const void *q, const void *k, const void *v, const float *g, const float *beta,
                                   float *S, int B, int H, int dk, int dv, gdn_dtype dtype, void *o, void *stream,
                                   bool raw) {
    if (B < 1) return fail(GDN_ERR_SHAPE, "B=%d must be >= 1", B);
    gdn_status s = check_common(q, k, v, g, beta, o, B, H, dk, dv, dtype);
    if (s != GDN_OK) return s;
    if (!S) return fail(GDN_ERR_NULL, "S is required");
    if (misaligned(S)) return fail(GDN_ERR_ALIGN, "S must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    ProfScope ps("decode_step", st);
    if (dtype == GDN_F32) {
        const float *qf = static_cast<const float *>(q), *kf = static_cast<const float *>(k),
                    *vf = static_cast<const float *>(v);
        float *of = static_cast<float *>(o);
        e = (dk == 64) ? gdn::launch_decode_step<float, 64>(qf, kf, vf, g, beta, S, B, H, of, st, raw)
                       : gdn::launch_decode_step<float, 128>(qf, kf, vf, g, beta, S, B, H, of, st, raw);
    } else {
        const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(q), *kb = static_cast<const __nv_bfloat16 *>(k),
                            *vb = static_cast<const __nv_bfloat16 *>(v);
        __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o);
        e = (dk == 64) ? gdn::launch_decode_step<__nv_bfloat16, 64>(qb, kb, vb, g, beta, S, B, H, ob, st, raw)
                       : gdn::launch_decode_step<__nv_bfloat16, 128>(qb, kb, vb, g, beta, S, B, H, ob, st, raw);
    }
    if (e != cudaSuccess) return cuda_fail(e, "decode step launch");
    return ok();
}

gdn_status gdn_decode_step(const void *q, const void *k, const void *v, const float *g, const float *beta, float *S,
                           int B, int H, int dk, int dv, gdn_dtype dtype, void *o, void *stream) {
    return decode_step_impl(q, k, v, g, beta, S, B, H, dk, dv, dtype, o, stream, false);
}

gdn_status gdn_decode_step_raw(const void *q_raw, const void *k_raw, const void *v, const float *a, const float *b,
                               float *S, int B, int H, int dk, int dv, gdn_dtype dtype, void *o, void *stream) {
    return decode_step_impl(q_raw, k_raw, v, a, b, S, B, H, dk, dv, dtype, o, stream, true);
}

gdn_status gdn_seq_scan(const void *q, const void *k, const void *v, const float *g, const float *beta,
                        const float *S0, const int32_t *cu_seqlens, int N, int T_tot, int H, int dk, int dv,
                        gdn_dtype dtype, void *o, float *S_T, void *stream) {
    gdn_status s = check_common(q, k, v, g, beta, o, T_tot, H, dk, dv, dtype);
    if (s != GDN_OK) return s;
    if (N < 1) return fail(GDN_ERR_SHAPE, "N=%d must be >= 1", N);
    if (!S_T) return fail(GDN_ERR_NULL, "S_T is required");
    if (misaligned(S0) || misaligned(S_T) || misaligned(cu_seqlens))
        return fail(GDN_ERR_ALIGN, "S0, S_T and cu_seqlens must be 16-byte aligned");
    if (!cu_seqlens && T_tot % N != 0)
        return fail(GDN_ERR_SEQLENS, "cu_seqlens is NULL and T_tot=%d is not a multiple of N=%d", T_tot, N);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    ProfScope ps("seq_scan", st);
    if (dtype == GDN_F32) {
        const float *qf = static_cast<const float *>(q), *kf = static_cast<const float *>(k),
                    *vf = static_cast<const float *>(v);
        float *of = static_cast<float *>(o);
        e = (dk == 64) ? gdn::launch_seq_scan<float, 64>(qf, kf, vf, g, beta, S0, cu_seqlens, N, T_tot, H, of, S_T, st)
                       : gdn::launch_seq_scan<float, 128>(qf, kf, vf, g, beta, S0, cu_seqlens, N, T_tot, H, of, S_T, st);
    } else {
        const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(q), *kb = static_cast<const __nv_bfloat16 *>(k),
                            *vb = static_cast<const __nv_bfloat16 *>(v);
        __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o);
        e = (dk == 64) ? gdn::launch_seq_scan<__nv_bfloat16, 64>(qb, kb, vb, g, beta, S0, cu_seqlens, N, T_tot, H, ob, S_T, st)
                       : gdn::launch_seq_scan<__nv_bfloat16, 128>(qb, kb, vb, g, beta, S0, cu_seqlens, N, T_tot, H, ob, S_T, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "sequential scan launch");
    return ok();
}

gdn_status gdn_proj_w8(const void *x, const int8_t *w, const float *scale, int T, int D, int H, int dk, int dv,
                       void *q_raw, void *k_raw, void *v, float *a, float *b, void *workspace, size_t ws_bytes,
                       void *stream) {
    if (T < 0 || D < 64 || D % 64 != 0 || H < 1 || dk < 1 || dv < 1 || (H * dk) % 8 != 0 || (H * dv) % 8 != 0)
        return fail(GDN_ERR_SHAPE, "T=%d D=%d H=%d dk=%d dv=%d unsupported (D a positive multiple of 64, H dk and "
                    "H dv multiples of 8)", T, D, H, dk, dv);
    if ((double)T * D >= 2.0e9 || (double)H * (2 * dk + dv) >= 1.0e6) return fail(GDN_ERR_SHAPE, "sizes overflow");
    if (T > 0 && (!x || !w || !scale || !q_raw || !k_raw || !v || !a || !b))
        return fail(GDN_ERR_NULL, "x, w, scale and every output are required");
    const void *p16[] = {x, w, scale, q_raw, k_raw, v};
    for (const void *p : p16)
        if (misaligned(p)) return fail(GDN_ERR_ALIGN, "pointer %p is not 16-byte aligned", p);
    if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 3u)
        return fail(GDN_ERR_ALIGN, "a and b must be 4-byte aligned");
    if (!workspace || ws_bytes < kErrWordBytes)
        return fail(GDN_ERR_WORKSPACE, "workspace of at least %zu bytes (the error word) needed", kErrWordBytes);
    const char *stage = "";
    const cudaError_t e = gdn::launch_proj_w8(
        static_cast<const __nv_bfloat16 *>(x), w, scale, T, D, H, dk, dv, static_cast<__nv_bfloat16 *>(q_raw),
        static_cast<__nv_bfloat16 *>(k_raw), static_cast<__nv_bfloat16 *>(v), a, b, static_cast<uint32_t *>(workspace),
        static_cast<cudaStream_t>(stream), &stage);
    if (e != cudaSuccess) return cuda_fail(e, stage);
    return ok();
}

gdn_status gdn_attn_fwd(const void *q, const void *k, const void *v, const int32_t *cu_seqlens, int N, int T_tot,
                        int H, int d, int max_len, float scale, gdn_dtype dtype, void *o, void *workspace,
                        size_t ws_bytes, void *stream) {
    if (dtype != GDN_BF16) return fail(GDN_ERR_DTYPE, "attention takes bf16 inputs only");
    if (d != 128) return fail(GDN_ERR_SHAPE, "attention head size d=%d unsupported (128)", d);
    if (N < 1 || H < 1 || T_tot < 0) return fail(GDN_ERR_SHAPE, "N=%d H=%d T=%d out of range", N, H, T_tot);
    if (!cu_seqlens && T_tot % N != 0)
        return fail(GDN_ERR_SEQLENS, "cu_seqlens is NULL and T_tot=%d is not a multiple of N=%d", T_tot, N);
    if (!cu_seqlens) max_len = T_tot / N;
    if (max_len < 0 || max_len > T_tot) return fail(GDN_ERR_SHAPE, "max_len=%d outside 0 .. T_tot", max_len);
    if ((double)T_tot * H * d >= 9.0e18 || (double)((max_len + 127) / 128) * H * N >= 2.0e9)
        return fail(GDN_ERR_SHAPE, "sizes overflow");
    if (T_tot > 0 && (!q || !k || !v || !o)) return fail(GDN_ERR_NULL, "q, k, v and o are required");
    const void *ptrs[] = {q, k, v, o, cu_seqlens};
    for (const void *p : ptrs)
        if (misaligned(p)) return fail(GDN_ERR_ALIGN, "pointer %p is not 16-byte aligned", p);
    if (!workspace || ws_bytes < kErrWordBytes)
        return fail(GDN_ERR_WORKSPACE, "workspace of at least %zu bytes (the error word) needed", kErrWordBytes);
    if (!(scale > 0.f)) scale = 1.f / sqrtf((float)d);
    const char *stage = "";
    const cudaError_t e = gdn::launch_attn_fwd(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), cu_seqlens, N, T_tot, H, max_len, scale,
        static_cast<__nv_bfloat16 *>(o), static_cast<uint32_t *>(workspace), static_cast<cudaStream_t>(stream), &stage);
    if (e != cudaSuccess) return cuda_fail(e, stage);
    return ok();
}

gdn_status gdn_debug_inject(int kind, unsigned wait_us) {
    if (kind != GDN_INJECT_NONE && kind != GDN_INJECT_WITHHOLD_LINK)
        return fail(GDN_ERR_SHAPE, "unknown injection kind %d", kind);
    if (kind != GDN_INJECT_NONE && (wait_us == 0 || wait_us > 1000000u))
        return fail(GDN_ERR_SHAPE, "wait_us=%u outside 1 .. 1000000", wait_us);
    gdn::g_inject_wait_ns.store((unsigned long long)wait_us * 1000ull);
    gdn::g_inject_kind.store(kind);
    return ok();
}

void gdn_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    g_prof.on = on != 0;
}

int gdn_profile_read(char *names, size_t names_len, float *ms, int *counts, int max_kernels) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    std::vector<std::string> keys;
    std::vector<float> tot;
    std::vector<int> cnt;
    for (const ProfRec &r : g_prof.recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
            t = -1.f;
        size_t i = 0;
        while (i < keys.size() && keys[i] != r.name) ++i;
        if (i == keys.size()) {
            keys.push_back(r.name);
            tot.push_back(0.f);
            cnt.push_back(0);
        }
        tot[i] += t;
        cnt[i] += 1;
        g_prof.pool.push_back(r.start);
        g_prof.pool.push_back(r.stop);
    }
    g_prof.recs.clear();
    std::string joined;
    int n = 0;
    for (size_t i = 0; i < keys.size() && n < max_kernels; ++i, ++n) {
        if (ms) ms[n] = tot[i];
        if (counts) counts[n] = cnt[i];
        joined += keys[i];
        joined += '\n';
    }
    if (names && names_len) {
        strncpy(names, joined.c_str(), names_len - 1);
        names[names_len - 1] = '\0';
    }
    return n;
}

}  // extern "C"
