"""ctypes binding of ``libgdn_b200.so`` (declared in ``include/gdn.h``).

Argument marshalling only: torch tensors become device pointers, sizes and
the current CUDA stream; every step of the computation runs in the library's
kernels. There is no CPU fallback: if the library is missing or a tensor is
not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# GDN_DEBUG_CHECKS=1 in the environment selects the index-checking build (see build.py --debug)
_LIB_PATH = os.path.join(_HERE, "libgdn_b200_debug.so" if os.environ.get("GDN_DEBUG_CHECKS") == "1"
                         else "libgdn_b200.so")
_lib = None

GDN_F32, GDN_BF16 = 0, 1
_DTYPE = {torch.float32: GDN_F32, torch.bfloat16: GDN_BF16}
STATUS = {0: "GDN_OK", 1: "GDN_ERR_NULL", 2: "GDN_ERR_SHAPE", 3: "GDN_ERR_DTYPE", 4: "GDN_ERR_ALIGN",
          5: "GDN_ERR_SEQLENS", 6: "GDN_ERR_WORKSPACE", 7: "GDN_ERR_CUDA", 8: "GDN_ERR_TIMEOUT",
          9: "GDN_ERR_BOUNDS"}

# Every symbol include/gdn.h declares, with its ctypes signature.
_VP, _SZ, _I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
SIGNATURES = {
    "gdn_version": (_I, []),
    "gdn_last_error": (ctypes.c_char_p, []),
    "gdn_chunk_fwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "gdn_chunk_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP, _VP, _VP, _SZ, _VP]),
    "gdn_chunk_fwd_raw": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP, _VP, _VP, _SZ, _VP]),
    "gdn_decode_step_raw": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _VP, _VP]),
    "gdn_chunk_fwd_check": (_I, [_VP, _SZ, _VP]),
    "gdn_attn_fwd": (_I, [_VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, ctypes.c_float, _I, _VP, _VP, _SZ, _VP]),
    "gdn_proj_w8": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "gdn_decode_step": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _VP, _VP]),
    "gdn_seq_scan": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP, _VP, _VP]),
    "gdn_diag_mma_tile": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP]),
    "gdn_diag_ut_solve": (_I, [_VP, _VP, _VP]),
    "gdn_chunk_fwd_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP, _VP, _VP]),
    "gdn_debug_inject": (_I, [_I, ctypes.c_uint]),
    "gdn_profile_enable": (None, [_I]),
    "gdn_profile_read": (_I, [ctypes.c_char_p, _SZ, _VP, _VP, _I]),
}


class GdnError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s: %s" % (STATUS.get(status, str(status)), msg))
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load (once) and return the ctypes handle; raises if the library was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise GdnError(-1, "CUDA library %s not built (run python -m "
                           "linear_attention_recurrent_chunked_b200.build)" % _LIB_PATH)
        lib = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(status: int):
    if status != 0:
        raise GdnError(status, load_library().gdn_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise GdnError(1, "tensors must be on a CUDA device (no CPU path)")
            if not t.is_contiguous():
                raise GdnError(2, "tensors must be contiguous")


def chunk_fwd_workspace_size(N: int, T_tot: int, H: int, dk: int, dv: int, dtype: torch.dtype) -> int:
    return int(load_library().gdn_chunk_fwd_workspace_size(N, T_tot, H, dk, dv, _DTYPE[dtype]))


_ws_cache = {}


def _workspace(nbytes: int, device) -> torch.Tensor:
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, N: Optional[int] = None, o=None, S_T=None,
              workspace=None, check: bool = False):
    """Chunked prefill. q,k [T,H,dk], v [T,H,dv] (fp32 or bf16); g,beta [T,H] fp32;
    S0 [N,H,dv,dk] fp32 or None; cu_seqlens [N+1] int32 (device) or None (then N
    equal sequences, N from ``N``, S0, else 1). Returns (o, S_T). With
    check=True the stream is synchronised and the device error word read."""
    lib = load_library()
    _need_cuda(q, k, v, g, beta, S0, cu_seqlens, o, S_T, workspace)
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
    elif N is None:
        N = S0.shape[0] if S0 is not None else 1
    if o is None:
        o = torch.empty((T_tot, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((N, H, dv, dk), dtype=torch.float32, device=q.device)
    dt = _DTYPE.get(q.dtype, 99)
    need = int(lib.gdn_chunk_fwd_workspace_size(N, T_tot, H, dk, dv, dt))
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check(lib.gdn_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                             N, T_tot, H, dk, dv, dt, _ptr(o), _ptr(S_T), _ptr(ws), ws.numel(), _stream()))
    if check:
        _check(lib.gdn_chunk_fwd_check(_ptr(ws), ws.numel(), _stream()))
    return o, S_T


def chunk_fwd_raw(q_raw, k_raw, v, a, b, S0=None, cu_seqlens=None, N: Optional[int] = None, o=None, S_T=None,
                  workspace=None, check: bool = False):
    """Chunked prefill from raw inputs (see include/gdn.h): q_raw, k_raw [T,H,dk] of any norm,
    v [T,H,dv]; a, b [T,H] fp32 gate logits (g = -softplus(a), beta = sigmoid(b)); the rest as
    chunk_fwd. The normalisation and gates run inside the library's kernels."""
    lib = load_library()
    _need_cuda(q_raw, k_raw, v, a, b, S0, cu_seqlens, o, S_T, workspace)
    T_tot, H, dk = q_raw.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
    elif N is None:
        N = S0.shape[0] if S0 is not None else 1
    if o is None:
        o = torch.empty((T_tot, H, dv), dtype=q_raw.dtype, device=q_raw.device)
    if S_T is None:
        S_T = torch.empty((N, H, dv, dk), dtype=torch.float32, device=q_raw.device)
    dt = _DTYPE.get(q_raw.dtype, 99)
    need = int(lib.gdn_chunk_fwd_workspace_size(N, T_tot, H, dk, dv, dt))
    ws = workspace if workspace is not None else _workspace(need, q_raw.device)
    _check(lib.gdn_chunk_fwd_raw(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a), _ptr(b), _ptr(S0), _ptr(cu_seqlens),
                                 N, T_tot, H, dk, dv, dt, _ptr(o), _ptr(S_T), _ptr(ws), ws.numel(), _stream()))
    if check:
        _check(lib.gdn_chunk_fwd_check(_ptr(ws), ws.numel(), _stream()))
    return o, S_T


def decode_step_raw(q_raw, k_raw, v, a, b, S, o=None):
    """One decode step from raw inputs (q, k normalised and gates applied in the kernel)."""
    lib = load_library()
    _need_cuda(q_raw, k_raw, v, a, b, S, o)
    B, H, dk = q_raw.shape
    dv = v.shape[2]
    if o is None:
        o = torch.empty((B, H, dv), dtype=q_raw.dtype, device=q_raw.device)
    _check(lib.gdn_decode_step_raw(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a), _ptr(b), _ptr(S), B, H, dk, dv,
                                   _DTYPE.get(q_raw.dtype, 99), _ptr(o), _stream()))
    return o


def proj_w8(x, w, scale, H: int, dk: int, dv: int, out=None, workspace=None, check: bool = False):
    """Input projection with int8 weights (see include/gdn.h): x [T, D] bf16, w [N, D] int8,
    scale [N] fp32, N = H (2 dk + dv) + 2 H. Returns (q_raw [T,H,dk], k_raw [T,H,dk], v [T,H,dv]
    bf16, a [T,H], b [T,H] fp32); ``out`` may pass those five tensors to write into."""
    lib = load_library()
    _need_cuda(x, w, scale, workspace)
    T, D = x.shape
    dev = x.device
    if out is None:
        out = (torch.empty((T, H, dk), dtype=torch.bfloat16, device=dev),
               torch.empty((T, H, dk), dtype=torch.bfloat16, device=dev),
               torch.empty((T, H, dv), dtype=torch.bfloat16, device=dev),
               torch.empty((T, H), dtype=torch.float32, device=dev),
               torch.empty((T, H), dtype=torch.float32, device=dev))
    _need_cuda(*out)
    ws = workspace if workspace is not None else _workspace(256, dev)
    _check(lib.gdn_proj_w8(_ptr(x), _ptr(w), _ptr(scale), T, D, H, dk, dv, *[_ptr(t) for t in out], _ptr(ws),
                           ws.numel(), _stream()))
    if check:
        _check(lib.gdn_chunk_fwd_check(_ptr(ws), ws.numel(), _stream()))
    return out


def attn_fwd(q, k, v, cu_seqlens=None, N: Optional[int] = None, max_len: Optional[int] = None,
             scale: float = 0.0, o=None, workspace=None, check: bool = False):
    """Causal attention (see include/gdn.h): q, k, v [T, H, 128] bf16; cu_seqlens [N+1] int32
    (device) or None (N equal sequences, N from ``N``, else 1); max_len bounds the sequence
    lengths (required with cu_seqlens); scale <= 0 means 1 / sqrt(128). Returns o [T, H, 128]."""
    lib = load_library()
    _need_cuda(q, k, v, cu_seqlens, o, workspace)
    T_tot, H, d = q.shape
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
        if max_len is None:
            raise GdnError(2, "max_len is required with cu_seqlens")
    else:
        N = 1 if N is None else N
        max_len = T_tot // N
    if o is None:
        o = torch.empty_like(q)
    ws = workspace if workspace is not None else _workspace(256, q.device)
    _check(lib.gdn_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), N, T_tot, H, d, max_len, float(scale),
                            _DTYPE.get(q.dtype, 99), _ptr(o), _ptr(ws), ws.numel(), _stream()))
    if check:
        _check(lib.gdn_chunk_fwd_check(_ptr(ws), ws.numel(), _stream()))
    return o


def chunk_fwd_noalloc(q, k, v, g, beta, S0=None, cu_seqlens=None, N: Optional[int] = None, o=None, S_T=None):
    """chunk_fwd without a workspace argument: the library's built-in scratch
    array is used instead (see include/gdn.h). o and S_T are allocated here
    only when the caller does not pass them."""
    lib = load_library()
    _need_cuda(q, k, v, g, beta, S0, cu_seqlens, o, S_T)
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
    elif N is None:
        N = S0.shape[0] if S0 is not None else 1
    if o is None:
        o = torch.empty((T_tot, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((N, H, dv, dk), dtype=torch.float32, device=q.device)
    _check(lib.gdn_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                                     N, T_tot, H, dk, dv, _DTYPE.get(q.dtype, 99), _ptr(o), _ptr(S_T), _stream()))
    return o, S_T


def decode_step(q, k, v, g, beta, S, o=None):
    """One decode step for B sequences: q,k [B,H,dk], v [B,H,dv], g,beta [B,H],
    S [B,H,dv,dk] fp32 updated in place. Returns o [B,H,dv]."""
    lib = load_library()
    _need_cuda(q, k, v, g, beta, S, o)
    B, H, dk = q.shape
    dv = v.shape[2]
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check(lib.gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), B, H, dk, dv,
                               _DTYPE.get(q.dtype, 99), _ptr(o), _stream()))
    return o


def seq_scan(q, k, v, g, beta, S0=None, cu_seqlens=None, N: Optional[int] = None, o=None, S_T=None):
    """Token-by-token scan on the GPU (comparator). Same arguments as chunk_fwd."""
    lib = load_library()
    _need_cuda(q, k, v, g, beta, S0, cu_seqlens, o, S_T)
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
    elif N is None:
        N = S0.shape[0] if S0 is not None else 1
    if o is None:
        o = torch.empty((T_tot, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((N, H, dv, dk), dtype=torch.float32, device=q.device)
    _check(lib.gdn_seq_scan(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                            N, T_tot, H, dk, dv, _DTYPE.get(q.dtype, 99), _ptr(o), _ptr(S_T), _stream()))
    return o, S_T


def diag_mma_tile(A, B, a_mn: int = 0, b_mn: int = 0, variant: int = 0):
    """Diagnostic single tensor-core tile: returns the [128, N] TMEM dump of
    A [M,K] @ B [N,K]^T (bf16 in, fp32 out). See include/gdn.h."""
    lib = load_library()
    _need_cuda(A, B)
    M, K = A.shape
    N = B.shape[0]
    D = torch.full((128, N), float("nan"), dtype=torch.float32, device=A.device)
    _check(lib.gdn_diag_mma_tile(_ptr(A), _ptr(B), _ptr(D), M, N, K, a_mn, b_mn, variant, _stream()))
    return D


def debug_inject(kind: int, wait_us: int = 0) -> None:
    """Failure injection for tests (see include/gdn.h): 0 = off, 1 = withhold the first
    segment's end state of head 0 so that the blocks waiting for it time out after wait_us."""
    _check(load_library().gdn_debug_inject(kind, wait_us))


def profile_enable(on: bool = True) -> None:
    """Record CUDA events around every kernel the library launches (see include/gdn.h)."""
    load_library().gdn_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """{kernel name: (total ms, launches)} since the last read; waits for the recorded events."""
    lib = load_library()
    n_max = 64
    names = ctypes.create_string_buffer(8192)
    ms = (ctypes.c_float * n_max)()
    cnt = (ctypes.c_int * n_max)()
    n = lib.gdn_profile_read(names, 8192, ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(cnt, ctypes.c_void_p), n_max)
    keys = names.value.decode().split("\n")[:n]
    return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(keys)}


def diag_ut_solve(A):
    """Diagnostic: the chunked path's (I + A)^{-1} for one strictly lower 64 x 64 fp32 matrix."""
    lib = load_library()
    _need_cuda(A)
    T = torch.full((64, 64), float("nan"), dtype=torch.float32, device=A.device)
    _check(lib.gdn_diag_ut_solve(_ptr(A), _ptr(T), _stream()))
    return T
