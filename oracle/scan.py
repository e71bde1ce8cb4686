"""ctypes wrapper around the fp64 sequential-scan oracle (``gdn_scan.c``).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The recurrence, per sequence and head (gated delta rule; the pages name it as
the recurrent layer of a "hybrid gated-delta-net backbone" and its
token-by-token "sequential scan", page 1 abstract result (i) and page 2
"Resumen Tecnico" / "Capas Recurrentes")::

    S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gdn_oracle_scan_f64.restype = ctypes.c_int
        lib.gdn_oracle_scan_f64.argtypes = [dp, dp, dp, dp, dp, dp,
                                            ctypes.POINTER(ctypes.c_int64),
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            dp, dp]
        lib.gdn_oracle_num_threads.restype = ctypes.c_int
        lib.gdn_oracle_set_num_threads.argtypes = [ctypes.c_int]
        _LIB = lib
    return _LIB


def as_f64(x):
    """Exact upcast of a CPU tensor / array (bf16, fp32, fp64) to a contiguous fp64 ndarray."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    """OpenMP threads the scan runs on."""
    return int(_lib().gdn_oracle_num_threads())


def set_num_threads(n: int) -> None:
    _lib().gdn_oracle_set_num_threads(int(n))


def scan(q, k, v, g, beta, S0=None, cu_seqlens=None, N=None):
    """fp64 sequential scan over packed sequences.

    q, k: [T_tot, H, dk]; v: [T_tot, H, dv]; g, beta: [T_tot, H] (natural-log
    decay g, alpha = exp(g)); S0: [N, H, dv, dk] or None (zero state);
    cu_seqlens: [N+1] offsets or None (then N equal sequences, N taken from
    ``N``, else from S0, else 1). Returns (o [T_tot, H, dv], S_T [N, H, dv, dk]),
    both fp64.
    """
    q, k, v, g, beta, S0 = (as_f64(x) for x in (q, k, v, g, beta, S0))
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        if N is None:
            N = S0.shape[0] if S0 is not None else 1
        if T_tot % N:
            raise ValueError("T_tot not divisible by N")
        cu = np.arange(N + 1, dtype=np.int64) * (T_tot // N)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
        N = cu.shape[0] - 1
    if cu[-1] != T_tot:
        raise ValueError("cu_seqlens[N] != T_tot")
    if S0 is not None and S0.shape != (N, H, dv, dk):
        raise ValueError("S0 shape %r != %r" % (S0.shape, (N, H, dv, dk)))
    if k.shape != q.shape or v.shape[:2] != (T_tot, H) or g.shape != (T_tot, H) or beta.shape != (T_tot, H):
        raise ValueError("inconsistent input shapes")
    o = np.zeros((T_tot, H, dv), dtype=np.float64)
    S_T = np.zeros((N, H, dv, dk), dtype=np.float64)
    rc = _lib().gdn_oracle_scan_f64(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
        _ptr(S0) if S0 is not None else None,
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        N, H, dk, dv, _ptr(o), _ptr(S_T))
    if rc != 0:
        raise RuntimeError("oracle scan failed with code %d" % rc)
    return o, S_T


def decode_step(q, k, v, g, beta, S):
    """One single-token state update per sequence: q,k [B,H,dk], v [B,H,dv],
    g,beta [B,H], S [B,H,dv,dk]. Returns (o [B,H,dv], S_new [B,H,dv,dk]) in fp64.
    It is the scan applied to B sequences of length one."""
    S = as_f64(S)
    B = S.shape[0]
    return scan(q, k, v, g, beta, S0=S, cu_seqlens=np.arange(B + 1, dtype=np.int64))
