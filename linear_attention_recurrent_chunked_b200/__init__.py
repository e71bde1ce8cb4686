"""Gated-delta-rule forward (chunked prefill + single-token decode) for NVIDIA B200.

The compute lives in a C-ABI shared library of hand-written sm_100a CUDA
kernels (``csrc/``, declared in ``include/gdn.h``); ``gdn`` is a thin ctypes
binding that only marshals torch tensors into pointers and the current CUDA
stream. There is no CPU fallback: calling into the binding without the built
library raises.

Public API (loaded lazily so that ``workloads`` can be imported on machines
without the library)::

    chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, o=None, S_T=None) -> (o, S_T)
    decode_step(q, k, v, g, beta, S, o=None) -> o           # S updated in place
    seq_scan(q, k, v, g, beta, S0=None, cu_seqlens=None) -> (o, S_T)
"""
_EXPORTS = ("chunk_fwd", "decode_step", "seq_scan", "chunk_fwd_workspace_size", "library_path",
            "GdnError", "load_library")


def __getattr__(name):
    if name in _EXPORTS:
        from . import gdn
        return getattr(gdn, name)
    raise AttributeError(name)


__all__ = list(_EXPORTS)
