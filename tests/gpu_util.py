"""Helpers for the GPU parity tests: move seeded CPU inputs to the device and
compare GPU results with the oracle (fp64) by the library's error measure
max|x_gpu - x_ref| / max|x_ref|, computed separately for o and for S_T."""
import numpy as np
import torch

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(x_gpu, x_ref) -> float:
    a = x_gpu.detach().double().cpu().numpy() if hasattr(x_gpu, "detach") else np.asarray(x_gpu, dtype=np.float64)
    b = np.asarray(x_ref, dtype=np.float64)
    den = float(np.max(np.abs(b))) if b.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(a))) if a.size else 0.0
    return float(np.max(np.abs(a - b)) / den)


def to_dev(w, keys=("q", "k", "v", "g", "beta", "S0", "cu_seqlens", "S")):
    out = dict(w)
    for key in keys:
        if out.get(key) is not None:
            out[key] = out[key].cuda()
    return out
