"""Oracle for the hybrid backbone's causal attention layer.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages' backbone interleaves the recurrent layers with causal attention layers, whose
O(N^2) kernel made prefill collapse at long context until it was rewritten as per-head GEMMs
(page 1, abstract: 17x faster prefill at 10k; page 2, "Resumen Tecnico", the attention
rewrite). The pages do not write the attention out; the plain reading is standard scaled
dot-product attention with a causal mask, per head h and query position t:

    s_tj = (q_t . k_j) * scale            for j <= t      (scale = 1 / sqrt(d) by default)
    p_tj = exp(s_tj - max_j s_tj) / sum_j exp(s_tj - max_j s_tj)
    o_t  = sum_{j <= t} p_tj v_j

computed here in fp64 over packed sequences (a query attends to the keys of its own sequence
at positions <= its own). Subtracting the row maximum does not change p; it only keeps exp in
range.
"""
from __future__ import annotations

import numpy as np

from .scan import as_f64


def causal_attention(q, k, v, scale=None, cu_seqlens=None, rows=None):
    """q, k [T, H, d], v [T, H, dv] -> o [T, H, dv] fp64. cu_seqlens [N+1] packs sequences (None:
    one sequence). rows: optional list of query positions to compute (others left zero)."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    T, H, d = q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(
        cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64)
    o = np.zeros((T, H, v.shape[2]))
    wanted = None if rows is None else set(int(r) for r in rows)
    for n in range(len(cu) - 1):
        a, b = int(cu[n]), int(cu[n + 1])
        for t in range(a, b):
            if wanted is not None and t not in wanted:
                continue
            for h in range(H):
                s = (k[a:t + 1, h] @ q[t, h]) * scale
                p = np.exp(s - s.max())
                o[t, h] = (p / p.sum()) @ v[a:t + 1, h]
    return o
