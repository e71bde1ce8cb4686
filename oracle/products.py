"""Second formulation of the gated delta rule: explicit transition-matrix products.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

With M_t = alpha_t (I - beta_t k_t k_t^T) (dk x dk), the recurrence
S_t = S_{t-1} M_t + beta_t v_t k_t^T unrolls to

    S_t = S_0 M_1 ... M_t + sum_{j<=t} beta_j v_j k_j^T M_{j+1} ... M_t,   o_t = S_t q_t.

This module builds every M_t and every suffix product explicitly (numpy
matmul as the only library step). It is O(T^2 dk^3) and meant for small T; it
shares no code with the sequential scan and pins it (they must agree to
rounding).
"""
from __future__ import annotations

import numpy as np

from .scan import as_f64


def transition_products(q, k, v, g, beta, S0=None):
    """Single sequence: q,k [T,H,dk], v [T,H,dv], g,beta [T,H], S0 [H,dv,dk] or None.
    Returns (o [T,H,dv], S_T [H,dv,dk]) in fp64."""
    q, k, v, g, beta = (as_f64(x) for x in (q, k, v, g, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    S0 = np.zeros((H, dv, dk)) if S0 is None else as_f64(S0).reshape(H, dv, dk)
    I = np.eye(dk)
    o = np.zeros((T, H, dv))
    S_T = np.zeros((H, dv, dk))
    for h in range(H):
        M = [np.exp(g[t, h]) * (I - beta[t, h] * np.outer(k[t, h], k[t, h])) for t in range(T)]
        for t in range(T):
            # R[j] = M_{j+1} ... M_t  (0-based: tokens j+1..t), built from the right.
            R = I.copy()
            S_t = np.zeros((dv, dk))
            for j in range(t, -1, -1):
                # term of token j uses the product of the transitions after it
                S_t += beta[j, h] * np.outer(v[j, h], k[j, h]) @ R
                R = M[j] @ R
            S_t += S0[h] @ R  # R is now M_0 ... M_t
            o[t, h] = S_t @ q[t, h]
            if t == T - 1:
                S_T[h] = S_t
        if T == 0:
            S_T[h] = S0[h]
    return o, S_T
