"""Third formulation: the chunked (intra-/inter-chunk) form, fp64, with stage dumps.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). It is a stage reference,
not the oracle: it must equal the sequential scan to rounding, which pins the
algebra below, and its per-stage dumps give the GPU kernels something to be
checked against stage by stage (the pages' "stage-validated" method: every
stage compared with a locally generated reference, page 1 abstract result (ii),
page 2 "Metodologia", "Portabilidad Validada por Etapas").

The pages name the rewrite only: the token-by-token scan becomes a chunked
delta-rule form with intra- and inter-chunk parts and a forward-substitution
step (page 1 abstract result (i); page 2 "Capas Recurrentes"). The algebra is
derived here from the recurrence. Inside one chunk (positions r, s = 1..C,
S_0 the state entering the chunk, all exponents <= 0):

    G_r = sum_{s<=r} g_s,   gamma_r = exp(G_r),   Gamma_rs = exp(G_r - G_s)
    A_rs = beta_r Gamma_rs (k_r . k_s)      for s <  r, else 0
    P_rs = Gamma_rs (q_r . k_s)             for s <= r, else 0
    T    = (I + A)^{-1}                     (unit lower triangular)
    W    = T diag(beta * gamma) K,   U = T diag(beta) V
    Delta = U - W S_0^T                     (row r = delta_r, the rank-1 write of token r)
    O     = diag(gamma) Q S_0^T + P Delta
    S_C   = gamma_C S_0 + Delta^T diag(exp(G_C - G_s)) K

Derivation: write S_r = alpha_r S_{r-1} + delta_r k_r^T with
delta_r = beta_r (v_r - alpha_r S_{r-1} k_r); unrolling gives
S_r = gamma_r S_0 + sum_{s<=r} Gamma_rs delta_s k_s^T; substituting into delta
gives (I + A) Delta = diag(beta) V - diag(beta gamma) K S_0^T; o_r = S_r q_r and
S_C follow.
"""
from __future__ import annotations

import numpy as np

from .scan import as_f64


def _forward_substitution(A):
    """T = (I + A)^{-1} for strictly lower-triangular A, row by row:
    T_r = e_r - sum_{s<r} A_rs T_s."""
    C = A.shape[0]
    T = np.zeros_like(A)
    for r in range(C):
        T[r] = -A[r, :r] @ T[:r] if r else 0.0
        T[r, r] = 1.0
    return T


def chunk_step(Qc, Kc, Vc, gc, bc, S0):
    """One chunk of one head. Qc,Kc [L,dk], Vc [L,dv], gc,bc [L], S0 [dv,dk].
    Returns (O [L,dv], S_C [dv,dk], dump dict)."""
    L = Kc.shape[0]
    G = np.cumsum(gc)
    gamma = np.exp(G)
    r = np.arange(L)
    lower_strict = r[:, None] > r[None, :]
    lower = r[:, None] >= r[None, :]
    # Gamma_rs = exp(G_r - G_s) only where s <= r (exponent <= 0 there).
    Gam = np.where(lower, np.exp(np.where(lower, G[:, None] - G[None, :], 0.0)), 0.0)
    A = np.where(lower_strict, bc[:, None] * Gam * (Kc @ Kc.T), 0.0)
    P = np.where(lower, Gam * (Qc @ Kc.T), 0.0)
    T = _forward_substitution(A)
    W = T @ ((bc * gamma)[:, None] * Kc)
    U = T @ (bc[:, None] * Vc)
    Delta = U - W @ S0.T
    O = gamma[:, None] * (Qc @ S0.T) + P @ Delta
    decay_to_end = np.exp(G[-1] - G) if L else np.zeros(0)
    S_C = (gamma[-1] if L else 1.0) * S0 + Delta.T @ (decay_to_end[:, None] * Kc)
    dump = dict(G=G, A=A, P=P, T=T, W=W, U=U, Delta=Delta, S0=S0.copy())
    return O, S_C, dump


def chunked(q, k, v, g, beta, S0=None, cu_seqlens=None, chunk=64, dump=False):
    """Chunked forward over packed sequences. Same arguments and results as
    ``oracle.scan``; chunks restart at every sequence start and the last chunk
    of a sequence may be partial. With dump=True also returns a list, per
    (n, h), of the per-chunk stage dictionaries."""
    q, k, v, g, beta, S0 = (as_f64(x) for x in (q, k, v, g, beta, S0))
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        N = S0.shape[0] if S0 is not None else 1
        cu = np.arange(N + 1) * (T_tot // N)
    else:
        cu = np.asarray(cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64)
        N = len(cu) - 1
    o = np.zeros((T_tot, H, dv))
    S_T = np.zeros((N, H, dv, dk))
    dumps = {}
    for n in range(N):
        for h in range(H):
            S = np.zeros((dv, dk)) if S0 is None else S0[n, h].copy()
            stages = []
            for c0 in range(int(cu[n]), int(cu[n + 1]), chunk):
                c1 = min(c0 + chunk, int(cu[n + 1]))
                O, S, d = chunk_step(q[c0:c1, h], k[c0:c1, h], v[c0:c1, h], g[c0:c1, h], beta[c0:c1, h], S)
                o[c0:c1, h] = O
                if dump:
                    stages.append(d)
            S_T[n, h] = S
            if dump:
                dumps[(n, h)] = stages
    return (o, S_T, dumps) if dump else (o, S_T)
