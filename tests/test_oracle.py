"""Pins for the oracle (CPU only).

The oracle is checked against things other than itself: a second and a third
formulation written independently, a hand-derived golden example, the
invariants and closed forms the gated delta rule fixes, a norm bound, a 2x2
brute force written from the matrix form, and mutation tests showing that
plausible mistakes (dropped term, wrong index, transposed operand) fail these
pins.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle.chunked import _forward_substitution

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel_err(a, b):
    a, b = np.asarray(a), np.asarray(b)
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def random_case(rng, T, H, dk, dv, s0=True, slow=False):
    q = unit_rows(rng.standard_normal((T, H, dk)))
    k = unit_rows(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    if slow:
        g = -0.01 * rng.random((T, H))
        beta = 1.0 / (1.0 + np.exp(-(rng.standard_normal((T, H)) + 3.0)))
    else:
        g = -np.log1p(np.exp(rng.standard_normal((T, H))))  # -softplus
        beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    S0 = 0.3 * rng.standard_normal((1, H, dv, dk)) if s0 else None
    return q, k, v, g, beta, S0


# ---------------------------------------------------------------- (i) formulations agree

@pytest.mark.parametrize("T,dk,dv", [(1, 8, 8), (5, 8, 6), (16, 6, 10), (16, 16, 16)])
def test_scan_equals_transition_products(T, dk, dv):
    rng = np.random.default_rng(100 + T + dk)
    q, k, v, g, beta, S0 = random_case(rng, T, 2, dk, dv)
    o1, S1 = oracle.scan(q, k, v, g, beta, S0=S0)
    o2, S2 = oracle.transition_products(q, k, v, g, beta, S0=S0[0])
    assert rel_err(o1, o2) < 1e-12
    assert rel_err(S1[0], S2) < 1e-12


@pytest.mark.parametrize("seqlens,chunk,dk,dv", [
    ([256], 64, 64, 64),          # tiny workload shape
    ([100], 16, 12, 20),          # ragged last chunk, dk != dv
    ([37, 0, 64, 129, 1], 32, 16, 8),  # packed, empty and one-token sequences
])
def test_scan_equals_chunked(seqlens, chunk, dk, dv):
    rng = np.random.default_rng(sum(seqlens) + chunk)
    T = sum(seqlens)
    q, k, v, g, beta, _ = random_case(rng, T, 2, dk, dv, s0=False)
    N = len(seqlens)
    S0 = 0.3 * rng.standard_normal((N, 2, dv, dk))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int64)
    o1, S1 = oracle.scan(q, k, v, g, beta, S0=S0, cu_seqlens=cu)
    o2, S2 = oracle.chunked(q, k, v, g, beta, S0=S0, cu_seqlens=cu, chunk=chunk)
    assert rel_err(o1, o2) < 1e-11
    assert rel_err(S1, S2) < 1e-11
    # empty sequence: S_T = S0
    for n, L in enumerate(seqlens):
        if L == 0:
            assert np.array_equal(S1[n], S0[n])


def test_chunked_slow_decay_long():
    """Slow decay and beta near one: the state carries over many chunks."""
    rng = np.random.default_rng(7)
    q, k, v, g, beta, S0 = random_case(rng, 700, 1, 16, 16, slow=True)
    o1, S1 = oracle.scan(q, k, v, g, beta, S0=S0)
    o2, S2 = oracle.chunked(q, k, v, g, beta, S0=S0, chunk=64)
    assert rel_err(o1, o2) < 1e-10
    assert rel_err(S1, S2) < 1e-10


def test_forward_substitution_is_the_inverse():
    rng = np.random.default_rng(3)
    A = np.tril(rng.standard_normal((64, 64)) * 0.3, -1)
    T = _forward_substitution(A)
    assert np.allclose(T, np.linalg.inv(np.eye(64) + A), rtol=0, atol=1e-10)
    assert np.allclose(np.triu(T, 1), 0) and np.allclose(np.diag(T), 1)


def test_chunk_size_independent():
    rng = np.random.default_rng(11)
    q, k, v, g, beta, S0 = random_case(rng, 200, 1, 8, 8)
    ref = oracle.chunked(q, k, v, g, beta, S0=S0, chunk=64)
    for c in (1, 7, 32, 200):
        o, S = oracle.chunked(q, k, v, g, beta, S0=S0, chunk=c)
        assert rel_err(o, ref[0]) < 1e-11 and rel_err(S, ref[1]) < 1e-11


# ---------------------------------------------------------------- golden worked example

def load_golden():
    rows, S_T = [], None
    with open(os.path.join(GOLDEN, "delta_rule_d2_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "S_T":
                S_T = np.array([float(x) for x in parts[1:]]).reshape(2, 2)
            else:
                rows.append([float(x) for x in parts[1:]])
    r = np.array(rows)
    g, beta = r[:, 0:1], r[:, 1:2]
    k, v, q, o = r[:, None, 2:4], r[:, None, 4:6], r[:, None, 6:8], r[:, None, 8:10]
    return q, k, v, g, beta, o, S_T


def test_golden_example_scan_and_products():
    q, k, v, g, beta, o_ref, S_ref = load_golden()
    o, S = oracle.scan(q, k, v, g, beta)
    assert np.allclose(o, o_ref, atol=1e-12) and np.allclose(S[0, 0], S_ref, atol=1e-12)
    o2, S2 = oracle.transition_products(q, k, v, g, beta)
    assert np.allclose(o2, o_ref, atol=1e-12) and np.allclose(S2[0], S_ref, atol=1e-12)


# ---------------------------------------------------------------- (ii) invariants

def test_beta0_alpha1_leaves_state_unchanged():
    rng = np.random.default_rng(1)
    q, k, v, g, beta, S0 = random_case(rng, 33, 3, 8, 5)
    g[:] = 0.0
    beta[:] = 0.0
    o, S = oracle.scan(q, k, v, g, beta, S0=S0)
    assert np.array_equal(S, S0)
    assert np.allclose(o, np.einsum("hvk,thk->thv", S0[0], q), atol=1e-14)


def test_orthonormal_keys_store_and_retrieve_exactly():
    rng = np.random.default_rng(2)
    d, T = 16, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    k = Qm[:T][:, None, :]  # T orthonormal keys
    v = rng.standard_normal((T, 1, d))
    # query token t with the key of an earlier (or the same) token j(t)
    j_of_t = np.array([rng.integers(0, t + 1) for t in range(T)])
    q = k[j_of_t]
    g = np.zeros((T, 1))
    beta = np.ones((T, 1))
    o, S = oracle.scan(q, k, v, g, beta)
    for j in range(T):
        assert np.allclose(S[0, 0] @ k[j, 0], v[j, 0], atol=1e-12)
    for t in range(T):
        assert np.allclose(o[t, 0], v[j_of_t[t], 0], atol=1e-12)


def test_alpha0_resets_state():
    rng = np.random.default_rng(4)
    q, k, v, g, beta, S0 = random_case(rng, 9, 2, 6, 7)
    g[5] = -np.inf  # token 5 forgets everything before it
    o, S = oracle.scan(q, k, v, g, beta, S0=S0)
    # after token 5 the state is beta_5 v_5 k_5^T, whatever came before
    o_tail, S_tail = oracle.scan(q[5:], k[5:], v[5:], g[5:], beta[5:], S0=np.zeros_like(S0))
    assert rel_err(o[5:], o_tail) < 1e-13 and rel_err(S, S_tail) < 1e-13
    for h in range(2):
        assert np.allclose(o[5, h], beta[5, h] * v[5, h] * (k[5, h] @ q[5, h]), atol=1e-14)


# ---------------------------------------------------------------- (iii) closed forms

def test_beta0_pure_decay_closed_form():
    rng = np.random.default_rng(5)
    q, k, v, g, beta, S0 = random_case(rng, 40, 2, 8, 8)
    beta[:] = 0.0
    o, S = oracle.scan(q, k, v, g, beta, S0=S0)
    for h in range(2):
        assert np.allclose(S[0, h], math.exp(g[:, h].sum()) * S0[0, h], rtol=1e-12, atol=0)
        G = np.cumsum(g[:, h])
        assert np.allclose(o[:, h], np.exp(G)[:, None] * (q[:, h] @ S0[0, h].T), rtol=1e-11, atol=1e-15)


def test_repeated_unit_key_is_scalar_ema():
    rng = np.random.default_rng(6)
    T, d = 50, 8
    kk = unit_rows(rng.standard_normal(d))
    k = np.tile(kk, (T, 1, 1))
    q = k.copy()  # o_t = S_t k
    v = rng.standard_normal((T, 1, d))
    g = -0.3 * rng.random((T, 1))
    beta = rng.random((T, 1))
    S0 = rng.standard_normal((1, 1, d, d))
    o, S = oracle.scan(q, k, v, g, beta, S0=S0)
    m = S0[0, 0] @ kk
    for t in range(T):
        a, b = math.exp(g[t, 0]), beta[t, 0]
        m = a * (1.0 - b) * m + b * v[t, 0]
        assert np.allclose(o[t, 0], m, atol=1e-12)
    assert np.allclose(S[0, 0] @ kk, m, atol=1e-12)


# ---------------------------------------------------------------- (iv) norm bound

def test_frobenius_bound_per_step():
    rng = np.random.default_rng(8)
    steps, B, H, d = 30, 3, 2, 8
    S = rng.standard_normal((B, H, d, d))
    for _ in range(steps):
        q, k, v, g, beta, _ = random_case(rng, B, H, d, d, s0=False)
        _, S_new = oracle.decode_step(q, k, v, g, beta, S)
        for b in range(B):
            for h in range(H):
                lhs = np.linalg.norm(S_new[b, h])
                rhs = math.exp(g[b, h]) * np.linalg.norm(S[b, h]) + beta[b, h] * np.linalg.norm(v[b, h])
                assert lhs <= rhs * (1 + 1e-12)
        S = S_new


# ---------------------------------------------------------------- (v) 2x2 brute force

def brute_force_2x2(q, k, v, g, beta, S0):
    """The matrix form alpha S (I - beta k k^T) + beta v k^T with every 2x2
    product written out entry by entry (not the expanded update the scan uses)."""
    S = [[S0[0][0], S0[0][1]], [S0[1][0], S0[1][1]]]
    outs = []
    for t in range(len(g)):
        a, b = math.exp(g[t]), beta[t]
        k0, k1 = k[t]
        M = [[a * (1 - b * k0 * k0), a * (-b * k0 * k1)],
             [a * (-b * k1 * k0), a * (1 - b * k1 * k1)]]
        W = [[b * v[t][0] * k0, b * v[t][0] * k1],
             [b * v[t][1] * k0, b * v[t][1] * k1]]
        S = [[S[i][0] * M[0][j] + S[i][1] * M[1][j] + W[i][j] for j in range(2)] for i in range(2)]
        outs.append([S[i][0] * q[t][0] + S[i][1] * q[t][1] for i in range(2)])
    return np.array(outs), np.array(S)


@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_brute_force_d2(T):
    rng = np.random.default_rng(20 + T)
    q, k, v, g, beta, S0 = random_case(rng, T, 1, 2, 2)
    o, S = oracle.scan(q, k, v, g, beta, S0=S0)
    o_bf, S_bf = brute_force_2x2(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0[0, 0])
    assert np.allclose(o[:, 0], o_bf, atol=1e-14) and np.allclose(S[0, 0], S_bf, atol=1e-14)


# ---------------------------------------------------------------- decode = scan of one-token sequences

def test_decode_step_chain_equals_scan():
    rng = np.random.default_rng(9)
    steps, H, d = 12, 2, 8
    q, k, v, g, beta, S0 = random_case(rng, steps, H, d, d)
    S = S0.copy()
    outs = []
    for t in range(steps):
        o_t, S = oracle.decode_step(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], beta[t:t + 1], S)
        outs.append(o_t[0])
    o, S_T = oracle.scan(q, k, v, g, beta, S0=S0)
    assert rel_err(np.stack(outs), o) < 1e-13 and rel_err(S, S_T) < 1e-13


# ---------------------------------------------------------------- mutation tests: the pins catch planted mistakes

def mutant_scan(q, k, v, g, beta, S0, mutation):
    """A scan with one planted mistake (CPU, test-local copy of the update)."""
    T, dk = k.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        a, b = math.exp(g[t]), beta[t]
        Sk = S @ k[t]
        if mutation == "output_before_update":
            o[t] = S @ q[t]
        if mutation == "no_alpha_on_erase":
            S = a * S - b * np.outer(Sk, k[t]) + b * np.outer(v[t], k[t])
        elif mutation == "no_beta_on_write":
            S = a * S - a * b * np.outer(Sk, k[t]) + np.outer(v[t], k[t])
        elif mutation == "transposed_write":
            S = a * S - a * b * np.outer(Sk, k[t]) + b * np.outer(k[t], v[t])
        elif mutation == "erase_sign":
            S = a * S + a * b * np.outer(Sk, k[t]) + b * np.outer(v[t], k[t])
        else:
            S = a * S - a * b * np.outer(Sk, k[t]) + b * np.outer(v[t], k[t])
        if mutation != "output_before_update":
            o[t] = S @ q[t]
    return o, S


def pins_pass(scan_fn):
    """Run a subset of the pins above against a single-head scan function."""
    q, k, v, g, beta, o_ref, S_ref = load_golden()
    o, S = scan_fn(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], np.zeros((2, 2)))
    if not (np.allclose(o, o_ref[:, 0], atol=1e-12) and np.allclose(S, S_ref, atol=1e-12)):
        return False
    # orthonormal store/retrieve
    rng = np.random.default_rng(2)
    Qm, _ = np.linalg.qr(rng.standard_normal((8, 8)))
    vv = rng.standard_normal((8, 8))
    o, S = scan_fn(Qm, Qm, vv, np.zeros(8), np.ones(8), np.zeros((8, 8)))
    return bool(np.allclose(S @ Qm.T, vv.T, atol=1e-10) and np.allclose(o, vv, atol=1e-10))


def test_pins_accept_the_rule():
    assert pins_pass(lambda *a: mutant_scan(*a, mutation=None))


@pytest.mark.parametrize("mutation", ["output_before_update", "no_alpha_on_erase", "no_beta_on_write",
                                      "transposed_write", "erase_sign"])
def test_pins_reject_planted_mistakes(mutation):
    assert not pins_pass(lambda *a: mutant_scan(*a, mutation=mutation))
