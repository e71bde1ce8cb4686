"""Pins for the oracle's causal attention (CPU only): closed forms (one key, equal scores give a
running mean, a dominant key selects its value, constant values pass through), causality and
packing as exact invariants, agreement with an independent formulation written without the
max shift, and mutation tests."""
import numpy as np
import pytest

from oracle import attention as at


def unshifted(q, k, v, scale):
    """The same definition written directly: exp(s) / sum exp(s) over j <= t (tiny inputs only)."""
    T, H, d = q.shape
    o = np.zeros((T, H, v.shape[2]))
    for t in range(T):
        for h in range(H):
            w = np.array([np.exp(scale * float(np.dot(q[t, h], k[j, h]))) for j in range(t + 1)])
            o[t, h] = sum(w[j] * v[j, h] for j in range(t + 1)) / w.sum()
    return o


def pins(attn):
    rng = np.random.default_rng(11)
    T, H, d = 7, 2, 4
    q, k, v = rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d)), rng.standard_normal((T, H, 3))
    o = attn(q, k, v)
    # the first position sees one key: o_0 = v_0
    assert np.allclose(o[0], v[0], rtol=0, atol=1e-14)
    # equal scores (q = 0): o_t is the mean of v_0 .. v_t
    o0 = attn(np.zeros_like(q), k, v)
    assert np.allclose(o0, np.cumsum(v, axis=0) / np.arange(1, T + 1)[:, None, None], atol=1e-14)
    # constant values pass through (the weights sum to one)
    assert np.allclose(attn(q, k, np.ones_like(v)), 1.0, atol=1e-14)
    # a dominant key selects its value from the positions that can see it
    k2 = k.copy()
    k2[3] = 60.0 * q[5]
    assert np.allclose(attn(q, k2, v)[5], v[3], atol=1e-9)
    # causality: changing the future leaves the past exactly unchanged
    k3, v3 = k.copy(), v.copy()
    k3[5:], v3[5:] = 9.0, -9.0
    assert np.array_equal(attn(q, k3, v3)[:5], o[:5])
    # the definition without the max shift, and the default scale 1 / sqrt(d)
    assert np.allclose(o, unshifted(q, k, v, 1.0 / np.sqrt(d)), rtol=1e-12, atol=1e-14)
    # packing: the second sequence equals a separate call on it
    op = attn(q, k, v, cu_seqlens=[0, 3, T])
    assert np.allclose(op[3:], attn(q[3:], k[3:], v[3:]), atol=1e-14)
    assert np.array_equal(op[:3], o[:3])


def test_pins_accept_the_oracle():
    pins(at.causal_attention)


def test_rows_subset_matches_full():
    rng = np.random.default_rng(12)
    q, k, v = (rng.standard_normal((20, 2, 8)) for _ in range(3))
    full = at.causal_attention(q, k, v)
    sub = at.causal_attention(q, k, v, rows=[0, 7, 19])
    assert np.array_equal(sub[[0, 7, 19]], full[[0, 7, 19]])


def _mask_off_by_one(q, k, v, scale=None, cu_seqlens=None, rows=None):
    q, k, v = at.as_f64(q), at.as_f64(k), at.as_f64(v)
    T = q.shape[0]
    kk = np.concatenate([k[1:], k[-1:]])  # each query also sees the next key
    return at.causal_attention(q, kk, np.concatenate([v[1:], v[-1:]]), scale, cu_seqlens, rows)


MUTANTS = {
    "no scale": lambda q, k, v, scale=None, cu_seqlens=None, rows=None: at.causal_attention(
        q, k, v, 1.0, cu_seqlens, rows),
    "mask shifted by one": _mask_off_by_one,
    "no causal mask": lambda q, k, v, scale=None, cu_seqlens=None, rows=None: np.stack(
        [at.causal_attention(q, k, v, scale, None)[-1]] * len(q)) if cu_seqlens is None else at.causal_attention(
        q, k, v, scale, None),
    "sequences not separated": lambda q, k, v, scale=None, cu_seqlens=None, rows=None: at.causal_attention(
        q, k, v, scale, None, rows),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistakes(name):
    with pytest.raises(AssertionError):
        pins(MUTANTS[name])
