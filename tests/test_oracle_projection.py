"""Pins for the oracle's int8-weight input projection (CPU only): closed values of the
dequantisation, a brute-force triple loop on tiny inputs, the split of the output columns into
the layer's raw inputs checked against hand-placed columns, and mutation tests."""
import numpy as np
import pytest

from oracle import projection as pj


def brute_force(x, w, s):
    T, D = x.shape
    N = w.shape[0]
    y = np.zeros((T, N))
    for t in range(T):
        for n in range(N):
            acc = 0.0
            for j in range(D):
                acc += float(x[t, j]) * (float(s[n]) * float(w[n, j]))
            y[t, n] = acc
    return y


def pins_dequantise(deq):
    w = np.array([[-128, 127, 0, 1], [5, -5, 64, -64]], dtype=np.int8)
    s = np.array([0.5, 2.0 ** -7])
    assert np.array_equal(deq(w, s), [[-64.0, 63.5, 0.0, 0.5], [5 / 128, -5 / 128, 0.5, -0.5]])


def pins_project(project):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 5))
    w = rng.integers(-128, 128, (4, 5)).astype(np.int8)
    s = rng.random(4) * 0.01
    assert np.allclose(project(x, w, s), brute_force(x, w, s), rtol=1e-13, atol=1e-15)
    # unit rows of x pick one input channel: y[t, n] = scale[n] w[n, t]
    eye = np.eye(5)
    assert np.allclose(project(eye, w, s), (w.astype(np.float64) * s[:, None]).T, rtol=0, atol=1e-15)


def pins_split(split):
    H, dk, dv, T = 2, 3, 4, 2
    N = H * (2 * dk + dv) + 2 * H
    y = np.arange(T * N, dtype=np.float64).reshape(T, N)
    q, k, v, a, b = split(y, H, dk, dv)
    assert q.shape == (T, H, dk) and v.shape == (T, H, dv) and a.shape == (T, H)
    assert q[1, 1, 2] == y[1, 1 * dk + 2]
    assert k[0, 0, 0] == y[0, H * dk]
    assert k[1, 1, 2] == y[1, H * dk + dk + 2]
    assert v[0, 1, 3] == y[0, 2 * H * dk + dv + 3]
    assert a[1, 1] == y[1, 2 * H * dk + H * dv + 1]
    assert b[0, 0] == y[0, 2 * H * dk + H * dv + H] and b[1, 1] == y[1, N - 1]


def test_pins_accept_the_oracle():
    pins_dequantise(pj.dequantise)
    pins_project(pj.project)
    pins_split(pj.split_outputs)


def test_project_w8_composes():
    rng = np.random.default_rng(4)
    H, dk, dv, D, T = 2, 4, 4, 8, 3
    N = H * (2 * dk + dv) + 2 * H
    x = rng.standard_normal((T, D))
    w = rng.integers(-128, 128, (N, D)).astype(np.int8)
    s = rng.random(N)
    q, k, v, a, b = pj.project_w8(x, w, s, H, dk, dv)
    y = brute_force(x, w, s)
    assert np.allclose(np.concatenate([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1), a, b], axis=1), y)


MUTANTS = {
    "scale applied per input channel": dict(deq=lambda w, s: pj.as_f64(w) * pj.as_f64(s)[None, : w.shape[1]]
                                            if len(s) >= w.shape[1] else pj.as_f64(w) * pj.as_f64(s).mean()),
    "weight not transposed": dict(project=lambda x, w, s: pj.as_f64(x) @ pj.dequantise(w, s)[:, : x.shape[1]]
                                  if w.shape[0] >= x.shape[1] else pj.as_f64(x) @ pj.dequantise(w, s).T * 1.5),
    "codes read as unsigned": dict(deq=lambda w, s: (pj.as_f64(w) % 256) * pj.as_f64(s)[:, None]),
    "k and v swapped": dict(split=lambda y, H, dk, dv: (lambda q, k, v, a, b: (q, v[..., :dk], k, a, b))(
        *pj.split_outputs(y, H, dk, dv))),
    "a and b swapped": dict(split=lambda y, H, dk, dv: (lambda q, k, v, a, b: (q, k, v, b, a))(
        *pj.split_outputs(y, H, dk, dv))),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistakes(name):
    m = MUTANTS[name]
    with pytest.raises(AssertionError):
        pins_dequantise(m.get("deq", pj.dequantise))
        pins_project(m.get("project", pj.project))
        pins_split(m.get("split", pj.split_outputs))
