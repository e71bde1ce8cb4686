"""The int8-weight input projection (gdn_proj_w8) against the fp64 oracle (oracle.projection).

Tolerance, from the arithmetic: the bf16 input x and the int8 codes are exact tensor-core
operands, products are exact and summed in fp32, the per-channel scale multiplies the fp32
sum, and q, k, v are rounded once to bf16 (half an ulp: 2^-9 of the value). So q, k, v must
agree to 4e-3 of max|y| (2^-8, twice the rounding bound) and the fp32 gate logits a, b to 1e-4
of max|y| (fp32 accumulation over D terms), measured as max|gpu - oracle| / max|oracle|."""
import numpy as np
import pytest
import torch

import oracle
from oracle.input_prep import prep_inputs
from oracle.projection import project_w8
from linear_attention_recurrent_chunked_b200 import gdn
from linear_attention_recurrent_chunked_b200.workloads import make_projection
from tests.gpu_util import TOL, rel_err

pytestmark = pytest.mark.gpu

TOL_BF16_OUT = 4e-3
TOL_F32_OUT = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gdn.load_library()


def run(p, rows=None):
    out = gdn.proj_w8(p["x"].cuda(), p["w"].cuda(), p["scale"].cuda(), p["H"], p["dk"], p["dv"], check=True)
    torch.cuda.synchronize()
    return [t.cpu() for t in out]


def check(p, got, rows=None):
    x = p["x"] if rows is None else p["x"][rows]
    ref = project_w8(x, p["w"], p["scale"], p["H"], p["dk"], p["dv"])
    scale_all = max(float(np.max(np.abs(r))) for r in ref)
    for name, g, r, tol in zip("qkvab", got, ref, [TOL_BF16_OUT] * 3 + [TOL_F32_OUT] * 2):
        g = g if rows is None else g[rows]
        err = float(np.max(np.abs(g.double().numpy() - r))) / scale_all if r.size else 0.0
        assert err <= tol, (name, err)


@pytest.mark.parametrize("T,D,H,dk,dv", [
    (200, 256, 2, 64, 64),    # partial token and channel tiles (N = 388)
    (130, 128, 2, 64, 128),   # dk != dv, N = 516
    (1, 64, 1, 8, 8),         # one token, one K step, N = 26
    (513, 320, 3, 40, 24),    # odd head sizes: a 32-column group straddles the q | k and v | a boundaries
    (3000, 256, 8, 64, 64),   # two token tiles per tile (enough tiles), ragged in tokens and channels (N = 1552)
])
def test_projection_small(T, D, H, dk, dv):
    p = make_projection(T, D, H, dk, dv, seed=T + D)
    check(p, run(p))


def test_projection_empty():
    p = make_projection(0, 128, 2, 64, 64)
    out = gdn.proj_w8(p["x"].cuda(), p["w"].cuda(), p["scale"].cuda(), 2, 64, 64, check=True)
    assert all(t.numel() == 0 for t in out)


def test_projection_full_size_2k():
    """The layer's projection at the prefill size: T = 2048, D = 1024, H = 16, dk = dv = 128."""
    p = make_projection(2048, seed=0)
    check(p, run(p))


def test_projection_10k_sampled_rows():
    """T = 10240: every output row computed, a sample of 384 rows (incl. first and last) checked."""
    p = make_projection(10240, seed=1)
    got = run(p)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 10239], rng.integers(0, 10240, 382)]))
    check(p, got, rows=torch.from_numpy(rows))
    assert all(torch.isfinite(t.float()).all() for t in got)


def test_projection_feeds_the_recurrence():
    """Hidden states -> int8 projection -> raw-input chunked forward, against the oracle chain
    (fp64 projection, the GPU's bf16 rounding of q, k, v reproduced, fp64 input prep, fp64 scan)."""
    T, H, d = 300, 2, 128
    p = make_projection(T, D=256, H=H, dk=d, dv=d, seed=5)
    q, k, v, a, b = gdn.proj_w8(p["x"].cuda(), p["w"].cuda(), p["scale"].cuda(), H, d, d, check=True)
    cu = torch.tensor([0, 120, T], dtype=torch.int32, device="cuda")
    o, S_T = gdn.chunk_fwd_raw(q, k, v, a, b, None, cu, check=True)
    qr, kr, vr, ar, br = project_w8(p["x"], p["w"], p["scale"], H, d, d)
    bf = lambda z: torch.from_numpy(z).to(torch.bfloat16)  # the projection's output rounding
    qh, kh, g, beta = prep_inputs(bf(qr), bf(kr), ar, br)
    o_ref, S_ref = oracle.scan(qh, kh, bf(vr), g, beta, S0=None, cu_seqlens=cu.cpu())
    assert rel_err(o, o_ref) <= TOL["bf16"] and rel_err(S_T, S_ref) <= TOL["bf16"]
