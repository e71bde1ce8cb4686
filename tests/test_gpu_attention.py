"""Causal attention of the hybrid's attention layers (gdn_attn_fwd) against the fp64 oracle
(oracle.attention), on the same seeded inputs. Error measure and bound as the recurrence's bf16
parity tests: max|gpu - oracle| / max|oracle| <= 2e-2 (bf16 inputs; the probabilities enter the
second product as bf16, and o is rounded to bf16)."""
import numpy as np
import pytest
import torch

from oracle.attention import causal_attention
from linear_attention_recurrent_chunked_b200 import gdn
from linear_attention_recurrent_chunked_b200.workloads import make_attention
from tests.gpu_util import TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gdn.load_library()


def run(w, scale=0.0):
    return gdn.attn_fwd(w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), w["cu_seqlens"].cuda(), max_len=w["max_len"],
                        scale=scale, check=True).cpu()


@pytest.mark.parametrize("seqlens,H", [([200], 2), ([1, 127, 128, 129, 300, 0], 2), ([640, 640], 3)])
def test_attention_small(seqlens, H):
    w = make_attention(seqlens, H=H, seed=sum(seqlens))
    o = run(w)
    ref = causal_attention(w["q"], w["k"], w["v"], cu_seqlens=w["cu_seqlens"])
    assert rel_err(o, ref) <= TOL["bf16"]


def test_attention_custom_scale_and_equal_split():
    w = make_attention([256, 256], H=2, seed=3)
    o = gdn.attn_fwd(w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), None, N=2, scale=0.05, check=True).cpu()
    ref = causal_attention(w["q"], w["k"], w["v"], scale=0.05, cu_seqlens=w["cu_seqlens"])
    assert rel_err(o, ref) <= TOL["bf16"]


@pytest.mark.parametrize("trend", ["rising", "falling"])
def test_attention_rescale_paths(trend):
    """Scores that grow along the keys make every key tile raise the row maximum (the running
    output is rescaled tile after tile); falling scores never rescale after the first tile."""
    T, H, d = 700, 2, 128
    w = make_attention([T], H=H, seed=4)
    gen = torch.Generator().manual_seed(5)
    u = torch.nn.functional.normalize(torch.randn(H, d, generator=gen), dim=-1)
    # scale * q . k reaches 30 * 8 / sqrt(128) ~ 21 (about 31 in log2 units): several rescales
    ramp = torch.linspace(0.0, 8.0, T) if trend == "rising" else torch.linspace(8.0, 0.0, T)
    w["q"] = (30.0 * u[None].expand(T, H, d)).to(torch.bfloat16).contiguous()
    w["k"] = (ramp[:, None, None] * u[None] + 0.1 * w["k"].float()).to(torch.bfloat16).contiguous()
    o = run(w)
    ref = causal_attention(w["q"], w["k"], w["v"], cu_seqlens=w["cu_seqlens"])
    assert rel_err(o, ref) <= TOL["bf16"]


def test_attention_full_2k():
    w = make_attention([2048], H=16, seed=0)
    o = run(w)
    ref = causal_attention(w["q"], w["k"], w["v"], cu_seqlens=w["cu_seqlens"])
    assert rel_err(o, ref) <= TOL["bf16"]


def test_attention_10k_sampled_rows():
    """T = 10240, 16 heads: every row computed, 48 rows (first, last, tile edges, random) checked
    against the oracle over all heads."""
    w = make_attention([10240], H=16, seed=1)
    o = run(w)
    rng = np.random.default_rng(0)
    rows = sorted(set([0, 1, 127, 128, 10111, 10112, 10239] + rng.integers(0, 10240, 41).tolist()))
    ref = causal_attention(w["q"], w["k"], w["v"], cu_seqlens=w["cu_seqlens"], rows=rows)
    assert rel_err(o[rows], ref[rows]) <= TOL["bf16"]
    assert torch.isfinite(o.float()).all()


def test_attention_malformed_seqlens_reported_not_written():
    w = make_attention([100, 100, 56], H=2, seed=6)
    bad = torch.tensor([0, 150, 100, 256], dtype=torch.int32, device="cuda")
    o = torch.full_like(w["q"].cuda(), 7.0)
    with pytest.raises(gdn.GdnError) as ei:
        gdn.attn_fwd(w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), bad, max_len=150, o=o, check=True)
    assert ei.value.status == 5
    assert bool((o == 7.0).all())
