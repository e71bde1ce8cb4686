"""Raw-input entry points (gdn_chunk_fwd_raw, gdn_decode_step_raw): the layer's input
preparation (q, k L2-normalised, g = -softplus(a), beta = sigmoid(b)) fused into the kernels,
checked against the oracle's fp64 preparation (oracle.input_prep) followed by the fp64 scan, on
the same seeded raw inputs. Tolerance as every parity test: max|gpu - oracle| / max|oracle| <=
1e-4 (fp32 inputs) or 2e-2 (bf16 inputs), for o and for the final state."""
import numpy as np
import pytest
import torch

import oracle
from oracle.input_prep import prep_inputs
from linear_attention_recurrent_chunked_b200 import gdn
from linear_attention_recurrent_chunked_b200.workloads import make_decode, make_prefill
from tests.gpu_util import TOL, rel_err

pytestmark = pytest.mark.gpu

RAW_KEYS = ("q_raw", "k_raw", "v", "a", "b", "S0", "cu_seqlens")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gdn.load_library()


def oracle_from_raw(w):
    q, k, g, beta = prep_inputs(w["q_raw"], w["k_raw"], w["a"], w["b"])
    return oracle.scan(q, k, w["v"], g, beta, S0=w["S0"], cu_seqlens=w["cu_seqlens"])


def run_raw(w, **kw):
    t = {key: (w[key].cuda() if w.get(key) is not None else None) for key in RAW_KEYS}
    return gdn.chunk_fwd_raw(t["q_raw"], t["k_raw"], t["v"], t["a"], t["b"], t["S0"], t["cu_seqlens"],
                             check=True, **kw)


def check(w, o, S_T, what):
    o_ref, S_ref = oracle_from_raw(w)
    eo, es = rel_err(o, o_ref), rel_err(S_T, S_ref)
    tol = TOL[w["dtype"]]
    assert eo <= tol and es <= tol, "%s: err(o)=%.3g err(S_T)=%.3g" % (what, eo, es)


@pytest.mark.parametrize("name", ["tiny", "prefill_2k", "prefill_10k", "varlen"])
def test_raw_prefill_full_configs(name):
    w = make_prefill(name, seed=0)
    o, S_T = run_raw(w)
    check(w, o, S_T, name + " from raw inputs")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64), ("bf16", 64), ("f32", 128)])
def test_raw_prefill_ragged(dtype, d):
    """Partial chunks, one-token and empty sequences: masked positions must stay inert
    (zero decay exponent and zero write strength, although softplus(0) = ln 2)."""
    w = make_prefill("varlen", seqlens=[1, 63, 64, 65, 0, 200], H=3, d=d, dtype=dtype, s0=True, seed=61)
    o, S_T = run_raw(w)
    check(w, o, S_T, "ragged raw")
    assert torch.equal(S_T[4].cpu(), w["S0"][4])


def test_raw_prefill_segmented_and_extremes():
    """A sequence split into parallel segments, with extreme logits (softplus and sigmoid
    saturate without overflow), a zero key (normalised to zero by the 1e-12 guard), keys of very
    different norms, and an unsplit short sequence."""
    w = make_prefill("varlen", seqlens=[1500, 40], H=2, d=128, dtype="bf16", s0=True, seed=62)
    w["a"][100:110] = 60.0     # alpha ~ exp(-60): reset
    w["a"][200:210] = -60.0    # alpha ~ 1
    w["b"][300:310] = -60.0    # beta ~ 0
    w["b"][400:410] = 60.0     # beta ~ 1
    w["k_raw"][500] = 0.0      # zero key
    w["k_raw"][600:700] *= 1e3
    w["q_raw"][700:800] *= 1e-3
    o, S_T = run_raw(w)
    check(w, o, S_T, "segmented raw with extremes")


def test_raw_matches_prepared_inputs():
    """From raw inputs, or prepared by the caller (fp32 normalisation, then the cast): the two
    differ only by the cast's rounding of the normalised q, k."""
    w = make_prefill("prefill_2k", seqlens=[700], H=4, s0=True, seed=63)
    o_raw, S_raw = run_raw(w)
    t = {key: (w[key].cuda() if w.get(key) is not None else None) for key in ("q", "k", "v", "g", "beta", "S0",
                                                                                "cu_seqlens")}
    o_pre, S_pre = gdn.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], t["cu_seqlens"], check=True)
    assert rel_err(o_raw, o_pre.double().cpu().numpy()) <= TOL["bf16"]
    assert rel_err(S_raw, S_pre.double().cpu().numpy()) <= TOL["bf16"]


def test_raw_needs_the_pipelined_workspace():
    w = make_prefill("prefill_2k", seqlens=[300], H=2, s0=True, seed=64)
    with pytest.raises(gdn.GdnError) as ei:
        run_raw(w, workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == 6


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_raw_decode_chain_small(dtype, d):
    w = make_decode(steps=6, B=3, H=2, d=d, dtype=dtype, seed=65)
    w["a"][2, 0] = 60.0
    w["k_raw"][3, 1, 0] = 0.0
    dw = {key: w[key].cuda() for key in ("q_raw", "k_raw", "v", "a", "b", "S")}
    S = dw["S"].clone()
    S_ref = w["S"].double().numpy()
    for t in range(w["steps"]):
        o = gdn.decode_step_raw(dw["q_raw"][t], dw["k_raw"][t], dw["v"][t], dw["a"][t], dw["b"][t], S)
        q, k, g, beta = prep_inputs(w["q_raw"][t], w["k_raw"][t], w["a"][t], w["b"][t])
        o_ref, S_ref = oracle.decode_step(q, k, w["v"][t], g, beta, S_ref)
        assert rel_err(o, o_ref) <= TOL[dtype], t
    assert rel_err(S, S_ref) <= TOL[dtype]


def test_raw_decode_full_size_all_pairs():
    """The decode workload (B=64, H=16, d=128, 256 steps) from raw inputs: every output of every
    step and every final state against the oracle (each sequence replayed as a 256-token scan)."""
    w = make_decode(seed=0)
    dw = {key: w[key].cuda() for key in ("q_raw", "k_raw", "v", "a", "b", "S")}
    S = dw["S"].clone()
    outs = torch.empty_like(dw["v"])
    for t in range(w["steps"]):
        gdn.decode_step_raw(dw["q_raw"][t], dw["k_raw"][t], dw["v"][t], dw["a"][t], dw["b"][t], S, o=outs[t])
    torch.cuda.synchronize()
    steps, B, H, d = w["q_raw"].shape
    q, k, g, beta = prep_inputs(w["q_raw"], w["k_raw"], w["a"], w["b"])
    seq = lambda x: np.ascontiguousarray(np.swapaxes(x, 0, 1).reshape((B * steps,) + x.shape[2:]))
    v = w["v"].double().numpy()
    o_ref, S_ref = oracle.scan(seq(q), seq(k), seq(v), seq(g), seq(beta), S0=w["S"],
                               cu_seqlens=np.arange(B + 1) * steps)
    o_ref = np.swapaxes(o_ref.reshape(B, steps, H, d), 0, 1)
    assert rel_err(outs, o_ref) <= TOL["bf16"]
    assert rel_err(S, S_ref) <= TOL["bf16"]
