"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs. Tolerance: max|gpu - oracle| / max|oracle| <= 1e-4 for
fp32 inputs and 2e-2 for bf16 inputs, for o and for the final state."""

import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrent_chunked_b200 import gdn
from linear_attention_recurrent_chunked_b200.workloads import make_decode, make_prefill
from tests.gpu_util import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gdn.load_library()


def run_oracle(w):
    return oracle.scan(w["q"], w["k"], w["v"], w["g"], w["beta"], S0=w["S0"], cu_seqlens=w["cu_seqlens"])


def check(o, S_T, o_ref, S_ref, dtype, what=""):
    eo, es = rel_err(o, o_ref), rel_err(S_T, S_ref)
    assert eo <= TOL[dtype] and es <= TOL[dtype], "%s: err(o)=%.3g err(S_T)=%.3g" % (what, eo, es)
    return eo, es


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_chain_small(dtype, d):
    w = make_decode(steps=6, B=3, H=2, d=d, dtype=dtype, seed=1)
    dw = to_dev(w)
    S = dw["S"].clone()
    S_ref = w["S"].double().numpy()
    for t in range(w["steps"]):
        o = gdn.decode_step(dw["q"][t], dw["k"][t], dw["v"][t], dw["g"][t], dw["beta"][t], S)
        o_ref, S_ref = oracle.decode_step(w["q"][t], w["k"][t], w["v"][t], w["g"][t], w["beta"][t], S_ref)
        assert rel_err(o, o_ref) <= TOL[dtype]
    assert rel_err(S, S_ref) <= TOL[dtype]


def test_decode_full_size_all_pairs():
    """Decode workload at full size (B=64, H=16, d=128, 256 chained steps): every output of
    every step and the final state of every (b, h) pair against the oracle. A chain of
    single-token steps is the scan over that sequence, so the oracle replays each of the 64
    sequences as one 256-token scan (all 16 heads) from the initial state."""
    w = make_decode(seed=0)
    dw = to_dev(w)
    S = dw["S"].clone()
    outs = torch.empty_like(dw["v"])
    for t in range(w["steps"]):
        gdn.decode_step(dw["q"][t], dw["k"][t], dw["v"][t], dw["g"][t], dw["beta"][t], S, o=outs[t])
    torch.cuda.synchronize()
    steps, B, H, d = w["q"].shape
    seq = lambda x: x.transpose(0, 1).reshape((B * steps,) + tuple(x.shape[2:]))  # [B * steps, H, ...]
    o_ref, S_ref = oracle.scan(seq(w["q"]), seq(w["k"]), seq(w["v"]), seq(w["g"]), seq(w["beta"]), S0=w["S"],
                               cu_seqlens=np.arange(B + 1) * steps)
    o_ref = o_ref.reshape(B, steps, H, d).transpose(1, 0, 2, 3)  # back to [steps, B, H, d]
    assert rel_err(outs, o_ref) <= TOL["bf16"]
    assert rel_err(S, S_ref) <= TOL["bf16"]
    # per step as well: no step may hide behind a larger one
    for t in range(steps):
        assert rel_err(outs[t], o_ref[t]) <= TOL["bf16"], t


# ------------------------------------------------------------------ sequential scan (GPU comparator)

@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 128)])
def test_seq_scan_varlen(dtype, d):
    w = make_prefill("varlen", seqlens=[1, 63, 0, 130], H=2, d=d, dtype=dtype, s0=True, seed=2)
    dw = to_dev(w)
    o, S_T = gdn.seq_scan(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], dw["S0"], dw["cu_seqlens"])
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, dtype, "seq_scan")


# ------------------------------------------------------------------ chunked prefill

def chunk(dw, **kw):
    return gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], dw["S0"], dw["cu_seqlens"], check=True, **kw)


def test_chunk_tiny_fp32_config():
    w = make_prefill("tiny", seed=0)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "f32", "tiny")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_chunk_ragged_small(dtype, d):
    # several tiles, partial chunks, one-token and empty sequences
    w = make_prefill("varlen", seqlens=[1, 63, 64, 65, 0, 200], H=3, d=d, dtype=dtype, s0=True, seed=3)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, dtype, "ragged")
    # empty sequence (index 4) returns its initial state exactly
    assert torch.equal(S_T[4].cpu(), w["S0"][4])


def test_chunk_no_initial_state_equal_split():
    w = make_prefill("prefill_2k", seqlens=[192, 192], H=2, s0=False, seed=4)
    dw = to_dev(w)
    o, S_T = gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], None, None, N=2, check=True)
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "bf16", "equal split")


def test_chunk_slow_decay_stress():
    """Slow decay, beta near one: the state carries information across many chunks."""
    w = make_prefill("prefill_2k", seqlens=[1500], H=2, s0=True, stress=True, seed=5)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "bf16", "stress")


@pytest.mark.parametrize("name", ["prefill_2k", "prefill_10k", "varlen"])
def test_chunk_full_configs(name):
    w = make_prefill(name, seed=0)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, w["dtype"], name)


@pytest.mark.parametrize("name", ["prefill_2k", "prefill_10k"])
def test_chunk_full_configs_equal_length_form(name):
    """The single-sequence workloads called without cu_seqlens (the form bench.py times): no plan
    kernel, offsets written by the prep kernel, item positions computed arithmetically."""
    w = make_prefill(name, seed=0)
    dw = to_dev(w)
    o, S_T = gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], dw["S0"], None, N=1, check=True)
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, w["dtype"], name + " (equal-length form)")


@pytest.mark.parametrize("T1", [64, 100])
def test_chunk_resume_from_state(T1):
    """Running [0, T) equals running [0, T1) then [T1, T) from S_T1 (on and off a chunk boundary)."""
    w = make_prefill("prefill_2k", seqlens=[300], H=2, s0=True, seed=6)
    dw = to_dev(w)
    o_full, S_full = chunk(dw)
    a = {k: (v[:T1] if k in ("q", "k", "v", "g", "beta") else v) for k, v in dw.items()}
    a["cu_seqlens"] = None
    o1, S1 = gdn.chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], dw["S0"], None, check=True)
    b = {k: (v[T1:].contiguous() if k in ("q", "k", "v", "g", "beta") else v) for k, v in dw.items()}
    o2, S2 = gdn.chunk_fwd(b["q"], b["k"], b["v"], b["g"], b["beta"], S1, None, check=True)
    ref = torch.cat([o1, o2]).float()
    assert rel_err(ref, o_full.double().cpu().numpy()) <= 1e-2
    assert rel_err(S2, S_full.double().cpu().numpy()) <= 1e-2


def test_chunk_in_place_state():
    """S0 may alias S_T."""
    w = make_prefill("varlen", seqlens=[100, 37], H=2, d=128, s0=True, seed=7)
    dw = to_dev(w)
    S = dw["S0"].clone()
    o, S_T = gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], S, dw["cu_seqlens"], S_T=S, check=True)
    o_ref, S_ref = run_oracle(w)
    check(o, S, o_ref, S_ref, "bf16", "in place")


def test_chunk_in_place_state_segmented():
    """S0 may alias S_T also when the sequence is split into segments: the first segment reads
    S0 while the last one writes S_T."""
    w = make_prefill("prefill_2k", seqlens=[2000], H=2, s0=True, stress=True, seed=9)
    dw = to_dev(w)
    S = dw["S0"].clone()
    o, S_T = gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], S, None, S_T=S, check=True)
    o_ref, S_ref = run_oracle(w)
    check(o, S, o_ref, S_ref, "bf16", "in place, segmented")


def test_chunk_equals_decode_steps():
    """Prefill over T tokens equals T decode steps (one sequence)."""
    w = make_prefill("prefill_2k", seqlens=[70], H=2, s0=True, seed=8)
    dw = to_dev(w)
    o, S_T = chunk(dw)
    S = dw["S0"].clone()
    outs = [gdn.decode_step(dw["q"][t:t + 1], dw["k"][t:t + 1], dw["v"][t:t + 1], dw["g"][t:t + 1],
                            dw["beta"][t:t + 1], S) for t in range(70)]
    assert rel_err(o, torch.cat(outs).double().cpu().numpy()) <= 2e-2
    assert rel_err(S_T, S.double().cpu().numpy()) <= 2e-2


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 128)])
def test_chunk_malformed_seqlens_reported_not_written(dtype, d):
    w = make_prefill("varlen", seqlens=[50, 50, 28], H=2, d=d, dtype=dtype, s0=True, seed=9)
    dw = to_dev(w)
    bad = torch.tensor([0, 100, 50, 128], dtype=torch.int32, device="cuda")  # decreasing offset
    o = torch.full_like(dw["v"], 7.0)
    S_T = torch.full_like(dw["S0"], 7.0)
    with pytest.raises(gdn.GdnError) as ei:
        gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], dw["S0"], bad, o=o, S_T=S_T, check=True)
    assert ei.value.status == 5
    assert bool((o == 7.0).all()) and bool((S_T == 7.0).all())


# ------------------------------------------------------------------ tensor-core tile diagnostics

@pytest.mark.parametrize("variant", [0, 1])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 0), (0, 1), (1, 1)])
@pytest.mark.parametrize("N,K", [(64, 128), (128, 64), (256, 32)])
def test_diag_mma_m128(variant, a_mn, b_mn, N, K):
    g = torch.Generator().manual_seed(N + K)
    A = torch.randn(128, K, generator=g).bfloat16()
    B = torch.randn(N, K, generator=g).bfloat16()
    D = gdn.diag_mma_tile(A.cuda(), B.cuda(), a_mn, b_mn, variant).cpu()
    ref = A.float() @ B.float().T
    assert torch.allclose(D, ref, atol=1e-3, rtol=1e-3), (D - ref).abs().max()


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 0), (0, 1), (1, 1)])
@pytest.mark.parametrize("N,K", [(64, 128), (128, 64), (128, 128)])
def test_diag_mma_m128_swizzled(a_mn, b_mn, N, K):
    """128-byte-swizzled operand tiles (the layout TMA writes with SWIZZLE_128B)."""
    g = torch.Generator().manual_seed(3 * N + K)
    A = torch.randn(128, K, generator=g).bfloat16()
    B = torch.randn(N, K, generator=g).bfloat16()
    D = gdn.diag_mma_tile(A.cuda(), B.cuda(), a_mn, b_mn, 2).cpu()
    ref = A.float() @ B.float().T
    assert torch.allclose(D, ref, atol=1e-3, rtol=1e-3), (D - ref).abs().max()


def test_diag_mma_m64_lane_map():
    """Where the rows of an M=64 accumulator land in TMEM: row i in lane (i % 16) + 32 (i / 16),
    the layout the prep kernel's epilogue reads."""
    g = torch.Generator().manual_seed(64)
    A = torch.randn(64, 64, generator=g).bfloat16()
    B = torch.randn(64, 64, generator=g).bfloat16()
    D = gdn.diag_mma_tile(A.cuda(), B.cuda(), 0, 0, 0).cpu()
    ref = A.float() @ B.float().T
    lanes = []
    for r in range(64):
        hit = [ln for ln in range(128) if torch.allclose(D[ln], ref[r], atol=1e-3, rtol=1e-3)]
        lanes.append(hit[0] if hit else -1)
    assert lanes == [(r % 16) + 32 * (r // 16) for r in range(64)], lanes


@pytest.mark.parametrize("kind", ["workload", "stress", "ones"])
def test_diag_ut_solve(kind):
    """The chunk solve T = (I + A)^{-1} against numpy's inverse (fp64)."""
    g = torch.Generator().manual_seed(5)
    if kind == "ones":  # keys all equal, beta = 1, no decay: A = strictly lower ones
        A = torch.tril(torch.ones(64, 64), -1)
    else:
        K = torch.nn.functional.normalize(torch.randn(64, 128, generator=g), dim=-1)
        beta = torch.sigmoid(torch.randn(64, generator=g) + (3.0 if kind == "stress" else 0.0))
        gl = -0.01 * torch.rand(64, generator=g) if kind == "stress" else -torch.nn.functional.softplus(
            torch.randn(64, generator=g))
        G = torch.cumsum(gl, 0)
        A = torch.tril(beta[:, None] * torch.exp(G[:, None] - G[None, :]) * (K @ K.T), -1)
    T = gdn.diag_ut_solve(A.cuda()).cpu().double()
    ref = np.linalg.inv(np.eye(64) + A.double().numpy())
    err = float(np.max(np.abs(T.numpy() - ref)) / np.max(np.abs(ref)))
    assert err < 2e-3, err
    assert torch.equal(torch.triu(T, 1), torch.zeros(64, 64, dtype=torch.float64))


# ------------------------------------------------------------------ segment-parallel prefill (few sequence-head pairs)

def test_segmented_varlen_mixed_segment_counts():
    """Few (sequence, head) pairs: the sequences are split into segments run in
    parallel (here 6, 1, 12 and 1 segments, one of them an empty sequence)."""
    w = make_prefill("varlen", seqlens=[700, 100, 1500, 0], H=2, d=128, s0=True, seed=21)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "bf16", "segmented varlen")
    assert torch.equal(S_T[3].cpu(), w["S0"][3])


def test_many_pairs_varlen_nothing_split():
    """Many (sequence, head) pairs, no sequence longer than 1.25x the average: the transition
    pass has no work (only its records flag is set) and every output CTA starts from it."""
    w = make_prefill("varlen", seqlens=[1000, 1010, 990, 1005, 995, 1000, 1002, 998], H=16, d=128, s0=True,
                     seed=25)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "bf16", "many pairs, nothing split")


def test_many_pairs_varlen_one_long_sequence_split():
    """Many pairs, one sequence 8x longer than the rest: only it is split (into four segments,
    so its first segment waits for its own end state) while the unsplit sequences' output CTAs
    start from the records flag."""
    w = make_prefill("varlen", seqlens=[512] * 7 + [4096], H=16, d=128, s0=True, stress=True, seed=26)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "bf16", "many pairs, one sequence split")


def test_many_pairs_one_sequence_in_six_segments():
    """[64] * 7 + [8192] over 16 heads: the many-pairs plan splits the long sequence into six
    segments, and the transition and output grids (224 blocks each) exceed one wave of the GPU.
    Transition blocks take their segments in the order they start (tickets), so a block only
    waits for blocks that are already running."""
    w = make_prefill("varlen", seqlens=[64] * 7 + [8192], H=16, d=128, s0=True, seed=27)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "bf16", "many pairs, six segments")


def test_segmented_slow_decay_stress():
    """Segment transitions matter when the state is remembered across segments."""
    w = make_prefill("prefill_2k", seqlens=[3000], H=1, s0=True, stress=True, seed=22)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "bf16", "segmented stress")


def test_segmented_last_segment_one_partial_chunk():
    """1034 tokens over 2 heads split 4 + 4 + 4 + 4 + 1 chunks: every later segment takes its start
    state from the one before it (copied into shared memory), and the last one is a single
    10-token chunk. Slow decay keeps each start state in the outputs."""
    w = make_prefill("prefill_2k", seqlens=[1034], H=2, s0=True, stress=True, seed=62)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "bf16", "last segment of one partial chunk")


def test_long_sequence_many_segments_long_fold():
    """One long sequence on one head: ~24 segments, so the last segment folds ~22 published parts
    (tf32 products) onto the first segment's end state; slow decay keeps the early state alive."""
    w = make_prefill("prefill_2k", seqlens=[24576], H=1, s0=True, stress=True, seed=61)
    o, S_T = chunk(to_dev(w))
    o_ref, S_ref = run_oracle(w)
    check(o, S_T, o_ref, S_ref, "bf16", "24 segments, long fold")


def test_medium_workspace_falls_back_correctly():
    """Workspaces between the error word and the preferred size select a plan that fits."""
    w = make_prefill("prefill_2k", seqlens=[1500], H=2, s0=True, stress=True, seed=24)
    dw = to_dev(w)
    need = gdn.chunk_fwd_workspace_size(1, 1500, 2, 128, 128, torch.bfloat16)
    o_ref, S_ref = run_oracle(w)
    for frac in (0.8, 0.5, 0.25):
        ws = torch.empty(int(need * frac) // 256 * 256, dtype=torch.uint8, device="cuda")
        o, S_T = chunk(dw, workspace=ws)
        check(o, S_T, o_ref, S_ref, "bf16", "workspace %.2f of preferred" % frac)


def test_small_workspace_selects_coarser_plan():
    """A workspace too small for the preferred segmentation gives the same results."""
    w = make_prefill("prefill_2k", seqlens=[1200], H=2, s0=True, seed=23)
    dw = to_dev(w)
    o_big, S_big = chunk(dw)
    small = torch.empty(256, dtype=torch.uint8, device="cuda")  # error word only: no segmentation
    o_small, S_small = chunk(dw, workspace=small)
    assert gdn.chunk_fwd_workspace_size(1, 1200, 2, 128, 128, torch.bfloat16) > 256
    o_ref, S_ref = run_oracle(w)
    check(o_small, S_small, o_ref, S_ref, "bf16", "unsegmented")
    check(o_big, S_big, o_ref, S_ref, "bf16", "segmented")
