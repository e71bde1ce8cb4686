"""Failure detection on the GPU without a GPU fault: a device-side wait that cannot complete
ends with an error status that the host reads, and the context stays usable.

The injection hook (gdn_debug_inject, C ABI) makes the transition block of head 0's first
segment withhold its end state. Every block that waits for it gives up after a short bound
(2 ms here, instead of 1 s), marks its own results failed so that the blocks waiting on them
give up too, records GDN_ERR_TIMEOUT in the workspace's error word and returns. Nothing traps,
faults or spins without a bound. The test then checks that the status is reported, that the
other head's results are complete and correct, and that a normal call afterwards on the same
stream and workspace matches the oracle."""
import ctypes
import time

import pytest
import torch

import oracle
from linear_attention_recurrent_chunked_b200 import gdn
from linear_attention_recurrent_chunked_b200.workloads import make_prefill
from tests.gpu_util import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_withheld_link_times_out_reports_and_recovers():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = gdn.load_library()
    # one 2000-token sequence, two heads: split into 7 parallel segments per head
    w = make_prefill("prefill_2k", seqlens=[2000], H=2, s0=True, seed=51)
    dw = to_dev(w)
    need = gdn.chunk_fwd_workspace_size(1, 2000, 2, 128, 128, torch.bfloat16)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o = torch.full_like(dw["v"], float("nan"))
    S_T = torch.full_like(dw["S0"], float("nan"))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    gdn.debug_inject(1, 2000)
    try:
        t0 = time.perf_counter()
        gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], dw["S0"], dw["cu_seqlens"], o=o, S_T=S_T,
                      workspace=ws)
        status = lib.gdn_chunk_fwd_check(_p(ws), ws.numel(), stream)
        message = lib.gdn_last_error()  # (the next successful call clears it)
        elapsed = time.perf_counter() - t0
    finally:
        gdn.debug_inject(0, 0)
    assert status == 8, (status, message)  # GDN_ERR_TIMEOUT
    # the message names the first wait that gave up: a wait for the withheld end-state flag
    assert b"flag word" in message, message
    assert elapsed < 5.0, elapsed  # the waits gave up after the injected bound, not after 1 s each
    o_ref, S_ref = oracle.scan(w["q"], w["k"], w["v"], w["g"], w["beta"], S0=w["S0"], cu_seqlens=w["cu_seqlens"])
    # head 1 never waits for head 0: its outputs and final state are complete and correct
    assert rel_err(o[:, 1], o_ref[:, 1]) <= TOL["bf16"]
    assert rel_err(S_T[:, 1], S_ref[:, 1]) <= TOL["bf16"]
    # the context is usable and the next call (same stream, same workspace) is correct
    o2, S2 = gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], dw["S0"], dw["cu_seqlens"],
                           workspace=ws, check=True)
    assert rel_err(o2, o_ref) <= TOL["bf16"] and rel_err(S2, S_ref) <= TOL["bf16"]


def test_injection_off_by_default_and_unsplit_calls_unaffected():
    """With the hook on, a call whose sequences are not split (many pairs, equal lengths) has
    no cross-block waits and completes normally."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = make_prefill("varlen", seqlens=[200] * 8, H=16, s0=True, seed=52)
    dw = to_dev(w)
    gdn.debug_inject(1, 2000)
    try:
        o, S_T = gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], dw["S0"], dw["cu_seqlens"],
                               check=True)
    finally:
        gdn.debug_inject(0, 0)
    o_ref, S_ref = oracle.scan(w["q"], w["k"], w["v"], w["g"], w["beta"], S0=w["S0"], cu_seqlens=w["cu_seqlens"])
    assert rel_err(o, o_ref) <= TOL["bf16"] and rel_err(S_T, S_ref) <= TOL["bf16"]
