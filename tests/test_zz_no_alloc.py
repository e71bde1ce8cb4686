"""gdn_chunk_fwd_noalloc: the chunked forward for callers that cannot allocate
device memory (a memory manager already owns the GPU's memory, or a
latency-critical path cannot take cudaMalloc's synchronisation). Its scratch is
an array built into the library instead of a caller-provided workspace. The
test calls it through the C ABI twice in a row (the array keeps the previous
call's contents) and compares each result with gdn_chunk_fwd's on the same
inputs and with the fp64 oracle, at the tolerances the parity tests use; it also
checks that a call leaves the device's free memory unchanged.

The cases cover the three plans the array can hold: the pipelined path without
segments (short sequences), the coarser segmentation of the single-kernel path
when the preferred workspace exceeds the array (2048 and 4096 tokens over 16
heads), the fp32 path, and a state updated in place (S0 aliasing S_T, which
needs the array's copy of S0 when the sequence is split)."""
import ctypes

import pytest
import torch

import oracle
from linear_attention_recurrent_chunked_b200 import gdn
from linear_attention_recurrent_chunked_b200.workloads import make_prefill
from tests.gpu_util import TOL, rel_err

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, t, w, H, d, dtype, o, S_T):
    N = len(w["seqlens"])
    return lib.gdn_chunk_fwd_noalloc(_p(t["q"]), _p(t["k"]), _p(t["v"]), _p(t["g"]), _p(t["beta"]), _p(t["S0"]),
                                     _p(t["cu_seqlens"]), N, w["T_tot"], H, d, d, 1 if dtype == "bf16" else 0,
                                     _p(o), _p(S_T), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype,d,seqlens,H", [
    ("bf16", 128, [130, 64, 1, 0], 3),
    ("f32", 64, [100, 29], 3),
    ("bf16", 128, [2048], 16),  # preferred workspace above the 8 MiB array: a coarser plan is used
    ("bf16", 128, [4096], 16),  # the single-kernel path with the segmentation that fits
])
def test_noalloc_matches_workspace_entry_twice(dtype, d, seqlens, H):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = gdn.load_library()
    for call, seed in enumerate((11, 12)):  # two calls in a row, different inputs
        w = make_prefill("varlen", seqlens=seqlens, H=H, d=d, dtype=dtype, s0=True, seed=seed)
        t = {k: (v.cuda() if hasattr(v, "cuda") else v) for k, v in w.items()}
        o_ref, S_ref = gdn.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], t["cu_seqlens"],
                                     check=True)
        o = torch.full_like(o_ref, float("nan"))
        S_T = torch.full_like(S_ref, float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        st = _noalloc(lib, t, w, H, d, dtype, o, S_T)
        assert st == 0, lib.gdn_last_error()
        torch.cuda.synchronize()
        if call == 1:  # after the first call (which may load the module), nothing is allocated
            assert torch.cuda.mem_get_info()[0] == free_before
        assert rel_err(o, o_ref.double().cpu().numpy()) <= TOL[dtype], call
        assert rel_err(S_T, S_ref.double().cpu().numpy()) <= TOL[dtype], call
        o_or, S_or = oracle.scan(w["q"], w["k"], w["v"], w["g"], w["beta"], S0=w["S0"], cu_seqlens=w["cu_seqlens"])
        assert rel_err(o, o_or) <= TOL[dtype] and rel_err(S_T, S_or) <= TOL[dtype], call


@pytest.mark.parametrize("seqlens,H", [([300, 41], 2), ([1500], 2)])
def test_noalloc_state_in_place(seqlens, H):
    """S0 may alias S_T through this entry point too: unsplit, and with the 1500-token sequence
    split into segments (that plan fits in the array and snapshots S0 there)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = gdn.load_library()
    for call, seed in enumerate((13, 14)):
        w = make_prefill("varlen", seqlens=seqlens, H=H, d=128, dtype="bf16", s0=True, seed=seed)
        t = {k: (v.cuda() if hasattr(v, "cuda") else v) for k, v in w.items()}
        S = t["S0"].clone()
        t["S0"] = S
        o = torch.full_like(t["v"], float("nan"))
        st = _noalloc(lib, t, w, H, 128, "bf16", o, S)
        assert st == 0, lib.gdn_last_error()
        torch.cuda.synchronize()
        o_or, S_or = oracle.scan(w["q"], w["k"], w["v"], w["g"], w["beta"], S0=w["S0"], cu_seqlens=w["cu_seqlens"])
        assert rel_err(o, o_or) <= TOL["bf16"] and rel_err(S, S_or) <= TOL["bf16"], call
