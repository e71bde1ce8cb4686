"""gdn_chunk_fwd_noalloc: the chunked forward for callers that cannot allocate
device memory (a memory manager already owns the GPU's memory, or a
latency-critical path cannot take cudaMalloc's synchronisation). Its scratch is
an array built into the library instead of a caller-provided workspace. The
test calls it through the C ABI twice in a row (the array keeps the previous
call's contents) and compares each result with gdn_chunk_fwd's on the same
inputs, at the tolerances the parity tests use."""
import ctypes

import pytest
import torch

from linear_attention_recurrent_chunked_b200 import gdn
from linear_attention_recurrent_chunked_b200.workloads import make_prefill
from tests.gpu_util import TOL, rel_err

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("dtype,d,seqlens,H", [
    ("bf16", 128, [130, 64, 1, 0], 3),
    ("f32", 64, [100, 29], 3),
    ("bf16", 128, [2048], 16),  # preferred workspace above the 8 MiB array: a coarser plan is used
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
        N = len(seqlens)
        st = lib.gdn_chunk_fwd_noalloc(_p(t["q"]), _p(t["k"]), _p(t["v"]), _p(t["g"]), _p(t["beta"]), _p(t["S0"]),
                                       _p(t["cu_seqlens"]), N, w["T_tot"], H, d, d,
                                       1 if dtype == "bf16" else 0, _p(o), _p(S_T),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, lib.gdn_last_error()
        torch.cuda.synchronize()
        assert rel_err(o, o_ref.double().cpu().numpy()) <= TOL[dtype], call
        assert rel_err(S_T, S_ref.double().cpu().numpy()) <= TOL[dtype], call
