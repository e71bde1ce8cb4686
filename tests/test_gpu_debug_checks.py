"""GPU: the GDN_DEBUG_CHECKS build (libgdn_b200_debug.so, whose kernels check every index into
the workspace's records, parts, links and states and every output row they write) on the
layouts that exercise those indices: a sequence split into segments (records, parts, the fold,
links), packed sequences with one split (the plan's offsets), equal-length calls without
cu_seqlens, and the full 2k call. Each case must report GDN_OK through gdn_chunk_fwd_check
(no failed check) and match the fp64 oracle. The cases run in a child process, which loads the
index-checking library instead of the normal one (the binding picks it at import from the
environment)."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, %(root)r)
import oracle
from linear_attention_recurrent_chunked_b200 import gdn
from linear_attention_recurrent_chunked_b200.workloads import make_prefill
from tests.gpu_util import TOL, rel_err, to_dev
assert gdn.library_path().endswith("libgdn_b200_debug.so"), gdn.library_path()
gdn.load_library()
cases = [
    ("segmented", dict(name="prefill_2k", seqlens=[1034], H=2, s0=True, stress=True, seed=71), True),
    ("packed, one split", dict(name="varlen", seqlens=[512] * 7 + [4096], H=16, d=128, s0=True, seed=72), True),
    ("mixed segment counts", dict(name="varlen", seqlens=[700, 100, 1500, 0], H=2, d=128, s0=True, seed=73), True),
    ("equal lengths", dict(name="prefill_2k", seqlens=[1000, 1000], H=4, s0=True, seed=74), False),
    ("prefill_2k", dict(name="prefill_2k", seed=0), False),
]
for what, kw, with_cu in cases:
    name = kw.pop("name")
    w = make_prefill(name, **kw)
    dw = to_dev(w)
    o, S_T = gdn.chunk_fwd(dw["q"], dw["k"], dw["v"], dw["g"], dw["beta"], dw["S0"],
                           dw["cu_seqlens"] if with_cu else None, N=w["N"], check=True)
    o_ref, S_ref = oracle.scan(w["q"], w["k"], w["v"], w["g"], w["beta"], S0=w["S0"], cu_seqlens=w["cu_seqlens"])
    eo, es = rel_err(o, o_ref), rel_err(S_T, S_ref)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (what, eo, es)
    print("%%s: GDN_OK, err(o)=%%.2e err(S_T)=%%.2e" %% (what, eo, es))
print("all cases ok")
"""


def test_index_checking_build_reports_ok_and_matches_the_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_chunked_b200 import build
    build.build(debug=True)
    env = dict(os.environ, GDN_DEBUG_CHECKS="1")
    r = subprocess.run([sys.executable, "-c", CHILD % {"root": ROOT}], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "all cases ok" in r.stdout
