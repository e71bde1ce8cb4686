"""Host-side tests of the C ABI (no GPU needed): the library builds and loads,
exports every symbol include/gdn.h declares, and rejects bad arguments with
the documented status codes before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    from linear_attention_recurrent_chunked_b200 import build, gdn
    build.build()
    return gdn.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("gdn_chunk_fwd", "gdn_decode_step", "gdn_chunk_fwd_workspace_size", "gdn_last_error",
                 "gdn_chunk_fwd_check", "gdn_seq_scan", "gdn_version"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    from linear_attention_recurrent_chunked_b200 import gdn
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (gdn_[a-z0-9_]+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert name in gdn.SIGNATURES, name
        assert getattr(lib, name) is not None


def test_debug_checks_variant_builds_and_exports_the_same_symbols():
    """The GDN_DEBUG_CHECKS build (kernels that check their indices into the workspace and the
    outputs, a failed check reported as GDN_ERR_BOUNDS) links, loads and exports the same C ABI."""
    from linear_attention_recurrent_chunked_b200 import build
    path = build.build(debug=True)
    assert os.path.basename(path) == "libgdn_b200_debug.so"
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (gdn_[a-z0-9_]+)", out))
    for name in declared_functions():
        assert name in exported, name
    dbg = ctypes.CDLL(path)
    assert dbg.gdn_version() == ctypes.CDLL(build.LIB).gdn_version()
    # the status the check entry point returns for a failed index check is declared
    assert re.search(r"GDN_ERR_BOUNDS\s*=\s*9", open(HEADER).read())


def test_header_compiles_as_c_and_cpp(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "gdn.h"\nint main(void){return gdn_version()==0;}\n')
    for cc in (["gcc", "-std=c99"], ["g++", "-x", "c++"]):
        r = subprocess.run(cc + ["-fsyntax-only", "-I", os.path.dirname(HEADER), str(src)], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails before any device work
FAKE_MIS = ctypes.c_void_p((1 << 20) + 4)


def chunk_args(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, S0=None, cu=None, N=1, T=128, H=2, dk=64, dv=64, dt=1,
             o=FAKE, S_T=FAKE, ws=ctypes.c_void_p(1 << 20), ws_bytes=1 << 20, stream=None)
    a.update(over)
    return [a[x] for x in ("q", "k", "v", "g", "beta", "S0", "cu", "N", "T", "H", "dk", "dv", "dt", "o", "S_T",
                           "ws", "ws_bytes", "stream")]


@pytest.mark.parametrize("over,status", [
    (dict(dt=7), 3),                      # dtype
    (dict(dk=96, dv=96), 2),              # head size
    (dict(dk=64, dv=128), 2),             # dk != dv
    (dict(N=0), 2),
    (dict(H=0), 2),
    (dict(q=None), 1),
    (dict(S_T=None), 1),
    (dict(k=FAKE_MIS), 4),                # alignment
    (dict(g=ctypes.c_void_p((1 << 20) + 2)), 4),
    (dict(N=3, T=128), 5),                # equal split impossible
    (dict(ws=None), 6),
    (dict(ws_bytes=8), 6),
    (dict(ws_bytes=255), 6),
    (dict(ws=ctypes.c_void_p((1 << 20) + 16)), 4),  # workspace must be 256-byte aligned
])
def test_chunk_fwd_rejects_bad_arguments(lib, over, status):
    assert lib.gdn_chunk_fwd(*chunk_args(**over)) == status
    assert len(lib.gdn_last_error()) > 0


def test_decode_rejects_bad_arguments(lib):
    # q, k, v, g, beta, S, B, H, dk, dv, dtype, o, stream
    assert lib.gdn_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 16, 128, 128, 1, FAKE, None) == 2
    assert lib.gdn_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 16, 128, 128, 1, FAKE, None) == 1
    assert lib.gdn_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE_MIS, 4, 16, 128, 128, 1, FAKE, None) == 4
    assert lib.gdn_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 16, 128, 128, 2, FAKE, None) == 3
    assert b"dtype" in lib.gdn_last_error()


def test_seq_scan_rejects_bad_arguments(lib):
    args = chunk_args(dk=32, dv=32)
    del args[15:17]  # no workspace
    assert lib.gdn_seq_scan(*args) == 2


def test_workspace_size_is_positive(lib):
    for N, T in ((1, 2048), (8, 18000), (1, 10240)):
        assert lib.gdn_chunk_fwd_workspace_size(N, T, 16, 128, 128, 1) >= 256


def test_workspace_size_covers_segment_states(lib):
    """Beyond the 9 KB per (chunk, head) records, a plan that splits sequences keeps 192 KB of
    segment states per (segment slot, head): the reported size must include them, both for few
    (sequence, head) pairs (every sequence split) and for many pairs of packed sequences, where
    only the longer ones are split."""
    rec = lambda N, T, H: ((T + 63 * N) // 64) * H * 9216
    for N, T, H in ((1, 2048, 16), (1, 10240, 16), (8, 19679, 16)):
        size = lib.gdn_chunk_fwd_workspace_size(N, T, H, 128, 128, 1)
        assert size >= rec(N, T, H) + 2 * H * 192 * 1024, (N, T, H, size)


def test_binding_refuses_cpu_tensors(lib):
    import torch
    from linear_attention_recurrent_chunked_b200 import gdn
    x = torch.zeros(4, 2, 64)
    gb = torch.zeros(4, 2)
    with pytest.raises(gdn.GdnError):
        gdn.chunk_fwd(x, x, x, gb, gb)
    with pytest.raises(gdn.GdnError):
        gdn.decode_step(x, x, x, gb, gb, torch.zeros(4, 2, 64, 64))


def test_failure_injection_arguments(lib):
    """The test-only failure injection accepts its documented kinds and bounds and nothing else
    (host logic only; the GPU side is tests/test_gpu_failure.py)."""
    assert lib.gdn_debug_inject(7, 1000) == 2
    assert lib.gdn_debug_inject(1, 0) == 2
    assert lib.gdn_debug_inject(1, 1000001) == 2
    assert lib.gdn_debug_inject(1, 2000) == 0
    assert lib.gdn_debug_inject(0, 0) == 0
