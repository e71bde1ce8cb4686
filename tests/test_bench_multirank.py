"""The multi-rank plumbing of bench.py on CPU (gloo, world size 2): ranks agree on
the max of their device times, and the JSON value is the whole-job aggregate
(replicas: N x tokens over the slowest rank's time)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist = bench.init_dist("gloo")
    ms = [3.0, 5.0][rank]
    got = bench.max_over_ranks(dist, ms)
    bench.barrier(dist)
    q.put((rank, got, bench.dist_info()))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [5.0, 5.0]
    assert res[1][2] == (2, 1, 1)


def test_single_process_identity():
    import bench
    assert bench.max_over_ranks(None, 2.5) == 2.5


def test_reference_arm_other_ranks_exit_quietly(capsys, monkeypatch):
    """Under torchrun with N > 1 only rank 0 runs the CPU reference; others print nothing."""
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.reference_arm(type("A", (), {"steps": 1, "warmup": 3})())
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("name,mbytes", [("prefill_2k", 34.865152), ("prefill_10k", 171.180032)])
def test_algorithmic_bytes(name, mbytes):
    import bench
    from linear_attention_recurrent_chunked_b200.workloads import make_prefill
    w = make_prefill(name, seed=0)
    assert abs(bench.prefill_bytes(w) / 1e6 - mbytes) < 1e-6
    assert bench.prefill_flops(w) == w["T_tot"] * 16 * 180224
    assert bench.decode_bytes(64, 16, 128) == 135274496
