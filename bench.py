#!/usr/bin/env python
"""Benchmark of the gated-delta-rule forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]

One JSON line on rank 0. A step is one chunked prefill call (validation +
chunked kernels: the whole prefill path) over the prefill_2k workload (B=1,
H=16, T=2048, d=128, bf16 inputs, fp32 state); `value` is tokens/s over all
ranks. The same line also carries, measured in the same run, the 10k and
packed-varlen prefills, the decode step (state GB/s, L2-cold with 4 rotated
state sets, 256 steps in a CUDA graph), the GPU sequential scan comparator,
the per-kernel roofline and the oracle timed on the host cores.

Multi-GPU (torchrun, N > 1): every rank runs its own replica of the workload
(the path shards into independent sequences and heads with no exchange);
value = N * tokens / max over ranks of the device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gated-delta-rule prefill tokens/s at T=2k/10k, % roofline; decode state GB/s"
CHUNK_ACCOUNTING = 64  # chunk length used as the accounting constant of the flop count
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------- accounting

def prefill_bytes(w) -> int:
    """Algorithmic HBM bytes of one prefill call: q,k,v,o once, g,beta once, S0 (if given) and S_T once."""
    e = 2 if w["dtype"] == "bf16" else 4
    T, H, d, N = w["T_tot"], w["H"], w["d"], w["N"]
    per_tok = (2 * d + d) * e + 8 + d * e
    states = N * H * d * d * 4 * (2 if w["S0"] is not None else 1)
    return T * H * per_tok + states


def prefill_flops(w) -> int:
    d, C = w["d"], CHUNK_ACCOUNTING
    return w["T_tot"] * w["H"] * (6 * d * d + 2 * C * (3 * d + 2 * d))


def decode_bytes(B, H, d) -> int:
    return B * H * (2 * d * d * 4 + 3 * d * 2 + 8 + d * 2)


def kernel_source_digest() -> str:
    """Digest of the CUDA sources and the C header: ties an ncu traffic figure to the kernels it was taken on."""
    import glob
    import hashlib
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "linear_attention_recurrent_chunked_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(pkg, "*.cu")) + glob.glob(os.path.join(pkg, "*.cuh")) +
                    glob.glob(os.path.join(pkg, "*.h")) + [os.path.join(ROOT, "include", "gdn.h")]):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of `kernel` on
    `workload` from the committed ncu capture in profiles/traffic.json, or None if that capture
    was taken on different kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("source_digest") != kernel_source_digest():
        return None
    v = t.get("bytes_per_launch", {}).get("%s@%s" % (kernel, workload))
    return float(v) if v is not None else None


def kernel_shares(w) -> dict:
    """Algorithmic bytes each launch of a bf16 prefill call must move itself (the method's
    inputs and outputs it touches; workspace records excluded): prep reads k, g, beta; the
    transition pass reads k and v (and S0); the output pass reads q, k, v (and S0) and writes o
    and S_T. The shares add up to more than the call's bytes, since k is read by all three."""
    e = 2 if w["dtype"] == "bf16" else 4
    T, H, d, N = w["T_tot"], w["H"], w["d"], w["N"]
    tok = T * H * d * e
    state = N * H * d * d * 4
    s0 = state if w["S0"] is not None else 0
    return {"ws_plan": 4 * (N + 1), "ws_prep": tok + 8 * T * H, "ws_trans": 2 * tok + s0,
            "ws_out": 4 * tok + s0 + state}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), src="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ----------------------------------------------------------------------------- distributed plumbing

def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str):
    import datetime

    import torch.distributed as dist
    ws, rank, _ = dist_info()
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if ws > 1 else None


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(dist, x: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (200 ms) while a load runs; summarised as the median SM clock."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- GPU arm

def gpu_arm(args):
    import torch

    from linear_attention_recurrent_chunked_b200 import gdn
    from linear_attention_recurrent_chunked_b200.workloads import make_decode, make_prefill

    ws, rank, local = dist_info()
    dist = init_dist("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    gdn.load_library()
    pk = peaks()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.random_(0, 255)  # writes 256 MiB: evicts the 126 MB L2

    def dev_inputs(w):
        t = {k: (v.to(dev) if hasattr(v, "to") else v) for k, v in w.items()}
        if t.get("N") == 1 and "cu_seqlens" in t:
            t["cu_seqlens"] = None  # one sequence: the equal-length form of the call (no offsets to read)
        return t

    def prefill_call(t, o, S_T):
        return lambda: gdn.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], t["cu_seqlens"],
                                     o=o, S_T=S_T)

    def time_steps(fn, steps, warmup, l2_flush=True):
        """Per-step device times (ms) with CUDA events; L2 flushed before each step, outside the events."""
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        barrier(dist, dev)
        torch.cuda.synchronize()
        st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            if l2_flush:
                flush()
            st[i].record()
            fn()
            en[i].record()
        torch.cuda.synchronize()
        barrier(dist, dev)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in zip(st, en)]

    def kernel_times(fn, reps):
        """Per-kernel device times recorded by the library's event hooks (L2 flushed before each call)."""
        gdn.profile_read()
        gdn.profile_enable(True)
        for _ in range(reps):
            flush()
            fn()
        torch.cuda.synchronize()
        gdn.profile_enable(False)
        return gdn.profile_read()

    def prefill_entry(name, steps, warmup, full=True):
        w = make_prefill(name, seed=0)
        t = dev_inputs(w)
        o = torch.empty_like(t["v"])
        S_T = torch.empty((w["N"], w["H"], w["d"], w["d"]), dtype=torch.float32, device=dev)
        fn = prefill_call(t, o, S_T)
        times = time_steps(fn, steps, warmup)
        # the device error word of the last call (malformed cu_seqlens, a bounded wait that gave up):
        # raises unless it reads GDN_OK
        gdn.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], t["cu_seqlens"], o=o, S_T=S_T,
                      check=True)
        ms = statistics.mean(times)
        ms_max = max_over_ranks(dist, ms, dev)
        tokens = w["T_tot"]
        reps = max(3, min(steps, 10))
        kt = kernel_times(fn, reps)
        nbytes, nflops = prefill_bytes(w), prefill_flops(w)
        # The whole call (plan, prep, transition and output launches) is the unit: its
        # algorithmic bytes over its device time. Per launch, each kernel's own share.
        gbs = nbytes / (ms_max * 1e-3) / 1e9
        shares = kernel_shares(w)
        per_kernel = {}
        for k, (tot, cnt) in kt.items():
            k_ms = tot / cnt
            own = shares.get(k)
            per_kernel[k] = {"ms_per_launch": k_ms, "launches_per_step": cnt // reps,
                             "own_bytes": own, "traffic": measured_traffic(k, name)}
            if own is not None:
                per_kernel[k]["achieved_GBs"] = own / (k_ms * 1e-3) / 1e9
                per_kernel[k]["frac"] = per_kernel[k]["achieved_GBs"] / pk["hbm"]
        traffic = [v["traffic"] for v in per_kernel.values()]
        traffic = sum(traffic) if traffic and all(x is not None for x in traffic) else None
        roofline_ms = max(nbytes / (pk["hbm"] * 1e9), nflops / (pk["bf16"] * 1e12)) * 1e3
        top = max(kt.items(), key=lambda kv: kv[1][0])
        entry = {
            "workload": name, "tokens": tokens, "seqs": w["N"], "H": w["H"], "d": w["d"], "dtype": w["dtype"],
            "ms_per_step": ms_max, "tokens_per_s": ws * tokens / (ms_max * 1e-3),
            "algorithmic_bytes": nbytes, "algorithmic_flops": nflops, "roofline_ms": roofline_ms,
            "kernels": per_kernel, "top_kernel": top[0],
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                         "frac": gbs / pk["hbm"], "traffic": traffic,
                         "traffic_over_algorithmic": traffic / nbytes if traffic is not None else None,
                         "peak_source": pk["src"], "kernel": "chunk_fwd call (%s)" % ", ".join(kt),
                         "scope": "algorithmic bytes of one call over the call's device time (CUDA events); "
                                  "traffic = DRAM bytes summed over the call's launches",
                         "tensor_tflops": nflops / (ms_max * 1e-3) / 1e12},
            "launches_per_step": sum(v[1] for v in kt.values()) // reps,
            "device_status": "GDN_OK",
        }
        entry["roofline_frac_step"] = roofline_ms / ms_max
        return w, t, fn, entry

    result = {}
    # ---------------- main workload: prefill_2k
    w2k, t2k, fn2k, e2k = prefill_entry("prefill_2k", args.steps, args.warmup)
    result["prefill_2k"] = e2k

    # clocks during a sustained window of the main step
    with ClockSampler(local) as cs:
        t_end = time.time() + (1.5 if not args.quick else 0.6)
        while time.time() < t_end:
            for _ in range(20):
                fn2k()
            torch.cuda.synchronize()
    clocks = cs.summary()

    # e2e: host (pinned) inputs -> device -> chunk_fwd -> host outputs, all inside the events
    host = {k: (w2k[k].pin_memory() if w2k[k] is not None else None) for k in ("q", "k", "v", "g", "beta", "S0",
                                                                              "cu_seqlens")}
    if w2k["N"] == 1:
        host["cu_seqlens"] = None  # one sequence: the equal-length form of the call, as in the device-timed loop
    dbuf = {k: (torch.empty_like(v, device=dev) if v is not None else None) for k, v in host.items()}
    o_dev = torch.empty_like(dbuf["v"])
    S_dev = torch.empty((w2k["N"], w2k["H"], w2k["d"], w2k["d"]), dtype=torch.float32, device=dev)
    o_host = torch.empty(o_dev.shape, dtype=o_dev.dtype).pin_memory()
    S_host = torch.empty(S_dev.shape, dtype=S_dev.dtype).pin_memory()

    def e2e_step():
        for k, v in host.items():
            if v is not None:
                dbuf[k].copy_(v, non_blocking=True)
        gdn.chunk_fwd(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["g"], dbuf["beta"], dbuf["S0"], dbuf["cu_seqlens"],
                      o=o_dev, S_T=S_dev)
        o_host.copy_(o_dev, non_blocking=True)
        S_host.copy_(S_dev, non_blocking=True)

    e2e_times = time_steps(e2e_step, args.steps, args.warmup)
    e2e_ms = max_over_ranks(dist, statistics.mean(e2e_times), dev)
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = o_host.numel() * o_host.element_size() + S_host.numel() * S_host.element_size()

    if not args.quick:
        for name in ("prefill_10k", "varlen"):
            _, _, _, e = prefill_entry(name, max(5, args.steps // 2), args.warmup)
            result[name] = e
        # input preparation fused into the kernels (raw q, k and gate logits) against the caller
        # preparing the inputs with torch on the GPU (a separate pass over q, k, g, beta) first
        import torch.nn.functional as F
        for name in ("prefill_2k", "prefill_10k"):
            w = make_prefill(name, seed=0)
            t = dev_inputs(w)
            o = torch.empty_like(t["v"])
            S_T = torch.empty((w["N"], w["H"], w["d"], w["d"]), dtype=torch.float32, device=dev)
            fused = lambda: gdn.chunk_fwd_raw(t["q_raw"], t["k_raw"], t["v"], t["a"], t["b"], t["S0"],
                                              t["cu_seqlens"], o=o, S_T=S_T)

            def separate():
                q = F.normalize(t["q_raw"].float(), dim=-1).to(t["q_raw"].dtype)
                k = F.normalize(t["k_raw"].float(), dim=-1).to(t["k_raw"].dtype)
                gdn.chunk_fwd(q, k, t["v"], -F.softplus(t["a"]), torch.sigmoid(t["b"]), t["S0"], t["cu_seqlens"],
                              o=o, S_T=S_T)

            ms_f = statistics.mean(time_steps(fused, max(5, args.steps // 2), args.warmup))
            ms_s = statistics.mean(time_steps(separate, max(5, args.steps // 2), args.warmup))
            result[name]["from_raw_inputs"] = {
                "fused_ms": ms_f, "torch_prep_then_chunk_fwd_ms": ms_s,
                "fused_tokens_per_s": w["T_tot"] / (ms_f * 1e-3),
                "note": "raw q, k (unnormalised) and gate logits a, b: g = -softplus(a), beta = sigmoid(b); "
                        "fused = gdn_chunk_fwd_raw, separate = torch normalise/softplus/sigmoid on the GPU, "
                        "then gdn_chunk_fwd"}
        # GPU sequential scan comparator (the pages' chunked-vs-sequential ratio)
        for name in ("prefill_2k", "prefill_10k"):
            w = make_prefill(name, seed=0)
            t = dev_inputs(w)
            o = torch.empty_like(t["v"])
            S_T = torch.empty((w["N"], w["H"], w["d"], w["d"]), dtype=torch.float32, device=dev)
            ts = time_steps(lambda: gdn.seq_scan(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"],
                                                 t["cu_seqlens"], o=o, S_T=S_T), 3, 1)
            result[name]["seq_scan_ms"] = statistics.mean(ts)
            result[name]["chunked_over_sequential"] = statistics.mean(ts) / result[name]["ms_per_step"]
        result["decode"] = decode_entry(args, torch, gdn, dev, dist, pk, make_decode)
        result["projection"] = projection_entry(args, torch, gdn, dev, dist, pk, time_steps)
        result["attention"] = attention_entry(args, torch, gdn, dev, dist, pk, time_steps)

    # ---------------- JSON line
    main = result["prefill_2k"]
    tokens = main["tokens"]
    line = {
        "metric": METRIC,
        "value": main["tokens_per_s"],
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": main["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded: q,k,v ~ N(0,1), q,k L2-normalised, g=-softplus(N(0,1)), beta=sigmoid(N(0,1)))",
        "config": {"workload": "prefill_2k", "seqs": 1, "H": 16, "seq_len": 2048, "d_k": 128, "d_v": 128,
                   "state": "fp32", "S0": None, "parallelism": "replicas" if ws > 1 else "single",
                   "l2": "flushed before every timed step (256 MiB write)"},
        "roofline": main["roofline"],
        "roofline_prefill_10k": (result["prefill_10k"]["roofline"] if "prefill_10k" in result else None),
        "e2e": {"value": ws * tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": main["launches_per_step"] * args.steps,
        "clocks": clocks,
        "workloads": result,
        "peaks": pk,
        "context": "pages (Tesla C2075, Fermi): chunked rewrite 2.8x faster than the sequential scan; "
                   "whole-model prefill 408 tok/s at 2k, 361 tok/s at 10k",
    }
    if rank == 0:
        if ws == 1:
            line["cpu_baseline"] = cpu_baseline(args)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier(device_ids=[dev.index])
        dist.destroy_process_group()


def projection_entry(args, torch, gdn, dev, dist, pk, time_steps):
    """The int8-weight input projection of the layer (x [T, 1024] -> q, k, v, a, b with H = 16,
    d = 128: N = 6176 channels) at the prefill sizes (tensor-bound: flops over the measured dense
    bf16 peak) and at the decode size T = 64 (one token for each of the 64 sequences: bound by
    reading the int8 weights; bytes over the measured HBM bandwidth). L2 flushed before each step."""
    from linear_attention_recurrent_chunked_b200.workloads import make_projection
    out = {}
    for T in (2048, 10240, 64):
        p = make_projection(T, seed=0)
        x, w, sc = p["x"].to(dev), p["w"].to(dev), p["scale"].to(dev)
        H, dk, dv, D, N = p["H"], p["dk"], p["dv"], p["D"], p["N"]
        bufs = gdn.proj_w8(x, w, sc, H, dk, dv)
        fn = lambda: gdn.proj_w8(x, w, sc, H, dk, dv, out=bufs)
        ms = max_over_ranks(dist, statistics.mean(time_steps(fn, max(5, args.steps // 2), args.warmup)), dev)
        gdn.proj_w8(x, w, sc, H, dk, dv, out=bufs, check=True)
        flops = 2.0 * T * D * N
        nbytes = T * D * 2 + N * D + N * 4 + T * (2 * H * dk + H * dv) * 2 + 2 * T * H * 4
        tflops = flops / (ms * 1e-3) / 1e12
        gbs = nbytes / (ms * 1e-3) / 1e9
        entry = {"T": T, "D": D, "N": N, "ms": ms, "tflops": tflops, "GB_per_s": gbs,
                 "algorithmic_flops": flops, "algorithmic_bytes": nbytes}
        if flops / nbytes > pk["bf16"] * 1e12 / (pk["hbm"] * 1e9):
            entry["roofline"] = {"bound": "tensor", "achieved": tflops, "peak": pk["bf16"], "unit": "TFLOP/s",
                                 "frac": tflops / pk["bf16"], "peak_source": pk["src"]}
        else:
            entry["roofline"] = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                                 "frac": gbs / pk["hbm"], "peak_source": pk["src"]}
        out["T%d" % T] = entry
    return out


def attention_entry(args, torch, gdn, dev, dist, pk, time_steps):
    """The hybrid's causal attention layer (H = 16 heads of d = 128, bf16) at 2k and 10k tokens:
    device time per call with L2 flushed, and the causal flop count 4 d T (T + 1) / 2 per head
    (Q K^T and P V over the pairs j <= t) against the measured dense bf16 peak."""
    from linear_attention_recurrent_chunked_b200.workloads import make_attention
    out = {}
    for T in (2048, 10240):
        w = make_attention([T], H=16, seed=0)
        q, k, v = w["q"].to(dev), w["k"].to(dev), w["v"].to(dev)
        o = torch.empty_like(q)
        fn = lambda: gdn.attn_fwd(q, k, v, None, N=1, o=o)
        ms = max_over_ranks(dist, statistics.mean(time_steps(fn, max(5, args.steps // 2), args.warmup)), dev)
        gdn.attn_fwd(q, k, v, None, N=1, o=o, check=True)
        flops = 4.0 * w["d"] * T * (T + 1) / 2 * w["H"]
        tflops = flops / (ms * 1e-3) / 1e12
        out["T%d" % T] = {"T": T, "H": w["H"], "d": w["d"], "ms": ms, "tokens_per_s": T / (ms * 1e-3),
                          "algorithmic_flops": flops,
                          "roofline": {"bound": "tensor", "achieved": tflops, "peak": pk["bf16"], "unit": "TFLOP/s",
                                       "frac": tflops / pk["bf16"], "peak_source": pk["src"]}}
    return out


def decode_entry(args, torch, gdn, dev, dist, pk, make_decode):
    """256 decode steps (B=64, H=16, d=128) in one CUDA graph; 4 independent state
    sets used round-robin (256 MiB, larger than L2) so the state streams from HBM."""
    w = make_decode(seed=0)
    steps = w["steps"]
    q, k, v, g, beta = (w[x].to(dev) for x in ("q", "k", "v", "g", "beta"))
    q_raw, k_raw, a, b = (w[x].to(dev) for x in ("q_raw", "k_raw", "a", "b"))
    sets = [w["S"].to(dev) for _ in range(4)]
    o = torch.empty_like(v)
    nbytes = decode_bytes(w["B"], w["H"], w["d"])

    def run(state_sets, raw=False):
        for t in range(steps):
            if raw:  # raw q, k and gate logits: normalisation and gates inside the decode kernel
                gdn.decode_step_raw(q_raw[t], k_raw[t], v[t], a[t], b[t], state_sets[t % len(state_sets)], o=o[t])
            else:
                gdn.decode_step(q[t], k[t], v[t], g[t], beta[t], state_sets[t % len(state_sets)], o=o[t])

    out = {}
    for label, ss, raw in (("l2_cold_4sets", sets, False), ("l2_resident_1set", sets[:1], False),
                           ("raw_inputs_l2_cold_4sets", sets, True)):
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            run(ss, raw)  # warm-up outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            run(ss, raw)
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        reps = 5
        st = torch.cuda.Event(enable_timing=True)
        en = torch.cuda.Event(enable_timing=True)
        st.record()
        for _ in range(reps):
            graph.replay()
        en.record()
        torch.cuda.synchronize()
        ms = max_over_ranks(dist, st.elapsed_time(en) / reps, dev)
        gbs = steps * nbytes / (ms * 1e-3) / 1e9
        out[label] = {"ms_per_256_steps": ms, "us_per_step": ms * 1e3 / steps, "GB_per_s": gbs,
                      "frac_hbm": gbs / pk["hbm"]}
        del graph
    # per-launch duration of the decode kernel itself (events around each launch)
    gdn.profile_read()
    gdn.profile_enable(True)
    run(sets)
    torch.cuda.synchronize()
    gdn.profile_enable(False)
    kt = gdn.profile_read()
    if "decode_step" in kt:
        ms, n = kt["decode_step"]
        out["kernel_us_per_launch"] = ms * 1e3 / n
        out["kernel_GB_per_s"] = nbytes / (ms / n * 1e-3) / 1e9
    out["bytes_per_step"] = nbytes
    out["value"] = out["l2_cold_4sets"]["GB_per_s"]
    out["unit"] = "GB/s"
    return out


# ----------------------------------------------------------------------------- CPU oracle arms

def _oracle_rate(run, units: float, budget_s: float) -> tuple:
    """Repeat run() until budget_s of wall time has passed (at least once); units per second."""
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        dt = time.perf_counter() - t0
        if dt > budget_s:
            return reps * units / dt, reps, dt


def cpu_baseline(args, budget_s: float = 2.0):
    """The oracle (fp64 scan, C + OpenMP) timed on the host cores, on all of them and on one,
    for three workloads, each on a bounded sample (about budget_s of repeats per figure):

    * prefill_2k: all cores, whole 2048-token passes over the 16 heads; one core, 2 of the heads;
    * prefill_10k: all cores, whole 10240-token passes; one core, 1 head;
    * decode (256 chained steps, B=64, H=16): all cores, 8 of the 64 sequences; one core, 1.
      A chain of single-token steps is the scan over that sequence (the oracle's decode step is
      the scan over length-one sequences), so each sequence runs as a 256-token scan from S.

    Prefill figures are tokens/s of the whole workload (token-heads/s / 16); decode figures are
    state GB/s (the decode step's algorithmic bytes per (sequence, head) and step)."""
    import oracle
    from linear_attention_recurrent_chunked_b200.workloads import make_decode, make_prefill
    cores = oracle.num_threads()
    figs = {}

    def prefill_fig(name, heads_1core):
        w = make_prefill(name, seed=0)
        H = w["H"]
        full = [oracle.as_f64(w[x]) for x in ("q", "k", "v", "g", "beta")]
        S0 = oracle.as_f64(w["S0"])
        cu = w["cu_seqlens"]
        rate, reps, dt = _oracle_rate(lambda: oracle.scan(*full, S0=S0, cu_seqlens=cu), w["T_tot"] * H, budget_s)
        figs["%s_all_cores" % name] = {"value": rate / H, "unit": "tokens/s", "cores": cores,
                                       "sample": "%d whole passes (%d tokens x %d heads) in %.1f s"
                                                 % (reps, w["T_tot"], H, dt)}
        part = [x[:, :heads_1core].copy() for x in full]
        S0p = S0[:, :heads_1core].copy() if S0 is not None else None
        oracle.set_num_threads(1)
        try:
            rate, reps, dt = _oracle_rate(lambda: oracle.scan(*part, S0=S0p, cu_seqlens=cu),
                                          w["T_tot"] * heads_1core, budget_s)
        finally:
            oracle.set_num_threads(cores)
        figs["%s_1_core" % name] = {"value": rate / H, "unit": "tokens/s", "cores": 1,
                                    "sample": "%d passes over %d of %d heads (%d tokens) in %.1f s"
                                              % (reps, heads_1core, H, w["T_tot"], dt)}

    prefill_fig("prefill_2k", 2)
    prefill_fig("prefill_10k", 1)

    d = make_decode(seed=0)
    steps, H, dd = d["steps"], d["H"], d["d"]
    per_pair_step = decode_bytes(1, 1, dd)

    def decode_sample(nseq):
        # [steps, B, H, d] -> sequences of `steps` tokens: [nseq * steps, H, d]
        seq = lambda x: oracle.as_f64(x[:, :nseq].transpose(0, 1).reshape((nseq * steps,) + tuple(x.shape[2:])))
        args_o = [seq(d[x]) for x in ("q", "k", "v", "g", "beta")]
        S = oracle.as_f64(d["S"][:nseq])
        cu = [steps * i for i in range(nseq + 1)]
        return lambda: oracle.scan(*args_o, S0=S, cu_seqlens=cu), nseq * H * steps

    for label, nseq, nthreads in (("decode_all_cores", 8, cores), ("decode_1_core", 1, 1)):
        run, units = decode_sample(nseq)
        oracle.set_num_threads(nthreads)
        try:
            rate, reps, dt = _oracle_rate(run, units, budget_s)
        finally:
            oracle.set_num_threads(cores)
        figs[label] = {"value": rate * per_pair_step / 1e9, "unit": "GB/s", "cores": nthreads,
                       "sample": "%d runs of 256 chained steps for %d of 64 sequences x %d heads in %.1f s"
                                 % (reps, nseq, H, dt)}
    main = figs["prefill_2k_all_cores"]
    return {"value": main["value"], "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "prefill_2k: " + main["sample"] + "; other workloads and one core under 'figures'",
            "figures": figs}


def reference_arm(args):
    ws, rank, _ = dist_info()
    if rank != 0:
        return
    import oracle
    from linear_attention_recurrent_chunked_b200.workloads import make_prefill
    w = make_prefill("prefill_2k", seed=0)
    args_o = [oracle.as_f64(w[x]) for x in ("q", "k", "v", "g", "beta")]
    for _ in range(args.warmup):
        oracle.scan(*args_o, S0=None, cu_seqlens=w["cu_seqlens"])
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.scan(*args_o, S0=None, cu_seqlens=w["cu_seqlens"])
        times.append(time.perf_counter() - t0)
    ms = statistics.mean(times) * 1e3
    val = w["T_tot"] / (ms * 1e-3)
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill_2k", "seqs": 1, "H": 16, "seq_len": 2048, "d_k": 128, "d_v": 128},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": "one full prefill_2k pass (2048 tokens x 16 heads) per step"},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def case_arm(args):
    """Run one workload's library calls back to back (for ncu / launch lists): WARMUP+STEPS calls."""
    import torch

    from linear_attention_recurrent_chunked_b200 import gdn
    from linear_attention_recurrent_chunked_b200.workloads import make_decode, make_prefill
    dev = torch.device("cuda", 0)
    gdn.load_library()
    n = args.warmup + args.steps
    if args.case.startswith("attn_"):  # attn_<T>: causal attention over one sequence of T tokens, 16 heads
        from linear_attention_recurrent_chunked_b200.workloads import make_attention
        w = make_attention([int(args.case[5:])], H=16, seed=0)
        q, k, v = w["q"].to(dev), w["k"].to(dev), w["v"].to(dev)
        for _ in range(n):
            gdn.attn_fwd(q, k, v, None, N=1)
    elif args.case.startswith("proj_"):  # proj_<T>: the int8-weight input projection for T tokens
        from linear_attention_recurrent_chunked_b200.workloads import make_projection
        p = make_projection(int(args.case[5:]), seed=0)
        x, w, sc = p["x"].to(dev), p["w"].to(dev), p["scale"].to(dev)
        for _ in range(n):
            gdn.proj_w8(x, w, sc, p["H"], p["dk"], p["dv"])
    elif args.case == "decode":
        w = make_decode(seed=0)
        t = {k: w[k].to(dev) for k in ("q", "k", "v", "g", "beta", "S")}
        for i in range(n):
            j = i % w["steps"]
            gdn.decode_step(t["q"][j], t["k"][j], t["v"][j], t["g"][j], t["beta"][j], t["S"])
    else:
        name = args.case[5:] if args.case.startswith("scan_") else args.case
        name = {"2k": "prefill_2k", "10k": "prefill_10k"}.get(name, name)
        w = make_prefill(name, seed=0)
        t = {k: (v.to(dev) if hasattr(v, "to") else v) for k, v in w.items()}
        if w["N"] == 1:
            t["cu_seqlens"] = None  # as the timed arm calls it
        fn = gdn.seq_scan if args.case.startswith("scan_") else gdn.chunk_fwd
        for _ in range(n):
            fn(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], t["cu_seqlens"])
    torch.cuda.synchronize()
    print("case %s: %d calls done" % (args.case, n))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="main workload only (no 10k/varlen/decode/scan extras)")
    ap.add_argument("--case", default=None,
                    help="profiling mode: run only WARMUP+STEPS calls of one workload (prefill_2k, prefill_10k, "
                         "varlen, tiny, decode, scan_2k, proj_<T>) and print nothing but a one-line summary")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.case:
        case_arm(args)
    elif args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
