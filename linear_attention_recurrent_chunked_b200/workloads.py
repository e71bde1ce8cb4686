"""Seeded synthetic workloads for the gated-delta-rule forward.

This module is the ONLY code shared by the CUDA path's tests/bench and the
oracle: it draws inputs and holds none of the method's arithmetic. Everything
is generated on the CPU with torch's own ``randn`` / ``F.normalize`` /
``softplus`` / ``sigmoid`` / dtype casts, so both sides consume the same,
already-cast values (the pages' rule of calling the reference operator rather
than re-implementing a rounding-sensitive step, page 1 abstract result (ii)).

The pages measure on no public dataset; the shapes below are the synthetic
workloads the library is benchmarked and tested on:

* ``tiny``        B=1, H=2,  T=256,   d=64,  fp32 inputs, S0 = 0
* ``prefill_2k``  B=1, H=16, T=2048,  d=128, bf16 inputs, S0 = 0
* ``prefill_10k`` B=1, H=16, T=10240, d=128, bf16 inputs, S0 ~ N(0, 0.02^2)
* ``varlen``      8 packed sequences, lengths uniform in [512, 4096], H=16,
                  d=128, bf16 inputs, per-sequence S0 ~ N(0, 0.02^2)
* ``decode``      B=64, H=16, d=128, fp32 state S ~ N(0, 0.02^2), 256 steps,
                  fresh bf16 q,k,v and fp32 g,beta per step

Value recipe (every config): q,k,v ~ N(0,1) drawn in fp32; q and k are
L2-normalised over the head dimension in fp32 (x / max(||x||, 1e-12)) and
then cast to the input dtype (round to nearest even); g = -softplus(N(0,1))
(natural-log decay, alpha = exp(g)); beta = sigmoid(N(0,1)); both fp32.
Draw order from one ``torch.Generator().manual_seed(seed)``: [varlen lengths],
q, k, v, g, beta, S0. The same draws before normalisation and activation (q_raw,
k_raw in the input dtype; gate logits a, b with g = -softplus(a), beta =
sigmoid(b)) are returned too, for the entry points that take raw inputs. ``stress=True`` replaces the decays by slow ones
(g ~ -U(0, 0.01)) and pushes beta towards one (sigmoid(N(0,1) + 3)), so the
state carries information across thousands of tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Prefill:
    name: str
    H: int
    d: int
    dtype: str  # "f32" or "bf16"
    seqlens: Optional[List[int]] = None  # fixed lengths; None => drawn (varlen)
    n_seqs: int = 1
    s0: bool = False
    len_range: tuple = (512, 4096)


@dataclass(frozen=True)
class Decode:
    name: str
    B: int
    H: int
    d: int
    steps: int
    dtype: str = "bf16"


PREFILL = {
    "tiny": Prefill("tiny", H=2, d=64, dtype="f32", seqlens=[256]),
    "prefill_2k": Prefill("prefill_2k", H=16, d=128, dtype="bf16", seqlens=[2048]),
    "prefill_10k": Prefill("prefill_10k", H=16, d=128, dtype="bf16", seqlens=[10240], s0=True),
    "varlen": Prefill("varlen", H=16, d=128, dtype="bf16", seqlens=None, n_seqs=8, s0=True),
}
DECODE = Decode("decode", B=64, H=16, d=128, steps=256)

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _unit(x: torch.Tensor) -> torch.Tensor:
    return F.normalize(x, p=2.0, dim=-1, eps=1e-12)


def draw_tokens(gen: torch.Generator, shape_qk, shape_v, shape_gate, dtype: str, stress: bool = False,
                raw_out: Optional[dict] = None):
    """q, k, v, g, beta in the draw order above. Returns CPU tensors. If ``raw_out`` is a dict,
    it also receives the same draws before normalisation and activation: q_raw, k_raw (the N(0,1)
    draws cast to the input dtype), a and b (the fp32 gate logits, so that g = -softplus(a) and
    beta = sigmoid(b); the stress recipe has no such logits and gives none)."""
    tdt = TORCH_DTYPE[dtype]
    q32 = torch.randn(shape_qk, generator=gen, dtype=torch.float32)
    k32 = torch.randn(shape_qk, generator=gen, dtype=torch.float32)
    q = _unit(q32).to(tdt)
    k = _unit(k32).to(tdt)
    v = torch.randn(shape_v, generator=gen, dtype=torch.float32).to(tdt)
    g_raw = torch.randn(shape_gate, generator=gen, dtype=torch.float32)
    b_raw = torch.randn(shape_gate, generator=gen, dtype=torch.float32)
    if stress:
        g = -0.01 * torch.rand(shape_gate, generator=gen, dtype=torch.float32)
        beta = torch.sigmoid(b_raw + 3.0)
    else:
        g = -F.softplus(g_raw)
        beta = torch.sigmoid(b_raw)
        if raw_out is not None:
            raw_out.update(q_raw=q32.to(tdt).contiguous(), k_raw=k32.to(tdt).contiguous(), a=g_raw.contiguous(),
                           b=b_raw.contiguous())
    return q.contiguous(), k.contiguous(), v.contiguous(), g.contiguous(), beta.contiguous()


def make_prefill(cfg, seed: int = 0, stress: bool = False, seqlens: Optional[List[int]] = None,
                 H: Optional[int] = None, d: Optional[int] = None, dtype: Optional[str] = None,
                 s0: Optional[bool] = None):
    """Inputs of a prefill workload (``cfg`` a name or a ``Prefill``); keyword
    overrides give the parity tests smaller shapes with the same recipe.

    Returns a dict of CPU tensors: q,k [T_tot,H,d] and v [T_tot,H,d] in the
    input dtype, g,beta [T_tot,H] fp32, S0 [N,H,d,d] fp32 or None, cu_seqlens
    [N+1] int32, plus ``name``, ``dtype``, ``N``, ``H``, ``d``, ``T_tot``.
    """
    if isinstance(cfg, str):
        cfg = PREFILL[cfg]
    H = cfg.H if H is None else H
    d = cfg.d if d is None else d
    dtype = cfg.dtype if dtype is None else dtype
    s0 = cfg.s0 if s0 is None else s0
    gen = torch.Generator().manual_seed(seed)
    if seqlens is None:
        seqlens = cfg.seqlens
    if seqlens is None:
        lo, hi = cfg.len_range
        seqlens = torch.randint(lo, hi + 1, (cfg.n_seqs,), generator=gen).tolist()
    seqlens = [int(x) for x in seqlens]
    N = len(seqlens)
    T_tot = sum(seqlens)
    raw = {}
    q, k, v, g, beta = draw_tokens(gen, (T_tot, H, d), (T_tot, H, d), (T_tot, H), dtype, stress, raw)
    S0 = (0.02 * torch.randn((N, H, d, d), generator=gen, dtype=torch.float32)).contiguous() if s0 else None
    cu = torch.zeros(N + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    return dict(name=cfg.name, dtype=dtype, N=N, H=H, d=d, T_tot=T_tot, seqlens=seqlens,
                q=q, k=k, v=v, g=g, beta=beta, S0=S0, cu_seqlens=cu, **raw)


def make_decode(cfg: Decode = DECODE, seed: int = 0, steps: Optional[int] = None, B: Optional[int] = None,
                H: Optional[int] = None, d: Optional[int] = None, dtype: Optional[str] = None,
                stress: bool = False):
    """Inputs of the decode workload: per-step q,k,v [steps,B,H,d], g,beta
    [steps,B,H], and the initial state S [B,H,d,d] fp32 ~ N(0, 0.02^2)."""
    steps = cfg.steps if steps is None else steps
    B = cfg.B if B is None else B
    H = cfg.H if H is None else H
    d = cfg.d if d is None else d
    dtype = cfg.dtype if dtype is None else dtype
    gen = torch.Generator().manual_seed(seed)
    raw = {}
    q, k, v, g, beta = draw_tokens(gen, (steps, B, H, d), (steps, B, H, d), (steps, B, H), dtype, stress, raw)
    S = (0.02 * torch.randn((B, H, d, d), generator=gen, dtype=torch.float32)).contiguous()
    return dict(name=cfg.name, dtype=dtype, B=B, H=H, d=d, steps=steps,
                q=q, k=k, v=v, g=g, beta=beta, S=S, **raw)


def make_projection(T: int, D: int = 1024, H: int = 16, dk: int = 128, dv: int = 128, seed: int = 0):
    """Inputs of the int8-weight input projection: hidden states x [T, D] ~ N(0, 1) in bf16, and a
    weight matrix W [N, D] ~ N(0, 1/D) (N = H (2 dk + dv) + 2 H output channels) quantised
    symmetrically per output channel to int8 codes w and fp32 scales (scale = max|W_n| / 127,
    w = round(W / scale)). Draw order: x, then W. Returns CPU tensors x, w, scale and the sizes."""
    gen = torch.Generator().manual_seed(seed)
    N = H * (2 * dk + dv) + 2 * H
    x = torch.randn((T, D), generator=gen, dtype=torch.float32).to(torch.bfloat16).contiguous()
    W = torch.randn((N, D), generator=gen, dtype=torch.float32) / float(D) ** 0.5
    scale = (W.abs().amax(dim=1) / 127.0).clamp_min(1e-12)
    w = torch.round(W / scale[:, None]).clamp(-127, 127).to(torch.int8).contiguous()
    return dict(x=x, w=w, scale=scale.contiguous(), T=T, D=D, H=H, dk=dk, dv=dv, N=N)


def make_attention(seqlens: List[int], H: int = 16, d: int = 128, seed: int = 0):
    """Inputs of the causal attention layer over packed sequences: q, k, v [T, H, d] ~ N(0, 1) in
    bf16 (draw order q, k, v), cu_seqlens [N+1] int32, and the sizes."""
    gen = torch.Generator().manual_seed(seed)
    T = int(sum(seqlens))
    q, k, v = (torch.randn((T, H, d), generator=gen, dtype=torch.float32).to(torch.bfloat16).contiguous()
               for _ in range(3))
    cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    return dict(q=q, k=k, v=v, cu_seqlens=cu, seqlens=[int(x) for x in seqlens], T=T, H=H, d=d,
                N=len(seqlens), max_len=max(seqlens) if seqlens else 0)
