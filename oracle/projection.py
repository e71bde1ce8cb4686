"""Oracle for the recurrent layer's input projection with int8 weights.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages' system keeps the language model's weights in 8-bit form and dequantises them for
an FP32 vendor GEMM (page 1, abstract: int8 weights dequantised once; page 2, "Resumen
Tecnico", the GEMM item). For the recurrent layer that projection turns the hidden states x
[T, D] into the layer's raw inputs: q, k, v (H heads of dk, dk, dv values) and the two gate
logits a, b (one per head), which the recurrence then normalises and activates. The pages give
neither the layout nor the quantisation scheme; the plain reading adopted here is one weight
matrix of N = H (2 dk + dv) + 2 H output channels, stored as int8 codes w[n, j] with one fp32
scale per output channel, so that the dequantised weight is scale[n] * w[n, j], and the output
channels in the order q, k, v, a, b (head-major inside each). Written from that definition in
fp64:

    y[t, n] = sum_j x[t, j] * (scale[n] * w[n, j])
    q_raw[t, h, :] = y[t, h dk : (h + 1) dk]                        (columns 0 .. H dk)
    k_raw[t, h, :] = y[t, H dk + h dk : ...]                         (columns H dk .. 2 H dk)
    v[t, h, :]     = y[t, 2 H dk + h dv : ...]                       (columns 2 H dk .. 2 H dk + H dv)
    a[t, h]        = y[t, 2 H dk + H dv + h],   b[t, h] = y[t, 2 H dk + H dv + H + h]
"""
from __future__ import annotations

import numpy as np

from .scan import as_f64


def dequantise(w_int8, scale):
    """scale[n] * w[n, j] in fp64 (w: [N, D] int8 codes, scale: [N])."""
    return as_f64(w_int8) * as_f64(scale)[:, None]


def project(x, w_int8, scale):
    """y = x W^T with W the dequantised weight: x [T, D], w [N, D], scale [N] -> y [T, N] fp64."""
    return as_f64(x) @ dequantise(w_int8, scale).T


def split_outputs(y, H, dk, dv):
    """The layer's raw inputs from the projection's output columns (q, k, v, a, b order)."""
    T = y.shape[0]
    o = 0
    q = y[:, o:o + H * dk].reshape(T, H, dk)
    o += H * dk
    k = y[:, o:o + H * dk].reshape(T, H, dk)
    o += H * dk
    v = y[:, o:o + H * dv].reshape(T, H, dv)
    o += H * dv
    a = y[:, o:o + H]
    b = y[:, o + H:o + 2 * H]
    return q, k, v, a, b


def project_w8(x, w_int8, scale, H, dk, dv):
    """(q_raw, k_raw, v, a, b) in fp64 from hidden states x and the int8 projection."""
    return split_outputs(project(x, w_int8, scale), H, dk, dv)
