"""Oracle for the layer's input preparation: from raw projections to the rule's inputs.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The gated delta rule consumes unit-norm queries and keys, a decay alpha_t = exp(g_t) in (0, 1)
and a write strength beta_t in (0, 1). In a gated-delta-net layer (the recurrent layer of the
"hybrid gated-delta-net backbone", page 1 abstract, result (i)) these come from raw per-token
projections: q and k are L2-normalised over the head dimension, the decay is
alpha = exp(-softplus(a)) of a raw gate logit a, and the write strength is beta = sigmoid(b)
of a raw logit b. The pages name the layer but print none of this; the recipe is the plain
reading of the layer's input contract and the one the synthetic workloads use. Every step is
written out from its definition, in fp64:

    x_hat     = x / max(||x||_2, eps)          (eps = 1e-12, per token and head)
    softplus  = log(1 + exp(a)),  evaluated as max(a, 0) + log(1 + exp(-|a|))
    g         = -softplus(a)                    (natural-log decay, alpha = exp(g))
    beta      = 1 / (1 + exp(-b)),  evaluated as exp(b) / (1 + exp(b)) for b < 0

(The two-branch forms are the same functions; they only avoid exp overflow.)
"""
from __future__ import annotations

import numpy as np

from .scan import as_f64

EPS = 1e-12


def l2_normalise(x, eps: float = EPS):
    """x / max(||x||, eps) over the last axis, fp64."""
    x = as_f64(x)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, eps)


def softplus(a):
    a = as_f64(a)
    return np.maximum(a, 0.0) + np.log1p(np.exp(-np.abs(a)))


def sigmoid(b):
    b = as_f64(b)
    z = np.exp(-np.abs(b))  # 1 / (1 + e^-b) for b >= 0, e^b / (1 + e^b) for b < 0: no overflow
    return np.where(b >= 0.0, 1.0 / (1.0 + z), z / (1.0 + z))


def prep_inputs(q_raw, k_raw, a, b):
    """(q, k, g, beta) of the rule from raw q, k [.., d] and raw gate logits a, b [..]: q and k
    normalised, g = -softplus(a), beta = sigmoid(b); all fp64."""
    return l2_normalise(q_raw), l2_normalise(k_raw), -softplus(a), sigmoid(b)
