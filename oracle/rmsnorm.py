"""Oracle: RMSNorm in front of the layer's first projection, forward and backward, fp64.

Test infrastructure only: nothing in the library calls this module.

The recipe's training stack normalizes each token with Liger's RMSNorm (Show HN:
LoRA over GGUF, "Things involved in the training") before the projections the layer implements. The
pages print no formula; this is the standard definition. For a token row x of K values, a frozen
gain g (part of the base model, never updated) and eps:

  forward   r = 1 / sqrt(mean_k(x_k^2) + eps)        (kept for the backward)
            x_n = x * r * g                           (the projection's input)
  backward  dL/dx_j = r g_j d_j - (r^3 x_j / K) sum_k x_k g_k d_k,   d = dL/dx_n

Rounding point (``mirror=True``): the layer stores x_n in bf16 (the projection's A operand is bf16), so
the forward returns the bf16 rounding of x_n; r and the backward stay fp64.
"""
from __future__ import annotations

import numpy as np

from .gguf_blocks import round_bf16


def rmsnorm_fwd(X, g, eps, mirror=True):
    """X [M, K], g [K] -> (Xn [M, K], r [M])."""
    X = np.asarray(X, np.float64)
    r = 1.0 / np.sqrt(np.mean(X * X, axis=1) + eps)
    Xn = X * r[:, None] * np.asarray(g, np.float64)[None, :]
    return (round_bf16(Xn) if mirror else Xn), r


def rmsnorm_bwd(X, g, r, dXn):
    """dX [M, K] from d = dXn [M, K]."""
    X = np.asarray(X, np.float64)
    g = np.asarray(g, np.float64)
    d = np.asarray(dXn, np.float64)
    K = X.shape[1]
    s = np.sum(X * g[None, :] * d, axis=1)
    return r[:, None] * g[None, :] * d - (r ** 3 / K)[:, None] * X * s[:, None]
