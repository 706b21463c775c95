"""Oracle: frozen block-quantized linear layer with a LoRA adapter, forward and backward, fp64.

Test infrastructure only: nothing in the library calls this module.

What it computes (the method's layer: a frozen GGUF base weight plus a trainable low-rank adapter,
whose backward the recipe takes from an Unsloth-style fast LoRA formula, Show HN: LoRA over GGUF,
"Things involved in the training"; the pages print no formula, so the one below is the plain chain
rule of the layer's definition):

  forward   H  = X A^T                       [M, r]   (kept for the backward)
            Y  = X deq(W)^T + s H B^T        [M, N]
  backward  G  = s dY B                      [M, r]
            dX = dY deq(W) + G A             [M, K]
            dA = G^T X                       [r, K]
            dB = s dY^T H                    [N, r]
  W is frozen: no gradient is formed for it.

deq(W) is the bf16 rounding of the exact decode (the bf16 weight tile is what the layer multiplies);
``round_weights=False`` uses the exact decode instead (used for finite-difference checks, which
need a smooth function of the inputs). Every sum is an fp64 matmul over exact input values.
"""
from __future__ import annotations

import numpy as np

from .gguf_blocks import decode_exact, deq_bf16


def weights(qtype, wq, N, K, round_weights=True) -> np.ndarray:
    return deq_bf16(qtype, wq, N, K) if round_weights else decode_exact(qtype, wq, N, K)


def linear_fwd(W: np.ndarray, X: np.ndarray, A: np.ndarray, B: np.ndarray, s: float):
    """Returns (Y, H). W [N,K] decoded weights; X [M,K]; A [r,K]; B [N,r]; all fp64."""
    H = X @ A.T
    Y = X @ W.T + s * (H @ B.T)
    return Y, H


def linear_bwd(W, X, dY, A, B, s, H=None):
    """Returns (dX, dA, dB, G)."""
    if H is None:
        H = X @ A.T
    G = s * (dY @ B)
    dX = dY @ W + G @ A
    dA = G.T @ X
    dB = s * (dY.T @ H)
    return dX, dA, dB, G
