"""Oracle: quantized lm_head with cross-entropy over the vocabulary, forward and backward, fp64.

Test infrastructure only: nothing in the library calls this module.

The recipe trains with a Liger-style chunked cross-entropy over the quantized matmul's logits (Show HN:
LoRA over GGUF, "Things involved in the training"): the logits of the quantized output projection
feed a per-token cross-entropy, chunked over tokens so the full logits never exist at once. Chunking
changes where the work happens, not what is computed, so the oracle is the plain definition:

  logits = X deq(W)^T                        [M, V]
  loss_t = logsumexp(logits_t) - logits_t[label_t]          (0 for a negative label: ignored)
  D      = (softmax(logits) - onehot(label)) * grad_scale   (zero rows for ignored tokens)
  dX     = D deq(W)                          the gradient of grad_scale * sum_t loss_t

deq(W) is the bf16 decode (oracle.gguf_blocks.deq_bf16). Rounding point (``mirror=True``): the layer
feeds D to the input-gradient matmul in bf16, so dX uses the bf16 rounding of D.
"""
from __future__ import annotations

import numpy as np

from .gguf_blocks import round_bf16


def lm_head_ce(W, X, labels, grad_scale=1.0, mirror=True):
    """W [V, K] decoded, X [M, K], labels [M] -> (loss [M], dX [M, K], D [M, V])."""
    W = np.asarray(W, np.float64)
    X = np.asarray(X, np.float64)
    labels = np.asarray(labels)
    M = X.shape[0]
    logits = X @ W.T
    mx = logits.max(axis=1, keepdims=True)
    lse = (mx + np.log(np.exp(logits - mx).sum(axis=1, keepdims=True)))[:, 0]
    keep = labels >= 0
    lab = np.where(keep, labels, 0)
    loss = np.where(keep, lse - logits[np.arange(M), lab], 0.0)
    D = np.exp(logits - lse[:, None])
    D[np.arange(M), lab] -= 1.0
    D = np.where(keep[:, None], D * grad_scale, 0.0)
    Dm = round_bf16(D) if mirror else D
    return loss, Dm @ W, D
