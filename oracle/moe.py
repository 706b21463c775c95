"""Oracle: MoE routing and the routed, per-expert SwiGLU layer with LoRA, forward and backward, fp64.

Test infrastructure only: nothing in the library calls this module.

Sources on the pages: MoE routing after OpenAI's Triton kernels, a grouped quantized matmul for the
experts, AITER's grouped matmuls for the non-quantized per-expert LoRA products, and the fast LoRA
backward for both the linear and the MoE layer (Show HN: LoRA over GGUF, "Things involved in the
training"); only active experts are loaded and their outputs are aggregated by a sparse reduce
(ai-manual.ru, "Fused dequant-matmul и MoE kernels: как это работает"); the load-balancing loss is
disabled (same Show HN list), so no auxiliary router loss appears here.

Routing (per token t, logits l_t over E experts):
  p_t = softmax(l_t); the k selected experts are the k largest logits, equal logits going to the
  lower expert index, in descending order (slot j = 0 is the largest); w_tj = p_{t,e_j} / sum of
  the selected p (equivalently the softmax over the k selected logits).
  counts_e = number of (token, slot) pairs routed to e; offsets = exclusive prefix sum of counts;
  perm lists the pairs (as t*k + j) sorted by (expert, token, slot); inv_perm is its inverse.

Expert e (x a token row, W_gu the fused [2I, H] gate/up weight with gate rows [0, I) and up rows
[I, 2I), W_d the [H, I] down weight, one LoRA adapter on each, s = alpha / r):
  gu = x W_gu^T + s (x A_gu^T) B_gu^T ; g = gu[:I], u = gu[I:]
  h  = silu(g) * u                          silu(g) = g / (1 + exp(-g))
  o  = h W_d^T + s (h A_d^T) B_d^T
  Y_t = sum over slots j (in slot order) of w_tj * o_tj
Backward, with dh_u = dY_t W_d + s (dY_t B_d) A_d (the down input-gradient before the routing
weight), dw_tj = <dh_u, h>, dh = w_tj dh_u, sigma = 1/(1+exp(-g)):
  dg = dh * u * sigma * (1 + g (1 - sigma)) ; du = dh * silu(g)
  dx_pair = d[g|u] W_gu + s (d[g|u] B_gu) A_gu ; dX_t = sum over slots of dx_pair
  dA_gu_e = sum_p (s d[g|u]_p B_gu)^T x_p      dB_gu_e = s sum_p d[g|u]_p^T (x_p A_gu^T)
  dA_d_e  = sum_p (s w_p dY_t B_d)^T h_p       dB_d_e  = s sum_p (w_p dY_t)^T (h_p A_d^T)
  d_logits on the k selected logits of token t: w_j (dw_j - sum_i w_i dw_i); zero elsewhere.

Rounding points (``mirror=True``): the layer stores h and d[g|u] in bf16 and feeds those stored
values to the matmuls that take them (h: the down projection and its adapter input h A_d^T;
d[g|u]: the gate/up input-gradient and its adapter input s d[g|u] B_gu); the oracle rounds the same
values at the same places. g and u are kept at fp32 accuracy (the layer saves them in fp32), so the
SwiGLU derivative takes them unrounded. The routing-weight gradient <dh_u, h> and the adapter
gradients dA_d and dB_gu (sums over an expert's pairs only) take h and d[g|u] at fp32 accuracy
(the layer carries them as a bf16 pair there), so the oracle uses the unrounded values for those. The weighted pair outputs w*o and the pair input-gradients dx_pair are kept in fp32 (no
rounding point). Weights are the bf16 decode. With ``mirror=False`` and ``round_weights=False`` the
function is smooth (finite-difference checks).

Why these are not rounding points: a bf16 rounding is a decision, and an fp32 and an fp64
evaluation of the same value land on neighbouring bf16 values now and then. A flipped g or u moves
the SwiGLU derivative by about 2^-8 relative in that entry, and for an expert with few pairs one
such entry can dominate an element of dB_gu (a sum over those pairs only). A flipped h moves one
term of <dh_u, h> by 2^-8 of itself, and single terms h_i dh_u_i are heavy-tailed (products of
near-Gaussian values): one flip can move a token's router-logit gradient by more than 1e-2 of its
RMS.
"""
from __future__ import annotations

import numpy as np

from .gguf_blocks import decode_exact, deq_bf16, round_bf16


def route(logits: np.ndarray, k: int):
    """logits [T, E] fp64 -> (idx [T,k] int32, w [T,k] fp64, counts [E], offsets [E+1], perm, inv_perm)."""
    T, E = logits.shape
    order = np.argsort(-logits, axis=1, kind="stable")      # ties keep the lower index first
    idx = order[:, :k].astype(np.int32)
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    psel = np.take_along_axis(p, idx, axis=1)
    w = psel / psel.sum(axis=1, keepdims=True)
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    pair = np.arange(T * k, dtype=np.int64)
    key = idx.ravel().astype(np.int64) * (T * k) + pair      # (expert, token, slot) order
    perm = np.argsort(key, kind="stable").astype(np.int32)
    inv_perm = np.empty_like(perm)
    inv_perm[perm] = np.arange(T * k, dtype=np.int32)
    return idx, w, counts, offsets, perm, inv_perm


def _silu(g):
    return g / (1.0 + np.exp(-g))


def _sigmoid(g):
    return 1.0 / (1.0 + np.exp(-g))


class LazyExpertWeights:
    """One expert's decoded weight matrix on demand (``W[e]``), keeping only the last one decoded:
    bounds host memory when the layer is evaluated at full size, where all experts' decoded
    weights would not fit."""

    def __init__(self, qtype, packed, rows, cols, round_weights=True):
        self.qtype, self.packed, self.rows, self.cols = qtype, packed, rows, cols
        self.dec = deq_bf16 if round_weights else decode_exact
        self._e, self._w = None, None

    def __getitem__(self, e):
        if e != self._e:
            self._w = None
            self._w = self.dec(self.qtype, self.packed[e], self.rows, self.cols)
            self._e = e
        return self._w


def expert_weights(qtype, w_gu, w_d, H, I, round_weights=True, experts=None, lazy=False):
    """Decoded (W_gu [E,2I,H], W_d [E,H,I]). With `experts`, only those are decoded (the others
    stay zero and must then be skipped by moe_fwd / moe_bwd through the same `experts`). With
    `lazy`, each expert is decoded when moe_fwd / moe_bwd reach it."""
    dec = deq_bf16 if round_weights else decode_exact
    E = w_gu.shape[0]
    if lazy:
        return (LazyExpertWeights(qtype, w_gu, 2 * I, H, round_weights),
                LazyExpertWeights(qtype, w_d, H, I, round_weights))
    if experts is None:
        Wgu = np.stack([dec(qtype, w_gu[e], 2 * I, H) for e in range(E)])
        Wd = np.stack([dec(qtype, w_d[e], H, I) for e in range(E)])
        return Wgu, Wd
    return ({e: dec(qtype, w_gu[e], 2 * I, H) for e in experts},
            {e: dec(qtype, w_d[e], H, I) for e in experts})


def moe_fwd(Wgu, Wd, X, idx, w, counts, offsets, perm, A_gu, B_gu, A_d, B_d, s, mirror=True, experts=None):
    """Grouped forward. Returns (Y [T,H], saved) where saved holds per-pair (perm order) tensors.
    With `experts`, only those experts' pairs are computed (Y is then complete only for tokens
    whose selected experts all lie in the subset)."""
    rb = round_bf16 if mirror else (lambda v: v)
    T, H = X.shape
    k = idx.shape[1]
    E = len(offsets) - 1
    I = B_gu.shape[1] // 2
    P = T * k
    tok = perm // k
    slot = perm % k
    wp = w[tok, slot]
    g = np.zeros((P, I)); u = np.zeros((P, I)); h = np.zeros((P, I)); h_exact = np.zeros((P, I))
    Hgu = np.zeros((P, A_gu.shape[1])); Hd = np.zeros((P, A_d.shape[1]))
    pair_out = np.zeros((P, H))
    for e in (range(E) if experts is None else experts):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        x = X[tok[a:b]]
        Hgu[a:b] = x @ A_gu[e].T
        gu = x @ Wgu[e].T + s * (Hgu[a:b] @ B_gu[e].T)
        ge, ue = gu[:, :I], gu[:, I:]
        h_exact[a:b] = _silu(ge) * ue
        h[a:b] = rb(h_exact[a:b])
        g[a:b] = ge
        u[a:b] = ue
        Hd[a:b] = h[a:b] @ A_d[e].T
        o = h[a:b] @ Wd[e].T + s * (Hd[a:b] @ B_d[e].T)
        pair_out[a:b] = wp[a:b, None] * o
    Y = np.zeros((T, H))
    inv = np.empty(P, np.int64)
    inv[perm] = np.arange(P)
    for j in range(k):                                   # slot order
        Y += pair_out[inv[np.arange(T) * k + j]]
    saved = dict(g=g, u=u, h=h, h_exact=h_exact, Hgu=Hgu, Hd=Hd, pair_out=pair_out)
    return Y, saved


def moe_bwd(Wgu, Wd, X, dY, idx, w, counts, offsets, perm, A_gu, B_gu, A_d, B_d, s, saved,
            mirror=True, experts=None):
    """Grouped backward. Returns dict(dX, dA_gu, dB_gu, dA_d, dB_d, d_logits_sel [T,k], dw [T,k]).
    `experts` restricts the work as in moe_fwd."""
    rb = round_bf16 if mirror else (lambda v: v)
    T, H = X.shape
    k = idx.shape[1]
    E = len(offsets) - 1
    I = B_gu.shape[1] // 2
    P = T * k
    tok = perm // k
    slot = perm % k
    wp = w[tok, slot]
    g, u, h, Hgu, Hd = saved["g"], saved["u"], saved["h"], saved["Hgu"], saved["Hd"]
    dA_gu = np.zeros_like(A_gu); dB_gu = np.zeros_like(B_gu)
    dA_d = np.zeros_like(A_d); dB_d = np.zeros_like(B_d)
    dw_p = np.zeros(P)
    dx_pair = np.zeros((P, H))
    for e in (range(E) if experts is None else experts):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        dy = dY[tok[a:b]]
        Gd = s * (dy @ B_d[e])
        dh_u = dy @ Wd[e] + Gd @ A_d[e]
        dw_p[a:b] = (dh_u * saved["h_exact"][a:b]).sum(axis=1)
        dh = wp[a:b, None] * dh_u
        sg = _sigmoid(g[a:b])
        dg = dh * u[a:b] * sg * (1.0 + g[a:b] * (1.0 - sg))
        du = dh * (g[a:b] * sg)
        dgu_exact = np.concatenate([dg, du], axis=1)
        dgu = rb(dgu_exact)
        dA_d[e] = (wp[a:b, None] * Gd).T @ saved["h_exact"][a:b]
        dB_d[e] = s * ((wp[a:b, None] * dy).T @ Hd[a:b])
        Ggu = s * (dgu @ B_gu[e])
        dx_pair[a:b] = dgu @ Wgu[e] + Ggu @ A_gu[e]
        dA_gu[e] = Ggu.T @ X[tok[a:b]]
        dB_gu[e] = s * (dgu_exact.T @ Hgu[a:b])
    inv = np.empty(P, np.int64)
    inv[perm] = np.arange(P)
    dX = np.zeros((T, H))
    dw = np.zeros((T, k))
    for j in range(k):
        sel = inv[np.arange(T) * k + j]
        dX += dx_pair[sel]
        dw[:, j] = dw_p[sel]
    d_logits_sel = w * (dw - (w * dw).sum(axis=1, keepdims=True))
    return dict(dX=dX, dA_gu=dA_gu, dB_gu=dB_gu, dA_d=dA_d, dB_d=dB_d, dw=dw,
                d_logits_sel=d_logits_sel, dx_pair=dx_pair)


def scatter_d_logits(idx, d_logits_sel, E):
    """Full [T, E] router-logit gradient (zero on unselected experts)."""
    T, k = idx.shape
    out = np.zeros((T, E))
    np.put_along_axis(out, idx.astype(np.int64), d_logits_sel, axis=1)
    return out
