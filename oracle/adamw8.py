"""Oracle: one AdamW step on the adapter parameters with 8-bit block-wise quantized moments.

Test infrastructure only: nothing in the library calls this module.

The recipe's optimizer is the bitsandbytes 8-bit AdamW (Show HN: LoRA over GGUF, "Things involved in
the training"). The pages give no formula; this is the plainest reading of that optimizer, written
from the published methods it combines:

* AdamW with decoupled weight decay (Loshchilov and Hutter): for gradient g at step t,
      m = b1 m + (1 - b1) g ;  v = b2 v + (1 - b2) g^2
      p = p - lr (m / c1 / (sqrt(v / c2) + eps) + wd p),   c1 = 1 - b1^t, c2 = 1 - b2^t.
* Block-wise 8-bit states (Dettmers et al., 8-bit optimizers via block-wise quantization): m and v
  live as one byte per value plus one fp32 absmax per block of 256 values; a byte q stands for
  absmax * T[q], T the block-normalized code table; after the update each block's new absmax is
  max |value| over the block and each value takes the code whose table entry is nearest to
  value / absmax (equal distances go to the smaller entry); a block whose values are all zero keeps
  absmax 0 and the zero code.
* Dynamic tree codes (the same paper; Dettmers, 8-bit approximations for parallelism): a code's
  bits after the optional sign bit are E zero bits (the decade, 10^-E), a one bit (the indicator)
  and F, the remaining B bits, a linear fraction of the decade:
      |T| = (0.1 + 0.9 (F + 1/2) / 2^B) / 10^E ;  all-zero bits (no indicator) code 0.
  m uses the signed table (bit 7 is the sign, 7 bits after it); v, never negative, the unsigned
  table (8 bits). Which table entries exist, their order and the tie rule are this module's
  reading; the step the layer takes must reproduce it.

Precision. The codes are integers decided by floating point, so this module takes every decision in
fp32 with a fixed order of operations (numpy fp32 scalars and arrays, each operation rounded to
nearest even, no fused multiply-add); the table entries are computed in fp64 from the formula above
and rounded once to fp32. With ``exact=True`` every value is fp64 and the states stay unquantized
(the plain AdamW step, for the closed-form pins).
"""
from __future__ import annotations

import numpy as np

QBLOCK = 256


def dynamic_table(signed: bool) -> np.ndarray:
    """The code table: T[q] for q in 0..255 as fp32 (signed: bit 7 = sign, code 0x80 = -0 -> 0)."""
    nbits = 7 if signed else 8
    vals = np.zeros(256, np.float64)
    for q in range(256):
        mag_bits = q & ((1 << nbits) - 1)
        neg = signed and (q >> 7) & 1
        if mag_bits == 0:
            v = 0.0
        else:
            E = nbits - mag_bits.bit_length()      # leading zeros below the top bit of the field
            B = nbits - E - 1                       # bits after the indicator
            F = mag_bits & ((1 << B) - 1)
            v = (0.1 + 0.9 * (F + 0.5) / 2.0 ** B) / float(10 ** E)
        vals[q] = -v if neg else v
    return vals.astype(np.float32)


def _sorted_codes(signed: bool):
    """Distinct table values in ascending order, with the code each stands for (the zero value is
    code 0; the signed table's -0 code 0x80 is never produced)."""
    T = dynamic_table(signed)
    order = np.argsort(T.astype(np.float64), kind="stable")
    vals, codes = [], []
    for q in order:
        if q == 0x80 and signed:
            continue
        vals.append(T[q])
        codes.append(q)
    return np.array(vals, np.float32), np.array(codes, np.uint8)


def encode(x: np.ndarray, signed: bool) -> np.ndarray:
    """Nearest code of each fp32 value x (|x| <= 1): the entry minimizing |x - T| in fp32, equal
    distances going to the smaller entry (brute force over the table)."""
    vals, codes = _sorted_codes(signed)
    x = np.asarray(x, np.float32)
    dist = np.abs(x[:, None] - vals[None, :])           # fp32
    return codes[np.argmin(dist, axis=1)]              # first minimum = smaller entry


def decode(q: np.ndarray, absmax: np.ndarray, signed: bool) -> np.ndarray:
    """fp32 values absmax[block] * T[q] (one fp32 multiplication)."""
    T = dynamic_table(signed)
    n = q.size
    a = np.repeat(np.asarray(absmax, np.float32), QBLOCK)[:n]
    return (a * T[q]).astype(np.float32)


def quantize_blocks(x: np.ndarray, signed: bool):
    """(codes, absmax) of fp32 values: absmax = max |x| per block; codes of x / absmax."""
    x = np.asarray(x, np.float32)
    n = x.size
    nb = (n + QBLOCK - 1) // QBLOCK
    pad = np.zeros(nb * QBLOCK, np.float32)
    pad[:n] = x
    absmax = np.abs(pad.reshape(nb, QBLOCK)).max(axis=1).astype(np.float32)
    a = np.repeat(absmax, QBLOCK)[:n]
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(a > 0, x / np.where(a > 0, a, np.float32(1)), np.float32(0)).astype(np.float32)
    return encode(y, signed), absmax


def adamw8_step(p, g, m_q, m_abs, v_q, v_abs, lr, b1, b2, eps, wd, c1, c2):
    """One step. p, g fp32 [n]; states as codes [n] uint8 and absmax [ceil(n/256)] fp32; c1, c2 the
    bias corrections 1 - b1^t, 1 - b2^t given as fp32. Returns (p, m_q, m_abs, v_q, v_abs)."""
    f = np.float32
    p = np.asarray(p, f)
    g = np.asarray(g, f)
    lr, b1, b2, eps, wd, c1, c2 = (f(x) for x in (lr, b1, b2, eps, wd, c1, c2))
    m = decode(m_q, m_abs, True)
    v = decode(v_q, v_abs, False)
    m = b1 * m + (f(1) - b1) * g
    v = b2 * v + (f(1) - b2) * (g * g)
    mh = m / c1
    vh = v / c2
    p = p - lr * (mh / (np.sqrt(vh) + eps) + wd * p)
    mq, ma = quantize_blocks(m, True)
    vq, va = quantize_blocks(v, False)
    return p.astype(f), mq, ma, vq, va


def adamw_exact_step(p, g, m, v, lr, b1, b2, eps, wd, t):
    """The plain AdamW step in fp64 with unquantized states (for the closed-form pins)."""
    p, g, m, v = (np.asarray(a, np.float64) for a in (p, g, m, v))
    m = b1 * m + (1 - b1) * g
    v = b2 * v + (1 - b2) * g * g
    c1, c2 = 1 - b1 ** t, 1 - b2 ** t
    p = p - lr * (m / c1 / (np.sqrt(v / c2) + eps) + wd * p)
    return p, m, v
