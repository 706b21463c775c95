"""Oracle: GGUF block decode (Q4_0, Q8_0, Q2_K, Q4_K, Q5_K, Q6_K), exact in fp64.

Test infrastructure only: nothing in the library calls this module.

The pages name GGUF as the frozen base format and say the training recipe runs a standalone
dequant function over it (Show HN: LoRA over GGUF, "Other notes": the GGUF dequant function;
aimodeling.com "GGUF steps up: a full kernel stack"). They do not print the block layouts; the
layouts below are the public GGUF/ggml encodings of these types, written out from their
definitions:

  Q4_0  18-byte block of 32: fp16 d; 16 bytes, byte j = q[j] | q[j+16] << 4; w = d * (q - 8).
  Q8_0  34-byte block of 32: fp16 d; 32 int8 q; w = d * q.
  Q4_K  144-byte superblock of 256: fp16 d, fp16 dmin, 12 bytes S of 6-bit (sc, m) pairs for
        8 sub-blocks of 32, 128 bytes of nibbles; w = d*sc_j*q - dmin*m_j. For j < 4,
        sc_j = S[j] & 63 and m_j = S[j+4] & 63; for j >= 4, sc_j = (S[j+4] & 15) | (S[j-4] >> 6) << 4
        and m_j = (S[j+4] >> 4) | (S[j] >> 6) << 4. Nibble group i (32 bytes) holds sub-block 2i
        in its low nibbles and sub-block 2i+1 in its high nibbles.
  Q5_K  176-byte superblock of 256: fp16 d, fp16 dmin, the same 12 scale bytes as Q4_K, 32 bytes
        qh, 128 bytes of nibbles laid out as in Q4_K. Weight l of sub-block j takes its fifth bit
        from bit j of qh[l]: q = nibble + 16 * ((qh[l] >> j) & 1) in [0, 32); w = d*sc_j*q - dmin*m_j.
  Q2_K  84-byte superblock of 256: 16 scale bytes (low nibble the scale, high nibble the min of one
        16-weight group), 64 bytes of 2-bit codes, fp16 d, fp16 dmin (bytes 80, 82). Each half h of
        128 weights uses qs[32h:32h+32]: its weight 32a + l (a in 0..3, l in 0..31) has the code
        (qs[32h + l] >> 2a) & 3 and the scale byte S = scales[8h + 2a + l // 16]:
        w = d * (S & 15) * q - dmin * (S >> 4).
  Q6_K  210-byte superblock of 256: 128 bytes ql, 64 bytes qh, 16 int8 scales, fp16 d (last).
        Each half h of 128 weights uses ql[64h:64h+64], qh[32h:32h+32] and scales[8h:8h+8]; its
        weight 32a + l (a in 0..3, l in 0..31) has low bits from ql[64h + 32(a & 1) + l] (low nibble
        for a < 2, high nibble otherwise), high bits (qh[32h + l] >> 2a) & 3, and scale
        scales[8h + 2a + l // 16]: q = low | high << 4 in [0, 64), w = d * scale * (q - 32).

Every decoded value is exact in fp64 (and, except the Q2_K / Q4_K / Q5_K difference, already in fp32:
at most 24 significant bits). ``deq_f32`` rounds the exact value once to fp32 (round to
nearest even); ``deq_bf16`` rounds that fp32 value to bf16 (round to nearest even). The layer
multiplies bf16 weight tiles, so ``deq_bf16`` is what the matmul oracles use.
"""
from __future__ import annotations

import numpy as np

Q4_0, Q8_0, Q2_K, Q4_K, Q5_K, Q6_K = 2, 8, 10, 12, 13, 14
_QK = {Q4_0: 32, Q8_0: 32, Q2_K: 256, Q4_K: 256, Q5_K: 256, Q6_K: 256}
_BB = {Q4_0: 18, Q8_0: 34, Q2_K: 84, Q4_K: 144, Q5_K: 176, Q6_K: 210}


def _fp16_at(blocks: np.ndarray, off: int) -> np.ndarray:
    """Little-endian fp16 at byte offset ``off`` of every block, as exact fp64."""
    u = blocks[:, off].astype(np.uint16) | (blocks[:, off + 1].astype(np.uint16) << np.uint16(8))
    return u.view(np.float16).astype(np.float64)


def _blocks(qtype, raw, rows, cols):
    if cols % _QK[qtype]:
        raise ValueError("cols must be a multiple of the block size")
    nb = cols // _QK[qtype]
    raw = np.ascontiguousarray(raw, dtype=np.uint8).reshape(rows, nb * _BB[qtype])
    return raw.reshape(rows * nb, _BB[qtype])


def decode_q4_0(raw, rows, cols) -> np.ndarray:
    b = _blocks(Q4_0, raw, rows, cols)
    d = _fp16_at(b, 0)
    qs = b[:, 2:18]
    q = np.concatenate([qs & 0x0F, qs >> 4], axis=1).astype(np.float64)   # elements 0..15, 16..31
    return (d[:, None] * (q - 8.0)).reshape(rows, cols)


def decode_q8_0(raw, rows, cols) -> np.ndarray:
    b = _blocks(Q8_0, raw, rows, cols)
    d = _fp16_at(b, 0)
    q = b[:, 2:34].view(np.int8).astype(np.float64)
    return (d[:, None] * q).reshape(rows, cols)


def q4_k_scales(S: np.ndarray):
    """(sc, m) for the 8 sub-blocks from the 12 packed scale bytes, shape [nb, 8] each."""
    S = S.astype(np.int64)
    sc = np.empty((S.shape[0], 8), np.int64)
    m = np.empty((S.shape[0], 8), np.int64)
    for j in range(8):
        if j < 4:
            sc[:, j] = S[:, j] & 63
            m[:, j] = S[:, j + 4] & 63
        else:
            sc[:, j] = (S[:, j + 4] & 15) | ((S[:, j - 4] >> 6) << 4)
            m[:, j] = (S[:, j + 4] >> 4) | ((S[:, j] >> 6) << 4)
    return sc, m


def decode_q4_k(raw, rows, cols) -> np.ndarray:
    b = _blocks(Q4_K, raw, rows, cols)
    d = _fp16_at(b, 0)
    dmin = _fp16_at(b, 2)
    sc, m = q4_k_scales(b[:, 4:16])
    qs = b[:, 16:144].reshape(-1, 4, 32)
    q = np.empty((b.shape[0], 8, 32), np.float64)
    for i in range(4):
        q[:, 2 * i, :] = qs[:, i, :] & 0x0F
        q[:, 2 * i + 1, :] = qs[:, i, :] >> 4
    w = d[:, None, None] * sc[:, :, None] * q - dmin[:, None, None] * m[:, :, None]
    return w.reshape(rows, cols)


def decode_q5_k(raw, rows, cols) -> np.ndarray:
    b = _blocks(Q5_K, raw, rows, cols)
    d = _fp16_at(b, 0)
    dmin = _fp16_at(b, 2)
    sc, m = q4_k_scales(b[:, 4:16])
    qh = b[:, 16:48].astype(np.int64)                  # [nb, 32]: bit j of qh[l] -> sub-block j
    qs = b[:, 48:176].reshape(-1, 4, 32).astype(np.int64)
    q = np.empty((b.shape[0], 8, 32), np.float64)
    for j in range(8):
        nib = (qs[:, j // 2, :] >> (4 * (j % 2))) & 0x0F
        q[:, j, :] = nib + 16 * ((qh >> j) & 1)
    w = d[:, None, None] * sc[:, :, None] * q - dmin[:, None, None] * m[:, :, None]
    return w.reshape(rows, cols)


def decode_q6_k(raw, rows, cols) -> np.ndarray:
    b = _blocks(Q6_K, raw, rows, cols)
    ql = b[:, 0:128].astype(np.int64)
    qh = b[:, 128:192].astype(np.int64)
    scales = b[:, 192:208].copy().view(np.int8).astype(np.float64)
    d = _fp16_at(b, 208)
    w = np.empty((b.shape[0], 256), np.float64)
    l = np.arange(32)
    for h in range(2):
        for a in range(4):
            low = (ql[:, 64 * h + 32 * (a & 1) + l] >> (4 * (a >> 1))) & 0x0F
            high = (qh[:, 32 * h + l] >> (2 * a)) & 3
            q = (low | (high << 4)).astype(np.float64)
            s = scales[:, 8 * h + 2 * a + l // 16]
            w[:, 128 * h + 32 * a + l] = d[:, None] * s * (q - 32.0)
    return w.reshape(rows, cols)


def decode_q2_k(raw, rows, cols) -> np.ndarray:
    b = _blocks(Q2_K, raw, rows, cols)
    S = b[:, 0:16].astype(np.int64)
    qs = b[:, 16:80].astype(np.int64)
    d = _fp16_at(b, 80)
    dmin = _fp16_at(b, 82)
    w = np.empty((b.shape[0], 256), np.float64)
    l = np.arange(32)
    for h in range(2):
        for a in range(4):
            q = ((qs[:, 32 * h + l] >> (2 * a)) & 3).astype(np.float64)
            sb = S[:, 8 * h + 2 * a + l // 16]
            w[:, 128 * h + 32 * a + l] = d[:, None] * (sb & 15) * q - dmin[:, None] * (sb >> 4)
    return w.reshape(rows, cols)


_DECODERS = {Q4_0: decode_q4_0, Q8_0: decode_q8_0, Q2_K: decode_q2_k, Q4_K: decode_q4_k, Q5_K: decode_q5_k,
             Q6_K: decode_q6_k}


def decode_exact(qtype, raw, rows, cols) -> np.ndarray:
    """Exact dequantized weights [rows, cols] in fp64."""
    return _DECODERS[qtype](raw, rows, cols)


def round_f32(x: np.ndarray) -> np.ndarray:
    """Round fp64 to fp32 (nearest even), returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest even) via fp32, returned as fp64. Inputs are finite.

    bf16 keeps the top 16 bits of an fp32 pattern; the discarded half is rounded to nearest with
    ties to the even kept pattern.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    keep = u >> np.uint64(16)
    rest = u & np.uint64(0xFFFF)
    up = (rest > 0x8000) | ((rest == 0x8000) & ((keep & np.uint64(1)) == 1))
    keep = keep + up.astype(np.uint64)
    return (keep.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def deq_f32(qtype, raw, rows, cols) -> np.ndarray:
    return round_f32(decode_exact(qtype, raw, rows, cols))


def deq_bf16(qtype, raw, rows, cols) -> np.ndarray:
    return round_bf16(deq_f32(qtype, raw, rows, cols))


def bf16_bits_to_f64(b) -> np.ndarray:
    """bf16 bit patterns (uint16) to exact fp64 values."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Exact bf16 values (fp64 holding bf16-representable numbers) to their bit patterns."""
    f = np.ascontiguousarray(round_bf16(x).astype(np.float32))
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
