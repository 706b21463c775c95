"""Seeded synthetic inputs and offline GGUF block packing.

Both sides of every parity test, and the benchmark, draw their inputs from here. This module holds
no step of the layer's own arithmetic (no block decode, no matmul, no routing): it draws random
tensors, stores them as bf16 bit patterns, and packs fp32 weights into GGUF blocks. Packing is the
offline quantization that happens before training starts (the recipe trains LoRA over a GGUF base
model to save memory, Show HN: LoRA over GGUF, opening paragraph); the layer itself only ever
reads the packed bytes.

Conventions
-----------
* bf16 tensors are ``np.uint16`` arrays of bit patterns (round-to-nearest-even from fp32).
* packed weights are ``np.uint8`` arrays of shape ``[rows, row_bytes]`` in GGUF block order.
* ``N(0, s)`` in the workload descriptions is read as a standard deviation ``s`` for X, dY, W and B,
  and ``A ~ N(0, 1/K)`` as the usual fan-in variance 1/K (standard deviation K**-0.5).
* Every generator takes a seed; the draw order is fixed and stated in each function.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# GGML type ids (the numbers the GGUF container uses for these block types).
Q4_0 = 2
Q8_0 = 8
Q2_K = 10
Q4_K = 12
Q5_K = 13
Q6_K = 14

QK = {Q4_0: 32, Q8_0: 32, Q2_K: 256, Q4_K: 256, Q5_K: 256, Q6_K: 256}          # elements per block
BLOCK_BYTES = {Q4_0: 18, Q8_0: 34, Q2_K: 84, Q4_K: 144, Q5_K: 176, Q6_K: 210}  # bytes per block
QTYPE_NAMES = {Q4_0: "q4_0", Q8_0: "q8_0", Q2_K: "q2_k", Q4_K: "q4_k", Q5_K: "q5_k", Q6_K: "q6_k"}
QTYPE_BY_NAME = {v: k for k, v in QTYPE_NAMES.items()}


def row_bytes(qtype: int, cols: int) -> int:
    """Bytes of one packed row of ``cols`` weights."""
    assert cols % QK[qtype] == 0
    return cols // QK[qtype] * BLOCK_BYTES[qtype]


# ---------------------------------------------------------------------------------------------
# bf16 storage
# ---------------------------------------------------------------------------------------------
def to_bf16_bits(x) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (inputs are finite)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    return ((b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------------------------
# GGUF block packing (offline; vectorised over blocks)
# ---------------------------------------------------------------------------------------------
def _round_half_away(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    f = np.floor(a)
    r = f + (a - f >= np.float32(0.5)).astype(a.dtype)
    return np.copysign(r, v)


def pack_q8_0(w: np.ndarray) -> np.ndarray:
    """Q8_0: per 32 weights, d = max|x|/127 (stored fp16), q = round-half-away(x/d) as int8."""
    rows, cols = w.shape
    x = np.ascontiguousarray(w, dtype=np.float32).reshape(-1, 32)
    d = (np.abs(x).max(axis=1) / np.float32(127)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(d != 0, np.float32(1) / d, np.float32(0)).astype(np.float32)
    q = _round_half_away(x * inv[:, None]).astype(np.int8)
    out = np.empty((x.shape[0], 34), np.uint8)
    out[:, 0:2] = d.astype(np.float16).view(np.uint8).reshape(-1, 2)
    out[:, 2:] = q.view(np.uint8)
    return out.reshape(rows, -1)


def pack_q4_0(w: np.ndarray) -> np.ndarray:
    """Q4_0: per 32 weights, d = (signed value of largest magnitude)/-8 (stored fp16),
    q = min(15, trunc(x/d + 8.5)); byte j holds q[j] (low nibble) and q[j+16] (high nibble)."""
    rows, cols = w.shape
    x = np.ascontiguousarray(w, dtype=np.float32).reshape(-1, 32)
    idx = np.argmax(np.abs(x), axis=1)
    amax = x[np.arange(x.shape[0]), idx]
    d = (amax / np.float32(-8)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(d != 0, np.float32(1) / d, np.float32(0)).astype(np.float32)
    q = np.minimum(np.float32(15), np.trunc(x * inv[:, None] + np.float32(8.5))).astype(np.uint8)
    out = np.empty((x.shape[0], 18), np.uint8)
    out[:, 0:2] = d.astype(np.float16).view(np.uint8).reshape(-1, 2)
    out[:, 2:] = q[:, :16] | (q[:, 16:] << np.uint8(4))
    return out.reshape(rows, -1)


def pack_q4_k(w: np.ndarray) -> np.ndarray:
    """Q4_K with a plain min/max encoder (any valid encoder serves: the layer reads bytes).

    Per 32-weight sub-block j: lo = min(0, min x), scale_j = (max x - lo)/15, min_j = -lo.
    d = max scale_j / 63 and dmin = max min_j / 63 (stored fp16); sc_j = round(scale_j/d),
    m_j = round(min_j/dmin) clamped to 6 bits; q = round((x + dmin*m_j)/(d*sc_j)) clamped to 4 bits.
    Byte layout: fp16 d, fp16 dmin, 12 bytes of packed 6-bit (sc, m), 128 bytes of nibbles.
    """
    rows, cols = w.shape
    x = np.ascontiguousarray(w, dtype=np.float32).reshape(-1, 8, 32)
    nb = x.shape[0]
    lo = np.minimum(np.float32(0), x.min(axis=2))
    hi = x.max(axis=2)
    scale = (hi - lo) / np.float32(15)
    mn = -lo
    d16 = (scale.max(axis=1) / np.float32(63)).astype(np.float16)
    dm16 = (mn.max(axis=1) / np.float32(63)).astype(np.float16)
    d = d16.astype(np.float32)[:, None]
    dm = dm16.astype(np.float32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        sc = np.where(d > 0, _round_half_away(scale / d), 0)
        m = np.where(dm > 0, _round_half_away(mn / dm), 0)
    sc = np.clip(sc, 0, 63).astype(np.uint8)
    m = np.clip(m, 0, 63).astype(np.uint8)
    step = (d * sc.astype(np.float32))[:, :, None]
    off = (dm * m.astype(np.float32))[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(step > 0, _round_half_away((x + off) / step), 0)
    q = np.clip(q, 0, 15).astype(np.uint8)
    out = np.empty((nb, 144), np.uint8)
    out[:, 0:2] = d16.view(np.uint8).reshape(-1, 2)
    out[:, 2:4] = dm16.view(np.uint8).reshape(-1, 2)
    S = np.zeros((nb, 12), np.uint8)
    for j in range(4):
        S[:, j] = (sc[:, j] & 63) | ((sc[:, j + 4] >> 4) << 6)
        S[:, j + 4] = (m[:, j] & 63) | ((m[:, j + 4] >> 4) << 6)
        S[:, j + 8] = (sc[:, j + 4] & 15) | ((m[:, j + 4] & 15) << 4)
    out[:, 4:16] = S
    for i in range(4):
        out[:, 16 + 32 * i:16 + 32 * (i + 1)] = q[:, 2 * i, :] | (q[:, 2 * i + 1, :] << np.uint8(4))
    return out.reshape(rows, -1)


def _k_scale_bytes(sc: np.ndarray, m: np.ndarray) -> np.ndarray:
    """The 12 bytes of eight 6-bit (sc, m) pairs shared by Q4_K and Q5_K, [nb, 12]."""
    S = np.zeros((sc.shape[0], 12), np.uint8)
    for j in range(4):
        S[:, j] = (sc[:, j] & 63) | ((sc[:, j + 4] >> 4) << 6)
        S[:, j + 4] = (m[:, j] & 63) | ((m[:, j + 4] >> 4) << 6)
        S[:, j + 8] = (sc[:, j + 4] & 15) | ((m[:, j + 4] & 15) << 4)
    return S


def pack_q5_k(w: np.ndarray) -> np.ndarray:
    """Q5_K with a plain min/max encoder, as pack_q4_k but with 5-bit codes (31 steps).

    Per 32-weight sub-block j: lo = min(0, min x), scale_j = (max x - lo)/31, min_j = -lo; d, dmin,
    sc_j, m_j as in pack_q4_k; q = round((x + dmin*m_j)/(d*sc_j)) clamped to [0, 31]. Byte layout:
    fp16 d, fp16 dmin, 12 scale bytes, 32 bytes qh (bit j of byte l = bit 4 of q of weight l of
    sub-block j), 128 bytes of low nibbles (group i: sub-block 2i low, 2i+1 high).
    """
    rows, cols = w.shape
    x = np.ascontiguousarray(w, dtype=np.float32).reshape(-1, 8, 32)
    nb = x.shape[0]
    lo = np.minimum(np.float32(0), x.min(axis=2))
    scale = (x.max(axis=2) - lo) / np.float32(31)
    mn = -lo
    d16 = (scale.max(axis=1) / np.float32(63)).astype(np.float16)
    dm16 = (mn.max(axis=1) / np.float32(63)).astype(np.float16)
    d = d16.astype(np.float32)[:, None]
    dm = dm16.astype(np.float32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        sc = np.where(d > 0, _round_half_away(scale / d), 0)
        m = np.where(dm > 0, _round_half_away(mn / dm), 0)
    sc = np.clip(sc, 0, 63).astype(np.uint8)
    m = np.clip(m, 0, 63).astype(np.uint8)
    step = d * sc.astype(np.float32)
    off = dm * m.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(step[:, :, None] > 0, _round_half_away((x + off[:, :, None]) / step[:, :, None]), 0)
    q = np.clip(q, 0, 31).astype(np.uint8)
    out = np.zeros((nb, 176), np.uint8)
    out[:, 0:2] = d16.view(np.uint8).reshape(-1, 2)
    out[:, 2:4] = dm16.view(np.uint8).reshape(-1, 2)
    out[:, 4:16] = _k_scale_bytes(sc, m)
    qh = np.zeros((nb, 32), np.uint8)
    for j in range(8):
        qh |= ((q[:, j, :] >> 4) & 1) << j
    out[:, 16:48] = qh
    for i in range(4):
        out[:, 48 + 32 * i:80 + 32 * i] = (q[:, 2 * i, :] & 15) | ((q[:, 2 * i + 1, :] & 15) << 4)
    return out.reshape(rows, -1)


def pack_q6_k(w: np.ndarray) -> np.ndarray:
    """Q6_K with a plain absmax encoder.

    Per 16-weight group g: scale_g = max|x| / 32; d = max scale_g / 127 (fp16); sc_g =
    round(scale_g / d) clamped to [-128, 127] (int8); q = round(x / (d*sc_g)) + 32 clamped to
    [0, 63] (32 where d*sc_g = 0). Byte layout: 128 bytes ql, 64 bytes qh, 16 int8 scales, fp16 d;
    weight 32a + l of half h (a in 0..3): low 4 bits in ql[64h + 32(a & 1) + l] (low nibble for
    a < 2), high 2 bits at bit 2a of qh[32h + l].
    """
    rows, cols = w.shape
    x = np.ascontiguousarray(w, dtype=np.float32).reshape(-1, 16, 16)
    nb = x.shape[0]
    scale = np.abs(x).max(axis=2) / np.float32(32)
    d16 = (scale.max(axis=1) / np.float32(127)).astype(np.float16)
    d = d16.astype(np.float32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        sc = np.where(d > 0, _round_half_away(scale / d), 0)
    sc = np.clip(sc, -128, 127).astype(np.int8)
    step = d * sc.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(step[:, :, None] != 0, _round_half_away(x / step[:, :, None]), 0) + 32
    q = np.clip(q, 0, 63).astype(np.uint8).reshape(nb, 256)
    out = np.zeros((nb, 210), np.uint8)
    l = np.arange(32)
    for h in range(2):
        for a in range(4):
            qa = q[:, 128 * h + 32 * a + l]
            out[:, 64 * h + 32 * (a & 1) + l] |= (qa & 15) << (4 * (a >> 1))
            out[:, 128 + 32 * h + l] |= (qa >> 4) << (2 * a)
    out[:, 192:208] = sc.view(np.uint8)
    out[:, 208:210] = d16.view(np.uint8).reshape(-1, 2)
    return out.reshape(rows, -1)


def pack_q2_k(w: np.ndarray) -> np.ndarray:
    """Q2_K with a plain min/max encoder.

    Per 16-weight group g: lo = min(0, min x), scale_g = (max x - lo) / 3, min_g = -lo; d = max
    scale_g / 15 and dmin = max min_g / 15 (fp16); sc_g = round(scale_g / d) and m_g =
    round(min_g / dmin), each clamped to [0, 15] with the fp16 d and dmin; q = round((x + dmin*m_g)
    / (d*sc_g)) clamped to [0, 3] (0 where d*sc_g = 0). Byte layout: 16 bytes sc_g | m_g << 4, 64
    bytes of codes (weight 32a + l of half h at bit 2a of qs[32h + l]), fp16 d, fp16 dmin.
    """
    rows, cols = w.shape
    x = np.ascontiguousarray(w, dtype=np.float32).reshape(-1, 16, 16)
    nb = x.shape[0]
    lo = np.minimum(np.float32(0), x.min(axis=2))
    scale = (x.max(axis=2) - lo) / np.float32(3)
    mn = -lo
    d16 = (scale.max(axis=1) / np.float32(15)).astype(np.float16)
    m16 = (mn.max(axis=1) / np.float32(15)).astype(np.float16)
    d = d16.astype(np.float32)[:, None]
    dm = m16.astype(np.float32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        sc = np.where(d > 0, _round_half_away(scale / d), 0)
        m = np.where(dm > 0, _round_half_away(mn / dm), 0)
    sc = np.clip(sc, 0, 15).astype(np.uint8)
    m = np.clip(m, 0, 15).astype(np.uint8)
    step = (d * sc.astype(np.float32))[:, :, None]
    off = (dm * m.astype(np.float32))[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(step != 0, _round_half_away((x + off) / step), 0)
    q = np.clip(q, 0, 3).astype(np.uint8).reshape(nb, 256)
    out = np.zeros((nb, 84), np.uint8)
    out[:, 0:16] = sc | (m << 4)
    l = np.arange(32)
    for h in range(2):
        for a in range(4):
            out[:, 16 + 32 * h + l] |= q[:, 128 * h + 32 * a + l] << (2 * a)
    out[:, 80:82] = d16.view(np.uint8).reshape(-1, 2)
    out[:, 82:84] = m16.view(np.uint8).reshape(-1, 2)
    return out.reshape(rows, -1)


PACKERS = {Q4_0: pack_q4_0, Q8_0: pack_q8_0, Q2_K: pack_q2_k, Q4_K: pack_q4_k, Q5_K: pack_q5_k,
           Q6_K: pack_q6_k}


def pack(qtype: int, w: np.ndarray) -> np.ndarray:
    return PACKERS[qtype](w)


# ---------------------------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------------------------
@dataclass
class LinearCase:
    """One dense LoRA linear problem: X [M,K], dY [M,N], packed W [N, row_bytes], A [r,K], B [N,r]."""
    name: str
    qtype: int
    M: int
    K: int
    N: int
    r: int
    alpha: float
    X: np.ndarray
    dY: np.ndarray
    wq: np.ndarray
    A: np.ndarray
    B: np.ndarray
    meta: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return self.alpha / self.r


def _normal(rng, shape, std):
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def linear_case(M, K, N, qtype, r, alpha, seed=0, outlier_frac=0.0, w_std=0.02, b_std=0.01,
                name=None, weights_first=False) -> LinearCase:
    """Draw order: X, dY, W, A, B, then (if outlier_frac > 0) the outlier rows of W (scaled x8).
    With weights_first: W, A, B, then X, dY (the weights then do not depend on M)."""
    rng = np.random.default_rng(seed)
    if weights_first:
        W = _normal(rng, (N, K), w_std)
        A = _normal(rng, (r, K), 1.0 / math.sqrt(K))
        B = _normal(rng, (N, r), b_std)
    X = _normal(rng, (M, K), 1.0)
    dY = _normal(rng, (M, N), 1.0)
    if not weights_first:
        W = _normal(rng, (N, K), w_std)
        A = _normal(rng, (r, K), 1.0 / math.sqrt(K))
        B = _normal(rng, (N, r), b_std)
    meta = {}
    if outlier_frac > 0:
        n_out = int(round(outlier_frac * N))
        rows = np.sort(rng.choice(N, size=n_out, replace=False))
        W[rows] *= np.float32(8)
        meta["outlier_rows"] = rows
    return LinearCase(name or f"linear_{QTYPE_NAMES[qtype]}_{M}x{K}x{N}", qtype, M, K, N, r, alpha,
                      to_bf16_bits(X), to_bf16_bits(dY), pack(qtype, W), to_bf16_bits(A),
                      to_bf16_bits(B), meta)


# The dense workloads of the method's benchmark set, named by what they are.
def q4_0_linear_64x256x512(seed=0):
    """Single Q4_0 LoRA linear: 64 tokens, K=256, N=512, rank 4, alpha 8."""
    return linear_case(64, 256, 512, Q4_0, 4, 8.0, seed, name="q4_0_linear_64x256x512_r4")


def dense_proj_2048x4096x4096(qtype=Q8_0, seed=0):
    """Dense projection at one 2048-token chunk: K = N = 4096, rank 16, alpha 32."""
    return linear_case(2048, 4096, 4096, qtype, 16, 32.0, seed,
                       name=f"dense_proj_{QTYPE_NAMES[qtype]}_2048x4096x4096_r16")


def decode_q4_0_8192(M, seed=0):
    """Decode-shaped Q4_0 linear: K = N = 8192 at M tokens (M in {1, 4, 16} in the benchmark set),
    rank 4, alpha 8; the weights are drawn first so they are the same for every M."""
    return linear_case(M, 8192, 8192, Q4_0, 4, 8.0, seed, name=f"decode_q4_0_{M}x8192x8192_r4",
                       weights_first=True)


def gate_up_q4_k_2048x2048x12288(seed=0):
    """Fused gate/up projection in Q4_K: 2048 tokens, K=2048, N=12288 with 1% outlier rows x8,
    rank 8, alpha 16."""
    return linear_case(2048, 2048, 12288, Q4_K, 8, 16.0, seed, outlier_frac=0.01,
                       name="gate_up_q4_k_2048x2048x12288_r8")


@dataclass
class MoECase:
    """One routed SwiGLU MoE layer. Expert e has a fused gate/up weight [2I, H] (rows [0,I) gate,
    [I,2I) up) and a down weight [H, I], both packed; one LoRA adapter on gate/up
    (A_gu [E,r,H], B_gu [E,2I,r]) and one on down (A_d [E,r,I], B_d [E,H,r])."""
    name: str
    qtype: int
    T: int
    H: int
    I: int
    E: int
    k: int
    r: int
    alpha: float
    X: np.ndarray
    dY: np.ndarray
    logits: np.ndarray
    w_gu: np.ndarray
    w_d: np.ndarray
    A_gu: np.ndarray
    B_gu: np.ndarray
    A_d: np.ndarray
    B_d: np.ndarray
    meta: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return self.alpha / self.r


def moe_case(T, H, I, E, k, qtype, r, alpha, seed=0, zipf_s=0.0, w_std=0.02, b_std=0.01,
             name=None) -> MoECase:
    """Draw order: X [T,H], dY [T,H], logits [T,E], then per expert e = 0..E-1: W_gu_e [2I,H],
    W_d_e [H,I]; then A_gu, B_gu, A_d, B_d. With zipf_s > 0 the logits get a popularity bias
    b_e = -zipf_s * ln(e + 1) (expert 0 most popular) before the bf16 cast."""
    rng = np.random.default_rng(seed)
    X = _normal(rng, (T, H), 1.0)
    dY = _normal(rng, (T, H), 1.0)
    logits = _normal(rng, (T, E), 1.0)
    if zipf_s > 0:
        logits = logits - np.float32(zipf_s) * np.log(np.arange(1, E + 1, dtype=np.float32))[None, :]
    w_gu = np.empty((E, 2 * I, row_bytes(qtype, H)), np.uint8)
    w_d = np.empty((E, H, row_bytes(qtype, I)), np.uint8)
    for e in range(E):
        w_gu[e] = pack(qtype, _normal(rng, (2 * I, H), w_std))
        w_d[e] = pack(qtype, _normal(rng, (H, I), w_std))
    A_gu = _normal(rng, (E, r, H), 1.0 / math.sqrt(H))
    B_gu = _normal(rng, (E, 2 * I, r), b_std)
    A_d = _normal(rng, (E, r, I), 1.0 / math.sqrt(I))
    B_d = _normal(rng, (E, H, r), b_std)
    return MoECase(name or f"moe_{QTYPE_NAMES[qtype]}_T{T}_H{H}_I{I}_E{E}_k{k}", qtype, T, H, I, E, k,
                   r, alpha, to_bf16_bits(X), to_bf16_bits(dY), to_bf16_bits(logits), w_gu, w_d,
                   to_bf16_bits(A_gu), to_bf16_bits(B_gu), to_bf16_bits(A_d), to_bf16_bits(B_d))


def synth_q4_k(rng, rows: int, cols: int) -> np.ndarray:
    """Valid Q4_K superblocks drawn directly as bytes, [rows x cols/256 x 144]: fp16 d uniform in
    [1.0e-4, 1.6e-4), fp16 dmin uniform in [0.8e-3, 1.2e-3), 6-bit sc and m uniform over all 64
    values (so both halves of the split of sub-blocks 4..7, whose top two bits live in bytes 0..7,
    occur), 4-bit codes uniform. The weights d sc q - dmin m then spread over about -0.07..0.14
    (std near 0.035), the scale of an N(0, 0.02) weight, without encoding the fp32 weights first."""
    nb = rows * (cols // 256)
    out = np.empty((nb, 144), np.uint8)
    d16 = rng.uniform(1.0e-4, 1.6e-4, nb).astype(np.float16)
    dm16 = rng.uniform(0.8e-3, 1.2e-3, nb).astype(np.float16)
    sc = rng.integers(0, 64, (nb, 8), dtype=np.uint8)
    m = rng.integers(0, 64, (nb, 8), dtype=np.uint8)
    out[:, 0:2] = d16.view(np.uint8).reshape(-1, 2)
    out[:, 2:4] = dm16.view(np.uint8).reshape(-1, 2)
    for j in range(4):
        out[:, 4 + j] = (sc[:, j] & 63) | ((sc[:, j + 4] >> 4) << 6)
        out[:, 8 + j] = (m[:, j] & 63) | ((m[:, j + 4] >> 4) << 6)
        out[:, 12 + j] = (sc[:, j + 4] & 15) | ((m[:, j + 4] & 15) << 4)
    out[:, 16:] = rng.integers(0, 256, (nb, 128), dtype=np.uint8)
    return out.reshape(rows, -1)


def synth_q8_0(rng, rows: int, cols: int) -> np.ndarray:
    """Valid Q8_0 blocks drawn directly as bytes, [rows x cols/32 x 34]: fp16 d uniform in
    [1.0e-4, 3.0e-4), int8 codes uniform in [-127, 127]. The weights d q then spread over about
    +-0.04 (std near 0.0135), without encoding fp32 weights first."""
    nb = rows * (cols // 32)
    out = np.empty((nb, 34), np.uint8)
    out[:, 0:2] = rng.uniform(1.0e-4, 3.0e-4, nb).astype(np.float16).view(np.uint8).reshape(-1, 2)
    out[:, 2:] = rng.integers(-127, 128, (nb, 32), dtype=np.int8).view(np.uint8)
    return out.reshape(rows, -1)


def lm_head_q8_0_128k(M=2048, seed=0):
    """Quantized lm_head workload: M tokens of hidden 2048, a 131072-entry vocabulary, Q8_0 weights
    drawn as blocks (synth_q8_0), labels uniform over the vocabulary. Draw order: W, X, labels."""
    V, K = 131072, 2048
    rng = np.random.default_rng(seed)
    wq = synth_q8_0(rng, V, K)
    X = to_bf16_bits(_normal(rng, (M, K), 1.0))
    labels = rng.integers(0, V, M).astype(np.int32)
    return dict(V=V, K=K, M=M, qtype=Q8_0, wq=wq, X=X, labels=labels)


_MOE256 = {}


def moe_q4_k_256x4096x1536(T, seed=0, E=256):
    """Skewed, weight-bound MoE: T tokens, hidden 4096, 256 experts of intermediate 1536, top-8,
    Q4_K, Zipf(1.1) popularity bias on the logits, rank 4, alpha 8 on gate/up and down.

    The layer shape is fixed and its weights are the same for every T: they and the adapters come
    from default_rng(seed), in the order W_gu_e, W_d_e for e = 0..E-1 (drawn as Q4_K blocks by
    synth_q4_k), then A_gu, B_gu, A_d, B_d; X, dY and the logits come from default_rng([seed, T]).
    The packed weights are kept between calls (2.7 GB). E < 256 gives the same expert shape with
    fewer experts (a profiling case small enough to capture with every counter)."""
    H, I, k, r = 4096, 1536, 8, 4
    key = (seed, E)
    if key not in _MOE256:
        rng = np.random.default_rng(seed)
        w_gu = np.empty((E, 2 * I, row_bytes(Q4_K, H)), np.uint8)
        w_d = np.empty((E, H, row_bytes(Q4_K, I)), np.uint8)
        for e in range(E):
            w_gu[e] = synth_q4_k(rng, 2 * I, H)
            w_d[e] = synth_q4_k(rng, H, I)
        A_gu = to_bf16_bits(_normal(rng, (E, r, H), 1.0 / math.sqrt(H)))
        B_gu = to_bf16_bits(_normal(rng, (E, 2 * I, r), 0.01))
        A_d = to_bf16_bits(_normal(rng, (E, r, I), 1.0 / math.sqrt(I)))
        B_d = to_bf16_bits(_normal(rng, (E, H, r), 0.01))
        _MOE256.clear()
        _MOE256[key] = (w_gu, w_d, A_gu, B_gu, A_d, B_d)
    w_gu, w_d, A_gu, B_gu, A_d, B_d = _MOE256[key]
    rng = np.random.default_rng([seed, T])
    X = _normal(rng, (T, H), 1.0)
    dY = _normal(rng, (T, H), 1.0)
    logits = _normal(rng, (T, E), 1.0) - np.float32(1.1) * np.log(np.arange(1, E + 1, dtype=np.float32))[None, :]
    return MoECase(f"moe_q4_k_T{T}_H4096_E{E}_I1536_k8_zipf", Q4_K, T, H, I, E, k, r, 8.0, to_bf16_bits(X),
                   to_bf16_bits(dY), to_bf16_bits(logits), w_gu, w_d, A_gu, B_gu, A_d, B_d)


def moe_q4_0_2048tok_128x768(seed=0):
    """Grouped MoE layer: 2048 tokens, hidden 2048, 128 experts of intermediate 768, top-8, Q4_0,
    rank 4, alpha 8 on gate/up and down."""
    return moe_case(2048, 2048, 768, 128, 8, Q4_0, 4, 8.0, seed, name="moe_q4_0_T2048_H2048_E128_I768_k8")
