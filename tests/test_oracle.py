"""Pins for the oracle: each check is independent of the oracle's own formulas (hand-packed blocks
with hand-computed values, an independent GGUF decoder, closed forms, finite differences,
brute-force loops), so a dropped term, a wrong sign or index, or a transposed operand fails one."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import gguf_blocks as gb
from oracle import lora_linear as ll
from oracle import moe as om
from quantized_base_lora_tma_b200 import inputs as inp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hand_blocks():
    out = []
    with open(os.path.join(GOLDEN, "gguf_hand_blocks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            t, hx, vals = [p.strip() for p in line.split("|")]
            raw = np.frombuffer(bytes.fromhex(hx.replace(" ", "")), np.uint8)
            out.append((t, raw, np.array([float(v) for v in vals.split()])))
    return out


@pytest.mark.parametrize("case", range(4))
def test_hand_packed_q4_0_q8_0(case):
    t, raw, want = _hand_blocks()[case]
    qt = {"q4_0": gb.Q4_0, "q8_0": gb.Q8_0}[t]
    got = gb.decode_exact(qt, raw, 1, 32)[0]
    assert np.array_equal(got, want)


def _hand_q4_k(d16, dmin16, sc, m, q):
    """Pack one Q4_K superblock byte by byte from (sc, m, q) chosen by hand."""
    S = [0] * 12
    for j in range(4):
        S[j] = (sc[j] & 63) | ((sc[j + 4] >> 4) << 6)
        S[j + 4] = (m[j] & 63) | ((m[j + 4] >> 4) << 6)
        S[j + 8] = (sc[j + 4] & 15) | ((m[j + 4] & 15) << 4)
    qs = []
    for i in range(4):
        qs += [q[2 * i][l] | (q[2 * i + 1][l] << 4) for l in range(32)]
    raw = bytes([d16 & 255, d16 >> 8, dmin16 & 255, dmin16 >> 8] + S + qs)
    assert len(raw) == 144
    return np.frombuffer(raw, np.uint8)


def test_hand_packed_q4_k_high_bit_split():
    # Scales and mins >= 16 in sub-blocks 4..7 exercise the split of their top 2 bits into S[0..7].
    sc = [1, 2, 3, 4, 17, 33, 50, 63]
    m = [0, 1, 2, 3, 16, 31, 47, 62]
    q = [[(l + j) % 16 for l in range(32)] for j in range(8)]
    raw = _hand_q4_k(0x3C00, 0x3800, sc, m, q)          # d = 1.0, dmin = 0.5
    # the 12 scale bytes, worked out by hand
    assert list(raw[4:16]) == [0x41, 0x82, 0xC3, 0xC4, 0x40, 0x41, 0x82, 0xC3, 0x01, 0xF1, 0xF2, 0xEF]
    got = gb.decode_exact(gb.Q4_K, raw, 1, 256)[0].reshape(8, 32)
    want = np.array([[1.0 * sc[j] * q[j][l] - 0.5 * m[j] for l in range(32)] for j in range(8)])
    assert np.array_equal(got, want)


def test_hand_packed_q5_k():
    """A Q5_K superblock written byte by byte from chosen (sc, m, q): the scales in the Q4_K packing,
    the fifth bit of weight l of sub-block j at bit j of qh[l], the low nibbles as in Q4_K."""
    sc = [1, 5, 9, 13, 17, 40, 51, 63]
    m = [2, 0, 7, 30, 33, 16, 48, 62]
    q = [[(3 * l + 5 * j) % 32 for l in range(32)] for j in range(8)]
    S = [0] * 12
    for j in range(4):
        S[j] = (sc[j] & 63) | ((sc[j + 4] >> 4) << 6)
        S[j + 4] = (m[j] & 63) | ((m[j + 4] >> 4) << 6)
        S[j + 8] = (sc[j + 4] & 15) | ((m[j + 4] & 15) << 4)
    qh = [sum(((q[j][l] >> 4) & 1) << j for j in range(8)) for l in range(32)]
    qs = []
    for i in range(4):
        qs += [(q[2 * i][l] & 15) | ((q[2 * i + 1][l] & 15) << 4) for l in range(32)]
    raw = np.frombuffer(bytes([0x00, 0x3C, 0x00, 0x38] + S + qh + qs), np.uint8)   # d = 1.0, dmin = 0.5
    assert raw.size == 176
    got = gb.decode_exact(gb.Q5_K, raw, 1, 256)[0].reshape(8, 32)
    want = np.array([[1.0 * sc[j] * q[j][l] - 0.5 * m[j] for l in range(32)] for j in range(8)])
    assert np.array_equal(got, want)


def test_hand_packed_q6_k():
    """A Q6_K superblock written byte by byte from chosen int8 scales and 6-bit codes: weight
    32a + l of half h has its low nibble in ql[64h + 32(a & 1) + l] (high nibble for a >= 2), its two
    high bits at bit 2a of qh[32h + l], and the scale scales[8h + 2a + l // 16]; d is the last fp16."""
    scales = [-128, -3, 0, 1, 7, 64, 127, -77, 5, -5, 33, -33, 100, 2, -1, 9]
    q = [(7 * i + 3) % 64 for i in range(256)]
    ql = [0] * 128
    qh = [0] * 64
    for h in range(2):
        for a in range(4):
            for l in range(32):
                v = q[128 * h + 32 * a + l]
                ql[64 * h + 32 * (a & 1) + l] |= (v & 15) << (4 * (a >> 1))
                qh[32 * h + l] |= (v >> 4) << (2 * a)
    sc_bytes = [x & 255 for x in scales]
    raw = np.frombuffer(bytes(ql + qh + sc_bytes + [0x00, 0x34]), np.uint8)          # d = 0.25
    assert raw.size == 210
    got = gb.decode_exact(gb.Q6_K, raw, 1, 256)[0]
    want = np.array([0.25 * scales[8 * (i // 128) + 2 * ((i % 128) // 32) + (i % 32) // 16] * (q[i] - 32)
                     for i in range(256)])
    assert np.array_equal(got, want)


def test_hand_packed_q2_k():
    """A Q2_K superblock written byte by byte from chosen 4-bit scales, 4-bit mins and 2-bit codes:
    weight 32a + l of half h has its code at bit 2a of qs[32h + l] and the scale byte
    scales[8h + 2a + l // 16] (low nibble the scale, high nibble the min); d and dmin are the fp16
    values at bytes 80 and 82."""
    sc = [0, 1, 2, 3, 5, 8, 13, 15, 7, 4, 9, 11, 6, 10, 12, 14]
    mn = [15, 0, 3, 7, 1, 2, 9, 4, 0, 15, 5, 6, 8, 10, 11, 13]
    q = [(5 * i + 2) % 4 for i in range(256)]
    qs = [0] * 64
    for h in range(2):
        for a in range(4):
            for l in range(32):
                qs[32 * h + l] |= q[128 * h + 32 * a + l] << (2 * a)
    scales = [s | (m << 4) for s, m in zip(sc, mn)]
    raw = np.frombuffer(bytes(scales + qs + [0x00, 0x34, 0x00, 0x38]), np.uint8)  # d = 0.25, dmin = 0.5
    assert raw.size == 84
    got = gb.decode_exact(gb.Q2_K, raw, 1, 256)[0]
    g = [8 * (i // 128) + 2 * ((i % 128) // 32) + (i % 32) // 16 for i in range(256)]
    want = np.array([0.25 * sc[g[i]] * q[i] - 0.5 * mn[g[i]] for i in range(256)])
    assert np.array_equal(got, want)


def _random_blocks(qtype, nblocks, rng):
    bb = {gb.Q4_0: 18, gb.Q8_0: 34, gb.Q2_K: 84, gb.Q4_K: 144, gb.Q5_K: 176, gb.Q6_K: 210}[qtype]
    raw = rng.integers(0, 256, size=(nblocks, bb), dtype=np.uint8)
    # finite fp16 scales only (random bytes could spell Inf/NaN): bytes 0-1 (and 2-3 for the
    # superblocks with a dmin), or the last two bytes of a Q6_K superblock
    offs = {gb.Q2_K: [80, 82], gb.Q4_K: [0, 2], gb.Q5_K: [0, 2], gb.Q6_K: [208]}.get(qtype, [0])
    for o in offs:
        d = (rng.standard_normal(nblocks) * 0.01).astype(np.float16)
        d[::7] = np.float16(6.0e-8)                    # include subnormal scales
        raw[:, o:o + 2] = d.view(np.uint8).reshape(-1, 2)
    return raw


@pytest.mark.parametrize("qtype,gtype", [(gb.Q4_0, "Q4_0"), (gb.Q8_0, "Q8_0"), (gb.Q4_K, "Q4_K"),
                                         (gb.Q5_K, "Q5_K"), (gb.Q6_K, "Q6_K"), (gb.Q2_K, "Q2_K")])
def test_decode_matches_gguf_py(qtype, gtype):
    """Independent codebase: gguf-py's dequantize (fp32) must equal the fp32 rounding of the exact
    decode, element by element."""
    gguf = pytest.importorskip("gguf")
    from gguf import quants
    rng = np.random.default_rng(7)
    qk = {gb.Q4_0: 32, gb.Q8_0: 32}.get(qtype, 256)
    rows, cols = 16, 4 * qk if qk == 256 else 16 * qk
    raw = _random_blocks(qtype, rows * cols // qk, rng).reshape(rows, -1)
    want = quants.dequantize(raw, getattr(gguf.GGMLQuantizationType, gtype)).astype(np.float32)
    got = gb.deq_f32(qtype, raw, rows, cols).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), want.reshape(rows, cols).view(np.uint32))


def test_decode_value_grid_closed_form():
    """Q4_0 values lie on d*{-8..7}; Q8_0 on d*{-128..127}."""
    rng = np.random.default_rng(3)
    for qt, lo, hi in [(gb.Q4_0, -8, 7), (gb.Q8_0, -128, 127)]:
        raw = _random_blocks(qt, 64, rng)
        d = raw[:, 0:2].copy().view(np.float16).astype(np.float64).ravel()
        w = gb.decode_exact(qt, raw, 64, 32)
        k = w / np.where(d == 0, 1, d)[:, None]
        assert np.all(k == np.round(k)) and k.min() >= lo and k.max() <= hi


@pytest.mark.parametrize("gtype", ["Q4_0", "Q8_0"])
def test_packers_match_gguf_py_bytes(gtype):
    """The input encoders agree byte for byte with gguf-py's quantize (pins the input recipe)."""
    gguf = pytest.importorskip("gguf")
    from gguf import quants
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((32, 512)) * 0.02).astype(np.float32)
    x[3, :32] = 0.0
    qt = {"Q4_0": inp.Q4_0, "Q8_0": inp.Q8_0}[gtype]
    assert np.array_equal(inp.pack(qt, x), quants.quantize(x, getattr(gguf.GGMLQuantizationType, gtype)))


def test_pack_q2_k_picks_the_nearest_code():
    """The Q2_K encoder: every weight decodes to the representable value d*sc*q - dmin*m (q in 0..3,
    from the block's own packed scale and min) nearest to it."""
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((8, 512)) * 0.02).astype(np.float32)
    x[2, :16] = 0.0
    x[5, 16:32] = np.abs(x[5, 16:32])        # a group with no negative values (min 0)
    raw = inp.pack(inp.Q2_K, x)
    w = gb.decode_exact(gb.Q2_K, raw, 8, 512)
    b = raw.reshape(-1, 84)
    d = b[:, 80:82].copy().view(np.float16).astype(np.float64).ravel()
    dm = b[:, 82:84].copy().view(np.float16).astype(np.float64).ravel()
    S = b[:, 0:16].astype(np.int64)
    step = d[:, None] * (S & 15)                           # [superblock, group]
    off = dm[:, None] * (S >> 4)
    grid = step[:, :, None] * np.arange(4) - off[:, :, None]   # [sb, group, 4]
    xs = x.astype(np.float64).reshape(-1, 16, 16)
    nearest = np.abs(xs[:, :, :, None] - grid[:, :, None, :]).min(axis=3)
    err = np.abs(w.reshape(-1, 16, 16) - xs)
    assert np.all(err <= nearest + 1e-6 * (step[:, :, None] + 1e-12))


@pytest.mark.parametrize("qtype", [inp.Q4_0, inp.Q8_0, inp.Q4_K, inp.Q5_K, inp.Q6_K])
def test_pack_roundtrip_error_bound(qtype):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((8, 512)) * 0.02).astype(np.float32)
    w = gb.decode_exact(qtype, inp.pack(qtype, x), 8, 512)
    err = np.abs(w - x)
    if qtype == inp.Q4_K:
        assert err.max() < 0.2 * (x.max() - x.min()) / 15 * 8
    elif qtype == inp.Q5_K:
        # per 32-weight sub-block: half a step of (max - min(0, min)) / 31, widened for the 6-bit
        # scale and min and their fp16 super-scales
        xs = x.reshape(-1, 32)
        step = (xs.max(axis=1) - np.minimum(0, xs.min(axis=1))) / 31
        assert np.all(err.reshape(-1, 32) <= step[:, None] * 1.5 + 1e-7)
    elif qtype == inp.Q6_K:
        # per 16-weight group with step = d * scale read from the packed bytes: half a step where
        # the code is not clipped, and the clipped excess |x| - 31 step (codes - 32 end at +31) or
        # |x| - 32 step (at -32) where it is
        b = inp.pack(qtype, x).reshape(-1, 210)
        d = b[:, 208:210].copy().view(np.float16).astype(np.float64).ravel()
        step = np.abs(d[:, None] * b[:, 192:208].copy().view(np.int8).astype(np.float64)).ravel()
        xs = x.reshape(-1, 16).astype(np.float64)
        clip = np.maximum(xs.max(axis=1) - 31 * step, -xs.min(axis=1) - 32 * step)
        bound = np.maximum(0.5 * step, clip)
        assert np.all(err.reshape(-1, 16) <= bound[:, None] * (1 + 1e-9) + 1e-9)
    else:
        qk = 32
        d = np.abs(inp.pack(qtype, x).reshape(-1, 18 if qtype == inp.Q4_0 else 34)[:, :2].copy()
                   .view(np.float16).astype(np.float64)).ravel()
        # half a step (a whole step at Q4_0's clipped top end) plus the fp16 rounding of d,
        # which the quantizer does not see: at most |q| * 2^-11 * |d|
        bound = d * (1 + 8 * 2.0 ** -11) if qtype == inp.Q4_0 else d * (0.5 + 127 * 2.0 ** -11)
        assert np.all(err.reshape(-1, qk) <= bound[:, None] * (1 + 1e-6) + 1e-12)


def test_round_bf16_ties_and_torch():
    one = 1.0
    assert gb.round_bf16(np.array([one + 2 ** -8]))[0] == 1.0                  # tie -> even
    assert gb.round_bf16(np.array([one + 3 * 2 ** -8]))[0] == one + 2 ** -6    # tie -> even (up)
    assert gb.round_bf16(np.array([one + 2 ** -8 + 2 ** -20]))[0] == one + 2 ** -7
    rng = np.random.default_rng(0)
    x = rng.standard_normal(100000).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(gb.round_bf16(x.astype(np.float64)), want)


# ------------------------------------------------------------------------------------------------
# dense linear
# ------------------------------------------------------------------------------------------------
def _small_linear(M=5, K=256, N=7, r=3, qtype=inp.Q4_0, seed=0):
    c = inp.linear_case(M, K, N, qtype, r, 2.0 * r, seed)
    f = gb.bf16_bits_to_f64
    return c, f(c.X), f(c.dY), f(c.A), f(c.B)


def test_linear_b_zero_is_base_gemm():
    """B = 0: Y is the dequantized base GEMM (computed here with gguf-py's decoder and torch),
    dA = 0 exactly and dB = s dY^T (X A^T)."""
    gguf = pytest.importorskip("gguf")
    from gguf import quants
    c, X, dY, A, B = _small_linear(M=9, K=512, N=33)
    B0 = np.zeros_like(B)
    W = ll.weights(c.qtype, c.wq, c.N, c.K)
    Y, H = ll.linear_fwd(W, X, A, B0, c.scale)
    Wg = quants.dequantize(c.wq, gguf.GGMLQuantizationType.Q4_0).astype(np.float32)
    Wg = torch.from_numpy(Wg).to(torch.bfloat16).double()
    Yt = torch.nn.functional.linear(torch.from_numpy(X), Wg).numpy()
    assert np.allclose(Y, Yt, rtol=0, atol=1e-12)
    dX, dA, dB, G = ll.linear_bwd(W, X, dY, A, B0, c.scale, H)
    assert np.all(dA == 0) and np.all(G == 0)
    dB_t = c.scale * torch.einsum("mn,mj->nj", torch.from_numpy(dY),
                                  torch.einsum("mk,jk->mj", torch.from_numpy(X), torch.from_numpy(A)))
    assert np.allclose(dB, dB_t.numpy(), rtol=1e-12, atol=1e-12)


def test_linear_lora_selector_closed_form():
    """A picks X's first r columns and B = c*[I_r; 0]: the LoRA term is s*c*X[:, n] for n < r and 0
    beyond, so a transposed operand, a missing s or a wrong index shows."""
    c, X, dY, A, B = _small_linear(M=6, K=256, N=9, r=3)
    r = c.r
    A = np.zeros_like(A); A[np.arange(r), np.arange(r)] = 1.0
    B = np.zeros_like(B); B[np.arange(r), np.arange(r)] = 0.75
    W0 = np.zeros((c.N, c.K))
    Y, H = ll.linear_fwd(W0, X, A, B, c.scale)
    want = np.zeros((c.M, c.N)); want[:, :r] = c.scale * 0.75 * X[:, :r]
    assert np.array_equal(Y, want)
    assert np.array_equal(H, X[:, :r])


@pytest.mark.parametrize("qtype", [inp.Q4_0, inp.Q8_0, inp.Q4_K])
def test_linear_grads_finite_differences(qtype):
    """Central differences of L = sum(dY * Y) against the analytic dX, dA, dB (fp64, exact decode)."""
    c, X, dY, A, B = _small_linear(M=3, K=256, N=5, r=2, qtype=qtype)
    s = c.scale
    W = ll.weights(qtype, c.wq, c.N, c.K, round_weights=False)

    def loss(X_, A_, B_):
        return float((dY * ll.linear_fwd(W, X_, A_, B_, s)[0]).sum())

    dX, dA, dB, _ = ll.linear_bwd(W, X, dY, A, B, s)
    h = 1e-4
    rng = np.random.default_rng(1)
    for name, T, grad in [("X", X, dX), ("A", A, dA), ("B", B, dB)]:
        for _ in range(12):
            i = tuple(rng.integers(0, n) for n in T.shape)
            Tp, Tm = T.copy(), T.copy()
            Tp[i] += h; Tm[i] -= h
            args_p = {"X": X, "A": A, "B": B}; args_m = dict(args_p)
            args_p[name] = Tp; args_m[name] = Tm
            fd = (loss(args_p["X"], args_p["A"], args_p["B"]) - loss(args_m["X"], args_m["A"], args_m["B"])) / (2 * h)
            assert abs(fd - grad[i]) <= 1e-6 * max(1.0, abs(grad[i])), (name, i, fd, grad[i])


# ------------------------------------------------------------------------------------------------
# routing
# ------------------------------------------------------------------------------------------------
def test_route_invariants_and_brute_force():
    rng = np.random.default_rng(2)
    T, E, k = 50, 16, 4
    logits = gb.bf16_bits_to_f64(inp.to_bf16_bits(rng.standard_normal((T, E)).astype(np.float32)))
    logits[3, :] = logits[3, 0]          # a token with all-equal logits
    logits[4, 5] = logits[4, 9] = 10.0   # a tie at the top
    idx, w, counts, offsets, perm, inv = om.route(logits, k)
    assert counts.sum() == T * k and offsets[-1] == T * k and np.all(np.diff(offsets) == counts)
    assert np.array_equal(np.sort(perm), np.arange(T * k))
    assert np.array_equal(perm[inv], np.arange(T * k))
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-15)
    assert list(idx[3]) == [0, 1, 2, 3]
    assert list(idx[4][:2]) == [5, 9]
    for t in range(T):
        assert len(set(idx[t])) == k
        # brute force: repeatedly take the largest remaining logit, lowest index on ties
        rem = list(range(E)); sel = []
        for _ in range(k):
            best = rem[0]
            for e in rem:
                if logits[t, e] > logits[t, best]:
                    best = e
            sel.append(best); rem.remove(best)
        assert list(idx[t]) == sel
        ex = [math.exp(logits[t, e]) for e in sel]
        assert np.allclose(w[t], np.array(ex) / sum(ex), rtol=1e-13)
    # pairs sorted by (expert, token, slot)
    keys = [(idx[p // k, p % k], p // k, p % k) for p in perm]
    assert keys == sorted(keys)


# ------------------------------------------------------------------------------------------------
# MoE
# ------------------------------------------------------------------------------------------------
def _small_moe(T=6, H=256, I=256, E=4, k=2, r=2, qtype=inp.Q4_0, seed=0):
    c = inp.moe_case(T, H, I, E, k, qtype, r, 2.0 * r, seed)
    f = gb.bf16_bits_to_f64
    return c, f(c.X), f(c.dY), f(c.logits), f(c.A_gu), f(c.B_gu), f(c.A_d), f(c.B_d)


def _brute_token_ffn(x, Wgu, Wd, Agu, Bgu, Ad, Bd, s, I):
    """One token through one expert, written as explicit per-element sums (no matmul)."""
    H = x.shape[0]
    r = Agu.shape[0]
    hg = [sum(x[kk] * Agu[j, kk] for kk in range(H)) for j in range(r)]
    gu = [sum(x[kk] * Wgu[n, kk] for kk in range(H)) + s * sum(hg[j] * Bgu[n, j] for j in range(r))
          for n in range(2 * I)]
    h = [gu[i] / (1 + math.exp(-gu[i])) * gu[I + i] for i in range(I)]
    hd = [sum(h[i] * Ad[j, i] for i in range(I)) for j in range(r)]
    return np.array([sum(h[i] * Wd[n, i] for i in range(I)) + s * sum(hd[j] * Bd[n, j] for j in range(r))
                     for n in range(H)])


def test_moe_fwd_vs_per_token_brute_force():
    c, X, dY, L, Agu, Bgu, Ad, Bd = _small_moe(T=5, H=256, I=256, E=4, k=2)
    Wgu, Wd = om.expert_weights(c.qtype, c.w_gu, c.w_d, c.H, c.I, round_weights=False)
    idx, w, counts, offsets, perm, inv = om.route(L, c.k)
    Y, _ = om.moe_fwd(Wgu, Wd, X, idx, w, counts, offsets, perm, Agu, Bgu, Ad, Bd, c.scale, mirror=False)
    for t in [0, 3]:
        want = np.zeros(c.H)
        for j in range(c.k):
            e = idx[t, j]
            want += w[t, j] * _brute_token_ffn(X[t], Wgu[e], Wd[e], Agu[e], Bgu[e], Ad[e], Bd[e], c.scale, c.I)
        assert np.allclose(Y[t], want, rtol=1e-10, atol=1e-12)


def test_moe_single_expert_is_dense_swiglu_with_lora():
    """E = 1, k = 1: the layer is one dense SwiGLU FFN built from the dense LoRA linear oracle."""
    c, X, dY, L, Agu, Bgu, Ad, Bd = _small_moe(T=7, E=1, k=1)
    Wgu, Wd = om.expert_weights(c.qtype, c.w_gu, c.w_d, c.H, c.I)
    idx, w, counts, offsets, perm, inv = om.route(L, 1)
    assert np.all(w == 1.0)
    Y, saved = om.moe_fwd(Wgu, Wd, X, idx, w, counts, offsets, perm, Agu, Bgu, Ad, Bd, c.scale, mirror=False)
    gu, _ = ll.linear_fwd(Wgu[0], X, Agu[0], Bgu[0], c.scale)
    g, u = gu[:, :c.I], gu[:, c.I:]
    sig = 1 / (1 + np.exp(-g))
    h = g * sig * u
    o, _ = ll.linear_fwd(Wd[0], h, Ad[0], Bd[0], c.scale)
    assert np.allclose(Y, o, rtol=1e-12, atol=1e-12)
    gr = om.moe_bwd(Wgu, Wd, X, dY, idx, w, counts, offsets, perm, Agu, Bgu, Ad, Bd, c.scale, saved, mirror=False)
    dh, dAd, dBd, _ = ll.linear_bwd(Wd[0], h, dY, Ad[0], Bd[0], c.scale)
    dgu = np.concatenate([dh * u * sig * (1 + g * (1 - sig)), dh * g * sig], axis=1)
    dX, dAgu, dBgu, _ = ll.linear_bwd(Wgu[0], X, dgu, Agu[0], Bgu[0], c.scale)
    for got, want in [(gr["dX"], dX), (gr["dA_d"][0], dAd), (gr["dB_d"][0], dBd),
                      (gr["dA_gu"][0], dAgu), (gr["dB_gu"][0], dBgu)]:
        assert np.allclose(got, want, rtol=1e-11, atol=1e-12)
    assert np.allclose(gr["d_logits_sel"], 0.0)      # one selected expert: weight is constant 1


def test_moe_grads_finite_differences():
    c, X, dY, L, Agu, Bgu, Ad, Bd = _small_moe(T=4, H=256, I=256, E=3, k=2, r=2)
    # separate the logits so that small perturbations never change the selection
    L = L + np.arange(c.E)[None, :] * 0.0 + np.array([[0.0, 0.7, 1.9]])
    Wgu, Wd = om.expert_weights(c.qtype, c.w_gu, c.w_d, c.H, c.I, round_weights=False)
    s = c.scale

    def run(X_, L_, Agu_, Bgu_, Ad_, Bd_):
        idx, w, counts, offsets, perm, inv = om.route(L_, c.k)
        Y, saved = om.moe_fwd(Wgu, Wd, X_, idx, w, counts, offsets, perm, Agu_, Bgu_, Ad_, Bd_, s, mirror=False)
        return Y, saved, (idx, w, counts, offsets, perm)

    Y, saved, (idx, w, counts, offsets, perm) = run(X, L, Agu, Bgu, Ad, Bd)
    gr = om.moe_bwd(Wgu, Wd, X, dY, idx, w, counts, offsets, perm, Agu, Bgu, Ad, Bd, s, saved, mirror=False)
    dL = om.scatter_d_logits(idx, gr["d_logits_sel"], c.E)
    names = ["X", "L", "Agu", "Bgu", "Ad", "Bd"]
    vals = dict(X=X, L=L, Agu=Agu, Bgu=Bgu, Ad=Ad, Bd=Bd)
    grads = dict(X=gr["dX"], L=dL, Agu=gr["dA_gu"], Bgu=gr["dB_gu"], Ad=gr["dA_d"], Bd=gr["dB_d"])
    rng = np.random.default_rng(4)
    h = 1e-5
    for name in names:
        T = vals[name]
        for _ in range(6):
            i = tuple(rng.integers(0, n) for n in T.shape)
            if name in ("Bgu", "Agu", "Ad", "Bd") and counts[i[0]] == 0:
                continue
            out = []
            for sgn in (1, -1):
                v = dict(vals)
                v[name] = T.copy(); v[name][i] += sgn * h
                out.append(float((dY * run(v["X"], v["L"], v["Agu"], v["Bgu"], v["Ad"], v["Bd"])[0]).sum()))
            fd = (out[0] - out[1]) / (2 * h)
            g = grads[name][i]
            assert abs(fd - g) <= 1e-5 * max(1.0, abs(g)), (name, i, fd, g)


def test_synth_q4_k_blocks_have_the_stated_fields():
    """The 256-expert workload's weights are drawn directly as Q4_K blocks: the 6-bit scales and
    mins take all 64 values (small and large ones in sub-blocks 4..7, whose top two bits sit in the
    first eight scale bytes), d and dmin lie in their stated ranges, and the weights spread over
    about -0.07..0.14 with a std near 0.035 (checked through the oracle's decoder and gguf-py's)."""
    rng = np.random.default_rng(3)
    raw = inp.synth_q4_k(rng, 64, 1024)
    assert raw.shape == (64, 4 * 144)
    b = raw.reshape(-1, 144)
    sc, m = gb.q4_k_scales(b[:, 4:16])
    assert sc.min() == 0 and sc.max() == 63 and m.min() == 0 and m.max() == 63
    assert (sc[:, 4:] < 16).any() and (sc[:, 4:] >= 48).any() and (m[:, 4:] < 16).any() and (m[:, 4:] >= 48).any()
    d = b[:, 0:2].copy().view(np.float16).astype(np.float64).ravel()
    dmin = b[:, 2:4].copy().view(np.float16).astype(np.float64).ravel()
    assert d.min() >= 0.99e-4 and d.max() <= 1.61e-4
    assert dmin.min() >= 0.79e-3 and dmin.max() <= 1.21e-3
    w = gb.decode_exact(inp.Q4_K, raw, 64, 1024)
    assert 0.025 < w.std() < 0.045
    assert -0.08 < w.min() and w.max() < 0.16
    try:
        import gguf
        from gguf import quants
    except ImportError:
        return
    want = quants.dequantize(raw, gguf.GGMLQuantizationType.Q4_K).astype(np.float32)
    got = gb.deq_f32(inp.Q4_K, raw, 64, 1024).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), want.reshape(64, 1024).view(np.uint32))


# ------------------------------------------------------------------------------------------------
# MoE rounding points (mirror=True)
# ------------------------------------------------------------------------------------------------
def _bf16_torch(v):
    """bf16 rounding of fp64 values through torch's own casts (fp64 -> fp32 -> bf16, nearest even):
    an implementation that shares nothing with the oracle's bit arithmetic."""
    return torch.from_numpy(np.asarray(v, dtype=np.float64)).to(torch.float32).to(torch.bfloat16).to(
        torch.float64).numpy()


def _brute_moe_rounded(X, dY, L, k, Wgu, Wd, Agu, Bgu, Ad, Bd, s, rb):
    """The routed SwiGLU layer, forward and backward, token by token and pair by pair with explicit
    scalar sums (no matmul, no sorting of pairs), with bf16 rounding `rb` applied where the layer
    stores a bf16 value that a later matmul reads: h (down projection, h A_d^T) and d[g|u] (gate/up
    input gradient, s d[g|u] B_gu). The routing-weight gradient <dh_u, h> and the adapter gradients
    dA_d and dB_gu take the unrounded h and d[g|u]; g and u are never rounded."""
    T, H = X.shape
    E, I, r = Wgu.shape[0], Wd.shape[2], Agu.shape[1]
    Y = np.zeros((T, H)); dX = np.zeros((T, H)); dL = np.zeros((T, E))
    dAgu = np.zeros_like(Agu); dBgu = np.zeros_like(Bgu); dAd = np.zeros_like(Ad); dBd = np.zeros_like(Bd)
    for t in range(T):
        sel = sorted(range(E), key=lambda e: (-L[t, e], e))[:k]
        z = [math.exp(L[t, e] - L[t, sel[0]]) for e in sel]
        w = [zi / sum(z) for zi in z]
        x, dy = X[t], dY[t]
        dws = []
        for j, e in enumerate(sel):
            hg = [sum(x[q] * Agu[e, a, q] for q in range(H)) for a in range(r)]
            gu = [sum(x[q] * Wgu[e, n, q] for q in range(H)) + s * sum(hg[a] * Bgu[e, n, a] for a in range(r))
                  for n in range(2 * I)]
            g, u = gu[:I], gu[I:]
            hx = [g[i] / (1.0 + math.exp(-g[i])) * u[i] for i in range(I)]
            h = list(rb(hx))
            hd = [sum(h[i] * Ad[e, a, i] for i in range(I)) for a in range(r)]
            for n in range(H):
                o = sum(h[i] * Wd[e, n, i] for i in range(I)) + s * sum(hd[a] * Bd[e, n, a] for a in range(r))
                Y[t, n] += w[j] * o
            Gd = [s * sum(dy[n] * Bd[e, n, a] for n in range(H)) for a in range(r)]
            dhu = [sum(dy[n] * Wd[e, n, i] for n in range(H)) + sum(Gd[a] * Ad[e, a, i] for a in range(r))
                   for i in range(I)]
            dws.append(sum(dhu[i] * hx[i] for i in range(I)))
            sg = [1.0 / (1.0 + math.exp(-g[i])) for i in range(I)]
            dgx = ([w[j] * dhu[i] * u[i] * sg[i] * (1.0 + g[i] * (1.0 - sg[i])) for i in range(I)]
                   + [w[j] * dhu[i] * g[i] * sg[i] for i in range(I)])
            dgr = list(rb(dgx))
            Ggu = [s * sum(dgr[n] * Bgu[e, n, a] for n in range(2 * I)) for a in range(r)]
            for q in range(H):
                dX[t, q] += (sum(dgr[n] * Wgu[e, n, q] for n in range(2 * I))
                             + sum(Ggu[a] * Agu[e, a, q] for a in range(r)))
            for a in range(r):
                for i in range(I):
                    dAd[e, a, i] += w[j] * Gd[a] * hx[i]
                for n in range(H):
                    dBd[e, n, a] += s * w[j] * dy[n] * hd[a]
                for q in range(H):
                    dAgu[e, a, q] += Ggu[a] * x[q]
                for n in range(2 * I):
                    dBgu[e, n, a] += s * dgx[n] * hg[a]
        tot = sum(w[i] * dws[i] for i in range(k))
        for j, e in enumerate(sel):
            dL[t, e] = w[j] * (dws[j] - tot)
    return dict(Y=Y, dX=dX, dA_gu=dAgu, dB_gu=dBgu, dA_d=dAd, dB_d=dBd, d_logits=dL)


def _tiny_moe_f64(seed=11, T=3, H=12, I=6, E=3, k=2, r=2):
    rng = np.random.default_rng(seed)
    n = lambda *shape, sd=1.0: rng.standard_normal(shape) * sd  # noqa: E731
    return dict(X=n(T, H), dY=n(T, H), L=n(T, E), Wgu=n(E, 2 * I, H, sd=0.4), Wd=n(E, H, I, sd=0.4),
                Agu=n(E, r, H, sd=0.3), Bgu=n(E, 2 * I, r, sd=0.3), Ad=n(E, r, I, sd=0.3), Bd=n(E, H, r, sd=0.3),
                s=1.5, k=k)


def _oracle_moe_f64(d, mirror):
    idx, w, counts, offsets, perm, inv = om.route(d["L"], d["k"])
    Y, saved = om.moe_fwd(d["Wgu"], d["Wd"], d["X"], idx, w, counts, offsets, perm, d["Agu"], d["Bgu"], d["Ad"],
                          d["Bd"], d["s"], mirror=mirror)
    gr = om.moe_bwd(d["Wgu"], d["Wd"], d["X"], d["dY"], idx, w, counts, offsets, perm, d["Agu"], d["Bgu"],
                    d["Ad"], d["Bd"], d["s"], saved, mirror=mirror)
    gr["Y"] = Y
    gr["d_logits"] = om.scatter_d_logits(idx, gr["d_logits_sel"], d["L"].shape[1])
    return gr, saved, (idx, w, perm)


@pytest.mark.parametrize("mirror", [True, False])
def test_moe_rounding_points_vs_brute_force(mirror):
    """Each bf16 rounding point of the MoE oracle, pinned by a scalar brute-force evaluation that
    applies torch's bf16 cast at the layer's storage points (or none, for mirror=False). Moving a
    rounding point (rounded h into dA_d or <dh_u, h>, rounded d[g|u] into dB_gu, a rounded g or u in
    the SwiGLU derivative, a rounded pair output) changes some output by about 2^-9 relative, far
    above the 1e-12 agreement asked here."""
    d = _tiny_moe_f64()
    rb = _bf16_torch if mirror else (lambda v: np.asarray(v, dtype=np.float64))
    want = _brute_moe_rounded(d["X"], d["dY"], d["L"], d["k"], d["Wgu"], d["Wd"], d["Agu"], d["Bgu"], d["Ad"],
                              d["Bd"], d["s"], rb)
    got, _, _ = _oracle_moe_f64(d, mirror)
    for name in want:
        scale = max(1.0, float(np.abs(want[name]).max()))
        assert np.allclose(got[name], want[name], rtol=1e-12, atol=1e-12 * scale), name


def test_moe_rounding_points_are_live_and_bounded():
    """mirror=True differs from mirror=False where a rounded value reaches the output (Y, dX, dA_gu,
    dB_d) and nowhere else (d_logits, dA_d, dB_gu), and by no more than the bf16 bound: Y depends on the rounding of h only through a linear map, so
    |Y_m - Y_x| <= sum_j w_j sum_i |dh_i| |Wd[:, i] + s Bd Ad[:, i]| with |dh_i| <= 2^-8 (1 + 2^-15) |h_i|
    (bf16 unit roundoff 2^-8, plus the fp32 step before it); dX likewise through the rounding of
    d[g|u] and W_gu + s B_gu A_gu."""
    d = _tiny_moe_f64(seed=12)
    gm, sm, (idx, w, perm) = _oracle_moe_f64(d, True)
    gx, sx, _ = _oracle_moe_f64(d, False)
    k = d["k"]
    u = 2.0 ** -8 * (1 + 2.0 ** -15)
    T, H = d["X"].shape
    for name in ["Y", "dX", "dA_gu", "dB_d"]:
        assert np.abs(gm[name] - gx[name]).max() > 1e-9, name      # the rounding reaches these outputs
    for name in ["d_logits", "dA_d", "dB_gu"]:
        assert np.array_equal(gm[name], gx[name]), name             # and these take no rounded value
    # g and u are not rounding points
    assert np.array_equal(sm["g"], sx["g"]) and np.array_equal(sm["u"], sx["u"])
    bY = np.zeros((T, H))
    bX = np.zeros((T, H))
    hx = sx["h"]
    for pos, pair in enumerate(perm):
        t, j = divmod(int(pair), k)
        e = idx[t, j]
        Md = np.abs(d["Wd"][e] + d["s"] * d["Bd"][e] @ d["Ad"][e])          # [H, I]
        bY[t] += w[t, j] * (Md @ (u * np.abs(hx[pos])))
        Mgu = np.abs(d["Wgu"][e] + d["s"] * d["Bgu"][e] @ d["Agu"][e])      # [2I, H]
        # d[g|u] of the pair without rounding: the smooth backward's value
        dgu_x = _pair_dgu(d, sx, pos, t, e, w[t, j])
        bX[t] += (u * np.abs(dgu_x)) @ Mgu
    assert np.all(np.abs(gm["Y"] - gx["Y"]) <= bY * (1 + 1e-9) + 1e-15)
    assert np.all(np.abs(gm["dX"] - gx["dX"]) <= bX * (1 + 1e-9) + 1e-15)


def _pair_dgu(d, saved, pos, t, e, w):
    """d[g|u] of one pair from the smooth (unrounded) forward values, written out elementwise."""
    g, uu = saved["g"][pos], saved["u"][pos]
    dy = d["dY"][t]
    Gd = d["s"] * (dy @ d["Bd"][e])
    dhu = dy @ d["Wd"][e] + Gd @ d["Ad"][e]
    sg = 1.0 / (1.0 + np.exp(-g))
    return np.concatenate([w * dhu * uu * sg * (1 + g * (1 - sg)), w * dhu * g * sg])


def test_synth_q8_0_blocks_have_the_stated_fields():
    """The lm_head workload's Q8_0 blocks are drawn as bytes: d in its range, codes in [-127, 127],
    and gguf-py decodes them to the oracle's values."""
    rng = np.random.default_rng(4)
    raw = inp.synth_q8_0(rng, 16, 512)
    b = raw.reshape(-1, 34)
    d = b[:, 0:2].copy().view(np.float16).astype(np.float64).ravel()
    q = b[:, 2:].view(np.int8)
    assert d.min() >= 0.99e-4 and d.max() <= 3.01e-4 and q.min() >= -127 and q.max() <= 127
    w = gb.decode_exact(inp.Q8_0, raw, 16, 512)
    assert 0.008 < w.std() < 0.02
    try:
        import gguf
        from gguf import quants
    except ImportError:
        return
    want = quants.dequantize(raw, gguf.GGMLQuantizationType.Q8_0).astype(np.float32)
    assert np.array_equal(gb.deq_f32(inp.Q8_0, raw, 16, 512).astype(np.float32).view(np.uint32),
                          want.reshape(16, 512).view(np.uint32))
