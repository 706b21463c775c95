"""Pins for the 8-bit AdamW oracle (oracle/adamw8.py): hand-computed code values, table invariants,
the quantization error bound, the closed form of the first step, and agreement with the plain fp64
AdamW over several steps."""
import numpy as np
import pytest

from oracle import adamw8 as aw


def test_table_hand_values():
    """Codes whose values follow from the bit layout by hand: sign, E leading zeros, indicator,
    B = bits after it, F = those bits; |T| = (0.1 + 0.9 (F + 1/2) / 2^B) / 10^E."""
    s = aw.dynamic_table(True)
    u = aw.dynamic_table(False)
    # signed: 0 | 1 111111 -> E 0, B 6, F 63
    assert s[0b01111111] == np.float32(0.1 + 0.9 * 63.5 / 64)
    # signed: 1 | 1 000000 -> negative, E 0, F 0
    assert s[0b11000000] == np.float32(-(0.1 + 0.9 * 0.5 / 64))
    # signed: 0 | 000000 1 -> E 6, B 0
    assert s[0b00000001] == np.float32(0.55e-6)
    # signed: 0 | 01 10101 -> E 1, B 5, F 21
    assert s[0b00110101] == np.float32((0.1 + 0.9 * 21.5 / 32) / 10)
    # unsigned: 1 0000000 -> E 0, B 7, F 0 ; 00000001 -> E 7, B 0 ; 0001 1111 -> E 3, B 4, F 15
    assert u[0b10000000] == np.float32(0.1 + 0.9 * 0.5 / 128)
    assert u[0b00000001] == np.float32(0.55e-7)
    assert u[0b00011111] == np.float32((0.1 + 0.9 * 15.5 / 16) / 1000)
    assert s[0] == 0 and s[0x80] == 0 and u[0] == 0


def test_table_invariants():
    for signed, n_distinct in [(True, 255), (False, 256)]:
        T = aw.dynamic_table(signed).astype(np.float64)
        assert len(np.unique(T)) == n_distinct
        assert np.abs(T).max() < 1.0
        if signed:
            assert np.array_equal(np.sort(T[0:128]), np.sort(-T[128:256]))  # symmetric
        else:
            assert T.min() == 0
        # decades tile: every entry of decade E lies in [0.1, 1) / 10^E
        for q in range(256):
            bits = q & (127 if signed else 255)
            if bits:
                E = (7 if signed else 8) - bits.bit_length()
                assert 0.1 / 10 ** E <= abs(T[q]) < 1.0 / 10 ** E


@pytest.mark.parametrize("signed", [True, False])
def test_quantize_error_bound(signed):
    """Each value comes back within half the gap to its neighbouring table entries (times absmax),
    and the block's absmax value itself comes back within half the gap below the top entry."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal(1000).astype(np.float32) * np.float32(0.01)
    x[512:768] = 0                                    # one all-zero block
    if not signed:
        x = np.abs(x)
    q, a = aw.quantize_blocks(x, signed)
    assert a[2] == 0 and np.all(q[512:768] == 0) and np.all(a[[0, 1, 3]] > 0)
    y = aw.decode(q, a, signed).astype(np.float64)
    vals = np.sort(np.unique(aw.dynamic_table(signed).astype(np.float64)))
    ar = np.repeat(a.astype(np.float64), aw.QBLOCK)[:x.size]
    xn = np.where(ar > 0, x / np.where(ar > 0, ar, 1), 0)
    i = np.clip(np.searchsorted(vals, xn), 1, len(vals) - 1)
    gap = np.maximum(vals[i] - vals[i - 1], 0)
    assert np.all(np.abs(y - x) <= (0.5 * gap * (1 + 1e-6) + 2e-7) * ar + 1e-30)
    assert np.all(y[x == 0] == 0)


def test_first_step_closed_form():
    """From zero states at t = 1 the bias corrections cancel: m/c1 = g and sqrt(v/c2) = |g|, so
    p' = p - lr (g / (|g| + eps) + wd p) up to fp32 rounding (the quantized states do not enter)."""
    rng = np.random.default_rng(4)
    n = 700
    p = rng.standard_normal(n).astype(np.float32)
    g = rng.standard_normal(n).astype(np.float32)
    nb = (n + 255) // 256
    zq, za = np.zeros(n, np.uint8), np.zeros(nb, np.float32)
    lr, b1, b2, eps, wd = 1e-3, 0.9, 0.999, 1e-8, 0.01
    c1, c2 = np.float32(1 - np.float32(b1)), np.float32(1 - np.float32(b2))
    p1, *_ = aw.adamw8_step(p, g, zq, za, zq, za, lr, b1, b2, eps, wd, c1, c2)
    want = p.astype(np.float64) - lr * (np.sign(g) * np.abs(g) / (np.abs(g) + eps) + wd * p.astype(np.float64))
    assert np.allclose(p1, want, rtol=0, atol=1e-6)


def test_steps_track_exact_adamw():
    """Ten steps with 8-bit states stay close to the plain fp64 AdamW: the coarse codes at the foot of
    each decade move single updates by up to several percent, so after ten steps of about lr each
    the parameters differ by well under one step (a wrong sign or a dropped moment term would move
    them by many steps)."""
    rng = np.random.default_rng(5)
    n = 1024
    p8 = rng.standard_normal(n).astype(np.float32) * np.float32(0.02)
    pe = p8.astype(np.float64)
    nb = n // 256
    mq, ma = np.zeros(n, np.uint8), np.zeros(nb, np.float32)
    vq, va = np.zeros(n, np.uint8), np.zeros(nb, np.float32)
    me, ve = np.zeros(n), np.zeros(n)
    lr, b1, b2, eps, wd = 1e-3, 0.9, 0.999, 1e-8, 0.0
    base = rng.standard_normal(n)
    for t in range(1, 11):
        g = (base + 0.3 * rng.standard_normal(n)).astype(np.float32) * np.float32(0.01)
        c1 = np.float32(1 - float(np.float32(b1)) ** t)
        c2 = np.float32(1 - float(np.float32(b2)) ** t)
        p8, mq, ma, vq, va = aw.adamw8_step(p8, g, mq, ma, vq, va, lr, b1, b2, eps, wd, c1, c2)
        pe, me, ve = aw.adamw_exact_step(pe, g, me, ve, lr, float(np.float32(b1)), float(np.float32(b2)), eps, wd, t)
    assert np.abs(p8 - pe).max() < 0.8 * lr
    assert np.abs(p8 - pe).mean() < 0.15 * lr
