"""GPU parity: gguf_dequant and the dense layer (forward + backward) through the C ABI, against the
oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

from oracle import gguf_blocks as gb
from oracle import lora_linear as ll
from quantized_base_lora_tma_b200 import inputs as inp

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import quantized_base_lora_tma_b200 as ql
    from tests.gpu_util import assert_close, bf16_f64, dev_bf16, dev_u8, f64


@pytest.fixture(autouse=True)
def _reset_status():
    ql.qlora_device_status(reset=True)
    yield
    rc, site = ql.qlora_device_status(reset=True)
    assert rc == 0, f"device status {rc} at site {site}"


def _random_packed(qtype, rows, cols, rng):
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    raw = inp.pack(qtype, w)
    # sprinkle subnormal and zero scales (d of Q4_0 / Q8_0 blocks, d of Q6_K and Q2_K superblocks)
    off = {inp.Q4_0: 0, inp.Q8_0: 0, inp.Q6_K: 208, inp.Q2_K: 80}.get(qtype)
    if off is not None:
        bb = inp.BLOCK_BYTES[qtype]
        v = raw.reshape(-1, bb)
        v[::5, off:off + 2] = np.frombuffer(np.float16(3.0e-6).tobytes(), np.uint8)
        v[::13, off:off + 2] = 0
    return raw


@pytest.mark.parametrize("qtype", [inp.Q4_0, inp.Q8_0, inp.Q4_K, inp.Q5_K, inp.Q6_K, inp.Q2_K])
def test_dequant_bit_exact(qtype):
    rng = np.random.default_rng(qtype)
    rows, cols = 37, 768
    raw = _random_packed(qtype, rows, cols, rng)
    wq = dev_u8(raw)
    for dt, ref in [(torch.float32, gb.deq_f32(qtype, raw, rows, cols)),
                    (torch.bfloat16, gb.deq_bf16(qtype, raw, rows, cols))]:
        out = torch.empty(rows, cols, dtype=dt, device="cuda")
        ql.gguf_dequant(qtype, wq, rows, cols, out)
        torch.cuda.synchronize()
        got = f64(out)
        assert np.array_equal(got, ref), f"{dt}: {np.sum(got != ref)} mismatches"


def run_linear(c, y_dtype=torch.float32, dx_dtype=torch.float32, with_dx=True):
    X, dY, A, B = dev_bf16(c.X), dev_bf16(c.dY), dev_bf16(c.A), dev_bf16(c.B)
    wq = dev_u8(c.wq)
    M, N, K, r = c.M, c.N, c.K, c.r
    ws = torch.empty(ql.qlora_linear_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    Y = torch.full((M, N), float("nan"), dtype=y_dtype, device="cuda")
    H = torch.empty(M, r, dtype=torch.float32, device="cuda")
    ql.qlora_linear_fwd(c.qtype, wq, N, K, X, A, B, r, c.scale, Y, H, ws)
    dX = torch.full((M, K), float("nan"), dtype=dx_dtype, device="cuda") if with_dx else None
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
    ql.qlora_linear_bwd(c.qtype, wq, N, K, X, dY, A, B, r, c.scale, H, dX, dA, dB, ws)
    torch.cuda.synchronize()
    return Y, H, dX, dA, dB


def oracle_linear(c, rows=None):
    W = ll.weights(c.qtype, c.wq, c.N, c.K)
    X, dY, A, B = bf16_f64(c.X), bf16_f64(c.dY), bf16_f64(c.A), bf16_f64(c.B)
    H = X @ A.T
    dX_rows = None
    if rows is None:
        Y, _ = ll.linear_fwd(W, X, A, B, c.scale)
        dX, dA, dB, _ = ll.linear_bwd(W, X, dY, A, B, c.scale, H)
        return Y, H, dX, dA, dB
    Y, _ = ll.linear_fwd(W, X[rows], A, B, c.scale)
    dX, _, _, _ = ll.linear_bwd(W, X[rows], dY[rows], A, B, c.scale, H[rows])
    G = c.scale * (dY @ B)
    dA = G.T @ X
    dB = c.scale * (dY.T @ H)
    return Y, H, dX, dA, dB


SMALL = [
    # (M, K, N, r): several tiles in every dimension and ragged tails
    (300, 512, 384, 4),
    (129, 768, 320, 16),
    (1, 256, 64, 1),
    (200, 256, 448, 40),   # r > 32: two LoRA k-blocks
    (64, 1024, 128, 64),
    (16, 2048, 512, 8),    # small M: the K range is split across CTAs (fwd and dX)
    (3, 1024, 1024, 4),
    (1100, 512, 4096, 8),  # more pair tiles than SM pairs: forward without a K split
    (1100, 4096, 512, 8),  # the same for the input-gradient GEMM
    (9, 1280, 192, 16),    # decode path: two token tiles, two adapter tiles, K steps not a multiple of the split
    (13, 768, 64, 12),     # decode path: one row block, ragged rank
    (7, 512, 384, 16),     # small-M backward: G in one CTA (Q4_0), full adapter tile
    (5, 768, 256, 12),     # the same with a ragged rank
    (4500, 256, 320, 8),   # adapter gradients from three row chunks (partials summed in chunk order)
    (2600, 256, 192, 40),  # the same with r > 32 (128-row tiles)
]


@pytest.mark.parametrize("qtype", [inp.Q4_0, inp.Q8_0, inp.Q4_K, inp.Q5_K])
@pytest.mark.parametrize("shape", SMALL)
def test_linear_parity_small(qtype, shape):
    M, K, N, r = shape
    c = inp.linear_case(M, K, N, qtype, r, 2.0 * r, seed=M + K + N + r)
    Y, H, dX, dA, dB = run_linear(c)
    Yr, Hr, dXr, dAr, dBr = oracle_linear(c)
    for got, ref, name in [(Y, Yr, "Y"), (H, Hr, "H"), (dX, dXr, "dX"), (dA, dAr, "dA"), (dB, dBr, "dB")]:
        assert_close(f64(got), ref, name)


def test_linear_q4_0_64x256x512_bf16_outputs():
    c = inp.q4_0_linear_64x256x512()
    Y, H, dX, dA, dB = run_linear(c, torch.bfloat16, torch.bfloat16)
    Yr, Hr, dXr, dAr, dBr = oracle_linear(c)
    assert_close(f64(Y), Yr, "Y", bf16_out=True)
    assert_close(f64(dX), dXr, "dX", bf16_out=True)
    assert_close(f64(dA), dAr, "dA")
    assert_close(f64(dB), dBr, "dB")


def test_linear_b_zero_gives_exact_zero_dA():
    c = inp.linear_case(130, 512, 256, inp.Q8_0, 8, 16.0, seed=3)
    c.B[:] = 0
    Y, H, dX, dA, dB = run_linear(c)
    assert torch.count_nonzero(dA).item() == 0
    Yr, Hr, dXr, dAr, dBr = oracle_linear(c)
    assert_close(f64(Y), Yr, "Y")
    assert_close(f64(dB), dBr, "dB")


@pytest.fixture
def unfused():
    """Row products in their own launch before each pair GEMM (the path without idle clusters)."""
    prev = ql.qlora_set_rows_fusion(False)
    try:
        yield
    finally:
        ql.qlora_set_rows_fusion(prev)


PAIR_SHAPES = [(300, 512, 384, 4), (129, 768, 320, 16), (200, 256, 448, 40), (1100, 512, 4096, 8),
               (4500, 256, 320, 8)]


@pytest.mark.parametrize("mask", [0, 3])
@pytest.mark.parametrize("qtype", [inp.Q8_0, inp.Q4_K])
@pytest.mark.parametrize("shape", PAIR_SHAPES)
def test_linear_parity_fusion_modes(qtype, shape, mask):
    """Row products in their own launches (mask 0) and inside both GEMMs (mask 3); the default
    (forward only) is what the other parity tests run."""
    M, K, N, r = shape
    c = inp.linear_case(M, K, N, qtype, r, 2.0 * r, seed=M + K + N + r)
    prev = ql.qlora_set_rows_fusion(mask)
    try:
        Y, H, dX, dA, dB = run_linear(c)
    finally:
        ql.qlora_set_rows_fusion(prev)
    Yr, Hr, dXr, dAr, dBr = oracle_linear(c)
    for got, ref, name in [(Y, Yr, "Y"), (H, Hr, "H"), (dX, dXr, "dX"), (dA, dAr, "dA"), (dB, dBr, "dB")]:
        assert_close(f64(got), ref, name)


def test_rows_fusion_engages():
    """With idle SM pairs the fused forward is one launch (GEMM with the row products) instead of two,
    and the fused backward two (GEMM, column reductions) instead of three; the results agree within
    the bar."""
    c = inp.linear_case(700, 1024, 768, inp.Q8_0, 16, 32.0, seed=5)
    counts, outs = [], []
    for mask in (3, 1, 0):
        prev = ql.qlora_set_rows_fusion(mask)
        try:
            n0 = ql.qlora_launch_count()
            outs.append([t.clone() for t in run_linear(c)])
            counts.append(ql.qlora_launch_count() - n0)
        finally:
            ql.qlora_set_rows_fusion(prev)
    assert counts == [3, 4, 5], counts
    refs = oracle_linear(c)
    for got in outs:
        for g, ref, name in zip(got, refs, ["Y", "H", "dX", "dA", "dB"]):
            assert_close(f64(g), ref, name)


@pytest.mark.parametrize("shape", [(300, 512, 384, 4), (2600, 256, 192, 40)])
def test_linear_bwd_without_dx(shape, unfused):
    """Without dX the adapter gradients follow the row kernel directly: with the row products in
    their own launch in both runs, the same values, bit for bit."""
    M, K, N, r = shape
    c = inp.linear_case(M, K, N, inp.Q8_0, r, 2.0 * r, seed=M + r)
    a = [t.clone() for t in run_linear(c)]
    b = run_linear(c, with_dx=False)
    assert b[2] is None
    for i in (0, 1, 3, 4):
        assert torch.equal(a[i], b[i])


@pytest.mark.parametrize("shape", [(300, 512, 384, 8), (2600, 256, 192, 40)])
def test_linear_bwd_without_dx_fused(shape):
    """The input-gradient GEMM computes G itself when fused; without dX the row kernel does: both
    sets of adapter gradients are within the bar of the oracle."""
    M, K, N, r = shape
    c = inp.linear_case(M, K, N, inp.Q8_0, r, 2.0 * r, seed=M + r)
    prev = ql.qlora_set_rows_fusion(3)
    try:
        a = [t.clone() for t in run_linear(c)]
        b = run_linear(c, with_dx=False)
    finally:
        ql.qlora_set_rows_fusion(prev)
    refs = oracle_linear(c)
    for run in (a, b):
        for i, name in [(3, "dA"), (4, "dB")]:
            assert_close(f64(run[i]), refs[i], name)


def test_linear_deterministic():
    c = inp.linear_case(257, 512, 256, inp.Q4_K, 8, 16.0, seed=9)
    a = [t.clone() for t in run_linear(c)]
    b = run_linear(c)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("name", ["dense_q8_0", "dense_q4_0", "gate_up_q4_k"])
def test_linear_full_size_sampled(name):
    """The benchmark's shapes and launch configuration: sampled rows of Y and dX, full dA and dB."""
    c = {"dense_q8_0": lambda: inp.dense_proj_2048x4096x4096(inp.Q8_0),
         "dense_q4_0": lambda: inp.dense_proj_2048x4096x4096(inp.Q4_0),
         "gate_up_q4_k": inp.gate_up_q4_k_2048x2048x12288}[name]()
    Y, H, dX, dA, dB = run_linear(c)
    rows = np.sort(np.random.default_rng(1).choice(c.M, size=24, replace=False))
    rows[0], rows[-1] = 0, c.M - 1
    Yr, Hr, dXr, dAr, dBr = oracle_linear(c, rows)
    assert_close(f64(Y)[rows], Yr, "Y")
    assert_close(f64(H), Hr, "H")
    assert_close(f64(dX)[rows], dXr, "dX")
    assert_close(f64(dA), dAr, "dA")
    assert_close(f64(dB), dBr, "dB")


def test_bounded_wait_self_check():
    ql.qlora_device_status(reset=True)
    ql.qlora_selftest_wait_timeout(20000)
    rc, site = ql.qlora_device_status(reset=True)
    assert rc == 7 and site == 99
    # the context is still usable
    c = inp.linear_case(64, 256, 128, inp.Q4_0, 4, 8.0, seed=1)
    Y, *_ = run_linear(c)
    Yr, *_ = oracle_linear(c)
    assert_close(f64(Y), Yr, "Y")


_W8192 = {}


def _small_m_case(M):
    c = inp.decode_q4_0_8192(M)
    if "W" not in _W8192:
        _W8192["W"] = (c.wq.copy(), ll.weights(c.qtype, c.wq, c.N, c.K))
    assert np.array_equal(_W8192["W"][0], c.wq)
    return c, _W8192["W"][1]


@pytest.mark.parametrize("M", [1, 4, 16])
def test_linear_decode_shape_q4_0_8192(M):
    """Weight-streaming shape: Q4_0, K = N = 8192, M in {1, 4, 16}; full Y, dX, dA, dB."""
    c, W = _small_m_case(M)
    Y, H, dX, dA, dB = run_linear(c)
    X, dY, A, B = bf16_f64(c.X), bf16_f64(c.dY), bf16_f64(c.A), bf16_f64(c.B)
    Yr, Hr = ll.linear_fwd(W, X, A, B, c.scale)
    dXr, dAr, dBr, _ = ll.linear_bwd(W, X, dY, A, B, c.scale, Hr)
    for got, ref, name in [(Y, Yr, "Y"), (H, Hr, "H"), (dX, dXr, "dX"), (dA, dAr, "dA"), (dB, dBr, "dB")]:
        assert_close(f64(got), ref, name)


@pytest.mark.parametrize("qtype", [inp.Q4_0, inp.Q8_0, inp.Q4_K])
def test_linear_repeated_launches_complete(qtype):
    """Many back-to-back forward + backward calls (both GEMM directions, BM = 256 tiles) finish
    without any bounded wait giving up, and give the same result every time."""
    c = inp.linear_case(512, 2048, 1024, qtype, 8, 16.0, seed=31)
    X, dY, A, B = dev_bf16(c.X), dev_bf16(c.dY), dev_bf16(c.A), dev_bf16(c.B)
    wq = dev_u8(c.wq)
    M, N, K, r = c.M, c.N, c.K, c.r
    ws = torch.empty(ql.qlora_linear_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    H = torch.empty(M, r, dtype=torch.float32, device="cuda")
    dX = torch.empty(M, K, dtype=torch.float32, device="cuda")
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
    first = None
    for i in range(60):
        ql.qlora_linear_fwd(c.qtype, wq, N, K, X, A, B, r, c.scale, Y, H, ws)
        ql.qlora_linear_bwd(c.qtype, wq, N, K, X, dY, A, B, r, c.scale, H, dX, dA, dB, ws)
        if i == 0:
            torch.cuda.synchronize()
            first = (Y.clone(), dX.clone())
    torch.cuda.synchronize()
    rc, site = ql.qlora_device_status(reset=False)
    assert rc == 0, f"bounded wait gave up at site {site}"
    assert torch.equal(first[0], Y) and torch.equal(first[1], dX)


def test_linear_cuda_graph_replay():
    """Forward and backward captured once into a CUDA graph and replayed with new inputs copied into
    the same buffers: every replay matches the oracle of its own inputs. (Under capture the row
    products run in their own launch: a fused launch's counter tag would repeat on every replay.)"""
    cases = [inp.linear_case(700, 1024, 768, inp.Q8_0, 16, 32.0, seed=s) for s in (21, 22)]
    c0 = cases[0]
    M, N, K, r = c0.M, c0.N, c0.K, c0.r
    X, dY, A, B = dev_bf16(c0.X), dev_bf16(c0.dY), dev_bf16(c0.A), dev_bf16(c0.B)
    wq = dev_u8(c0.wq)
    ws = torch.empty(ql.qlora_linear_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    H = torch.empty(M, r, dtype=torch.float32, device="cuda")
    dX = torch.empty(M, K, dtype=torch.float32, device="cuda")
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")

    def step():
        ql.qlora_linear_fwd(c0.qtype, wq, N, K, X, A, B, r, c0.scale, Y, H, ws)
        ql.qlora_linear_bwd(c0.qtype, wq, N, K, X, dY, A, B, r, c0.scale, H, dX, dA, dB, ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside the capture (lazy per-kernel set-up)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for c in cases + cases[:1]:
        X.copy_(dev_bf16(c.X))
        dY.copy_(dev_bf16(c.dY))
        A.copy_(dev_bf16(c.A))
        B.copy_(dev_bf16(c.B))
        wq.copy_(dev_u8(c.wq))
        g.replay()
        torch.cuda.synchronize()
        refs = oracle_linear(c)
        for got, ref, name in zip([Y, H, dX, dA, dB], refs, ["Y", "H", "dX", "dA", "dB"]):
            assert_close(f64(got), ref, name)
    del g
