"""The forward entry point that allocates nothing (qlora_linear_fwd_noalloc) against the regular
forward with a caller-provided workspace and against the oracle.

Some callers cannot allocate device memory (their device pool is owned by a caching allocator, or
an allocation's device-wide synchronisation is not acceptable where they run), so they cannot pass a
workspace; this entry point uses the library's own static device scratch instead. This file is
collected last so that a run that stops at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

from quantized_base_lora_tma_b200 import inputs as inp

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import quantized_base_lora_tma_b200 as ql
    from tests.gpu_util import assert_close, dev_bf16, dev_u8, f64

from oracle import gguf_blocks as gb
from oracle import lora_linear as ll


def _forward_both(c):
    X, A, B = dev_bf16(c.X), dev_bf16(c.A), dev_bf16(c.B)
    wq = dev_u8(c.wq)
    M, N, K, r = c.M, c.N, c.K, c.r
    ws = torch.empty(ql.qlora_linear_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    Y_ws = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    H_ws = torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda")
    ql.qlora_linear_fwd(c.qtype, wq, N, K, X, A, B, r, c.scale, Y_ws, H_ws, ws)
    Y_na = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    H_na = torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda")
    ql.qlora_linear_fwd_noalloc(c.qtype, wq, N, K, X, A, B, r, c.scale, Y_na, H_na)
    torch.cuda.synchronize()
    return f64(Y_ws), f64(H_ws), f64(Y_na), f64(H_na)


def _oracle_fwd(c):
    W = ll.weights(c.qtype, c.wq, c.N, c.K)
    f = gb.bf16_bits_to_f64
    return ll.linear_fwd(W, f(c.X), f(c.A), f(c.B), c.scale)


# (M, K, N, qtype, r): pair-tile sizes, the decode-sized and single-tile sizes where the regular
# forward takes the weight stream or a K split and this one the plain single-CTA GEMM, and a size
# whose adapter operands fill the 4 MiB array exactly ((512 + 32256) rows x 128 bytes).
NOALLOC_CASES = [(300, 512, 384, inp.Q4_K, 16), (129, 768, 320, inp.Q8_0, 40), (4, 1024, 512, inp.Q4_0, 16),
                 (64, 512, 640, inp.Q4_K, 8), (512, 256, 32256, inp.Q4_0, 4)]


def test_noalloc_forward_matches_workspace_forward_twice():
    ql.qlora_device_status(reset=True)
    # calls in a row, each with other sizes and values than the one before
    for i, (M, K, N, qt, r) in enumerate(NOALLOC_CASES):
        c = inp.linear_case(M, K, N, qt, r, 2.0 * r, seed=21 + i)
        Y_ws, H_ws, Y_na, H_na = _forward_both(c)
        assert_close(Y_na, Y_ws, f"Y vs workspace forward {M}x{K}x{N}")
        assert_close(H_na, H_ws, f"H vs workspace forward {M}x{K}x{N}")
        Yr, Hr = _oracle_fwd(c)
        assert_close(Y_na, Yr, f"Y vs oracle {M}x{K}x{N}")
        assert_close(H_na, Hr, f"H vs oracle {M}x{K}x{N}")
    rc, site = ql.qlora_device_status(reset=True)
    assert rc == 0, (rc, site)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = ql.lib()
    fake = 1 << 20
    # M + N far beyond the 4 MiB of static scratch: refused before any launch
    before = ql.qlora_launch_count()
    rc = lib.qlora_linear_fwd_noalloc(inp.Q4_0, fake, 65536, 256, fake, 65536, fake, fake, 16, 2.0, fake, 0,
                                      fake, None)
    assert rc == 5
    # one 64-row block past the exact fit of the last case above
    rc = lib.qlora_linear_fwd_noalloc(inp.Q4_0, fake, 32320, 256, fake, 512, fake, fake, 4, 2.0, fake, 0,
                                      fake, None)
    assert rc == 5
    assert ql.qlora_launch_count() == before
