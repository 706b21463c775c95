"""The forward entry point that allocates nothing (qlora_linear_fwd_noalloc) against the regular
forward with a caller-provided workspace.

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


def test_noalloc_forward_matches_workspace_forward_twice():
    ql.qlora_device_status(reset=True)
    # two calls in a row, the second with other sizes and values than the first
    cases = [inp.linear_case(300, 512, 384, inp.Q4_K, 16, 32.0, seed=21),
             inp.linear_case(129, 768, 320, inp.Q8_0, 40, 80.0, seed=22)]
    for c in cases:
        Y_ws, H_ws, Y_na, H_na = _forward_both(c)
        assert_close(Y_na, Y_ws, "Y")
        assert_close(H_na, H_ws, "H")
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
    assert ql.qlora_launch_count() == before
