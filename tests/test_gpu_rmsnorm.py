"""GPU parity: RMSNorm forward and backward (qlora_rmsnorm_fwd / _bwd) against the oracle, alone and
in front of the quantized LoRA projection (norm -> linear forward -> linear backward -> norm
backward)."""
import numpy as np
import pytest
import torch

from oracle import gguf_blocks as gb
from oracle import lora_linear as ll
from oracle import rmsnorm as rn
from quantized_base_lora_tma_b200 import inputs as inp

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import quantized_base_lora_tma_b200 as ql
    from tests.gpu_util import assert_close, dev_bf16, dev_u8, f64


@pytest.fixture(autouse=True)
def _status():
    ql.qlora_device_status(reset=True)
    yield
    rc, site = ql.qlora_device_status(reset=True)
    assert rc == 0, f"device status {rc} at site {site}"


@pytest.mark.parametrize("M,K", [(37, 768), (2048, 4096), (3, 8)])
def test_rmsnorm_alone(M, K):
    rng = np.random.default_rng(M + K)
    X = inp.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) * np.float32(2.0))
    gam = inp.to_bf16_bits((1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32))
    d = rng.standard_normal((M, K)).astype(np.float32)
    eps = 1e-6
    Xd, gd = dev_bf16(X), dev_bf16(gam)
    Xn = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    r = torch.empty(M, dtype=torch.float32, device="cuda")
    ql.qlora_rmsnorm_fwd(Xd, gd, eps, Xn, r)
    dX = torch.empty(M, K, dtype=torch.float32, device="cuda")
    ql.qlora_rmsnorm_bwd(Xd, gd, r, torch.from_numpy(d).cuda(), dX)
    torch.cuda.synchronize()
    Xf, gf = gb.bf16_bits_to_f64(X), gb.bf16_bits_to_f64(gam)
    Xn_ref, r_ref = rn.rmsnorm_fwd(Xf, gf, eps)
    assert np.allclose(f64(r), r_ref, rtol=2e-6, atol=0)
    assert_close(f64(Xn), Xn_ref, "Xn", bf16_out=True)
    assert_close(f64(dX), rn.rmsnorm_bwd(Xf, gf, r_ref, d.astype(np.float64)), "dX")


def test_rmsnorm_before_the_projection():
    """x -> RMSNorm -> Q4_K LoRA projection, forward and backward, against the oracle chain (the
    oracle feeds its own bf16 x_n to the linear oracle)."""
    M, K, N, r = 300, 512, 384, 8
    c = inp.linear_case(M, K, N, inp.Q4_K, r, 16.0, seed=9)
    rng = np.random.default_rng(10)
    gam = inp.to_bf16_bits((1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32))
    eps = 1e-5
    Xd, gd = dev_bf16(c.X), dev_bf16(gam)
    wq, A, B, dY = dev_u8(c.wq), dev_bf16(c.A), dev_bf16(c.B), dev_bf16(c.dY)
    Xn = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    rs = torch.empty(M, dtype=torch.float32, device="cuda")
    ws = torch.empty(ql.qlora_linear_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    H = torch.empty(M, r, dtype=torch.float32, device="cuda")
    dXn = torch.empty(M, K, dtype=torch.float32, device="cuda")
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
    dX = torch.empty(M, K, dtype=torch.float32, device="cuda")
    ql.qlora_rmsnorm_fwd(Xd, gd, eps, Xn, rs)
    ql.qlora_linear_fwd(c.qtype, wq, N, K, Xn, A, B, r, c.scale, Y, H, ws)
    ql.qlora_linear_bwd(c.qtype, wq, N, K, Xn, dY, A, B, r, c.scale, H, dXn, dA, dB, ws)
    ql.qlora_rmsnorm_bwd(Xd, gd, rs, dXn, dX)
    torch.cuda.synchronize()
    f = gb.bf16_bits_to_f64
    Xn_ref, r_ref = rn.rmsnorm_fwd(f(c.X), f(gam), eps)
    W = ll.weights(c.qtype, c.wq, N, K)
    Y_ref, H_ref = ll.linear_fwd(W, Xn_ref, f(c.A), f(c.B), c.scale)
    dXn_ref, dA_ref, dB_ref, _ = ll.linear_bwd(W, Xn_ref, f(c.dY), f(c.A), f(c.B), c.scale, H_ref)
    dX_ref = rn.rmsnorm_bwd(f(c.X), f(gam), r_ref, dXn_ref)
    for got, ref, name in [(Y, Y_ref, "Y"), (dA, dA_ref, "dA"), (dB, dB_ref, "dB"), (dX, dX_ref, "dX")]:
        assert_close(f64(got), ref, name)
