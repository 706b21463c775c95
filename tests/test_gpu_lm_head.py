"""GPU parity: the quantized lm_head with chunked cross-entropy (qlora_lm_head_ce) against the
oracle: per-token losses and the input gradient, with ragged chunks and ignored tokens."""
import numpy as np
import pytest
import torch

from oracle import gguf_blocks as gb
from oracle import lm_head as lh
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


@pytest.mark.parametrize("M,V,K,chunk,qtype", [(300, 1024, 512, 128, inp.Q8_0), (600, 32000, 1024, 256, inp.Q4_K),
                                               (5, 4096, 256, 64, inp.Q5_K), (260, 2048, 256, 260, inp.Q4_0),
                                               (700, 4160, 512, 384, inp.Q8_0)])  # a partial last column tile
def test_lm_head_ce_matches_oracle(M, V, K, chunk, qtype):
    rng = np.random.default_rng(M + V)
    W = (rng.standard_normal((V, K)) * 0.05).astype(np.float32)
    wq = inp.pack(qtype, W)
    X = inp.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    labels = rng.integers(0, V, M).astype(np.int32)
    labels[::17] = -100
    ws = torch.empty(ql.qlora_lm_head_ce_workspace_bytes(M, V, K, chunk), dtype=torch.uint8, device="cuda")
    loss = torch.full((M,), float("nan"), dtype=torch.float32, device="cuda")
    dX = torch.full((M, K), float("nan"), dtype=torch.float32, device="cuda")
    ql.qlora_lm_head_ce(qtype, dev_u8(wq), V, K, dev_bf16(X), torch.from_numpy(labels).cuda(), chunk, 1.0 / M,
                        loss, dX, ws)
    torch.cuda.synchronize()
    Wd = gb.deq_bf16(qtype, wq, V, K)
    loss_r, dX_r, _ = lh.lm_head_ce(Wd, gb.bf16_bits_to_f64(X), labels, grad_scale=1.0 / M)
    assert_close(f64(loss), loss_r, "loss")
    assert_close(f64(dX), dX_r, "dX")
