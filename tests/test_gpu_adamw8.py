"""GPU parity: the 8-bit AdamW step (qlora_adamw8_step) against the oracle. The codes and scales are
integers and exact maxima decided in fp32 by both sides in the same order, so they must agree bit
for bit; so must the fp32 parameters and their bf16 copy."""
import numpy as np
import pytest
import torch

from oracle import adamw8 as aw

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import quantized_base_lora_tma_b200 as ql


@pytest.fixture(autouse=True)
def _status():
    ql.qlora_device_status(reset=True)
    yield
    rc, site = ql.qlora_device_status(reset=True)
    assert rc == 0, f"device status {rc} at site {site}"


@pytest.mark.parametrize("n,start", [(1000, "random"), (256 * 7, "zero"), (33, "random"), (131072, "random")])
def test_adamw8_matches_oracle(n, start):
    rng = np.random.default_rng(n)
    nb = (n + 255) // 256
    p = rng.standard_normal(n).astype(np.float32) * np.float32(0.02)
    if start == "zero":
        mq, ma = np.zeros(n, np.uint8), np.zeros(nb, np.float32)
        vq, va = np.zeros(n, np.uint8), np.zeros(nb, np.float32)
    else:  # every code of both tables appears, with varied block scales (one block all zero)
        mq = rng.integers(0, 256, n).astype(np.uint8)
        vq = rng.integers(0, 256, n).astype(np.uint8)
        ma = (rng.uniform(0.0, 0.02, nb)).astype(np.float32)
        va = (rng.uniform(0.0, 4e-4, nb)).astype(np.float32)
        ma[0] = va[0] = 0
    lr, b1, b2, eps, wd = 1e-3, 0.9, 0.999, 1e-8, 0.01
    st = ql.Adamw8State(n)
    st.m_q.copy_(torch.from_numpy(mq))
    st.v_q.copy_(torch.from_numpy(vq))
    st.m_absmax.copy_(torch.from_numpy(ma))
    st.v_absmax.copy_(torch.from_numpy(va))
    pd = torch.from_numpy(p.copy()).cuda()
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    for t in range(1, 5):
        g = (rng.standard_normal(n) * 0.01).astype(np.float32)
        if t == 2:
            g[:min(n, 300)] = 0  # zero gradients: the moments only decay
        ql.qlora_adamw8_step(pd, torch.from_numpy(g).cuda(), st, t, lr, b1, b2, eps, wd, p_bf16=pb)
        c1 = np.float32(1.0 - float(np.float32(b1)) ** t)
        c2 = np.float32(1.0 - float(np.float32(b2)) ** t)
        p, mq, ma, vq, va = aw.adamw8_step(p, g, mq, ma, vq, va, lr, b1, b2, eps, wd, c1, c2)
        torch.cuda.synchronize()
        assert np.array_equal(st.m_absmax.cpu().numpy(), ma), t
        assert np.array_equal(st.v_absmax.cpu().numpy(), va), t
        assert np.array_equal(st.m_q.cpu().numpy(), mq), (t, int((st.m_q.cpu().numpy() != mq).sum()))
        assert np.array_equal(st.v_q.cpu().numpy(), vq), (t, int((st.v_q.cpu().numpy() != vq).sum()))
        assert np.array_equal(pd.cpu().numpy().view(np.uint32), p.view(np.uint32)), t
        want_b = torch.from_numpy(p.copy()).to(torch.bfloat16)
        assert torch.equal(pb.cpu(), want_b), t
