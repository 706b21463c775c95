"""GPU parity: MoE routing (exact) and the routed SwiGLU expert layer with LoRA, forward and
backward, through the C ABI against the oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

from oracle import gguf_blocks as gb
from oracle import moe as om
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


def _check_route(R, logits_bits, k):
    L = gb.bf16_bits_to_f64(logits_bits)
    idx, w, counts, offsets, perm, inv = om.route(L, k)
    assert np.array_equal(R.topk_idx.cpu().numpy(), idx)
    assert np.array_equal(R.counts.cpu().numpy(), counts)
    assert np.array_equal(R.offsets.cpu().numpy(), offsets)
    assert np.array_equal(R.perm.cpu().numpy(), perm)
    assert np.array_equal(R.inv_perm.cpu().numpy(), inv)
    mblk = np.zeros(len(counts) + 1, np.int64)
    mblk[1:] = np.cumsum((counts + 127) // 128)
    assert np.array_equal(R.mblk.cpu().numpy(), mblk)
    assert np.abs(R.topk_w.cpu().numpy().astype(np.float64) - w).max() <= 1e-6
    return idx, w, counts, offsets, perm, inv


@pytest.mark.parametrize("T,E,k,zipf", [(2048, 128, 8, 0.0), (4096, 256, 8, 1.1), (37, 16, 3, 0.0), (5, 4, 4, 0.0),
                                        (1000, 256, 16, 1.1), (777, 33, 1, 0.0)])
def test_route_exact(T, E, k, zipf):
    rng = np.random.default_rng(T + E)
    L = rng.standard_normal((T, E)).astype(np.float32)
    if zipf:
        L -= np.float32(zipf) * np.log(np.arange(1, E + 1, dtype=np.float32))
    L[0, :] = 0.25            # all-equal row: experts 0..k-1
    a, b = min(3, E - 2), min(7, E - 1)
    L[1, a] = L[1, b] = 9.0   # a tie at the top
    bits = inp.to_bf16_bits(L)
    R = ql.qlora_moe_route(dev_bf16(bits), k)
    torch.cuda.synchronize()
    idx, *_ = _check_route(R, bits, k)
    assert list(idx[0]) == list(range(k))
    if k >= 2:
        assert list(idx[1][:2]) == [a, b]


def run_moe(c, y_dtype=torch.float32, dx_dtype=torch.float32):
    T, H, I, E, k, r = c.T, c.H, c.I, c.E, c.k, c.r
    X, dY, logits = dev_bf16(c.X), dev_bf16(c.dY), dev_bf16(c.logits)
    w_gu, w_d = dev_u8(c.w_gu), dev_u8(c.w_d)
    A_gu, B_gu, A_d, B_d = dev_bf16(c.A_gu), dev_bf16(c.B_gu), dev_bf16(c.A_d), dev_bf16(c.B_d)
    R = ql.qlora_moe_route(logits, k)
    saved = torch.empty(ql.qlora_moe_saved_bytes(T, k, H, I, r), dtype=torch.uint8, device="cuda")
    ws = torch.empty(ql.qlora_moe_workspace_bytes(T, k, E, H, I, r), dtype=torch.uint8, device="cuda")
    Y = torch.full((T, H), float("nan"), dtype=y_dtype, device="cuda")
    ql.qlora_moe_fwd(c.qtype, w_gu, w_d, E, H, I, X, R, A_gu, B_gu, A_d, B_d, r, c.scale, Y, saved, ws)
    dX = torch.full((T, H), float("nan"), dtype=dx_dtype, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    dA_gu = torch.full((E, r, H), float("nan"), **f32)
    dB_gu = torch.full((E, 2 * I, r), float("nan"), **f32)
    dA_d = torch.full((E, r, I), float("nan"), **f32)
    dB_d = torch.full((E, H, r), float("nan"), **f32)
    dL = torch.full((T, E), float("nan"), **f32)
    ql.qlora_moe_bwd(c.qtype, w_gu, w_d, E, H, I, X, dY, R, A_gu, B_gu, A_d, B_d, r, c.scale, saved, dX, dA_gu, dB_gu,
                     dA_d, dB_d, dL, ws)
    torch.cuda.synchronize()
    return R, dict(Y=Y, dX=dX, dA_gu=dA_gu, dB_gu=dB_gu, dA_d=dA_d, dB_d=dB_d, d_logits=dL)


def oracle_moe(c, experts=None, lazy=False):
    """The oracle on the case's inputs; `experts` restricts the work to those experts' pairs and
    `lazy` decodes one expert at a time (full-size cases)."""
    f = gb.bf16_bits_to_f64
    L = f(c.logits)
    idx, w, counts, offsets, perm, inv = om.route(L, c.k)
    Wgu, Wd = om.expert_weights(c.qtype, c.w_gu, c.w_d, c.H, c.I, experts=None if lazy else experts, lazy=lazy)
    X, dY = f(c.X), f(c.dY)
    A_gu, B_gu, A_d, B_d = f(c.A_gu), f(c.B_gu), f(c.A_d), f(c.B_d)
    Y, saved = om.moe_fwd(Wgu, Wd, X, idx, w, counts, offsets, perm, A_gu, B_gu, A_d, B_d, c.scale, experts=experts)
    gr = om.moe_bwd(Wgu, Wd, X, dY, idx, w, counts, offsets, perm, A_gu, B_gu, A_d, B_d, c.scale, saved,
                    experts=experts)
    gr["Y"] = Y
    gr["d_logits"] = om.scatter_d_logits(idx, gr["d_logits_sel"], c.E)
    return gr, (idx, w, counts, offsets, perm, inv)


def _check_full(got, ref, counts, experts, tokens):
    """Y, dX and d_logits on `tokens`; per-expert adapter gradients on `experts` (exact zeros for an
    expert without tokens)."""
    for name in ["Y", "dX", "d_logits"]:
        assert_close(f64(got[name])[tokens], ref[name][tokens], f"{name}[tokens]")
    for name in ["dA_gu", "dB_gu", "dA_d", "dB_d"]:
        g = f64(got[name])
        for e in experts:
            if counts[e] == 0:
                assert np.all(g[e] == 0), (name, e)
            else:
                assert_close(g[e], ref[name][e], f"{name}[{e}]")


SMALL = [
    # T, H, I, E, k, qtype, r, zipf
    (150, 256, 256, 8, 2, inp.Q4_0, 4, 0.0),      # ragged segments, several n tiles
    (40, 512, 256, 16, 2, inp.Q4_K, 8, 2.0),      # skewed: experts with no tokens
    (600, 256, 512, 4, 2, inp.Q8_0, 16, 0.0),     # segments spanning several 128-row blocks
    (33, 256, 256, 1, 1, inp.Q4_0, 4, 0.0),       # one expert, k = 1: a dense SwiGLU layer
    (64, 256, 256, 8, 8, inp.Q4_K, 40, 0.0),      # k = E (every expert every token), r > 32
    (300, 512, 256, 8, 4, inp.Q5_K, 8, 1.0),      # Q5_K experts, skewed
]


@pytest.mark.parametrize("case", SMALL)
def test_moe_parity_small(case):
    T, H, I, E, k, qt, r, zipf = case
    c = inp.moe_case(T, H, I, E, k, qt, r, 2.0 * r, seed=T + E, zipf_s=zipf)
    R, got = run_moe(c)
    ref, route = oracle_moe(c)
    _check_route(R, c.logits, k)
    for name in ["Y", "dX", "dA_gu", "dB_gu", "dA_d", "dB_d", "d_logits"]:
        g = f64(got[name])
        if name in ("dA_gu", "dB_gu", "dA_d", "dB_d"):
            counts = route[2]
            for e in range(E):   # per expert; experts without tokens are exactly zero
                if counts[e] == 0:
                    assert np.all(g[e] == 0), (name, e)
                else:
                    assert_close(g[e], ref[name][e], f"{name}[{e}]")
        else:
            assert_close(g, ref[name], name)


def test_moe_bf16_outputs():
    c = inp.moe_case(96, 256, 256, 8, 2, inp.Q4_0, 4, 8.0, seed=5)
    R, got = run_moe(c, torch.bfloat16, torch.bfloat16)
    ref, _ = oracle_moe(c)
    assert_close(f64(got["Y"]), ref["Y"], "Y", bf16_out=True)
    assert_close(f64(got["dX"]), ref["dX"], "dX", bf16_out=True)


def test_moe_deterministic():
    c = inp.moe_case(150, 256, 256, 8, 2, inp.Q4_K, 4, 8.0, seed=6)
    _, a = run_moe(c)
    a = {k_: v.clone() for k_, v in a.items()}
    _, b = run_moe(c)
    for name in a:
        assert torch.equal(a[name], b[name]), name


def test_moe_q4_0_2048tok_128x768_full():
    """The benchmark's MoE shape (2048 tokens, hidden 2048, 128 experts of 768, top-8, Q4_0, rank 4)
    in the launch configuration the benchmark uses, checked in full: every token's output,
    input-gradient and router-logit gradient, and every expert's four adapter gradients (the oracle
    decodes one expert at a time)."""
    c = inp.moe_q4_0_2048tok_128x768()
    R, got = run_moe(c)
    ref, route = oracle_moe(c, lazy=True)
    _check_route(R, c.logits, c.k)
    counts = route[2]
    assert (counts > 0).sum() == c.E
    _check_full(got, ref, counts, range(c.E), np.arange(c.T))


@pytest.mark.parametrize("T", [8, 64, 4096])
def test_moe_q4_k_256x4096x1536_zipf(T):
    """The skewed, weight-bound MoE shape (256 experts of 1536, hidden 4096, top-8, Q4_K, Zipf(1.1)
    popularity, rank 4) at 8, 64 and 4096 tokens, with exact routing for every token.
    At 8 and 64 tokens everything is checked: every token's output, input gradient and router-logit
    gradient and every expert's adapter gradients (zeros for the experts no token chose). At 4096
    tokens the oracle evaluates a sample of experts, the experts of tokens 0..3 plus the least and a
    middling popular expert among those chosen at all (each expert's gradients summed over every
    pair it received), and checks tokens 0..3 and those experts."""
    c = inp.moe_q4_k_256x4096x1536(T)
    R, got = run_moe(c)
    L = gb.bf16_bits_to_f64(c.logits)
    idx_all, _, counts, *_ = om.route(L, c.k)
    if T <= 64:
        experts, tokens = list(range(c.E)), np.arange(T)
        ref, route = oracle_moe(c, lazy=True)
    else:
        tokens = np.arange(4)
        used = np.flatnonzero(counts)
        by_pop = used[np.argsort(counts[used], kind="stable")]
        experts = sorted(set(int(e) for e in idx_all[tokens].ravel()) | {int(by_pop[0]), int(by_pop[len(by_pop) // 2])})
        ref, route = oracle_moe(c, experts=experts, lazy=True)
    _check_route(R, c.logits, c.k)
    _check_full(got, ref, counts, experts, tokens)
