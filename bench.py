"""Benchmark of the frozen-GGUF-base + LoRA layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step is one forward + backward of the layer on one batch: for the default workload the
2048-token dense projection K = N = 4096 with a Q8_0 base and a rank-16 adapter (alpha 32):
H = X A^T, Y = X deq(W)^T + s H B^T, then G = s dY B, dX = dY deq(W) + G A, dA = G^T X,
dB = s dY^T H. Inputs are seeded synthetic tensors of that shape (X, dY ~ N(0,1); W ~ N(0, 0.02)
packed once; A ~ N(0, 1/K); B ~ N(0, 0.01)).

Timing: W untimed warm-up steps, then K steps each bracketed by CUDA events on the launch stream;
the L2 cache is flushed (a 256 MiB write) between steps, outside the events. With N > 1 each rank
runs its own batch (weak scaling) and the adapter gradients are summed across ranks with one NCCL
all-reduce per step (the data-parallel exchange); the step time is the max over ranks.

The JSON line also carries: the dominant kernel's roofline (its algorithmic FLOPs over its
event-timed duration against the measured bf16 peak), the end-to-end number through the public
API with host buffers, the CPU oracle timed on a sample of the same workload, the count of the
library's own kernel launches and the SM clocks sampled during the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_base_lora_tma_b200 import inputs as inp  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "quantized-LoRA fwd+bwd tokens/s and TFLOP/s (% bf16 peak); small-M weight GB/s"

WORKLOADS = {
    "dense_q8_0": ("dense_proj_q8_0_2048x4096x4096_r16", lambda seed: inp.dense_proj_2048x4096x4096(inp.Q8_0, seed)),
    "dense_q4_0": ("dense_proj_q4_0_2048x4096x4096_r16", lambda seed: inp.dense_proj_2048x4096x4096(inp.Q4_0, seed)),
    "gate_up_q4_k": ("gate_up_q4_k_2048x2048x12288_r8", lambda seed: inp.gate_up_q4_k_2048x2048x12288(seed)),
    "decode_q4_0_m1": ("decode_q4_0_1x8192x8192_r4", lambda seed: inp.decode_q4_0_8192(1, seed)),
    "decode_q4_0_m16": ("decode_q4_0_16x8192x8192_r4", lambda seed: inp.decode_q4_0_8192(16, seed)),
}


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "quantized_base_lora_tma_b200", "csrc")
    for fn in sorted(os.listdir(d)):
        with open(os.path.join(d, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload][kernel]
        if e.get("source_hash") == kernel_source_hash():
            return float(e["dram_bytes"])
    except Exception:
        pass
    return None


# ------------------------------------------------------------------------------------------------
# clocks
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML every `period` seconds while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period: float = 0.01):
        self.period = period
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------------
# our implementation
# ------------------------------------------------------------------------------------------------
def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


class DenseLayerRun:
    """Device buffers and one fwd+bwd step of the dense layer through the C ABI."""

    def __init__(self, case):
        import quantized_base_lora_tma_b200 as ql
        self.ql = ql
        self.c = c = case
        self.X = bf16_dev(c.X)
        self.dY = bf16_dev(c.dY)
        self.A = bf16_dev(c.A)
        self.B = bf16_dev(c.B)
        self.wq = torch.from_numpy(c.wq).cuda()
        M, N, K, r = c.M, c.N, c.K, c.r
        self.ws = torch.empty(ql.qlora_linear_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
        self.Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        self.H = torch.empty(M, r, dtype=torch.float32, device="cuda")
        self.dX = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
        self.dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
        self.dB = torch.empty(N, r, dtype=torch.float32, device="cuda")

    def fwd(self, X=None):
        c, ql = self.c, self.ql
        X = self.X if X is None else X
        ql.qlora_linear_fwd(c.qtype, self.wq, c.N, c.K, X, self.A, self.B, c.r, c.scale, self.Y, self.H, self.ws)

    def bwd(self, X=None, dY=None):
        c, ql = self.c, self.ql
        X = self.X if X is None else X
        dY = self.dY if dY is None else dY
        ql.qlora_linear_bwd(c.qtype, self.wq, c.N, c.K, X, dY, self.A, self.B, c.r, c.scale, self.H, self.dX,
                            self.dA, self.dB, self.ws)

    def step(self, X=None, dY=None):
        self.fwd(X)
        self.bwd(X, dY)

    def flops(self):
        c = self.c
        base = 2 * 2.0 * c.M * c.N * c.K           # forward and input-gradient GEMMs (W is frozen)
        lora = 6.0 * c.r * (c.K + c.N) * c.M
        return base + lora

    def gemm_flops(self, slot):
        c = self.c
        return 2.0 * c.M * c.N * c.K + 2.0 * c.M * c.r * (c.N if slot == 0 else c.K)


class MoERun:
    """Device buffers and one step (route + forward + backward) of the routed MoE layer."""

    _dev_weights = {}  # packed expert stacks already on the device, by host array identity

    def __init__(self, case):
        import quantized_base_lora_tma_b200 as ql
        self.ql = ql
        self.c = c = case
        T, H, I, E, k, r = c.T, c.H, c.I, c.E, c.k, c.r
        self.X, self.dY, self.logits = bf16_dev(c.X), bf16_dev(c.dY), bf16_dev(c.logits)
        key = (id(c.w_gu), id(c.w_d))
        if key not in MoERun._dev_weights:
            MoERun._dev_weights.clear()
            MoERun._dev_weights[key] = (torch.from_numpy(c.w_gu).cuda(), torch.from_numpy(c.w_d).cuda())
        self.w_gu, self.w_d = MoERun._dev_weights[key]
        self.A_gu, self.B_gu = bf16_dev(c.A_gu), bf16_dev(c.B_gu)
        self.A_d, self.B_d = bf16_dev(c.A_d), bf16_dev(c.B_d)
        self.route = ql.MoeRoute(T, E, k)
        self.saved = torch.empty(ql.qlora_moe_saved_bytes(T, k, H, I, r), dtype=torch.uint8, device="cuda")
        self.ws = torch.empty(ql.qlora_moe_workspace_bytes(T, k, E, H, I, r), dtype=torch.uint8, device="cuda")
        f32 = dict(dtype=torch.float32, device="cuda")
        self.Y = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        self.dX = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        self.dA_gu = torch.empty(E, r, H, **f32)
        self.dB_gu = torch.empty(E, 2 * I, r, **f32)
        self.dA_d = torch.empty(E, r, I, **f32)
        self.dB_d = torch.empty(E, H, r, **f32)
        self.dL = torch.empty(T, E, **f32)

    def fwd(self):
        """Routing and the forward: one pass over the touched experts' weights."""
        c, ql = self.c, self.ql
        ql.qlora_moe_route(self.logits, c.k, self.route)
        ql.qlora_moe_fwd(c.qtype, self.w_gu, self.w_d, c.E, c.H, c.I, self.X, self.route, self.A_gu, self.B_gu,
                         self.A_d, self.B_d, c.r, c.scale, self.Y, self.saved, self.ws)

    def bwd(self):
        """The backward (second pass over the touched experts' weights)."""
        c, ql = self.c, self.ql
        ql.qlora_moe_bwd(c.qtype, self.w_gu, self.w_d, c.E, c.H, c.I, self.X, self.dY, self.route, self.A_gu,
                         self.B_gu, self.A_d, self.B_d, c.r, c.scale, self.saved, self.dX, self.dA_gu, self.dB_gu,
                         self.dA_d, self.dB_d, self.dL, self.ws)

    def step(self):
        self.fwd()
        self.bwd()

    def flops(self):
        c = self.c
        P = c.T * c.k
        return 12.0 * P * c.H * c.I + 6.0 * c.r * (2 * c.H + 3 * c.I) * P

    def touched_weight_bytes(self):
        """Packed weight bytes of the experts that received at least one pair (one pass)."""
        c = self.c
        used = int((self.route.counts > 0).sum().item())
        return used, used * (c.w_gu[0].nbytes + c.w_d[0].nbytes)


def allreduce_adapter_grads(grads):
    """The data-parallel exchange of the layer: every rank holds the adapter gradients of its own
    tokens; dA and dB are sums over tokens, so their sum over ranks is the full-batch gradient."""
    for g in grads:
        torch.distributed.all_reduce(g, op=torch.distributed.ReduceOp.SUM)


LM_CHUNK = 1024  # token rows per cross-entropy chunk of the lm_head workload
EV_EVERY = 8  # kernel events on one timed step in this many (as for the headline)


def time_steps(fn, steps, warmup, flush, slots=()):
    """Mean device time (ms) of fn() over `steps` calls, L2 flushed before each, and per-slot GEMM
    means. The GEMM events are recorded on one step in EV_EVERY only: an event between two kernels
    stops the next one from starting while the previous one drains (programmatic launch), so those
    steps are slower; they stay in the step mean, as in the headline."""
    import quantized_base_lora_tma_b200 as ql
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    nev = (steps + EV_EVERY - 1) // EV_EVERY
    gev = {s: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nev)]
           for s in slots}
    for i in range(steps):
        flush.zero_()
        for s in slots:
            if i % EV_EVERY == 0:
                ql.qlora_set_kernel_events(s, gev[s][i // EV_EVERY][0], gev[s][i // EV_EVERY][1])
            else:
                ql.qlora_set_kernel_events(s, None, None)
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    for s in slots:
        ql.qlora_set_kernel_events(s, None, None)
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    return ms, {s: statistics.mean(a.elapsed_time(b) for a, b in gev[s]) for s in slots}


def device_status_ok(where):
    import quantized_base_lora_tma_b200 as ql
    st, site = ql.qlora_device_status(reset=True)
    if st != 0:
        raise RuntimeError(f"device status {st} (wait site {site}) after {where}")


def also_measurements(flush, steps, pk):
    """Single-GPU measurements of the other shapes of the benchmark set (not the headline)."""
    import quantized_base_lora_tma_b200 as ql
    out = {}
    # routed MoE layer, fwd + bwd incl. routing
    c = inp.moe_q4_0_2048tok_128x768()
    m = MoERun(c)
    ms, g = time_steps(m.step, max(5, steps // 4), 3, flush, slots=(2, 3, 4, 5))
    tf = m.flops() / (ms / 1e3) / 1e12
    out["moe_q4_0_T2048_H2048_E128_I768_k8_r4"] = {
        "tokens_per_s": c.T / (ms / 1e3), "ms_per_step": ms, "tflops": tf, "frac_of_bf16_peak": tf / pk["bf16_tflops"],
        "gemm_ms": {"gate_up": g[2], "down": g[3], "down_dx": g[4], "gate_up_dx": g[5]},
        "experts_touched": int((m.route.counts > 0).sum().item())}
    device_status_ok("moe")
    del m
    torch.cuda.empty_cache()
    # 8-bit AdamW on the headline layer's adapters (A [16 x 4096] and B [4096 x 16])
    torch.manual_seed(0)
    n = 2 * 16 * 4096
    st = ql.Adamw8State(n)
    pp = torch.zeros(n, dtype=torch.float32, device="cuda")
    gg = torch.randn(n, dtype=torch.float32, device="cuda") * 0.01
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    t_ = [0]

    def adam_step():
        t_[0] += 1
        ql.qlora_adamw8_step(pp, gg, st, t_[0], 1e-4, 0.9, 0.999, 1e-8, 0.01, p_bf16=pb)
    ms_a, _ = time_steps(adam_step, steps, 3, flush)
    abytes = n * (4 + 4 + 4 + 1 + 1 + 1 + 1 + 2) + 4 * 4 * ((n + 255) // 256)  # p r/w, g, codes r/w, bf16 copy
    out["adamw8_adapters_r16_4096x4096"] = {"params": n, "ms": ms_a, "gbs": abytes / (ms_a / 1e3) / 1e9}
    device_status_ok("adamw8")
    del st, pp, gg, pb
    # RMSNorm before the headline projection: 2048 tokens x 4096, forward (x -> bf16 x_n, rstd) and
    # backward (fp32 d -> fp32 dx)
    M_, K_ = 2048, 4096
    xr = torch.randn(M_, K_, device="cuda").to(torch.bfloat16)
    gr = torch.ones(K_, device="cuda").to(torch.bfloat16)
    xn_ = torch.empty(M_, K_, dtype=torch.bfloat16, device="cuda")
    rs_ = torch.empty(M_, dtype=torch.float32, device="cuda")
    dxn_ = torch.randn(M_, K_, device="cuda")
    dx_ = torch.empty(M_, K_, dtype=torch.float32, device="cuda")
    ms_nf, _ = time_steps(lambda: ql.qlora_rmsnorm_fwd(xr, gr, 1e-6, xn_, rs_), steps, 3, flush)
    ms_nb, _ = time_steps(lambda: ql.qlora_rmsnorm_bwd(xr, gr, rs_, dxn_, dx_), steps, 3, flush)
    out["rmsnorm_2048x4096"] = {"fwd_ms": ms_nf, "bwd_ms": ms_nb,
                                "fwd_gbs": (M_ * K_ * 4) / (ms_nf / 1e3) / 1e9,
                                "bwd_gbs": (M_ * K_ * (2 + 4 + 4)) / (ms_nb / 1e3) / 1e9}
    device_status_ok("rmsnorm")
    del xr, gr, xn_, rs_, dxn_, dx_
    # quantized lm_head with chunked cross-entropy: 2048 tokens, hidden 2048, 128K vocabulary, Q8_0, in
    # chunks of 1024 tokens (512-row pair tiles for the logits GEMM; 0.8 GB of workspace)
    lm = inp.lm_head_q8_0_128k()
    lr_ = LmHeadRun(lm, LM_CHUNK)
    ms_l, _ = time_steps(lr_.step, max(5, steps // 4), 3, flush)
    lflops = 4.0 * lm["M"] * lm["V"] * lm["K"]
    out[f"lm_head_ce_q8_0_2048x2048x131072_chunk{LM_CHUNK}"] = {
        "ms": ms_l, "tokens_per_s": lm["M"] / (ms_l / 1e3), "tflops": lflops / (ms_l / 1e3) / 1e12,
        "frac_of_bf16_peak": lflops / (ms_l / 1e3) / 1e12 / pk["bf16_tflops"]}
    device_status_ok("lm_head")
    del lm, lr_
    torch.cuda.empty_cache()
    # routing alone at 4096 tokens, 256 experts, top-8 (the skewed workload's logits)
    c = inp.moe_q4_k_256x4096x1536(4096)
    lg = bf16_dev(c.logits)
    R = ql.MoeRoute(c.T, c.E, c.k)
    ms_r, _ = time_steps(lambda: ql.qlora_moe_route(lg, c.k, R), steps, 3, flush)
    out["moe_route_T4096_E256_k8"] = {"ms": ms_r, "logit_gbs": c.logits.nbytes / (ms_r / 1e3) / 1e9}
    device_status_ok("route")
    del R, lg
    # skewed 256-expert Q4_K MoE: weight-bound at 8 and 64 tokens, tensor-bound at 4096
    for T in (8, 64, 4096):
        c = inp.moe_q4_k_256x4096x1536(T)
        m = MoERun(c)
        n = max(5, steps // 4) if T == 4096 else steps
        ms, g = time_steps(m.step, n, 3, flush, slots=(2, 3, 4, 5))
        ms_f, _ = time_steps(m.fwd, n, 3, flush)
        ms_b, _ = time_steps(m.bwd, n, 3, flush)
        used, wb = m.touched_weight_bytes()
        counts = m.route.counts.cpu().numpy()
        tf = m.flops() / (ms / 1e3) / 1e12
        out[f"moe_q4_k_T{T}_H4096_E256_I1536_k8_r4_zipf"] = {
            "tokens_per_s": T / (ms / 1e3), "ms_per_step": ms, "fwd_ms": ms_f, "bwd_ms": ms_b,
            "tflops": tf, "frac_of_bf16_peak": tf / pk["bf16_tflops"],
            "experts_touched": used, "weight_bytes_per_pass": wb,
            "fwd_weight_gbs": wb / (ms_f / 1e3) / 1e9, "bwd_weight_gbs": wb / (ms_b / 1e3) / 1e9,
            "fwd_frac_of_hbm": wb / (ms_f / 1e3) / 1e9 / pk["hbm_gbs"],
            "bwd_frac_of_hbm": wb / (ms_b / 1e3) / 1e9 / pk["hbm_gbs"],
            "gemm_ms": {"gate_up": g[2], "down": g[3], "down_dx": g[4], "gate_up_dx": g[5]},
            "top_expert_counts": sorted((int(x) for x in counts), reverse=True)[:8]}
        device_status_ok(f"moe256 T={T}")
        del m
        torch.cuda.empty_cache()
    MoERun._dev_weights.clear()
    torch.cuda.empty_cache()
    # decode-shaped linear: weight streaming
    for M in (1, 4, 16):
        c = inp.decode_q4_0_8192(M)
        d = DenseLayerRun(c)
        wbytes = c.wq.nbytes
        # no kernel events inside the call: they would serialize its three launches
        ms_f, _ = time_steps(lambda: d.ql.qlora_linear_fwd(c.qtype, d.wq, c.N, c.K, d.X, d.A, d.B, c.r, c.scale, d.Y,
                                                          d.H, d.ws), steps, 3, flush, slots=())
        ms_b, gb = time_steps(lambda: d.ql.qlora_linear_bwd(c.qtype, d.wq, c.N, c.K, d.X, d.dY, d.A, d.B, c.r, c.scale,
                                                           d.H, d.dX, d.dA, d.dB, d.ws), steps, 3, flush, slots=(1,))
        act_f = c.M * (c.K + c.N) * 2
        out[f"decode_q4_0_M{M}_8192x8192"] = {
            "fwd_ms": ms_f, "bwd_ms": ms_b, "dx_gemm_ms": gb[1],
            "fwd_weight_gbs": (wbytes + act_f) / (ms_f / 1e3) / 1e9,
            "dx_gemm_weight_gbs": (wbytes + act_f) / (gb[1] / 1e3) / 1e9,
            "fwd_frac_of_hbm": (wbytes + act_f) / (ms_f / 1e3) / 1e9 / pk["hbm_gbs"]}
        device_status_ok(f"decode M={M}")
        del d
    torch.cuda.empty_cache()
    # the other dense shapes
    for key in ("dense_q4_0", "gate_up_q4_k"):
        name, make = WORKLOADS[key]
        d = DenseLayerRun(make(0))
        ms, g = time_steps(d.step, steps, 3, flush, slots=(0, 1))
        tf = d.flops() / (ms / 1e3) / 1e12
        out[name] = {"tokens_per_s": d.c.M / (ms / 1e3), "ms_per_step": ms, "tflops": tf,
                     "frac_of_bf16_peak": tf / pk["bf16_tflops"], "gemm_ms": {"fwd": g[0], "dx": g[1]}}
        device_status_ok(name)
        del d
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import quantized_base_lora_tma_b200 as ql
    from quantized_base_lora_tma_b200 import build
    build.build()
    torch.cuda.set_device(local_rank)
    wl_name, make = WORKLOADS[args.workload]
    # weights identical on every rank (replicated frozen base); tokens differ per rank
    case = make(0)
    if rank != 0:
        rng = np.random.default_rng(1000 + rank)
        case.X = inp.to_bf16_bits(rng.standard_normal(case.X.shape, dtype=np.float32))
        case.dY = inp.to_bf16_bits(rng.standard_normal(case.dY.shape, dtype=np.float32))
    run = DenseLayerRun(case)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    ql.qlora_device_status(reset=True)

    def allreduce_grads():
        if world > 1:
            allreduce_adapter_grads([run.dA, run.dB])

    for _ in range(args.warmup):
        run.step()
        allreduce_grads()
    torch.cuda.synchronize()

    # --- device-timed steps with per-kernel events for the two tensor-core GEMMs ---
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    gev = {s: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
           for s in (0, 1)}
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = ql.qlora_launch_count()
    sampler = ClockSampler(local_rank)
    wall0 = time.perf_counter()
    # The GEMM events are recorded on every eighth step only: an event between two kernels of the
    # step stops the next kernel from starting while the previous one drains (programmatic launch),
    # so those steps are slower; they stay in the step mean, which is therefore slightly pessimistic.
    EV_EVERY = 8
    ev_steps = list(range(0, K, EV_EVERY))
    with sampler:
        for i in range(K):
            flush.zero_()
            for s in (0, 1):
                if i % EV_EVERY == 0:
                    ql.qlora_set_kernel_events(s, gev[s][i // EV_EVERY][0], gev[s][i // EV_EVERY][1])
                else:
                    ql.qlora_set_kernel_events(s, None, None)
            ev[i][0].record(stream)
            run.step()
            allreduce_grads()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    launches = ql.qlora_launch_count() - launches0
    for s in (0, 1):
        ql.qlora_set_kernel_events(s, None, None)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    st, site = ql.qlora_device_status(reset=True)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site}")
    step_ms = [a.elapsed_time(b) for a, b in ev]
    gemm_ms = {s: [gev[s][j][0].elapsed_time(gev[s][j][1]) for j in range(len(ev_steps))] for s in (0, 1)}
    ms = statistics.mean(step_ms)
    if world > 1:
        t = torch.tensor([ms], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())

    # --- end to end through the public API with host buffers ---
    E = max(3, min(K, 50))
    X_h = torch.from_numpy(np.ascontiguousarray(case.X).view(np.int16)).view(torch.bfloat16).pin_memory()
    dY_h = torch.from_numpy(np.ascontiguousarray(case.dY).view(np.int16)).view(torch.bfloat16).pin_memory()
    dA_h = torch.empty(run.dA.shape, dtype=torch.float32).pin_memory()
    dB_h = torch.empty(run.dB.shape, dtype=torch.float32).pin_memory()
    Xd = torch.empty_like(run.X)
    dYd = torch.empty_like(run.dY)
    e2e_ms = []
    # X first on the compute stream; dY on a copy stream once X is in, so that its transfer
    # overlaps the forward; the backward waits for it
    copy_stream = torch.cuda.Stream()
    for i in range(E + 2):
        flush.zero_()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev_x, ev_dy = torch.cuda.Event(), torch.cuda.Event()
        a.record(stream)
        Xd.copy_(X_h, non_blocking=True)
        ev_x.record(stream)
        copy_stream.wait_event(ev_x)
        with torch.cuda.stream(copy_stream):
            dYd.copy_(dY_h, non_blocking=True)
        ev_dy.record(copy_stream)
        run.fwd(Xd)
        stream.wait_event(ev_dy)
        run.bwd(Xd, dYd)
        allreduce_grads()
        dA_h.copy_(run.dA, non_blocking=True)
        dB_h.copy_(run.dB, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= 2:
            e2e_ms.append(a.elapsed_time(b))
    e2e = statistics.mean(e2e_ms)
    if world > 1:
        t = torch.tensor([e2e], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e = float(t.item())

    c = case
    tokens = c.M * world
    value = tokens / (ms / 1e3)
    pk, pk_kind = peaks()
    # dominant kernel: the tensor-core GEMM with the larger share of the step
    g_mean = {s: statistics.mean(gemm_ms[s]) for s in (0, 1)}
    dom = max(g_mean, key=g_mean.get)
    dom_name = {0: "qgemm_fwd (dequant-in-SMEM tcgen05 cta_group::2 GEMM, 512x256 pair tiles, K-major B)",
                1: "qgemm_dx (dequant-in-SMEM tcgen05 cta_group::2 GEMM, 512x256 pair tiles, MN-major B)"}[dom]
    achieved = run.gemm_flops(dom) / (g_mean[dom] / 1e3) / 1e12
    step_tflops = run.flops() / (ms / 1e3) / 1e12
    traffic = profiled_traffic(args.workload, "qgemm_fwd" if dom == 0 else "qgemm_dx")
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights packed once to GGUF)",
        "config": {"workload": wl_name, "tokens_per_gpu": c.M, "K": c.K, "N": c.N, "qtype": inp.QTYPE_NAMES[c.qtype],
                   "rank": c.r, "alpha": c.alpha, "global_batch_tokens": tokens,
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": "flushed between steps (256 MiB write outside the timed events)"},
        "tflops": step_tflops,
        "frac_of_bf16_peak": step_tflops / pk["bf16_tflops"],
        "roofline": {"kernel": dom_name, "bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"], "traffic": traffic,
                     "peak_kind": f"{pk_kind} burst bf16 (cuBLAS)",
                     "kernel_ms": {"qgemm_fwd": g_mean[0], "qgemm_dx": g_mean[1]}},
        "e2e": {"value": tokens / (e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(run.X.numel() * 2 + run.dY.numel() * 2),
                "d2h_bytes_per_step": int((run.dA.numel() + run.dB.numel()) * 4),
                "ms_per_step": e2e},
        "gpu_launches": int(launches),
        "clocks": sampler.summary(),
        "wall_s_timed_region": wall,
    }
    if rank == 0 and world == 1 and not args.no_also:
        out["also"] = also_measurements(flush, max(20, K // 4), pk)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(case, target_s=args.cpu_seconds)
    return out


# ------------------------------------------------------------------------------------------------
# CPU oracle (baseline leg and the reference arm)
# ------------------------------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def _cpu_model():
    """The host CPU's model name (first processor entry of /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_step(case, rows):
    """The oracle's forward + backward restricted to a sample of token rows (dA, dB over those rows)."""
    from oracle import gguf_blocks as gb
    from oracle import lora_linear as ll
    W = ll.weights(case.qtype, case.wq, case.N, case.K)
    X = gb.bf16_bits_to_f64(case.X[rows])
    dY = gb.bf16_bits_to_f64(case.dY[rows])
    A = gb.bf16_bits_to_f64(case.A)
    B = gb.bf16_bits_to_f64(case.B)
    Y, H = ll.linear_fwd(W, X, A, B, case.scale)
    return ll.linear_bwd(W, X, dY, A, B, case.scale, H)


def cpu_baseline(case, target_s=15.0, max_rows=None):
    rows_total = case.M
    n = 64
    t0 = time.perf_counter()
    oracle_step(case, np.arange(n))
    t1 = time.perf_counter() - t0
    n = int(min(rows_total if max_rows is None else max_rows, max(64, n * target_s / max(t1, 1e-3))))
    t0 = time.perf_counter()
    oracle_step(case, np.arange(n))
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": _blas_threads(), "cpu_model": _cpu_model(),
            "kind": "oracle", "sample": f"fp64 numpy oracle fwd+bwd on the first {n} of {rows_total} token rows "
                      f"(weights decoded once per call), {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    wl_name, make = WORKLOADS[args.workload]
    case = make(0)
    cores = _blas_threads()
    n = max(32, int(args.ref_rows))
    for _ in range(args.warmup):
        oracle_step(case, np.arange(n))
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(case, np.arange(n))
        times.append(time.perf_counter() - t0)
    ms = statistics.mean(times) * 1e3
    value = n / (ms / 1e3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl_name, "tokens_per_step_sample": n},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "cpu_model": _cpu_model(),
                         "kind": "oracle", "sample": f"fp64 numpy oracle fwd+bwd on {n} token rows per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


class LmHeadRun:
    """Device buffers and one call of the quantized lm_head with chunked cross-entropy."""

    def __init__(self, lm, chunk=None):
        chunk = LM_CHUNK if chunk is None else chunk
        import quantized_base_lora_tma_b200 as ql
        self.ql, self.lm, self.chunk = ql, lm, chunk
        self.w = torch.from_numpy(lm["wq"]).cuda()
        self.x = bf16_dev(lm["X"])
        self.lab = torch.from_numpy(lm["labels"]).cuda()
        self.ws = torch.empty(ql.qlora_lm_head_ce_workspace_bytes(lm["M"], lm["V"], lm["K"], chunk),
                              dtype=torch.uint8, device="cuda")
        self.loss = torch.empty(lm["M"], dtype=torch.float32, device="cuda")
        self.dx = torch.empty(lm["M"], lm["K"], dtype=torch.bfloat16, device="cuda")

    def step(self):
        lm = self.lm
        self.ql.qlora_lm_head_ce(lm["qtype"], self.w, lm["V"], lm["K"], self.x, self.lab, self.chunk, 1.0 / lm["M"],
                                 self.loss, self.dx, self.ws)

    fwd = step


PROFILE_CASES = {
    "moe_q4_k_e32_t4096": lambda: MoERun(inp.moe_q4_k_256x4096x1536(4096, E=32)),
    "lm_head": lambda: LmHeadRun(inp.lm_head_q8_0_128k()),
    "dense_q8_0": lambda: DenseLayerRun(inp.dense_proj_2048x4096x4096(inp.Q8_0)),
    "dense_q4_0": lambda: DenseLayerRun(inp.dense_proj_2048x4096x4096(inp.Q4_0)),
    "gate_up_q4_k": lambda: DenseLayerRun(inp.gate_up_q4_k_2048x2048x12288()),
    "moe_q4_0": lambda: MoERun(inp.moe_q4_0_2048tok_128x768()),
    "moe256_t8": lambda: MoERun(inp.moe_q4_k_256x4096x1536(8)),
    "moe256_t64": lambda: MoERun(inp.moe_q4_k_256x4096x1536(64)),
    "moe256_t4096": lambda: MoERun(inp.moe_q4_k_256x4096x1536(4096)),
    "decode_m1": lambda: DenseLayerRun(inp.decode_q4_0_8192(1)),
    "decode_m4": lambda: DenseLayerRun(inp.decode_q4_0_8192(4)),
    "decode_m16": lambda: DenseLayerRun(inp.decode_q4_0_8192(16)),
}


def profile_calls(name, calls=3, fwd_only=False):
    """`calls` steps (or forwards) of a named workload and nothing else: the launches a profiler
    captures. No timing, no JSON line."""
    from quantized_base_lora_tma_b200 import build
    build.build()
    run = PROFILE_CASES[name]()
    for _ in range(calls):
        run.fwd() if fwd_only else run.step()
    torch.cuda.synchronize()
    device_status_ok(name)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="dense_q8_0", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-also", action="store_true", help="skip the other shapes of the benchmark set")
    ap.add_argument("--calls", default=None, choices=sorted(PROFILE_CASES),
                    help="profiling driver: run three steps of the named workload and exit (no timing, no JSON line)")
    ap.add_argument("--fwd-only", action="store_true", help="with --calls: forwards only")
    ap.add_argument("--ncalls", type=int, default=3, help="with --calls: how many")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.calls:
        profile_calls(args.calls, args.ncalls, args.fwd_only)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
