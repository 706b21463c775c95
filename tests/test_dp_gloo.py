"""The multi-GPU path on CPU: two gloo ranks each take half the tokens of one batch, compute their
adapter gradients with the oracle, and sum them with the benchmark's all-reduce; the result is the
full-batch gradient (dA and dB are sums over tokens). The frozen base weights are replicated and
never exchanged."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from oracle import gguf_blocks as gb
        from oracle import lora_linear as ll
        from quantized_base_lora_tma_b200 import inputs as inp
        c = inp.linear_case(64, 256, 128, inp.Q4_0, 4, 8.0, seed=3)
        W = ll.weights(c.qtype, c.wq, c.N, c.K)
        f = gb.bf16_bits_to_f64
        X, dY, A, B = f(c.X), f(c.dY), f(c.A), f(c.B)
        rows = slice(rank * 32, (rank + 1) * 32)          # this rank's tokens
        _, dA, dB, _ = ll.linear_bwd(W, X[rows], dY[rows], A, B, c.scale)
        tA, tB = torch.from_numpy(dA.copy()), torch.from_numpy(dB.copy())
        bench.allreduce_adapter_grads([tA, tB])
        if rank == 0:
            _, dA_full, dB_full, _ = ll.linear_bwd(W, X, dY, A, B, c.scale)
            q.put((float(np.abs(tA.numpy() - dA_full).max()), float(np.abs(tB.numpy() - dB_full).max())))
    finally:
        dist.destroy_process_group()


def test_two_rank_adapter_gradient_allreduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    ea, eb = q.get(timeout=10)
    assert ea < 1e-12 and eb < 1e-12
