"""Helpers for the GPU parity tests: upload seeded inputs, compare against the oracle."""
import numpy as np
import torch

from oracle import gguf_blocks as gb

TOL = 1e-2  # max|err| <= TOL * RMS(ref), per tensor (fp32 outputs)


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def rms(a):
    return float(np.sqrt(np.mean(np.square(a)))) if a.size else 0.0


def assert_close(got, ref, name, tol=TOL, bf16_out=False):
    """max|got - ref| <= tol * RMS(ref) (+ half a bf16 ulp of ref for bf16-rounded outputs)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), name
    err = np.abs(got - ref)
    bound = tol * rms(ref)
    if bf16_out:
        e = np.floor(np.log2(np.maximum(np.abs(ref), 1e-38)))
        bound = bound + 2.0 ** (e - 8)
    worst = float(np.max(err - bound)) if err.size else 0.0
    assert worst <= 0, f"{name}: max err {err.max():.3e} vs bound {np.max(bound):.3e} (rms {rms(ref):.3e})"
    return float(err.max() / max(rms(ref), 1e-300)) if err.size else 0.0


def bf16_f64(bits):
    return gb.bf16_bits_to_f64(bits)
