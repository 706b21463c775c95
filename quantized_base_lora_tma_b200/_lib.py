"""ctypes binding of libqlora.so: the C ABI in include/qlora.h, same names, argument marshalling only.

Tensors are torch tensors on the GPU (torch supplies device memory and streams); every number the
layer computes comes from the library's kernels. If the library is not built, loading fails loudly:
there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqlora.so")

Q4_0, Q8_0, Q2_K, Q4_K, Q5_K, Q6_K = 2, 8, 10, 12, 13, 14
QL_F32, QL_BF16 = 0, 1
QL_OK = 0
STATUS = {0: "QL_OK", 1: "QL_ERR_INVALID_ARG", 2: "QL_ERR_UNSUPPORTED", 3: "QL_ERR_SHAPE",
          4: "QL_ERR_ALIGNMENT", 5: "QL_ERR_WORKSPACE", 6: "QL_ERR_CUDA", 7: "QL_ERR_TIMEOUT"}

_c_i64 = ctypes.c_int64
_c_vp = ctypes.c_void_p
_c_int = ctypes.c_int
_c_f = ctypes.c_float
_c_sz = ctypes.c_size_t

# name -> (restype, argtypes); must match include/qlora.h
SIGNATURES = {
    "qlora_status_string": (ctypes.c_char_p, [_c_int]),
    "qlora_launch_count": (ctypes.c_uint64, []),
    "qlora_device_status": (_c_int, [ctypes.POINTER(_c_int), _c_int]),
    "qlora_set_kernel_events": (_c_int, [_c_int, _c_vp, _c_vp]),
    "qlora_set_rows_fusion": (_c_int, [_c_int]),
    "qlora_selftest_wait_timeout": (_c_int, [_c_i64, _c_vp]),
    "gguf_dequant": (_c_int, [_c_int, _c_vp, _c_i64, _c_i64, _c_vp, _c_int, _c_vp]),
    "qlora_linear_workspace_bytes": (_c_sz, [_c_i64, _c_i64, _c_i64, _c_int]),
    "qlora_linear_fwd": (_c_int, [_c_int, _c_vp, _c_i64, _c_i64, _c_vp, _c_i64, _c_vp, _c_vp, _c_int, _c_f,
                                  _c_vp, _c_int, _c_vp, _c_vp, _c_sz, _c_vp]),
    "qlora_moe_route_workspace_bytes": (_c_sz, [_c_i64, _c_int, _c_int]),
    "qlora_moe_route": (_c_int, [_c_vp, _c_i64, _c_int, _c_int, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp,
                                 _c_vp, _c_sz, _c_vp]),
    "qlora_moe_saved_bytes": (_c_sz, [_c_i64, _c_int, _c_i64, _c_i64, _c_int]),
    "qlora_moe_workspace_bytes": (_c_sz, [_c_i64, _c_int, _c_int, _c_i64, _c_i64, _c_int]),
    "qlora_moe_fwd": (_c_int, [_c_int, _c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_vp, _c_i64, _c_int, _c_vp, _c_vp,
                               _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_f, _c_vp, _c_int,
                               _c_vp, _c_sz, _c_vp, _c_sz, _c_vp]),
    "qlora_moe_bwd": (_c_int, [_c_int, _c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_vp, _c_vp, _c_i64, _c_int, _c_vp,
                               _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_f, _c_vp,
                               _c_sz, _c_vp, _c_int, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_sz, _c_vp]),
    "qlora_lm_head_ce_workspace_bytes": (_c_sz, [_c_i64, _c_i64, _c_i64, _c_i64]),
    "qlora_lm_head_ce": (_c_int, [_c_int, _c_vp, _c_i64, _c_i64, _c_vp, _c_i64, _c_vp, _c_i64, _c_f, _c_vp, _c_vp,
                                  _c_int, _c_vp, _c_sz, _c_vp]),
    "qlora_rmsnorm_fwd": (_c_int, [_c_vp, _c_vp, _c_i64, _c_i64, _c_f, _c_vp, _c_vp, _c_vp]),
    "qlora_rmsnorm_bwd": (_c_int, [_c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_vp, _c_int, _c_vp]),
    "qlora_adamw8_step": (_c_int, [_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_f, _c_f, _c_f, _c_f, _c_f,
                                   _c_i64, _c_vp, _c_vp]),
    "qlora_linear_fwd_noalloc": (_c_int, [_c_int, _c_vp, _c_i64, _c_i64, _c_vp, _c_i64, _c_vp, _c_vp, _c_int,
                                          _c_f, _c_vp, _c_int, _c_vp, _c_vp]),
    "qlora_linear_bwd": (_c_int, [_c_int, _c_vp, _c_i64, _c_i64, _c_vp, _c_vp, _c_i64, _c_vp, _c_vp, _c_int,
                                  _c_f, _c_vp, _c_vp, _c_int, _c_vp, _c_vp, _c_vp, _c_sz, _c_vp]),
}

_lib = None


class QloraError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m quantized_base_lora_tma_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return _c_vp(t.data_ptr())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _s(stream):
    if stream is None:
        if _raw_stream is not None:  # the current stream's handle without building a Stream object
            return _c_vp(_raw_stream(torch.cuda.current_device()))
        stream = torch.cuda.current_stream()
    return _c_vp(stream.cuda_stream)


def _dt(t):
    if t.dtype == torch.float32:
        return QL_F32
    if t.dtype == torch.bfloat16:
        return QL_BF16
    raise ValueError(f"unsupported output dtype {t.dtype}")


def _check(rc, where):
    if rc != QL_OK:
        raise QloraError(rc, where)


def qlora_status_string(code: int) -> str:
    return lib().qlora_status_string(code).decode()


def qlora_launch_count() -> int:
    return int(lib().qlora_launch_count())


def qlora_device_status(reset: bool = False):
    site = _c_int(0)
    rc = lib().qlora_device_status(ctypes.byref(site), 1 if reset else 0)
    return rc, site.value


def qlora_set_rows_fusion(mask) -> int:
    """Which dense pair GEMMs compute the adapter row products in their own launch: bit 0 the
    forward, bit 1 the input gradient (True = both, False = neither); returns the previous mask."""
    m = 3 if mask is True else (0 if mask is False else int(mask))
    return int(lib().qlora_set_rows_fusion(m))


def qlora_set_kernel_events(slot: int, start=None, stop=None):
    """start / stop: torch.cuda.Event (created with enable_timing=True) or None to clear."""
    def h(e):
        if e is None:
            return None
        if e.cuda_event == 0:          # torch creates the event lazily
            e.record()
        return _c_vp(e.cuda_event)
    _check(lib().qlora_set_kernel_events(slot, h(start), h(stop)), "qlora_set_kernel_events")


def qlora_selftest_wait_timeout(limit_us: int, stream=None):
    _check(lib().qlora_selftest_wait_timeout(limit_us, _s(stream)), "qlora_selftest_wait_timeout")


def gguf_dequant(qtype, wq, rows, cols, out, stream=None):
    _check(lib().gguf_dequant(qtype, _p(wq), rows, cols, _p(out), _dt(out), _s(stream)), "gguf_dequant")


def qlora_linear_workspace_bytes(M, N, K, r) -> int:
    return int(lib().qlora_linear_workspace_bytes(M, N, K, r))


def qlora_linear_fwd(qtype, wq, N, K, X, A, B, r, scale, Y, H, ws, stream=None):
    M = X.shape[0]
    _check(lib().qlora_linear_fwd(qtype, _p(wq), N, K, _p(X), M, _p(A), _p(B), r, scale, _p(Y), _dt(Y), _p(H),
                                  _p(ws), ws.numel() * ws.element_size(), _s(stream)), "qlora_linear_fwd")


def qlora_linear_fwd_noalloc(qtype, wq, N, K, X, A, B, r, scale, Y, H, stream=None):
    """qlora_linear_fwd without a workspace: the library's own static device scratch is used."""
    M = X.shape[0]
    _check(lib().qlora_linear_fwd_noalloc(qtype, _p(wq), N, K, _p(X), M, _p(A), _p(B), r, scale, _p(Y), _dt(Y),
                                          _p(H), _s(stream)), "qlora_linear_fwd_noalloc")


def qlora_linear_bwd(qtype, wq, N, K, X, dY, A, B, r, scale, H, dX, dA, dB, ws, stream=None):
    M = X.shape[0]
    dxt = _dt(dX) if dX is not None else QL_F32
    _check(lib().qlora_linear_bwd(qtype, _p(wq), N, K, _p(X), _p(dY), M, _p(A), _p(B), r, scale, _p(H), _p(dX),
                                  dxt, _p(dA), _p(dB), _p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "qlora_linear_bwd")


class MoeRoute:
    """Device buffers written by qlora_moe_route."""

    def __init__(self, T, E, k, device="cuda"):
        P = T * k
        i32 = torch.int32
        self.T, self.E, self.k = T, E, k
        self.topk_idx = torch.empty(T, k, dtype=i32, device=device)
        self.topk_w = torch.empty(T, k, dtype=torch.float32, device=device)
        self.counts = torch.empty(E, dtype=i32, device=device)
        self.offsets = torch.empty(E + 1, dtype=i32, device=device)
        self.perm = torch.empty(P, dtype=i32, device=device)
        self.inv_perm = torch.empty(P, dtype=i32, device=device)
        self.mblk = torch.empty(E + 1, dtype=i32, device=device)
        self.ws = torch.empty(max(1, qlora_moe_route_workspace_bytes(T, E, k)), dtype=torch.uint8,
                              device=device)


def qlora_moe_route(logits, k, route=None, stream=None) -> MoeRoute:
    T, E = logits.shape
    if route is None:
        route = MoeRoute(T, E, k, logits.device)
    _check(lib().qlora_moe_route(_p(logits), T, E, k, _p(route.topk_idx), _p(route.topk_w), _p(route.counts),
                                 _p(route.offsets), _p(route.perm), _p(route.inv_perm), _p(route.mblk),
                                 _p(route.ws), route.ws.numel(), _s(stream)),
           "qlora_moe_route")
    return route


def qlora_moe_route_workspace_bytes(T, E, k) -> int:
    return int(lib().qlora_moe_route_workspace_bytes(T, E, k))


def qlora_moe_saved_bytes(T, k, H, I, r) -> int:
    return int(lib().qlora_moe_saved_bytes(T, k, H, I, r))


def qlora_moe_workspace_bytes(T, k, E, H, I, r) -> int:
    return int(lib().qlora_moe_workspace_bytes(T, k, E, H, I, r))


def _nb(t):
    return t.numel() * t.element_size()


def qlora_moe_fwd(qtype, w_gu, w_d, E, H, I, X, route, A_gu, B_gu, A_d, B_d, r, scale, Y, saved, ws, stream=None):
    T = X.shape[0]
    R = route
    _check(lib().qlora_moe_fwd(qtype, _p(w_gu), _p(w_d), E, H, I, _p(X), T, R.k, _p(R.topk_idx), _p(R.topk_w),
                               _p(R.offsets), _p(R.perm), _p(R.inv_perm), _p(R.mblk), _p(A_gu), _p(B_gu), _p(A_d),
                               _p(B_d), r, scale, _p(Y), _dt(Y), _p(saved), _nb(saved), _p(ws), _nb(ws), _s(stream)),
           "qlora_moe_fwd")


def qlora_moe_bwd(qtype, w_gu, w_d, E, H, I, X, dY, route, A_gu, B_gu, A_d, B_d, r, scale, saved, dX, dA_gu, dB_gu,
                  dA_d, dB_d, d_logits, ws, stream=None):
    T = X.shape[0]
    R = route
    _check(lib().qlora_moe_bwd(qtype, _p(w_gu), _p(w_d), E, H, I, _p(X), _p(dY), T, R.k, _p(R.topk_idx),
                               _p(R.topk_w), _p(R.offsets), _p(R.perm), _p(R.inv_perm), _p(R.mblk), _p(A_gu), _p(B_gu),
                               _p(A_d), _p(B_d), r, scale, _p(saved), _nb(saved), _p(dX), _dt(dX), _p(dA_gu),
                               _p(dB_gu), _p(dA_d), _p(dB_d), _p(d_logits), _p(ws), _nb(ws), _s(stream)),
           "qlora_moe_bwd")


class Adamw8State:
    """Device buffers of the 8-bit AdamW moments for n parameters (zeros: before the first step)."""

    def __init__(self, n, device="cuda"):
        nb = (n + 255) // 256
        self.n = n
        self.m_q = torch.zeros(n, dtype=torch.uint8, device=device)
        self.v_q = torch.zeros(n, dtype=torch.uint8, device=device)
        self.m_absmax = torch.zeros(nb, dtype=torch.float32, device=device)
        self.v_absmax = torch.zeros(nb, dtype=torch.float32, device=device)


def qlora_adamw8_step(p, grad, state, step, lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0,
                      p_bf16=None, stream=None):
    _check(lib().qlora_adamw8_step(_p(p), _p(grad), _p(state.m_q), _p(state.m_absmax), _p(state.v_q),
                                   _p(state.v_absmax), p.numel(), lr, beta1, beta2, eps, weight_decay, step,
                                   _p(p_bf16) if p_bf16 is not None else None, _s(stream)),
           "qlora_adamw8_step")


def qlora_rmsnorm_fwd(X, gamma, eps, Xn, rstd, stream=None):
    M, K = X.shape
    _check(lib().qlora_rmsnorm_fwd(_p(X), _p(gamma), M, K, eps, _p(Xn), _p(rstd), _s(stream)), "qlora_rmsnorm_fwd")


def qlora_rmsnorm_bwd(X, gamma, rstd, dXn, dX, stream=None):
    M, K = X.shape
    _check(lib().qlora_rmsnorm_bwd(_p(X), _p(gamma), _p(rstd), _p(dXn), _dt(dXn), M, K, _p(dX), _dt(dX), _s(stream)),
           "qlora_rmsnorm_bwd")


def qlora_lm_head_ce_workspace_bytes(M, V, K, chunk) -> int:
    return int(lib().qlora_lm_head_ce_workspace_bytes(M, V, K, chunk))


def qlora_lm_head_ce(qtype, wq, V, K, X, labels, chunk, grad_scale, loss, dX, ws, stream=None):
    M = X.shape[0]
    _check(lib().qlora_lm_head_ce(qtype, _p(wq), V, K, _p(X), M, _p(labels), chunk, grad_scale, _p(loss),
                                  _p(dX) if dX is not None else None, _dt(dX) if dX is not None else QL_F32,
                                  _p(ws), _nb(ws), _s(stream)),
           "qlora_lm_head_ce")
