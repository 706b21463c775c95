"""Host-side checks of the C ABI (no GPU): the library loads, exports every function the public
header declares, and rejects bad arguments with the documented status before launching anything."""
import os
import re

import pytest

import quantized_base_lora_tma_b200 as ql
from quantized_base_lora_tma_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    from quantized_base_lora_tma_b200 import build
    build.build()
    return _lib.lib()


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = _header_functions()
    assert {"gguf_dequant", "qlora_linear_fwd", "qlora_linear_bwd"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(_lib.SIGNATURES), names ^ set(_lib.SIGNATURES)


def test_every_entry_point_has_a_binding_of_the_same_name(lib):
    missing = [n for n in _lib.SIGNATURES if not callable(getattr(ql, n, None))]
    assert not missing, missing


def test_status_strings(lib):
    for code, name in _lib.STATUS.items():
        assert ql.qlora_status_string(code) == name
    assert ql.qlora_status_string(1234) == "QL_UNKNOWN_STATUS"


def test_workspace_query(lib):
    a = ql.qlora_linear_workspace_bytes(2048, 4096, 4096, 16)
    b = ql.qlora_linear_workspace_bytes(4096, 4096, 4096, 16)
    assert 0 < a < b
    assert ql.qlora_linear_workspace_bytes(0, 4096, 4096, 16) == 0
    assert ql.qlora_linear_workspace_bytes(16, 4096, 4096, 65) == 0


FAKE = 1 << 20  # a 16-byte aligned non-null address that is never dereferenced


def test_dequant_argument_errors(lib):
    L = lib
    s = None
    assert L.gguf_dequant(5, FAKE, 4, 256, FAKE, 0, s) == 2          # unsupported qtype
    assert L.gguf_dequant(2, None, 4, 256, FAKE, 0, s) == 1          # null
    assert L.gguf_dequant(2, FAKE, 4, 100, FAKE, 0, s) == 3          # cols % 256
    assert L.gguf_dequant(2, FAKE + 2, 4, 256, FAKE, 0, s) == 4      # misaligned
    assert L.gguf_dequant(2, FAKE, 0, 256, FAKE, 0, s) == 1          # empty
    assert L.gguf_dequant(2, FAKE, 4, 256, FAKE, 7, s) == 1          # bad dtype


def test_linear_argument_errors(lib):
    L = lib
    ws_need = ql.qlora_linear_workspace_bytes(64, 512, 256, 4)
    args = dict(qt=2, wq=FAKE, N=512, K=256, X=FAKE, M=64, A=FAKE, B=FAKE, r=4, s=2.0, Y=FAKE, yd=0, H=FAKE,
                ws=FAKE, wsb=ws_need)

    def fwd(**kw):
        a = dict(args, **kw)
        return L.qlora_linear_fwd(a["qt"], a["wq"], a["N"], a["K"], a["X"], a["M"], a["A"], a["B"], a["r"],
                                  a["s"], a["Y"], a["yd"], a["H"], a["ws"], a["wsb"], None)

    assert fwd(K=300) == 3
    assert fwd(N=100) == 3
    assert fwd(r=0) == 2
    assert fwd(r=65) == 2
    assert fwd(qt=3) == 2
    assert fwd(qt=14) == 2  # Q6_K: gguf_dequant only (its 210-byte superblocks are not TMA-copied)
    assert fwd(qt=10) == 2  # Q2_K: likewise (84-byte superblocks)
    assert fwd(X=None) == 1
    assert fwd(M=0) == 1
    assert fwd(X=FAKE + 8) == 4
    assert fwd(wsb=ws_need - 1) == 5
    assert fwd(ws=None) == 5
    assert fwd(yd=3) == 1

    def bwd(**kw):
        a = dict(args, **kw)
        return L.qlora_linear_bwd(a["qt"], a["wq"], a["N"], a["K"], a["X"], FAKE, a["M"], a["A"], a["B"],
                                  a["r"], a["s"], a["H"], FAKE, 0, FAKE, FAKE, a["ws"], a["wsb"], None)

    assert bwd(K=512 + 128) == 3
    assert bwd(H=None) == 1
    assert bwd(wsb=16) == 5
    assert ql.qlora_launch_count() == 0    # nothing above reached a launch


def test_rows_fusion_switch(lib):
    """The fusion mask is process-wide host state: set, read back through the previous value, and
    restored (no launch, no device call)."""
    prev = ql.qlora_set_rows_fusion(0)
    try:
        assert ql.qlora_set_rows_fusion(3) == 0
        assert ql.qlora_set_rows_fusion(True) == 3
        assert ql.qlora_set_rows_fusion(False) == 3
        assert ql.qlora_set_rows_fusion(6) == 0      # only bits 0 and 1 are kept
        assert ql.qlora_set_rows_fusion(1) == 2
    finally:
        ql.qlora_set_rows_fusion(prev)
    assert prev == 1  # the default: the forward only


def test_moe_argument_errors(lib):
    """Routing and the MoE layer reject bad arguments on the host (no launch)."""
    L = lib
    s = None
    before = ql.qlora_launch_count()
    wsr = ql.qlora_moe_route_workspace_bytes(64, 8, 2)
    r6 = [FAKE] * 7  # topk_idx, topk_w, counts, offsets, perm, inv_perm, mblk

    def route(**kw):
        a = dict(lg=FAKE, T=64, E=8, k=2, ws=FAKE, wsb=wsr)
        a.update(kw)
        return L.qlora_moe_route(a["lg"], a["T"], a["E"], a["k"], *r6, a["ws"], a["wsb"], s)

    assert route(lg=None) == 1
    assert route(E=257) == 2 and route(k=17) == 2 and route(k=9) == 2 and route(k=0) == 2
    assert route(T=0) == 1
    assert route(wsb=wsr - 1) == 5 and route(ws=None) == 5
    assert route(ws=FAKE + 4) == 4

    T, k, E, H, I, r = 64, 2, 8, 256, 256, 4
    sv = ql.qlora_moe_saved_bytes(T, k, H, I, r)
    wsm = ql.qlora_moe_workspace_bytes(T, k, E, H, I, r)

    def fwd(**kw):
        a = dict(qt=2, E=E, H=H, I=I, X=FAKE, T=T, k=k, r=r, Y=FAKE, yd=0, sv=FAKE, svb=sv, ws=FAKE, wsb=wsm)
        a.update(kw)
        return L.qlora_moe_fwd(a["qt"], FAKE, FAKE, a["E"], a["H"], a["I"], a["X"], a["T"], a["k"], FAKE, FAKE,
                               FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, a["r"], 2.0, a["Y"], a["yd"],
                               a["sv"], a["svb"], a["ws"], a["wsb"], s)

    assert fwd(qt=14) == 2          # Q6_K: dequantization only
    assert fwd(E=300) == 2 and fwd(k=9) == 2 and fwd(r=65) == 2
    assert fwd(H=300) == 3 and fwd(I=128) == 3
    assert fwd(X=FAKE + 2) == 4
    assert fwd(Y=None) == 1 and fwd(yd=5) == 1
    assert fwd(svb=sv - 1) == 5 and fwd(wsb=wsm - 1) == 5

    def bwd(**kw):
        a = dict(dX=FAKE, dxd=0, dl=FAKE, svb=sv, wsb=wsm)
        a.update(kw)
        return L.qlora_moe_bwd(2, FAKE, FAKE, E, H, I, FAKE, FAKE, T, k, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                               FAKE, FAKE, FAKE, r, 2.0, FAKE, a["svb"], a["dX"], a["dxd"], FAKE, FAKE, FAKE, FAKE,
                               a["dl"], FAKE, a["wsb"], s)

    assert bwd(dX=None) == 1 and bwd(dxd=4) == 1
    assert bwd(dl=FAKE + 4) == 4
    assert bwd(svb=16) == 5 and bwd(wsb=16) == 5
    assert ql.qlora_launch_count() == before


def test_lm_head_rmsnorm_adamw_argument_errors(lib):
    """The lm_head, RMSNorm and 8-bit AdamW entry points reject bad arguments on the host."""
    L = lib
    s = None
    before = ql.qlora_launch_count()
    M, V, K, C = 300, 1024, 512, 128
    wsl = ql.qlora_lm_head_ce_workspace_bytes(M, V, K, C)
    assert wsl > 0 and ql.qlora_lm_head_ce_workspace_bytes(0, V, K, C) == 0

    def lm(**kw):
        a = dict(qt=8, V=V, K=K, X=FAKE, M=M, lab=FAKE, C=C, loss=FAKE, dX=FAKE, dxd=0, ws=FAKE, wsb=wsl)
        a.update(kw)
        return L.qlora_lm_head_ce(a["qt"], FAKE, a["V"], a["K"], a["X"], a["M"], a["lab"], a["C"], 1.0, a["loss"],
                                  a["dX"], a["dxd"], a["ws"], a["wsb"], s)

    assert lm(lab=None) == 1 and lm(loss=None) == 1 and lm(C=0) == 1
    assert lm(qt=5) == 2
    assert lm(V=1000) == 3 and lm(K=300) == 3
    assert lm(dxd=3) == 1
    assert lm(X=FAKE + 8) == 4
    assert lm(wsb=wsl - 1) == 5 and lm(ws=None) == 5

    assert L.qlora_rmsnorm_fwd(None, FAKE, 4, 64, 1e-6, FAKE, FAKE, s) == 1
    assert L.qlora_rmsnorm_fwd(FAKE, FAKE, 4, 60, 1e-6, FAKE, FAKE, s) == 3
    assert L.qlora_rmsnorm_fwd(FAKE, FAKE, 4, 64, -1.0, FAKE, FAKE, s) == 1
    assert L.qlora_rmsnorm_fwd(FAKE + 2, FAKE, 4, 64, 1e-6, FAKE, FAKE, s) == 4
    assert L.qlora_rmsnorm_bwd(FAKE, FAKE, FAKE, FAKE, 7, 4, 64, FAKE, 0, s) == 1
    assert L.qlora_rmsnorm_bwd(FAKE, FAKE, FAKE, FAKE, 0, 4, 68, FAKE, 0, s) == 3

    def adam(**kw):
        a = dict(p=FAKE, n=1000, b1=0.9, b2=0.999, eps=1e-8, t=1)
        a.update(kw)
        return L.qlora_adamw8_step(a["p"], FAKE, FAKE, FAKE, FAKE, FAKE, a["n"], 1e-3, a["b1"], a["b2"], a["eps"],
                                   0.01, a["t"], None, s)

    assert adam(p=None) == 1 and adam(n=0) == 1 and adam(t=0) == 1
    assert adam(b1=1.0) == 1 and adam(b2=-0.1) == 1 and adam(eps=0.0) == 1
    assert ql.qlora_launch_count() == before
