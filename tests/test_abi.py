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
