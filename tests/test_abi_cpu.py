"""The C-ABI library builds, loads and exports every declared symbol; host-side
argument checks return their codes before touching a GPU (CPU only)."""
import ctypes as C
import os
import re
import subprocess

import pytest

from mixture_experts_layer_counts_b200 import _lib
from mixture_experts_layer_counts_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, re.M)))


def test_exports_match_header(L):
    decl = declared_functions()
    assert set(decl) == set(_lib.EXPORTS)
    syms = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                          text=True, check=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", syms))
    for name in decl:
        assert name in exported, name
        assert getattr(L, name) is not None


def test_workspace_size(L):
    a = L.moe_workspace_size(16, 2048, 64, 1024, 8, 0)
    b = L.moe_workspace_size(32, 2048, 64, 1024, 8, 0)
    assert 0 < a < b
    assert L.moe_workspace_size(16, 2048, 64, 1024, 8, 1) > 0
    assert L.moe_workspace_size(16, 2000, 64, 1024, 8, 0) == 0      # H not a multiple of 128
    assert L.moe_workspace_size(16, 2048, 64, 1024, 65, 0) == 0     # top_k > E
    assert L.moe_workspace_size(0, 2048, 64, 1024, 8, 0) == 0
    assert L.moe_workspace_size(16, 2048, 2048, 1024, 8, 0) == 0    # E > 1024


def test_status_strings(L):
    for code in range(8):
        assert L.moe_status_string(code)
    assert L.moe_status_string(99) == b"unknown status"


def _fwd(L, **kw):
    args = dict(hidden=16, router_w=16, bias=None, w13=16, w2=16, s13=None, s2=None, T=4, H=256,
                E=8, I=512, k=2, dtype=0, out=16, ws=16, ws_bytes=1 << 40)
    args.update(kw)
    p = lambda v: None if v is None else C.c_void_p(v)
    return L.moe_forward(p(args["hidden"]), p(args["router_w"]), p(args["bias"]), p(args["w13"]),
                         p(args["w2"]), p(args["s13"]), p(args["s2"]), args["T"], args["H"],
                         args["E"], args["I"], args["k"], args["dtype"], p(args["out"]),
                         p(args["ws"]), args["ws_bytes"], None, None)


def test_argument_errors_before_any_launch(L):
    assert _fwd(L, hidden=None) == 1
    assert _fwd(L, dtype=7) == 1
    assert _fwd(L, k=9) == 1
    assert _fwd(L, H=200) == 2
    assert _fwd(L, I=100) == 2
    assert _fwd(L, T=0) == 2
    assert _fwd(L, dtype=1) == 1                 # FP8 without scales
    assert _fwd(L, w13=0x1008) == 7              # not 16-byte aligned
    assert _fwd(L, ws_bytes=1024) == 3
    assert L.moe_workspace_init(None, 0, None) == 1
    assert L.moe_align(None, 4, 8, 2, None, None, None, None, None, 0, None) == 1
    assert L.moe_align(C.c_void_p(16), 4, 2000, 2, None, None, None, None, None, 0, None) == 2


def test_inv_rope_argument_errors(L):
    p = C.c_void_p
    f = L.moe_inv_rope_fp8_quant
    assert f(None, p(16), p(16), p(16), 4, 2, 128, 10, p(16), p(16), None) == 1      # NULL x
    assert f(p(16), p(16), p(16), p(16), 4, 2, 96, 10, p(16), p(16), None) == 2      # head_dim 96
    assert f(p(16), p(16), p(16), p(16), 0, 2, 128, 10, p(16), p(16), None) == 2     # T = 0
    assert f(p(24), p(16), p(16), p(16), 4, 2, 128, 10, p(16), p(16), None) == 7     # x not 16-byte aligned
    assert f(p(16), p(16), p(16), p(16), 4, 2, 128, 10, p(16), p(18), None) == 7     # scales not 4-byte aligned
