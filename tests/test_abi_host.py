"""The C-ABI library loads, exports every symbol include/jmoe.h declares, and rejects bad
arguments on the host (no GPU needed: these calls return before touching a device)."""
import ctypes
import os
import re

import pytest

import int8_expert_weight_b200 as jm
from int8_expert_weight_b200 import build as jbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    jbuild.build()
    return jm.load_library()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(jamba_(?:moe|mlp)_[a-z_0-9]+)\s*\(", src, re.M))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "jamba_moe_forward" in names and "jamba_moe_quantize" in names and "jamba_mlp_forward" in names
    for n in names:
        assert hasattr(lib, n), n


def test_workspace_size(lib):
    assert jm.jamba_moe_workspace_size(32, 4096, 14336) > 32 * 2 * 4096 * 4
    assert jm.jamba_moe_workspace_size(0, 4096, 14336) > 0      # no token: valid, nothing to do
    assert jm.jamba_moe_workspace_size(-1, 4096, 14336) == 0
    assert jm.jamba_moe_workspace_size(8, 4000, 14336) == 0      # d not a multiple of 128
    assert jm.jamba_moe_workspace_size(8, 4096, 14336, 8, 2) == 0  # only 16 experts
    assert jm.jamba_moe_workspace_size(8, 4096, 14336, 16, 1) == 0  # only top-2
    a = jm.jamba_moe_workspace_size(100, 256, 512)
    b = jm.jamba_moe_workspace_size(200, 256, 512)
    assert b > a and a % 256 == 0


def test_status_strings(lib):
    for s in range(8):
        assert jm.jamba_moe_status_string(s)
    assert jm.jamba_moe_status_string(99) == "unknown status"


FAKE = 0x10000  # a 256-aligned non-null value; never dereferenced because validation fails first


def fwd(lib, T=8, d=256, F=512, E=16, K=2, x=FAKE, ws=FAKE, wsb=1 << 40, path=0, y=FAKE):
    p = [x, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE]
    return lib.jamba_moe_forward_path(*p, T, d, F, E, K, y, None, None, ws, wsb, None, path)


def test_forward_argument_errors(lib):
    assert fwd(lib, x=None) == 1
    assert fwd(lib, y=None) == 1
    assert fwd(lib, ws=None) == 1
    assert fwd(lib, E=8) == 2
    assert fwd(lib, K=1) == 2
    assert fwd(lib, d=200) == 2
    assert fwd(lib, F=100) == 2
    assert fwd(lib, T=-1) == 2
    assert fwd(lib, T=0) == 0                      # no token: nothing launched
    assert fwd(lib, T=0, x=None, y=None, ws=None, wsb=0) == 0  # and no pointer read
    assert fwd(lib, T=0, d=200) == 2               # sizes are still checked
    assert fwd(lib, path=7) == 2
    assert fwd(lib, x=FAKE + 8) == 7
    assert fwd(lib, ws=FAKE + 16) == 3
    assert fwd(lib, wsb=1024) == 3


def mlp(lib, T=8, d=256, F=512, x=FAKE, ws=FAKE, wsb=1 << 40, path=0, y=FAKE, s=FAKE):
    return lib.jamba_mlp_forward_path(x, FAKE, s, FAKE, FAKE, FAKE, FAKE, T, d, F, y, ws, wsb, None, path)


def test_mlp_workspace_and_argument_errors(lib):
    a = jm.jamba_mlp_workspace_size(32, 4096, 14336)
    assert a > 128 * 14336 * 2 and a % 256 == 0
    assert a < jm.jamba_moe_workspace_size(32, 4096, 14336)
    assert jm.jamba_mlp_workspace_size(-1, 4096, 14336) == 0
    assert jm.jamba_mlp_workspace_size(8, 4096, 14300) == 0
    assert mlp(lib, x=None) == 1
    assert mlp(lib, s=None) == 1
    assert mlp(lib, ws=None) == 1
    assert mlp(lib, T=-1) == 2
    assert mlp(lib, T=0, x=None, y=None, ws=None, s=None) == 0
    assert mlp(lib, d=200) == 2
    assert mlp(lib, path=5) == 2
    assert mlp(lib, y=FAKE + 2) == 7
    assert mlp(lib, s=FAKE + 2) == 7
    assert mlp(lib, ws=FAKE + 64) == 3
    assert mlp(lib, wsb=4096) == 3


def test_fp8_workspace_and_argument_errors(lib):
    assert jm.jamba_moe_workspace_size_fp8(32, 4096, 14336) > 0
    assert jm.jamba_moe_workspace_size_fp8(8, 4000, 14336) == 0
    p = [FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE]
    f = lib.jamba_moe_forward_fp8
    assert f(None, *p[1:], 8, 256, 512, 16, 2, FAKE, None, None, FAKE, 1 << 40, None, 0) == 1
    assert f(*p, 8, 256, 512, 8, 2, FAKE, None, None, FAKE, 1 << 40, None, 0) == 2
    assert f(*p, 8, 256, 512, 16, 2, FAKE + 4, None, None, FAKE, 1 << 40, None, 0) == 7
    assert f(*p, 8, 256, 512, 16, 2, FAKE, None, None, FAKE, 1024, None, 0) == 3
    assert f(*p, 8, 256, 512, 16, 2, FAKE, None, None, FAKE, 1 << 40, None, 9) == 2
    q = lib.jamba_moe_quantize_fp8
    assert q(None, 1, 4, 16, FAKE, FAKE, None) == 1
    assert q(FAKE, 1, 4, 10, FAKE, FAKE, None) == 2


def test_quantize_argument_errors(lib):
    q = lib.jamba_moe_quantize
    assert q(None, 1, 4, 16, FAKE, FAKE, None) == 1
    assert q(FAKE, 1, 4, 10, FAKE, FAKE, None) == 2
    assert q(FAKE, 0, 4, 16, FAKE, FAKE, None) == 2
    assert q(FAKE + 4, 1, 4, 16, FAKE, FAKE, None) == 7


def test_oracle_and_product_share_no_code():
    """The CUDA path and the oracle never import, include or link each other."""
    imp_oracle = re.compile(r"^\s*(import|from)\s+oracle\b|#include\s+[\"<][^\">]*oracle", re.M)
    imp_prod = re.compile(r"^\s*(import|from)\s+int8_expert_weight_b200\b|#include\s+[\"<][^\">]*(jmoe|csrc)", re.M)
    for dirpath, _, files in os.walk(os.path.join(ROOT, "int8_expert_weight_b200")):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                assert not imp_oracle.search(open(os.path.join(dirpath, f)).read()), f
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".c", ".h")):
            assert not imp_prod.search(open(os.path.join(ROOT, "oracle", f)).read()), f
