"""The C-ABI library loads and exports every function include/gmm_fp8.h
declares; host-side argument checks return their status codes before any
CUDA call (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

from moe_fp8_grouped_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gmm_fp8.h")


@pytest.fixture(scope="module")
def L():
    from moe_fp8_grouped_b200 import build
    build.build()
    return B.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_header_declares_the_binding_exports():
    assert sorted(B.EXPORTS) == declared_functions()


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_pure_host_queries(L):
    ws_fwd = L.gmm_workspace_bytes(0, 16384, 4096, 28672, 8)
    assert ws_fwd >= 16384 * 4096 + 4 * 16384 * 32
    assert L.gmm_workspace_bytes(0, 0, 128, 128, 1) == 0
    assert L.gmm_workspace_bytes(0, 10, 100, 128, 1) == 0
    assert L.gmm_workspace_bytes(2, 300, 256, 256, 3) > 0
    assert L.gmm_workspace_bytes(7, 300, 256, 256, 3) == 0
    assert L.gmm_chunk_capacity(256, 8) == 2 + 8
    assert L.gmm_chunk_capacity(257, 8) == 3 + 8
    for s in range(10):
        assert L.gmm_status_string(s)
    assert b"unknown" in L.gmm_status_string(99)


def _op(data, dtype, scale, rule):
    return B.Operand(data, dtype, scale, rule)


FAKE = 0x100000  # a 16-byte aligned fake device address; never dereferenced


def test_host_errors(L):
    lhs = _op(FAKE, B.DT_BF16, FAKE, B.Q_STATIC)
    rhs = _op(FAKE, B.DT_E4M3, FAKE, B.Q_NONE)
    gs, out, ws = FAKE, FAKE, FAKE
    big = 1 << 40
    f = L.gmm_fwd
    assert f(lhs, rhs, 0, gs, 8, 0, 512, 512, out, B.DT_BF16, ws, big, None) == 2  # M = 0
    assert f(lhs, rhs, 0, gs, 8, 256, 500, 512, out, B.DT_BF16, ws, big, None) == 2  # K % 128
    assert f(lhs, rhs, 0, gs, 8, 256, 512, 200, out, B.DT_BF16, ws, big, None) == 2  # N % 128
    assert f(lhs, rhs, 0, gs, 2000, 256, 512, 512, out, B.DT_BF16, ws, big, None) == 5  # G > 1024
    assert f(lhs, rhs, 0, gs, 8, 65528 * 128 + 1, 512, 512, out, B.DT_BF16, ws, big, None) == 5  # chunks > 65535
    assert f(lhs, rhs, 0, gs, 8, 65527 * 128, 512, 512, out, B.DT_BF16, ws, 1024, None) == 9  # at the limit
    assert f(lhs, rhs, 0, None, 8, 256, 512, 512, out, B.DT_BF16, ws, big, None) == 1  # no group_sizes
    assert f(_op(FAKE, B.DT_BF16, None, B.Q_STATIC), rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big,
             None) == 1  # static rule without its scale
    assert f(lhs, _op(FAKE, B.DT_E4M3, None, B.Q_NONE), 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big,
             None) == 1  # fp8 rhs without scales
    assert f(_op(FAKE, B.DT_BF16, None, B.Q_NONE), rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big,
             None) == 1  # rule NONE with an e4m3 operand
    assert f(lhs, rhs, 0, gs, 8, 256, 512, 512, out, B.DT_E4M3, ws, big, None) == 1  # fp8 output
    assert f(_op(FAKE + 2, B.DT_BF16, FAKE, B.Q_STATIC), rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big,
             None) == 3  # misaligned
    assert f(lhs, rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, 1024, None) == 9  # workspace too small
    assert f(lhs, rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, None, big, None) == 9  # no workspace
    assert f(_op(FAKE, B.DT_E4M3, None, B.Q_DYNAMIC), rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big,
             None) == 1  # pre-quantized lhs without its scales
    sw = L.gmm_fwd_swiglu
    assert sw(lhs, rhs, 0, gs, 8, 256, 512, 384, out, B.DT_BF16, ws, big, None) == 2  # N = 2F, F % 128
    assert sw(lhs, rhs, 0, gs, 8, 256, 512, 0, out, B.DT_BF16, ws, big, None) == 2
    assert sw(lhs, rhs, 0, None, 8, 256, 512, 512, out, B.DT_BF16, ws, big, None) == 1
    assert sw(lhs, rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, 1024, None) == 9
    kl = L.gmm_fwd_keep_lhs
    assert kl(lhs, rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big, None, None, None) == 1  # no codes buffer
    assert kl(_op(FAKE, B.DT_BF16, None, B.Q_DYNAMIC), rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big, FAKE,
              None, None) == 1  # dynamic rule without a scales buffer
    assert kl(lhs, rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big, FAKE + 2, None, None) == 3
    bw = L.gmm_backward
    dop = _op(FAKE, B.DT_BF16, None, B.Q_DYNAMIC)
    assert bw(lhs, dop, rhs, 0, gs, 8, 256, 500, 512, out, B.DT_BF16, out, B.DT_F32, ws, big, None) == 2  # K % 128
    assert bw(lhs, dop, rhs, 0, gs, 8, 256, 512, 512, None, B.DT_BF16, out, B.DT_F32, ws, big, None) == 1
    assert bw(lhs, dop, rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, out, B.DT_F32, ws, 1024, None) == 9
    assert bw(lhs, _op(FAKE, B.DT_BF16, None, B.Q_STATIC), rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, out,
              B.DT_F32, ws, big, None) == 1  # gradients are dynamic
    d = L.gmm_dlhs
    assert d(_op(FAKE, B.DT_E4M3, FAKE, B.Q_DYNAMIC), rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big,
             None) == 1  # dout must be bf16 (the rhs scale is folded in)
    assert d(_op(FAKE, B.DT_BF16, None, B.Q_STATIC), rhs, 0, gs, 8, 256, 512, 512, out, B.DT_BF16, ws, big,
             None) == 1  # gradients are dynamic
    t = L.tgmm_drhs
    dout = _op(FAKE, B.DT_BF16, None, B.Q_DYNAMIC)
    assert t(lhs, _op(FAKE, B.DT_BF16, None, B.Q_STATIC), gs, 8, 256, 512, 512, out, B.DT_F32, ws, big,
             None) == 1  # dout must be dynamic
    assert t(lhs, dout, gs, 8, 256, 512, 512, out, B.DT_F32, ws, 4096, None) == 9
    q = L.gmm_quantize
    assert q(FAKE, 256, 512, 3, 1, None, None, 0, None, FAKE, FAKE, FAKE, big, None) == 1  # bad rule
    assert q(FAKE, 256, 512, B.Q_STATIC, 1, None, None, 0, None, FAKE, FAKE, FAKE, big, None) == 1
    assert q(FAKE, 256, 512, B.Q_DYNAMIC, 0, None, None, 0, None, FAKE, FAKE, FAKE, big, None) == 1  # axis 0
    assert L.gmm_quantize_rhs(None, 8, 512, 512, 0, FAKE, FAKE, None) == 1
    assert L.gmm_quantize_rhs(FAKE, 8, 500, 512, 0, FAKE, FAKE, None) == 2
    assert L.gmm_read_device_status(None, None, None) == 1
    assert L.gmm_selftest_timeout(None, 1000, None) == 1
