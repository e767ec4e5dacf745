"""ctypes wrapper around ``oracle.c`` (the plain CPU reference).

TEST INFRASTRUCTURE: imported only by tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``.  It builds ``liboracle.so`` with gcc on
first use (no ``-ffast-math``; ``-ffp-contract=off`` so that every fp32
operation in the quantizers is a single IEEE round-to-nearest-even step).

Arrays are numpy.  bf16 inputs may be given as torch bfloat16 CPU tensors or as
numpy uint16 bit patterns.  Every function cites, in ``oracle.c``, the page
passage it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

Q_NONE, Q_STATIC, Q_DYNAMIC = 0, 1, 2
FLAG_GROUP_SIZES, FLAG_SCALE = 1, 2
BLOCK = 128

_lib = None


_CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it; returns the path."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.run(["gcc", *_CFLAGS, "-o", _LIB_PATH, _SRC, "-lm"], check=True)
    return _LIB_PATH


def source_text() -> str:
    """The C source of this oracle."""
    with open(_SRC) as f:
        return f.read()


def build_variant(src_text: str, directory: str, name: str) -> str:
    """Compile a variant of the C source (same flags) into directory/name.so."""
    c_path = os.path.join(directory, name + ".c")
    so_path = os.path.join(directory, name + ".so")
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", *_CFLAGS, "-o", so_path, c_path, "-lm"], check=True)
    return so_path


def _P(t):
    return ctypes.POINTER(t)


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def load_variant(so_path: str):
    """A separately compiled build of this oracle's C source (for example a
    copy with a deliberate mistake, made by a test to show that the pins
    reject it), with the same signatures bound.  Pass it as ``_L`` to the
    wrappers that take one."""
    return _bind(ctypes.CDLL(so_path))


def _bind(L):
    i32, i64, f32, u8, u16, f64 = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_uint8,
                                   ctypes.c_uint16, ctypes.c_double)
    L.gmo_num_threads.restype = ctypes.c_int
    L.gmo_e4m3_decode.argtypes = [u8]
    L.gmo_e4m3_decode.restype = f64
    L.gmo_e4m3_encode.argtypes = [f64]
    L.gmo_e4m3_encode.restype = u8
    L.gmo_static_scale_ok.argtypes = [f32]
    L.gmo_static_scale_ok.restype = ctypes.c_int
    L.gmo_plan.argtypes = [_P(i32), i32, i64, _P(i64), _P(i32)]
    L.gmo_quantize_rows.argtypes = [_P(u16), i64, i64, i32, f32, _P(u8), _P(f32), _P(i32)]
    L.gmo_quantize_rows_scaled.argtypes = [_P(u16), i64, i64, _P(f32), _P(i32), i32, _P(u8), _P(f32)]
    L.gmo_quantize_rhs.argtypes = [_P(u16), i32, i64, i64, _P(u8), _P(f32)]
    L.gmo_quantize_rhs_blocks.argtypes = [_P(u16), i32, i64, i64, i32, _P(u8), _P(f32)]
    L.gmo_gmm_fwd_blockwise.argtypes = [_P(u16), i32, f32, _P(u8), _P(f32), _P(i32), i32, i64, i64, i64,
                                        _P(i64), i64, _P(f64), _P(f64)]
    L.gmo_gmm_dlhs_blockwise.argtypes = [_P(u16), _P(u8), _P(f32), _P(i32), i32, i64, i64, i64, _P(i64), i64,
                                         _P(f64), _P(f64)]
    L.gmo_num_chunks.argtypes = [_P(i32), i32, i64]
    L.gmo_num_chunks.restype = i64
    L.gmo_quantize_chunks.argtypes = [_P(u16), i64, i64, i32, f32, _P(i32), i32, _P(u8), _P(f32)]
    L.gmo_gmm_fwd.argtypes = [_P(u16), i32, f32, _P(u8), _P(f32), _P(i32), i32, i64, i64, i64,
                              _P(i64), i64, _P(f64), _P(f64)]
    L.gmo_gmm_dlhs.argtypes = [_P(u16), _P(u8), _P(f32), _P(i32), i32, i64, i64, i64, _P(i64), i64,
                               _P(f64), _P(f64)]
    L.gmo_tgmm_drhs.argtypes = [_P(u16), i32, f32, _P(u16), _P(i32), i32, i64, i64, i64, _P(i64), i64,
                                _P(f64), _P(f64)]
    L.gmo_gmm_fwd_bf16.argtypes = [_P(u16), _P(u16), _P(i32), i32, i64, i64, i64, _P(i64), i64,
                                   _P(f64), _P(f64)]
    L.gmo_gmm_dlhs_bf16.argtypes = L.gmo_gmm_fwd_bf16.argtypes
    L.gmo_tgmm_drhs_bf16.argtypes = L.gmo_gmm_fwd_bf16.argtypes
    return L


# ----------------------------------------------------------------- helpers

def _bf16_bits(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(ctypes.POINTER(t))


def _sizes(group_sizes) -> np.ndarray:
    if not isinstance(group_sizes, np.ndarray):
        group_sizes = np.asarray(group_sizes.cpu() if hasattr(group_sizes, "cpu") else group_sizes)
    return np.ascontiguousarray(group_sizes.astype(np.int32))


def _rows(rows, M):
    if rows is None:
        return np.arange(M, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def num_threads() -> int:
    return lib().gmo_num_threads()


# ----------------------------------------------------------------- formats

def e4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    L = lib()
    table = np.array([L.gmo_e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[codes]


def e4m3_encode(values) -> np.ndarray:
    values = np.asarray(values, dtype=np.float64)
    L = lib()
    flat = values.reshape(-1)
    out = np.fromiter((L.gmo_e4m3_encode(float(v)) for v in flat), dtype=np.uint8, count=flat.size)
    return out.reshape(values.shape)


def static_scale_ok(s: float) -> bool:
    return bool(lib().gmo_static_scale_ok(float(s)))


# -------------------------------------------------------------------- plan

def plan(group_sizes, M: int):
    """Clamped group row offsets [G+1] and the flags word."""
    gs = _sizes(group_sizes)
    offs = np.zeros(gs.size + 1, dtype=np.int64)
    flags = ctypes.c_int32(0)
    lib().gmo_plan(_ptr(gs, ctypes.c_int32), gs.size, M, _ptr(offs, ctypes.c_int64), ctypes.byref(flags))
    return offs, flags.value


# ---------------------------------------------------------------- quantize

def quantize_rows(x, rule: int, static_scale: float = 0.0):
    """Codes [R, C] and scales [R, C/128] (128-blocks along each row)."""
    xb = _bf16_bits(x)
    R, C = xb.shape
    codes = np.empty((R, C), dtype=np.uint8)
    scales = np.empty((R, C // BLOCK), dtype=np.float32)
    flags = ctypes.c_int32(0)
    lib().gmo_quantize_rows(_ptr(xb, ctypes.c_uint16), R, C, rule, static_scale,
                            _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_float), ctypes.byref(flags))
    return codes, scales, flags.value


def quantize_rows_scaled(dout, sr: np.ndarray, group_sizes):
    """dlhs operand: fl32(dout * s_r[g(m), n]) in dynamic 128-blocks along n."""
    db = _bf16_bits(dout)
    M, N = db.shape
    sr = np.ascontiguousarray(sr, dtype=np.float32)
    gs = _sizes(group_sizes)
    codes = np.empty((M, N), dtype=np.uint8)
    scales = np.empty((M, N // BLOCK), dtype=np.float32)
    lib().gmo_quantize_rows_scaled(_ptr(db, ctypes.c_uint16), M, N, _ptr(sr, ctypes.c_float),
                                   _ptr(gs, ctypes.c_int32), gs.size, _ptr(codes, ctypes.c_uint8),
                                   _ptr(scales, ctypes.c_float))
    return codes, scales


def quantize_rhs(w):
    """W [G, K, N] bf16 -> codes [G, K, N], per-(g, n) scales [G, N]."""
    wb = _bf16_bits(w)
    G, K, N = wb.shape
    codes = np.empty((G, K, N), dtype=np.uint8)
    scales = np.empty((G, N), dtype=np.float32)
    lib().gmo_quantize_rhs(_ptr(wb, ctypes.c_uint16), G, K, N, _ptr(codes, ctypes.c_uint8),
                           _ptr(scales, ctypes.c_float))
    return codes, scales


def quantize_rhs_blocks(w, axis: int):
    """W [G, K, N] bf16 -> codes [G, K, N] and block-wise scales: axis 0
    [G, K/128, N] (blocks along K), axis 1 [G, N/128, K] (blocks along N)."""
    wb = _bf16_bits(w)
    G, K, N = wb.shape
    codes = np.empty((G, K, N), dtype=np.uint8)
    scales = np.empty((G, K // BLOCK, N) if axis == 0 else (G, N // BLOCK, K), dtype=np.float32)
    lib().gmo_quantize_rhs_blocks(_ptr(wb, ctypes.c_uint16), G, K, N, axis, _ptr(codes, ctypes.c_uint8),
                                  _ptr(scales, ctypes.c_float))
    return codes, scales


def num_chunks(group_sizes, M: int) -> int:
    gs = _sizes(group_sizes)
    return int(lib().gmo_num_chunks(_ptr(gs, ctypes.c_int32), gs.size, M))


def quantize_chunks(x, rule: int, static_scale: float, group_sizes):
    """tgmm operand: codes [M, C] in x's layout, scales [num_chunks, C]."""
    xb = _bf16_bits(x)
    M, C = xb.shape
    gs = _sizes(group_sizes)
    nch = num_chunks(gs, M)
    codes = np.empty((M, C), dtype=np.uint8)
    scales = np.empty((max(nch, 1), C), dtype=np.float32)
    lib().gmo_quantize_chunks(_ptr(xb, ctypes.c_uint16), M, C, rule, static_scale, _ptr(gs, ctypes.c_int32),
                              gs.size, _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_float))
    return codes, scales[:nch]


# ------------------------------------------------------------------ passes

def gmm_fwd(lhs, rule: int, static_scale: float, qr: np.ndarray, sr: np.ndarray, group_sizes, rows=None):
    """Forward gmm on the given rows (all by default) -> (out, absum) fp64."""
    lb = _bf16_bits(lhs)
    M, K = lb.shape
    G, K2, N = qr.shape
    assert K2 == K
    gs = _sizes(group_sizes)
    r = _rows(rows, M)
    qr = np.ascontiguousarray(qr, dtype=np.uint8)
    sr = np.ascontiguousarray(sr, dtype=np.float32)
    out = np.empty((r.size, N), dtype=np.float64)
    ab = np.empty((r.size, N), dtype=np.float64)
    lib().gmo_gmm_fwd(_ptr(lb, ctypes.c_uint16), rule, static_scale, _ptr(qr, ctypes.c_uint8),
                      _ptr(sr, ctypes.c_float), _ptr(gs, ctypes.c_int32), G, M, K, N, _ptr(r, ctypes.c_int64),
                      r.size, _ptr(out, ctypes.c_double), _ptr(ab, ctypes.c_double))
    return out, ab


def gmm_dlhs(dout, qr: np.ndarray, sr: np.ndarray, group_sizes, rows=None):
    """Backward gmm wrt lhs on the given rows -> (dlhs, absum) fp64 [rows, K]."""
    db = _bf16_bits(dout)
    M, N = db.shape
    G, K, N2 = qr.shape
    assert N2 == N
    gs = _sizes(group_sizes)
    r = _rows(rows, M)
    qr = np.ascontiguousarray(qr, dtype=np.uint8)
    sr = np.ascontiguousarray(sr, dtype=np.float32)
    out = np.empty((r.size, K), dtype=np.float64)
    ab = np.empty((r.size, K), dtype=np.float64)
    lib().gmo_gmm_dlhs(_ptr(db, ctypes.c_uint16), _ptr(qr, ctypes.c_uint8), _ptr(sr, ctypes.c_float),
                       _ptr(gs, ctypes.c_int32), G, M, K, N, _ptr(r, ctypes.c_int64), r.size,
                       _ptr(out, ctypes.c_double), _ptr(ab, ctypes.c_double))
    return out, ab


def tgmm_drhs(x, rule: int, static_scale: float, dout, group_sizes, sel=None):
    """Weight gradient on selected (g, k) rows (index g*K + k; all by default).

    Returns (dW, absum) fp64: [G, K, N] when sel is None, else [len(sel), N].
    """
    xb = _bf16_bits(x)
    db = _bf16_bits(dout)
    M, K = xb.shape
    M2, N = db.shape
    assert M2 == M
    gs = _sizes(group_sizes)
    G = gs.size
    s = np.arange(G * K, dtype=np.int64) if sel is None else np.ascontiguousarray(np.asarray(sel, np.int64))
    out = np.empty((s.size, N), dtype=np.float64)
    ab = np.empty((s.size, N), dtype=np.float64)
    lib().gmo_tgmm_drhs(_ptr(xb, ctypes.c_uint16), rule, static_scale, _ptr(db, ctypes.c_uint16),
                        _ptr(gs, ctypes.c_int32), G, M, K, N, _ptr(s, ctypes.c_int64), s.size,
                        _ptr(out, ctypes.c_double), _ptr(ab, ctypes.c_double))
    if sel is None:
        return out.reshape(G, K, N), ab.reshape(G, K, N)
    return out, ab


def gmm_fwd_blockwise(lhs, rule: int, static_scale: float, qr: np.ndarray, srb: np.ndarray, group_sizes,
                      rows=None):
    """Forward gmm with block-wise rhs scales srb [G, K/128, N] -> (out, absum)."""
    lb = _bf16_bits(lhs)
    M, K = lb.shape
    G, K2, N = qr.shape
    assert K2 == K and srb.shape == (G, K // BLOCK, N)
    gs, r = _sizes(group_sizes), _rows(rows, M)
    qr = np.ascontiguousarray(qr, dtype=np.uint8)
    srb = np.ascontiguousarray(srb, dtype=np.float32)
    out = np.empty((r.size, N)); ab = np.empty((r.size, N))
    lib().gmo_gmm_fwd_blockwise(_ptr(lb, ctypes.c_uint16), rule, static_scale, _ptr(qr, ctypes.c_uint8),
                                _ptr(srb, ctypes.c_float), _ptr(gs, ctypes.c_int32), G, M, K, N,
                                _ptr(r, ctypes.c_int64), r.size, _ptr(out, ctypes.c_double),
                                _ptr(ab, ctypes.c_double))
    return out, ab


def gmm_dlhs_blockwise(dout, qr: np.ndarray, srb: np.ndarray, group_sizes, rows=None):
    """dlhs with block-wise rhs scales along N, srb [G, N/128, K] -> (dlhs, absum)."""
    db = _bf16_bits(dout)
    M, N = db.shape
    G, K, N2 = qr.shape
    assert N2 == N and srb.shape == (G, N // BLOCK, K)
    gs, r = _sizes(group_sizes), _rows(rows, M)
    qr = np.ascontiguousarray(qr, dtype=np.uint8)
    srb = np.ascontiguousarray(srb, dtype=np.float32)
    out = np.empty((r.size, K)); ab = np.empty((r.size, K))
    lib().gmo_gmm_dlhs_blockwise(_ptr(db, ctypes.c_uint16), _ptr(qr, ctypes.c_uint8), _ptr(srb, ctypes.c_float),
                                 _ptr(gs, ctypes.c_int32), G, M, K, N, _ptr(r, ctypes.c_int64), r.size,
                                 _ptr(out, ctypes.c_double), _ptr(ab, ctypes.c_double))
    return out, ab


# ------------------------------------------------------------------ SwiGLU

# max over the reals of |silu'(z)|, reached near z = 2.3994 (value 1.09984);
# rounded up.  Bounds how an error in the gate moves silu(gate).
SILU_LIPSCHITZ = 1.1


def silu(z):
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z)), fp64, elementwise: the
    activation of the SwiGLU MLP whose gate and up projections the merged gmm
    computes ("FP8 Megablox for batch split", maxtext PR #3770, Description
    (2): W0 and W1 concatenated into one gmm).  exp(-z) overflows to inf for
    z below about -709, which gives -0.0, the limit."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def gmm_fwd_swiglu(lhs, rule: int, static_scale: float, qr: np.ndarray, sr: np.ndarray, group_sizes,
                   rows=None):
    """SwiGLU of the merged forward.  qr / sr are the codes and scales of the
    merged rhs [W0 | W1] ([G, K, 2F], [G, 2F]).  The forward h is this
    module's gmm_fwd (fp64); the result is silu(h[:, :F]) * h[:, F:].

    Returns (out [rows, F], (gate, up, absum_gate, absum_up)); the second item
    feeds the propagated tolerance of a reduced-precision implementation."""
    h, ab = gmm_fwd(lhs, rule, static_scale, qr, sr, group_sizes, rows)
    F = h.shape[1] // 2
    gate, up = h[:, :F], h[:, F:]
    return silu(gate) * up, (gate, up, ab[:, :F], ab[:, F:])


def gmm_fwd_bf16(lhs, w, group_sizes, rows=None, _L=None):
    """bf16-family forward: out[m, :] = lhs[m, :] @ W[g(m)] with the bf16
    operands widened exactly, fp64 sums -> (out, absum)."""
    lb, wb = _bf16_bits(lhs), _bf16_bits(w)
    M, K = lb.shape
    G, _, N = wb.shape
    gs, r = _sizes(group_sizes), _rows(rows, M)
    out = np.empty((r.size, N)); ab = np.empty((r.size, N))
    (_L or lib()).gmo_gmm_fwd_bf16(_ptr(lb, ctypes.c_uint16), _ptr(wb, ctypes.c_uint16), _ptr(gs, ctypes.c_int32), G,
                           M, K, N, _ptr(r, ctypes.c_int64), r.size, _ptr(out, ctypes.c_double),
                           _ptr(ab, ctypes.c_double))
    return out, ab


def gmm_dlhs_bf16(dout, w, group_sizes, rows=None, _L=None):
    """bf16-family dlhs: dlhs[m, :] = dout[m, :] @ W[g(m)]^T -> (dlhs, absum)."""
    db, wb = _bf16_bits(dout), _bf16_bits(w)
    M, N = db.shape
    G, K, _ = wb.shape
    gs, r = _sizes(group_sizes), _rows(rows, M)
    out = np.empty((r.size, K)); ab = np.empty((r.size, K))
    (_L or lib()).gmo_gmm_dlhs_bf16(_ptr(db, ctypes.c_uint16), _ptr(wb, ctypes.c_uint16), _ptr(gs, ctypes.c_int32), G,
                            M, K, N, _ptr(r, ctypes.c_int64), r.size, _ptr(out, ctypes.c_double),
                            _ptr(ab, ctypes.c_double))
    return out, ab


def tgmm_drhs_bf16(x, dout, group_sizes, sel=None, _L=None):
    """bf16-family tgmm: dW[g] = x[rows of g]^T @ dout[rows of g] on the
    selected (g, k) rows (index g*K + k; all by default) -> (dW, absum)."""
    xb, db = _bf16_bits(x), _bf16_bits(dout)
    M, K = xb.shape
    _, N = db.shape
    gs = _sizes(group_sizes)
    G = gs.size
    s = np.arange(G * K, dtype=np.int64) if sel is None else np.ascontiguousarray(np.asarray(sel, np.int64))
    out = np.empty((s.size, N)); ab = np.empty((s.size, N))
    (_L or lib()).gmo_tgmm_drhs_bf16(_ptr(xb, ctypes.c_uint16), _ptr(db, ctypes.c_uint16), _ptr(gs, ctypes.c_int32), G,
                             M, K, N, _ptr(s, ctypes.c_int64), s.size, _ptr(out, ctypes.c_double),
                             _ptr(ab, ctypes.c_double))
    if sel is None:
        return out.reshape(G, K, N), ab.reshape(G, K, N)
    return out, ab
