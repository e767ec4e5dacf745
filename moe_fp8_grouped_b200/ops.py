"""Torch-facing binding of the C-ABI in include/gmm_fp8.h, with the same names.

Marshalling only: every step runs in libgmm_fp8.so on the tensors' CUDA
device and on torch's current stream.  torch provides device memory (outputs
and a reusable workspace) and the stream.
"""
from __future__ import annotations

import ctypes

import torch

from . import _binding as B


class GmmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = B.STATUS_NAMES.get(status, str(status))
        text = B.lib().gmm_status_string(status).decode()
        super().__init__(f"{where}: {name} ({text})")


class QRule:
    NONE, STATIC, DYNAMIC = B.Q_NONE, B.Q_STATIC, B.Q_DYNAMIC
    by_name = {"none": B.Q_NONE, "static": B.Q_STATIC, "dynamic": B.Q_DYNAMIC}


class DType:
    BF16, F32, E4M3 = B.DT_BF16, B.DT_F32, B.DT_E4M3


_TORCH_DT = {torch.bfloat16: B.DT_BF16, torch.float32: B.DT_F32, torch.uint8: B.DT_E4M3,
             torch.float8_e4m3fn: B.DT_E4M3}


def _rule(rule) -> int:
    return QRule.by_name[rule] if isinstance(rule, str) else int(rule)


def _check(status: int, where: str):
    if status != B.GMM_OK:
        raise GmmError(status, where)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


_ws_cache: dict = {}


def workspace(nbytes: int, device) -> torch.Tensor:
    """A reusable uint8 workspace on ``device`` of at least ``nbytes``."""
    dev = torch.device(device)
    key = (dev.type, dev.index if dev.index is not None else torch.cuda.current_device())
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 1 << 16), dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    return ws


def gmm_workspace_bytes(op: int, M: int, K: int, N: int, G: int) -> int:
    return int(B.lib().gmm_workspace_bytes(op, M, K, N, G))


def gmm_chunk_capacity(rows: int, G: int) -> int:
    return int(B.lib().gmm_chunk_capacity(rows, G))


def gmm_status_string(status: int) -> str:
    return B.lib().gmm_status_string(status).decode()


def last_launch_count() -> int:
    return int(B.lib().gmm_last_launch_count())


def gmm_quantize_rhs(w: torch.Tensor, transpose_out: bool = False):
    """W [G, K, N] bf16 -> (codes uint8 [G, K, N] or [G, N, K], scales fp32 [G, N])."""
    G, K, N = w.shape
    codes = torch.empty((G, N, K) if transpose_out else (G, K, N), dtype=torch.uint8, device=w.device)
    scales = torch.empty((G, N), dtype=torch.float32, device=w.device)
    st = B.lib().gmm_quantize_rhs(_dev(w, "w", torch.bfloat16), G, K, N, int(transpose_out), codes.data_ptr(),
                                  scales.data_ptr(), _stream(w))
    _check(st, "gmm_quantize_rhs")
    return codes, scales


def gmm_quantize(x: torch.Tensor, rule="dynamic", axis: int = 1, static_scale: torch.Tensor | None = None,
                 group_sizes: torch.Tensor | None = None, col_scale: torch.Tensor | None = None,
                 ws: torch.Tensor | None = None):
    """Quantize x [rows, cols] bf16; see gmm_quantize in include/gmm_fp8.h for
    the layouts.  Returns (codes, scales)."""
    rows, cols = x.shape
    G = int(group_sizes.numel()) if group_sizes is not None else 1
    r = _rule(rule)
    if axis == 1:
        codes = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
        scales = torch.empty((cols // 128, rows), dtype=torch.float32, device=x.device)
    else:
        cap = gmm_chunk_capacity(rows, G)
        codes = torch.empty((cap, cols, 128), dtype=torch.uint8, device=x.device)
        scales = torch.empty((cap, cols), dtype=torch.float32, device=x.device)
    nbytes = gmm_workspace_bytes(B.OP_FWD, rows, cols, cols, G)
    if ws is None:
        ws = workspace(nbytes, x.device)
    st = B.lib().gmm_quantize(
        _dev(x, "x", torch.bfloat16), rows, cols, r, axis,
        _dev(static_scale, "static_scale", torch.float32) if static_scale is not None else None,
        _dev(group_sizes, "group_sizes", torch.int32) if group_sizes is not None else None, G,
        _dev(col_scale, "col_scale", torch.float32) if col_scale is not None else None,
        codes.data_ptr(), scales.data_ptr(), ws.data_ptr(), ws.numel(), _stream(x))
    _check(st, "gmm_quantize")
    return codes, scales


def _operand(data, dtype_code, scale, rule):
    return B.Operand(data, dtype_code, scale, rule)


def _rhs_operand(rhs, rhs_scales):
    """rhs with its scales: 2-D scales [G, N] are per channel (rule NONE), 3-D
    scales block-wise (rule DYNAMIC, from gmm_quantize_rhs_blocks)."""
    blockwise = rhs_scales is not None and rhs_scales.dim() == 3
    return _operand(_dev(rhs, "rhs"), _TORCH_DT[rhs.dtype],
                    _dev(rhs_scales, "rhs_scales", torch.float32) if rhs_scales is not None else None,
                    B.Q_DYNAMIC if blockwise else B.Q_NONE)


def gmm_quantize_rhs_blocks(w: torch.Tensor, axis: int = 0):
    """W [G, K, N] bf16 -> (codes uint8 [G, K, N], block-wise scales fp32):
    axis 0 [G, K/128, N] for gmm_fwd, axis 1 [G, N/128, K] for gmm_dlhs."""
    G, K, N = w.shape
    codes = torch.empty((G, K, N), dtype=torch.uint8, device=w.device)
    scales = torch.empty((G, K // 128, N) if axis == 0 else (G, N // 128, K), dtype=torch.float32, device=w.device)
    st = B.lib().gmm_quantize_rhs_blocks(_dev(w, "w", torch.bfloat16), G, K, N, int(axis), codes.data_ptr(),
                                         scales.data_ptr(), _stream(w))
    _check(st, "gmm_quantize_rhs_blocks")
    return codes, scales


def gmm_fwd(lhs: torch.Tensor, rhs: torch.Tensor, rhs_scales: torch.Tensor | None, group_sizes: torch.Tensor,
            rule="static", static_scale: torch.Tensor | None = None, transpose_rhs: bool = False,
            out_dtype=torch.bfloat16, out: torch.Tensor | None = None, ws: torch.Tensor | None = None,
            lhs_scales: torch.Tensor | None = None):
    """Forward gmm: out[m] = lhs[m] @ rhs[g(m)] with lhs quantized inside the
    call (rule "static" with ``static_scale``, or "dynamic"); rule "none"
    runs the bf16 family (rhs bf16, no scales).  A uint8 / float8 ``lhs`` is
    taken as already-quantized E4M3 codes: its scale is ``static_scale``
    (static) or ``lhs_scales`` [K/128, M] (dynamic, as gmm_quantize writes)."""
    return _fwd(lhs, rhs, rhs_scales, group_sizes, rule, static_scale, transpose_rhs, out_dtype, out, ws,
                lhs_scales, swiglu=False)


def gmm_fwd_keep_lhs(lhs: torch.Tensor, rhs: torch.Tensor, rhs_scales: torch.Tensor | None,
                     group_sizes: torch.Tensor, rule="static", static_scale: torch.Tensor | None = None,
                     transpose_rhs: bool = False, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                     ws: torch.Tensor | None = None, lhs_codes: torch.Tensor | None = None,
                     lhs_scales: torch.Tensor | None = None):
    """gmm_fwd that also returns the E4M3 codes [M, K] (and, for the dynamic
    rule, the block scales [K/128, M]) it made for lhs: (out, codes, scales),
    written into ``lhs_codes`` / ``lhs_scales`` when given.
    With the static rule the codes can be passed as the lhs of tgmm_drhs /
    gmm_backward, which then skip their own quantization of lhs."""
    M, K = lhs.shape
    G, K2, N = (rhs.shape[0], rhs.shape[2], rhs.shape[1]) if transpose_rhs else rhs.shape
    assert K2 == K, "lhs / rhs contraction mismatch"
    r = _rule(rule)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=lhs.device)
    if ws is None:
        ws = workspace(gmm_workspace_bytes(B.OP_FWD, M, K, N, G), lhs.device)
    codes = lhs_codes if lhs_codes is not None else torch.empty((M, K), dtype=torch.uint8, device=lhs.device)
    scales = None
    if r == B.Q_DYNAMIC:
        scales = lhs_scales if lhs_scales is not None else torch.empty((K // 128, M), dtype=torch.float32,
                                                                         device=lhs.device)
    a = _operand(_dev(lhs, "lhs", torch.bfloat16), B.DT_BF16,
                 _dev(static_scale, "static_scale", torch.float32) if static_scale is not None else None, r)
    st = B.lib().gmm_fwd_keep_lhs(a, _rhs_operand(rhs, rhs_scales), int(transpose_rhs),
                                  _dev(group_sizes, "group_sizes", torch.int32), G, M, K, N,
                                  _dev(out, "out", (torch.bfloat16, torch.float32)), _TORCH_DT[out.dtype],
                                  ws.data_ptr(), ws.numel(), _dev(codes, "lhs_codes", torch.uint8),
                                  _dev(scales, "lhs_scales", torch.float32) if scales is not None else None,
                                  _stream(lhs))
    _check(st, "gmm_fwd_keep_lhs")
    return out, codes, scales


def gmm_fwd_swiglu(lhs: torch.Tensor, rhs: torch.Tensor, rhs_scales: torch.Tensor | None,
                   group_sizes: torch.Tensor, rule="static", static_scale: torch.Tensor | None = None,
                   transpose_rhs: bool = False, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                   ws: torch.Tensor | None = None, lhs_scales: torch.Tensor | None = None):
    """Merged gate|up forward with SwiGLU fused: rhs is [W0 | W1] along N
    (N = 2F); returns out[M, F] = silu(h[:, :F]) * h[:, F:] with h the merged
    product, which is never written.  Arguments as for gmm_fwd."""
    return _fwd(lhs, rhs, rhs_scales, group_sizes, rule, static_scale, transpose_rhs, out_dtype, out, ws,
                lhs_scales, swiglu=True)


def _fwd(lhs, rhs, rhs_scales, group_sizes, rule, static_scale, transpose_rhs, out_dtype, out, ws, lhs_scales,
         swiglu):
    M, K = lhs.shape
    if transpose_rhs:
        G, N, K2 = rhs.shape
    else:
        G, K2, N = rhs.shape
    assert K2 == K, "lhs / rhs contraction mismatch"
    r = _rule(rule)
    if out is None:
        out = torch.empty((M, N // 2 if swiglu else N), dtype=out_dtype, device=lhs.device)
    if ws is None:
        ws = workspace(gmm_workspace_bytes(B.OP_FWD, M, K, N, G), lhs.device)
    if lhs.dtype in (torch.uint8, torch.float8_e4m3fn):
        sc = static_scale if r == B.Q_STATIC else lhs_scales
        a = _operand(_dev(lhs, "lhs"), B.DT_E4M3, _dev(sc, "lhs scale", torch.float32) if sc is not None else None, r)
    else:
        a = _operand(_dev(lhs, "lhs", torch.bfloat16), B.DT_BF16,
                     _dev(static_scale, "static_scale", torch.float32) if static_scale is not None else None, r)
    b = _rhs_operand(rhs, rhs_scales)
    fn = B.lib().gmm_fwd_swiglu if swiglu else B.lib().gmm_fwd
    st = fn(a, b, int(transpose_rhs), _dev(group_sizes, "group_sizes", torch.int32), G, M, K, N,
            _dev(out, "out", (torch.bfloat16, torch.float32)), _TORCH_DT[out.dtype], ws.data_ptr(),
            ws.numel(), _stream(lhs))
    _check(st, "gmm_fwd_swiglu" if swiglu else "gmm_fwd")
    return out


def gmm_dlhs(dout: torch.Tensor, rhs: torch.Tensor, rhs_scales: torch.Tensor | None, group_sizes: torch.Tensor,
             transpose_rhs: bool = False, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
             ws: torch.Tensor | None = None, rule="dynamic"):
    """Backward gmm wrt lhs: dlhs[m] = dout[m] @ rhs[g(m)]^T, dout quantized
    with dynamic 128-blocks after folding the rhs column scale in."""
    M, N = dout.shape
    if transpose_rhs:
        G, N2, K = rhs.shape
    else:
        G, K, N2 = rhs.shape
    assert N2 == N, "dout / rhs mismatch"
    r = _rule(rule)
    if out is None:
        out = torch.empty((M, K), dtype=out_dtype, device=dout.device)
    if ws is None:
        ws = workspace(gmm_workspace_bytes(B.OP_DLHS, M, K, N, G), dout.device)
    a = _operand(_dev(dout, "dout", torch.bfloat16), B.DT_BF16, None, r)
    b = _rhs_operand(rhs, rhs_scales)
    st = B.lib().gmm_dlhs(a, b, int(transpose_rhs), _dev(group_sizes, "group_sizes", torch.int32), G, M, K, N,
                          _dev(out, "out", (torch.bfloat16, torch.float32)), _TORCH_DT[out.dtype], ws.data_ptr(),
                          ws.numel(), _stream(dout))
    _check(st, "gmm_dlhs")
    return out


def tgmm_drhs(lhs: torch.Tensor, dout: torch.Tensor, group_sizes: torch.Tensor, rule="static",
              static_scale: torch.Tensor | None = None, out_dtype=torch.float32, out: torch.Tensor | None = None,
              ws: torch.Tensor | None = None):
    """Weight gradient dW[g] = lhs[rows of g]^T @ dout[rows of g] ([G, K, N]),
    both operands quantized per 128-row chunk of each group.  With rule
    "static" a uint8 / float8 ``lhs`` is taken as the forward's E4M3 codes
    (scale ``static_scale``) and only re-laid out."""
    M, K = lhs.shape
    M2, N = dout.shape
    assert M2 == M
    G = int(group_sizes.numel())
    r = _rule(rule)
    if out is None:
        out = torch.empty((G, K, N), dtype=out_dtype, device=lhs.device)
    if ws is None:
        ws = workspace(gmm_workspace_bytes(B.OP_DRHS, M, K, N, G), lhs.device)
    sc = _dev(static_scale, "static_scale", torch.float32) if static_scale is not None else None
    if lhs.dtype in (torch.uint8, torch.float8_e4m3fn):
        a = _operand(_dev(lhs, "lhs"), B.DT_E4M3, sc, r)
    else:
        a = _operand(_dev(lhs, "lhs", torch.bfloat16), B.DT_BF16, sc, r)
    d = _operand(_dev(dout, "dout", torch.bfloat16), B.DT_BF16, None, B.Q_NONE if r == B.Q_NONE else B.Q_DYNAMIC)
    st = B.lib().tgmm_drhs(a, d, _dev(group_sizes, "group_sizes", torch.int32), G, M, K, N,
                           _dev(out, "out", (torch.bfloat16, torch.float32)), _TORCH_DT[out.dtype], ws.data_ptr(),
                           ws.numel(), _stream(lhs))
    _check(st, "tgmm_drhs")
    return out


def gmm_backward(lhs: torch.Tensor, dout: torch.Tensor, rhs: torch.Tensor, rhs_scales: torch.Tensor | None,
                 group_sizes: torch.Tensor, rule="static", static_scale: torch.Tensor | None = None,
                 transpose_rhs: bool = False, dlhs_dtype=torch.bfloat16, drhs_dtype=torch.float32,
                 dlhs: torch.Tensor | None = None, drhs: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """Both backward passes in one call (dout read once): returns (dlhs [M, K],
    dW [G, K, N]) equal bit for bit to gmm_dlhs and tgmm_drhs.  ``rule`` and
    ``static_scale`` describe lhs as for tgmm_drhs ("none": bf16 family)."""
    M, K = lhs.shape
    M2, N = dout.shape
    assert M2 == M
    G = int(group_sizes.numel())
    r = _rule(rule)
    if dlhs is None:
        dlhs = torch.empty((M, K), dtype=dlhs_dtype, device=lhs.device)
    if drhs is None:
        drhs = torch.empty((G, K, N), dtype=drhs_dtype, device=lhs.device)
    if ws is None:
        ws = workspace(gmm_workspace_bytes(B.OP_BWD, M, K, N, G), lhs.device)
    sc = _dev(static_scale, "static_scale", torch.float32) if static_scale is not None else None
    if lhs.dtype in (torch.uint8, torch.float8_e4m3fn):
        a = _operand(_dev(lhs, "lhs"), B.DT_E4M3, sc, r)
    else:
        a = _operand(_dev(lhs, "lhs", torch.bfloat16), B.DT_BF16, sc, r)
    d = _operand(_dev(dout, "dout", torch.bfloat16), B.DT_BF16, None, B.Q_NONE if r == B.Q_NONE else B.Q_DYNAMIC)
    b = _rhs_operand(rhs, rhs_scales)
    st = B.lib().gmm_backward(a, d, b, int(transpose_rhs), _dev(group_sizes, "group_sizes", torch.int32), G, M, K, N,
                              _dev(dlhs, "dlhs", (torch.bfloat16, torch.float32)), _TORCH_DT[dlhs.dtype],
                              _dev(drhs, "drhs", (torch.bfloat16, torch.float32)), _TORCH_DT[drhs.dtype],
                              ws.data_ptr(), ws.numel(), _stream(lhs))
    _check(st, "gmm_backward")
    return dlhs, drhs


def gmm_read_device_status(ws: torch.Tensor):
    """(status, bits) left in ``ws`` by the last call; synchronizes the stream."""
    bits = ctypes.c_uint32(0)
    st = B.lib().gmm_read_device_status(ws.data_ptr(), ctypes.byref(bits), _stream(ws))
    return st, bits.value


def gmm_selftest_timeout(ws: torch.Tensor, limit_ns: int):
    _check(B.lib().gmm_selftest_timeout(ws.data_ptr(), limit_ns, _stream(ws)), "gmm_selftest_timeout")


def gmm_set_wait_limit_ns(limit_ns: int):
    B.lib().gmm_set_wait_limit_ns(limit_ns)


TILES = {"auto": B.TILES_AUTO, "one_cta": B.TILES_ONE_CTA, "cta_pairs": B.TILES_CTA_PAIRS,
         "cta_pairs_narrow": B.TILES_CTA_PAIRS_NARROW}


def gmm_set_tiles(mode="auto"):
    """GEMM tile choice for the calls that follow: "auto", "one_cta" (128-row
    tiles), "cta_pairs" (256-row tiles over a two-CTA cluster) or
    "cta_pairs_narrow" (CTA pairs; 256 x 128 tiles for the promoted passes
    with K-major weights)."""
    _check(B.lib().gmm_set_tiles(TILES[mode] if isinstance(mode, str) else int(mode)), "gmm_set_tiles")


def gmm_plan(group_sizes: torch.Tensor, M: int):
    """Host-side helper (no kernel): clamped row offsets of the groups, as
    int64 CPU tensor [G + 1] (same rule as the device plan)."""
    gs = group_sizes.detach().to("cpu", torch.int64).clamp(min=0)
    offs = torch.zeros(gs.numel() + 1, dtype=torch.int64)
    offs[1:] = torch.cumsum(gs, 0).clamp(max=M)
    return offs


def profile_enable(on: bool = True):
    """Bracket every library kernel launch with CUDA events (benchmarks)."""
    B.lib().gmm_profile_enable(int(on))


def profile_collect() -> dict:
    """{kernel name: (launches, total ms)} since the last collect."""
    arr = (B.ProfileEntry * 32)()
    n = B.lib().gmm_profile_collect(arr, 32)
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(n)}
