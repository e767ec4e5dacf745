"""Shared helpers for the GPU parity tests (CUDA path vs the CPU oracle).

Tolerance: an output element may differ from the oracle by at most
2e-3 * A, where A = sum_k |a_k * b_k| over the dequantized terms of that
element (the oracle's absum).  A bf16 output additionally carries its own
round-to-nearest error, up to 2^-8 of the value.
"""
import numpy as np
import torch

import oracle

TOL = 2e-3


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(gpu: torch.Tensor, ref: np.ndarray, absum: np.ndarray, what: str = ""):
    g = to_np(gpu).reshape(ref.shape)
    bound = TOL * absum + (2.0 ** -8 * np.abs(ref) if gpu.dtype == torch.bfloat16 else 0.0)
    err = np.abs(g - ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        worst = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside 2e-3*A; first {idx.tolist()}; "
            f"worst at {worst}: gpu={g[worst]!r} ref={ref[worst]!r} A={absum[worst]!r}")
    return float((err / np.maximum(absum, 1e-300)).max())


def rule_code(rule: str) -> int:
    return {"static": oracle.Q_STATIC, "dynamic": oracle.Q_DYNAMIC}[rule]


def untranspose_chunks(codes_t: torch.Tensor, scales: torch.Tensor, offs: np.ndarray, M: int):
    """GPU axis-0 layout (codes [cap, C, 128] chunk-major, scales [cap, C]) ->
    the oracle's (codes [M, C] in row order, scales [num_chunks, C])."""
    ct = codes_t.cpu().numpy()
    sc = scales.cpu().numpy()
    C = ct.shape[1]
    out = np.zeros((M, C), dtype=np.uint8)
    j = 0
    for g in range(len(offs) - 1):
        for a in range(int(offs[g]), int(offs[g + 1]), 128):
            b = min(a + 128, int(offs[g + 1]))
            out[a:b] = ct[j, :, :b - a].T
            # pad rows of the chunk must be zero codes
            assert not ct[j, :, b - a:].any(), "chunk padding not zero"
            j += 1
    return out, sc[:j]


def guarded(shape, dtype, device="cuda", fill=0x5A):
    """A tensor view with 4 KiB guard bands on both sides filled with a
    canary byte; check_guards() verifies nothing wrote outside the view."""
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    pad = 4096
    raw = torch.full((n + 2 * pad,), fill, dtype=torch.uint8, device=device)
    view = raw[pad: pad + n].view(dtype).view(*shape)
    return raw, view, pad, n


def check_guards(raw: torch.Tensor, pad: int, n: int, fill=0x5A):
    r = raw.cpu()
    assert bool((r[:pad] == fill).all()), "write before the output buffer"
    assert bool((r[pad + n:] == fill).all()), "write past the output buffer"


def swiglu_bound(gpu_dtype, terms, ref, eps: float = TOL):
    """Elementwise bound for out = silu(g) * u when the gate g and the up value
    u each carry the forward's error, |dg| <= eps * A_g and |du| <= eps * A_u:
      |silu(g + dg)(u + du) - silu(g) u|
        <= L eps A_g |u| + (|silu(g)| + L eps A_g) eps A_u,
    with L = max |silu'| (oracle.SILU_LIPSCHITZ).  Added: the output's own
    bf16 rounding (2^-8 |ref|) and 1e-5 |ref| for the fp32 evaluation of silu
    and the product."""
    gate, up, ag, au = terms
    L = oracle.SILU_LIPSCHITZ
    b = L * eps * ag * np.abs(up) + (np.abs(oracle.silu(gate)) + L * eps * ag) * eps * au
    b = b + 1e-5 * np.abs(ref)
    if gpu_dtype == torch.bfloat16:
        b = b + 2.0 ** -8 * np.abs(ref)
    return b


def assert_within(gpu: torch.Tensor, ref: np.ndarray, bound: np.ndarray, what: str = ""):
    g = to_np(gpu).reshape(ref.shape)
    err = np.abs(g - ref)
    bad = ~(err <= bound)  # NaN fails too
    if bad.any():
        worst = np.unravel_index(np.argmax(np.where(np.isnan(err), np.inf, err - bound)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements outside the bound; worst at "
                             f"{worst}: gpu={g[worst]!r} ref={ref[worst]!r} bound={bound[worst]!r}")
