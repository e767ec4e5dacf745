"""Pins for the oracle's forward gmm, dlhs gmm and tgmm drhs.

Each pass is checked against routes that do not go through its own loops:
numpy fp64 matmul of the dequantized operands per group (a library
primitive), the G=1 case as one ordinary GEMM, the rules for empty groups and
unrouted rows, the merged gate|up identity, and torch.autograd of the fp64
dequantized forward (the analogue of the pages' value-and-gradient
equivalence test).

Sources: "Support quantization for tokamax gmm v2" (maxtext PR #4451),
Description (fwd gmm, dlhs gmm, drhs tgmm; value and gradient equivalence
test) and review thread on ops.py (dlhs is a gmm with transpose_rhs flipped);
"FP8 Megablox for batch split" (maxtext PR #3770), Description (merged W0|W1
gating doubles the local N).
"""
import numpy as np
import pytest
import torch

import oracle
from moe_fp8_grouped_b200 import synth

QS, QD = oracle.Q_STATIC, oracle.Q_DYNAMIC


def dec(c):
    return oracle.e4m3_decode(c)


def deq_rows(codes, scales):
    return dec(codes) * np.repeat(scales.astype(np.float64), 128, axis=1)


def offsets(sizes, M):
    return oracle.plan(sizes, M)[0]


def ref_fwd(inp, rule, s):
    """Per-group numpy matmul of dequantized lhs and rhs."""
    qr, sr = oracle.quantize_rhs(inp.w)
    ql, sl, _ = oracle.quantize_rows(inp.lhs, rule, s)
    xl = deq_rows(ql, sl)
    wt = dec(qr) * sr[:, None, :].astype(np.float64)
    M, N = inp.lhs.shape[0], inp.w.shape[2]
    out = np.zeros((M, N))
    offs = offsets(inp.group_sizes, M)
    for g in range(inp.w.shape[0]):
        a, b = offs[g], offs[g + 1]
        out[a:b] = xl[a:b] @ wt[g]
    return out, (qr, sr)


CASES = [
    # G, M, K, N, sizes
    (4, 200, 256, 384, [60, 0, 100, 40]),
    (3, 300, 512, 256, [1, 128, 150]),  # sums to 279: 21 unrouted rows
    (1, 130, 384, 128, None),
]


@pytest.mark.parametrize("G,M,K,N,sizes", CASES)
@pytest.mark.parametrize("rule", [QS, QD])
def test_fwd_matches_numpy_matmul(G, M, K, N, sizes, rule):
    inp = synth.small_case(G, M, K, N, seed=11, sizes=sizes)
    ref, (qr, sr) = ref_fwd(inp, rule, inp.static_scale)
    out, ab = oracle.gmm_fwd(inp.lhs, rule, inp.static_scale, qr, sr, inp.group_sizes)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * ab.max())
    assert np.all(ab >= np.abs(out) * (1 - 1e-12))


def test_fwd_G1_is_one_gemm_and_rows_subset():
    inp = synth.small_case(1, 96, 256, 128, seed=12, sizes=[96])
    qr, sr = oracle.quantize_rhs(inp.w)
    ql, sl, _ = oracle.quantize_rows(inp.lhs, QD)
    full, _ = oracle.gmm_fwd(inp.lhs, QD, 0.0, qr, sr, inp.group_sizes)
    ref = deq_rows(ql, sl) @ (dec(qr[0]) * sr[0].astype(np.float64))
    assert np.allclose(full, ref, rtol=1e-12, atol=1e-14)
    sub, _ = oracle.gmm_fwd(inp.lhs, QD, 0.0, qr, sr, inp.group_sizes, rows=[5, 77, 0])
    assert np.array_equal(sub, full[[5, 77, 0]])


def test_fwd_empty_group_and_unrouted_rows_are_zero():
    inp = synth.small_case(4, 100, 128, 128, seed=13, sizes=[30, 0, 40, 20])
    qr, sr = oracle.quantize_rhs(inp.w)
    out, ab = oracle.gmm_fwd(inp.lhs, QS, inp.static_scale, qr, sr, inp.group_sizes)
    assert np.all(out[90:] == 0) and np.all(ab[90:] == 0)
    assert np.all(np.any(out[:90] != 0, axis=1))


def test_fwd_sizes_past_M_are_clamped():
    inp = synth.small_case(3, 50, 128, 128, seed=14, sizes=[20, 40, 30])
    qr, sr = oracle.quantize_rhs(inp.w)
    out, _ = oracle.gmm_fwd(inp.lhs, QS, inp.static_scale, qr, sr, inp.group_sizes)
    inp2 = synth.small_case(3, 50, 128, 128, seed=14, sizes=[20, 30, 0])
    out2, _ = oracle.gmm_fwd(inp2.lhs, QS, inp.static_scale, qr, sr, inp2.group_sizes)
    assert np.array_equal(out, out2)


def ref_dlhs(inp):
    qr, sr = oracle.quantize_rhs(inp.w)
    qt, st = oracle.quantize_rows_scaled(inp.dout, sr, inp.group_sizes)
    t = deq_rows(qt, st)
    M, K = inp.lhs.shape
    out = np.zeros((M, K))
    offs = offsets(inp.group_sizes, M)
    for g in range(inp.w.shape[0]):
        a, b = offs[g], offs[g + 1]
        out[a:b] = t[a:b] @ dec(qr[g]).T  # the same codes with the transposed role
    return out, (qr, sr)


@pytest.mark.parametrize("G,M,K,N,sizes", CASES)
def test_dlhs_matches_numpy_matmul(G, M, K, N, sizes):
    inp = synth.small_case(G, M, K, N, seed=21, sizes=sizes)
    ref, (qr, sr) = ref_dlhs(inp)
    out, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * ab.max())


def ref_drhs(inp, rule, s):
    M, K = inp.lhs.shape
    N = inp.dout.shape[1]
    G = inp.w.shape[0]
    qx, sx = oracle.quantize_chunks(inp.lhs, rule, s, inp.group_sizes)
    qd, sd = oracle.quantize_chunks(inp.dout, QD, 0.0, inp.group_sizes)
    offs = offsets(inp.group_sizes, M)
    out = np.zeros((G, K, N))
    c = 0
    for g in range(G):
        for a in range(offs[g], offs[g + 1], 128):
            b = min(a + 128, offs[g + 1])
            xa = dec(qx[a:b]) * sx[c].astype(np.float64)
            da = dec(qd[a:b]) * sd[c].astype(np.float64)
            out[g] += xa.T @ da
            c += 1
    return out


@pytest.mark.parametrize("G,M,K,N,sizes", CASES)
@pytest.mark.parametrize("rule", [QS, QD])
def test_drhs_matches_numpy_matmul(G, M, K, N, sizes, rule):
    inp = synth.small_case(G, M, K, N, seed=31, sizes=sizes)
    ref = ref_drhs(inp, rule, inp.static_scale)
    out, ab = oracle.tgmm_drhs(inp.lhs, rule, inp.static_scale, inp.dout, inp.group_sizes)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * ab.max())


def test_drhs_empty_group_is_zero_and_selection():
    inp = synth.small_case(4, 100, 128, 256, seed=32, sizes=[30, 0, 60, 0])
    out, ab = oracle.tgmm_drhs(inp.lhs, QD, 0.0, inp.dout, inp.group_sizes)
    assert np.all(out[1] == 0) and np.all(out[3] == 0) and np.all(ab[1] == 0)
    assert np.any(out[0] != 0) and np.any(out[2] != 0)
    sel = [2 * 128 + 5, 0 * 128 + 127, 1 * 128 + 3]
    sub, _ = oracle.tgmm_drhs(inp.lhs, QD, 0.0, inp.dout, inp.group_sizes, sel=sel)
    assert np.array_equal(sub, out.reshape(-1, 256)[sel])


def test_merged_gate_up_identity():
    """W = W0 | W1 along N: fwd and drhs split exactly into the two separate
    calls; dlhs is the sum of the two separate dlhs calls."""
    inp = synth.small_case(3, 120, 256, 512, seed=41, sizes=[50, 0, 70])
    w0, w1 = inp.w[:, :, :256].contiguous(), inp.w[:, :, 256:].contiguous()
    d0, d1 = inp.dout[:, :256].contiguous(), inp.dout[:, 256:].contiguous()
    qr, sr = oracle.quantize_rhs(inp.w)
    q0, s0 = oracle.quantize_rhs(w0)
    q1, s1 = oracle.quantize_rhs(w1)
    assert np.array_equal(qr, np.concatenate([q0, q1], axis=2))
    for rule in (QS, QD):
        f, _ = oracle.gmm_fwd(inp.lhs, rule, inp.static_scale, qr, sr, inp.group_sizes)
        f0, _ = oracle.gmm_fwd(inp.lhs, rule, inp.static_scale, q0, s0, inp.group_sizes)
        f1, _ = oracle.gmm_fwd(inp.lhs, rule, inp.static_scale, q1, s1, inp.group_sizes)
        assert np.array_equal(f, np.concatenate([f0, f1], axis=1))
        r, _ = oracle.tgmm_drhs(inp.lhs, rule, inp.static_scale, inp.dout, inp.group_sizes)
        r0, _ = oracle.tgmm_drhs(inp.lhs, rule, inp.static_scale, d0, inp.group_sizes)
        r1, _ = oracle.tgmm_drhs(inp.lhs, rule, inp.static_scale, d1, inp.group_sizes)
        assert np.array_equal(r, np.concatenate([r0, r1], axis=2))
    dl, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
    dl0, _ = oracle.gmm_dlhs(d0, q0, s0, inp.group_sizes)
    dl1, _ = oracle.gmm_dlhs(d1, q1, s1, inp.group_sizes)
    assert np.allclose(dl, dl0 + dl1, rtol=0, atol=1e-13 * ab.max())


@pytest.mark.parametrize("rule", [QS, QD])
def test_gradients_match_autograd_of_dequantized_forward(rule):
    """dlhs and drhs equal the autograd gradients of y = x~ @ W~[g] (fp64,
    dequantized operands) up to the E4M3 rounding of the gradient operands:
    half a spacing, 2^-4 relative in the normal range."""
    inp = synth.small_case(3, 160, 256, 256, seed=51, sizes=[70, 10, 60])
    M, K = inp.lhs.shape
    qr, sr = oracle.quantize_rhs(inp.w)
    ql, sl, _ = oracle.quantize_rows(inp.lhs, rule, inp.static_scale)
    x = torch.tensor(deq_rows(ql, sl), requires_grad=True)
    W = torch.tensor(dec(qr) * sr[:, None, :].astype(np.float64), requires_grad=True)
    offs = offsets(inp.group_sizes, M)
    ys = [x[offs[g]:offs[g + 1]] @ W[g] for g in range(3)]
    y = torch.cat(ys + [torch.zeros(M - offs[3], W.shape[2], dtype=torch.float64)])
    dout = torch.tensor(inp.dout.to(torch.float32).numpy().astype(np.float64))
    y.backward(dout)

    dl, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
    gx = x.grad.numpy()
    assert np.all(np.abs(dl - gx) <= 2.0 ** -4 * ab * 1.001 + 1e-9)
    assert np.abs(dl - gx).max() > 0  # the gradient really was quantized

    dw, abw = oracle.tgmm_drhs(inp.lhs, rule, inp.static_scale, inp.dout, inp.group_sizes)
    gw = W.grad.numpy()
    if rule == QS:
        # x codes are the forward codes: only dout's rounding separates them
        assert np.all(np.abs(dw - gw) <= 2.0 ** -4 * abw * 1.001 + 1e-9)
    else:
        # x is re-quantized per 128-row chunk: both operands carry rounding
        assert np.all(np.abs(dw - gw) <= (2.0 ** -4 + 2.0 ** -4 + 2.0 ** -3) * abw * 1.001 + 1e-9)
