"""Pins for the oracle's SwiGLU of the merged gate|up forward.

silu is checked against closed forms and identities of the logistic function;
the fused result against a per-group numpy matmul of the dequantized operands
followed by the activation, and against two separate gate / up forward calls
(the merged-weights identity).  The tolerance's Lipschitz constant is checked
against the derivative on a fine grid.

Source: "FP8 Megablox for batch split" (maxtext PR #3770), Description (2):
the gate and up projections of the SwiGLU MLP, W0 and W1, concatenated into
one gmm call.
"""
import math

import numpy as np
import pytest

import oracle
from moe_fp8_grouped_b200 import synth

QS, QD = oracle.Q_STATIC, oracle.Q_DYNAMIC


def test_silu_closed_forms():
    # sigmoid(ln 3) = 3/4, sigmoid(0) = 1/2, sigmoid(-ln 3) = 1/4
    l3 = math.log(3.0)
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(l3) - 0.75 * l3) <= 1e-15
    assert abs(oracle.silu(-l3) + 0.25 * l3) <= 1e-15
    # saturation: silu(z) -> z for large z, -> -0 for very negative z
    assert oracle.silu(60.0) == 60.0
    v = oracle.silu(-1000.0)
    assert v == 0.0 and not np.isnan(v)


def test_silu_reflection_identity():
    """sigmoid(-z) = 1 - sigmoid(z) gives silu(-z) = silu(z) - z."""
    z = np.linspace(-30, 30, 6001)
    assert np.allclose(oracle.silu(-z), oracle.silu(z) - z, rtol=0, atol=1e-13)


def test_silu_lipschitz_constant():
    """The tolerance uses L >= max |silu'|; the maximum is about 1.0998."""
    z = np.linspace(-20, 20, 400001)
    s = 1.0 / (1.0 + np.exp(-z))
    d = s * (1.0 + z * (1.0 - s))  # derivative of z * sigmoid(z)
    # the analytic derivative agrees with a central difference of the oracle
    h = 1e-6
    fd = (oracle.silu(z + h) - oracle.silu(z - h)) / (2 * h)
    assert np.allclose(fd, d, atol=1e-8)
    m = np.abs(d).max()
    assert 1.0998 < m <= oracle.SILU_LIPSCHITZ
    assert abs(z[np.argmax(d)] - 2.3994) < 1e-3


def ref_swiglu(inp, rule, s):
    """Per-group numpy matmul of the dequantized operands, then silu(gate) * up."""
    qr, sr = oracle.quantize_rhs(inp.w)
    ql, sl, _ = oracle.quantize_rows(inp.lhs, rule, s)
    xl = oracle.e4m3_decode(ql) * np.repeat(sl.astype(np.float64), 128, axis=1)
    wt = oracle.e4m3_decode(qr) * sr[:, None, :].astype(np.float64)
    M, N = inp.lhs.shape[0], inp.w.shape[2]
    F = N // 2
    offs = oracle.plan(inp.group_sizes, M)[0]
    out = np.zeros((M, F))
    for g in range(inp.w.shape[0]):
        a, b = offs[g], offs[g + 1]
        h = xl[a:b] @ wt[g]
        gate, up = h[:, :F], h[:, F:]
        out[a:b] = gate / (1.0 + np.exp(-gate)) * up
    return out, (qr, sr)


@pytest.mark.parametrize("G,M,K,N,sizes", [(4, 200, 256, 512, [60, 0, 100, 30]), (1, 130, 384, 256, None)])
@pytest.mark.parametrize("rule", [QS, QD])
def test_swiglu_matches_numpy_matmul(G, M, K, N, sizes, rule):
    inp = synth.small_case(G, M, K, N, seed=17, sizes=sizes)
    ref, (qr, sr) = ref_swiglu(inp, rule, inp.static_scale)
    out, (gate, up, ag, au) = oracle.gmm_fwd_swiglu(inp.lhs, rule, inp.static_scale, qr, sr, inp.group_sizes)
    assert out.shape == (M, N // 2)
    scale = (np.abs(gate) * np.abs(up) + ag * au).max()
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * scale)
    # unrouted rows and rows of empty groups are zero
    routed = int(np.sum(inp.group_sizes.numpy()))
    assert not out[routed:].any()


def test_swiglu_equals_separate_gate_and_up_calls():
    inp = synth.small_case(3, 150, 256, 512, seed=43, sizes=[40, 0, 90])
    qr, sr = oracle.quantize_rhs(inp.w)
    q0, s0 = oracle.quantize_rhs(inp.w[:, :, :256].contiguous())
    q1, s1 = oracle.quantize_rhs(inp.w[:, :, 256:].contiguous())
    for rule in (QS, QD):
        out, _ = oracle.gmm_fwd_swiglu(inp.lhs, rule, inp.static_scale, qr, sr, inp.group_sizes)
        g, _ = oracle.gmm_fwd(inp.lhs, rule, inp.static_scale, q0, s0, inp.group_sizes)
        u, _ = oracle.gmm_fwd(inp.lhs, rule, inp.static_scale, q1, s1, inp.group_sizes)
        assert np.array_equal(out, oracle.silu(g) * u)


def test_swiglu_bound_catches_a_dropped_gate_scale():
    """The propagated bound used by the GPU tests is tight enough to reject a
    result whose gate lost its column scale, or one with gate and up swapped
    (plausible epilogue slips)."""
    import torch
    from parity import swiglu_bound
    inp = synth.small_case(2, 256, 256, 512, seed=5, sizes=[128, 128])
    qr, sr = oracle.quantize_rhs(inp.w)
    out, terms = oracle.gmm_fwd_swiglu(inp.lhs, QS, inp.static_scale, qr, sr, inp.group_sizes)
    gate, up, _, _ = terms
    g = np.repeat(np.arange(2), 128)
    wrong = oracle.silu(gate / sr[g, :256]) * up
    bound = swiglu_bound(torch.float32, terms, out)
    assert (np.abs(wrong - out) > bound).mean() > 0.9
    swapped = oracle.silu(up) * gate
    assert (np.abs(swapped - out) > bound).mean() > 0.3  # near 0 silu(z) ~ z/2 is symmetric
