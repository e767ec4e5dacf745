"""Pins for the oracle's block-wise rhs scales (one scale per 128-block of the
weights along a contraction axis) and the forward / dlhs that use them.

The quantizer is checked against the per-channel quantizer (weights whose
blocks share their column's absolute maximum give the same codes and
scales), against closed forms (a block's largest element maps to +-448, an
all-zero block to scale 0), against its own other axis on the transposed
weights, and against the E4M3 rounding bound.  The passes are checked against
a numpy matmul of the dequantized operands per group, and against the exact
bf16 product within the FP8 quantization error.

Source: "Support quantization for tokamax gmm v2" (maxtext PR #4451), review
thread on the rhs scale: a 2-D scale is per channel, a 3-D one block-wise.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_fp8_grouped_b200 import synth

QS, QD = oracle.Q_STATIC, oracle.Q_DYNAMIC


def dec(c):
    return oracle.e4m3_decode(c)


def f64(t):
    return t.double().numpy()


def expand_k(srb, K):
    """[G, K/128, N] -> [G, K, N]"""
    return np.repeat(srb.astype(np.float64), 128, axis=1)[:, :K]


def expand_n(srb, N):
    """[G, N/128, K] -> [G, K, N]"""
    return np.repeat(srb.astype(np.float64), 128, axis=1).transpose(0, 2, 1)[:, :, :N]


def test_blocks_sharing_the_column_max_reduce_to_per_channel():
    g = torch.Generator().manual_seed(3)
    w = (torch.randn(2, 384, 256, generator=g) * 0.02).bfloat16()
    cmax = w.float().abs().amax(dim=1, keepdim=True)  # [G, 1, N]
    for kb in range(3):  # plant the column maximum in every block
        w[:, kb * 128 + 5, :] = cmax[:, 0, :].bfloat16()
    qb, sb = oracle.quantize_rhs_blocks(w, 0)
    qc, sc = oracle.quantize_rhs(w)
    assert np.array_equal(qb, qc)
    assert np.array_equal(sb, np.repeat(sc[:, None, :], 3, axis=1))


@pytest.mark.parametrize("axis", [0, 1])
def test_block_max_maps_to_448_and_zero_blocks(axis):
    g = torch.Generator().manual_seed(4)
    w = (torch.randn(2, 256, 384, generator=g) * 0.05).bfloat16()
    w[1, :128, :] = 0  # all-zero blocks along K (axis 0) / rows whose n-blocks are all zero (axis 1)
    q, s = oracle.quantize_rhs_blocks(w, axis)
    wf = f64(w)
    G, K, N = wf.shape
    if axis == 0:
        blocks = wf.reshape(G, K // 128, 128, N)
        codes = q.reshape(G, K // 128, 128, N)
        arg = np.abs(blocks).argmax(axis=2)
        top = np.take_along_axis(codes, arg[:, :, None, :], axis=2)[:, :, 0, :]
        assert np.array_equal(s, (np.abs(blocks).max(axis=2) / np.float32(448)).astype(np.float32))
        zero = s[1, 0] == 0
        assert zero.all() and not codes[1, 0].any()
    else:
        blocks = wf.reshape(G, K, N // 128, 128)
        codes = q.reshape(G, K, N // 128, 128)
        arg = np.abs(blocks).argmax(axis=3)
        top = np.take_along_axis(codes, arg[..., None], axis=3)[..., 0].transpose(0, 2, 1)
        assert (s[1, :, :128] == 0).all() and not codes[1, :128].any()
    nz = s > 0
    assert np.all(np.abs(dec(top[nz])) == 448.0)


def test_axis1_is_axis0_of_the_transposed_weights():
    g = torch.Generator().manual_seed(5)
    w = (torch.randn(3, 256, 384, generator=g) * 0.02).bfloat16()
    q1, s1 = oracle.quantize_rhs_blocks(w, 1)
    qt, st = oracle.quantize_rhs_blocks(w.transpose(1, 2).contiguous(), 0)
    assert np.array_equal(s1, st)
    assert np.array_equal(q1, qt.transpose(0, 2, 1))


@pytest.mark.parametrize("axis", [0, 1])
def test_roundtrip_within_e4m3_rounding(axis):
    g = torch.Generator().manual_seed(6)
    w = (torch.randn(2, 256, 256, generator=g) * 0.02).bfloat16()
    q, s = oracle.quantize_rhs_blocks(w, axis)
    sx = expand_k(s, 256) if axis == 0 else expand_n(s, 256)
    err = np.abs(dec(q) * sx - f64(w))
    # half an E4M3 ulp: 2^-4 relative for normals, 2^-10 * scale below 2^-6 * scale
    assert np.all(err <= 2.0 ** -4 * np.abs(f64(w)) * (1 + 1e-6) + 2.0 ** -10 * sx)


CASES = [(4, 200, 256, 384, [60, 0, 100, 30]), (1, 130, 384, 256, None)]


@pytest.mark.parametrize("G,M,K,N,sizes", CASES)
@pytest.mark.parametrize("rule", [QS, QD])
def test_fwd_blockwise_matches_numpy_matmul(G, M, K, N, sizes, rule):
    inp = synth.small_case(G, M, K, N, seed=21, sizes=sizes)
    q, sb = oracle.quantize_rhs_blocks(inp.w, 0)
    ql, sl, _ = oracle.quantize_rows(inp.lhs, rule, inp.static_scale)
    xl = dec(ql) * np.repeat(sl.astype(np.float64), 128, axis=1)
    wt = dec(q) * expand_k(sb, K)
    offs = oracle.plan(inp.group_sizes, M)[0]
    ref = np.zeros((M, N))
    for g in range(G):
        ref[offs[g]:offs[g + 1]] = xl[offs[g]:offs[g + 1]] @ wt[g]
    out, ab = oracle.gmm_fwd_blockwise(inp.lhs, rule, inp.static_scale, q, sb, inp.group_sizes)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * ab.max())
    assert np.all(ab >= np.abs(out) * (1 - 1e-12))
    # rows past the groups are zero; an empty group's rows do not exist
    assert not out[int(offs[-1]):].any()


def test_fwd_blockwise_equals_per_channel_when_blocks_agree():
    inp = synth.small_case(2, 150, 256, 256, seed=22, sizes=[70, 80])
    w = inp.w.clone()
    cmax = w.float().abs().amax(dim=1)
    w[:, 3, :] = cmax.bfloat16()
    w[:, 131, :] = cmax.bfloat16()
    qb, sb = oracle.quantize_rhs_blocks(w, 0)
    qc, sc = oracle.quantize_rhs(w)
    for rule in (QS, QD):
        a, _ = oracle.gmm_fwd_blockwise(inp.lhs, rule, inp.static_scale, qb, sb, inp.group_sizes)
        b, ab = oracle.gmm_fwd(inp.lhs, rule, inp.static_scale, qc, sc, inp.group_sizes)
        assert np.allclose(a, b, rtol=1e-13, atol=1e-13 * ab.max())


@pytest.mark.parametrize("G,M,K,N,sizes", CASES)
def test_dlhs_blockwise_matches_numpy_matmul(G, M, K, N, sizes):
    inp = synth.small_case(G, M, K, N, seed=23, sizes=sizes)
    q, sb = oracle.quantize_rhs_blocks(inp.w, 1)
    qd, sd, _ = oracle.quantize_rows(inp.dout, QD)
    dd = dec(qd) * np.repeat(sd.astype(np.float64), 128, axis=1)
    wt = dec(q) * expand_n(sb, N)  # [G, K, N]
    offs = oracle.plan(inp.group_sizes, M)[0]
    ref = np.zeros((M, K))
    for g in range(G):
        ref[offs[g]:offs[g + 1]] = dd[offs[g]:offs[g + 1]] @ wt[g].T
    out, ab = oracle.gmm_dlhs_blockwise(inp.dout, q, sb, inp.group_sizes)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * ab.max())
    assert not out[int(offs[-1]):].any()


def test_blockwise_passes_track_the_exact_product():
    """Both passes stay within the FP8 error of the exact bf16 products:
    each operand carries at most half an E4M3 ulp (2^-4 relative) plus its
    subnormal floor, so |err| <= ~2^-3 * sum |a| |b| (checked with slack)."""
    inp = synth.small_case(2, 256, 256, 384, seed=24, sizes=[100, 156])
    offs = oracle.plan(inp.group_sizes, 256)[0]
    x, d, w = f64(inp.lhs), f64(inp.dout), f64(inp.w)
    q0, s0 = oracle.quantize_rhs_blocks(inp.w, 0)
    q1, s1 = oracle.quantize_rhs_blocks(inp.w, 1)
    f, _ = oracle.gmm_fwd_blockwise(inp.lhs, QD, 0.0, q0, s0, inp.group_sizes)
    dl, _ = oracle.gmm_dlhs_blockwise(inp.dout, q1, s1, inp.group_sizes)
    for g in range(2):
        r = slice(offs[g], offs[g + 1])
        assert np.all(np.abs(f[r] - x[r] @ w[g]) <= 0.14 * (np.abs(x[r]) @ np.abs(w[g])) + 1e-9)
        assert np.all(np.abs(dl[r] - d[r] @ w[g].T) <= 0.14 * (np.abs(d[r]) @ np.abs(w[g]).T) + 1e-9)
