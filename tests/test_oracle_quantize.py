"""Pins for the oracle's quantizers and group plan.

Sources: "add static LHS scaling support for GMM v2 FWD" (maxtext PR #4735),
review threads on the LhsRef docstring (qvalue = clip(lhs / scale), per-tensor
[1, 1] scale) and on inner_kernel (block_scale_inv is 0 where block_scale is
0, lhs * block_scale_inv cast to the fp8 dtype); "FP8 Megablox for batch
split" (maxtext PR #3770), Description (weights quantized manually, per
channel in "Support quantization for tokamax gmm v2", review thread on the
2-D rhs scale).
"""
import numpy as np
import torch

import oracle
from moe_fp8_grouped_b200 import synth


def bf16(a):
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def f32(x):
    return x.to(torch.float32).numpy().astype(np.float64)


def test_block_with_amax_448_has_unit_scale():
    gen = torch.Generator().manual_seed(3)
    x = (torch.rand(2, 128, generator=gen) * 800 - 400).to(torch.bfloat16)
    x[0, 17] = 448.0
    x[1, 5] = -448.0
    codes, scales, _ = oracle.quantize_rows(x, oracle.Q_DYNAMIC)
    assert np.all(scales == 1.0)
    # with s = 1 the codes are the plain E4M3 rounding of x (torch's cast)
    ref = x.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def test_zero_block_gives_zero_scale_and_codes():
    x = torch.zeros(3, 256, dtype=torch.bfloat16)
    x[1, 200] = 1.0  # only the second block of row 1 is nonzero
    codes, scales, _ = oracle.quantize_rows(x, oracle.Q_DYNAMIC)
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and scales[1, 0] == 0 and scales[2, 1] == 0
    assert scales[1, 1] == np.float32(1.0) / np.float32(448.0)
    assert np.count_nonzero(codes) == 1 and codes[1, 200] == 0x7E


def test_static_scale_4_over_448():
    s = np.float32(4.0) / np.float32(448.0)
    x = bf16([[4.0, -4.0, 2.0, 0.0, 8.0, -100.0] + [0.0] * 122])
    codes, scales, flags = oracle.quantize_rows(x, oracle.Q_STATIC, float(s))
    assert flags == 0 and scales[0, 0] == s
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0xFE  # 4 * fl32(1/s) ~ 448
    assert codes[0, 4] == 0x7E and codes[0, 5] == 0xFE  # clipped
    assert oracle.e4m3_decode(codes[0, 2]) == 224.0  # 2 -> ~224 -> exactly 224
    assert codes[0, 3] == 0


def test_invalid_static_scale_flags_and_zeroes():
    x = bf16(np.ones((1, 128)))
    for bad in [0.0, -1.0, float("inf"), float("nan"), 1e-39]:
        codes, scales, flags = oracle.quantize_rows(x, oracle.Q_STATIC, bad)
        assert flags == oracle.FLAG_SCALE
        assert np.all(codes == 0) and np.all(scales == 0)
    assert oracle.static_scale_ok(1e-30) and not oracle.static_scale_ok(1e-39)


def test_scale_whose_inverse_overflows_is_zero():
    tiny = torch.tensor([2.0 ** -133], dtype=torch.float32).to(torch.bfloat16)  # bf16 subnormal
    x = torch.zeros(1, 128, dtype=torch.bfloat16)
    x[0, 0] = tiny
    codes, scales, _ = oracle.quantize_rows(x, oracle.Q_DYNAMIC)
    assert scales[0, 0] == 0.0 and np.all(codes == 0)


def _dequant_error_ok(x, codes, scale):
    """E4M3 rounding error bound: half a spacing, i.e. 2^-4 relative in the
    normal range and 2^-10 absolute (in code units) in the subnormal range,
    plus the fp32 rounding of x * (1/s)."""
    v = oracle.e4m3_decode(codes) * scale
    q = np.abs(x) / np.where(scale == 0, 1, scale)
    bound_units = np.maximum(2.0 ** -4 * q, 2.0 ** -10) + 2.0 ** -20 * q
    return np.all(np.abs(v - x) <= bound_units * scale + 1e-300)


def test_dynamic_rows_error_bound_and_amax_maps_to_448():
    inp = synth.small_case(4, 64, 512, 128, seed=5)
    x = inp.lhs
    codes, scales, _ = oracle.quantize_rows(x, oracle.Q_DYNAMIC)
    xf = f32(x)
    s_full = np.repeat(scales.astype(np.float64), 128, axis=1)
    assert _dequant_error_ok(xf, codes, s_full)
    # the element holding the block's absolute maximum maps to +-448
    xb = np.abs(xf).reshape(64, 4, 128)
    cb = codes.reshape(64, 4, 128)
    arg = xb.argmax(axis=2)
    picked = np.take_along_axis(cb, arg[..., None], axis=2)[..., 0]
    assert np.all((picked & 0x7F) == 0x7E)
    expect = (xb.max(axis=2).astype(np.float32) / np.float32(448.0))
    assert np.array_equal(scales, expect)


def test_rhs_per_column_scale():
    inp = synth.small_case(3, 16, 256, 384, seed=6)
    codes, scales = oracle.quantize_rhs(inp.w)
    wf = f32(inp.w)
    assert scales.shape == (3, 384)
    expect = np.abs(wf).max(axis=1).astype(np.float32) / np.float32(448.0)
    assert np.array_equal(scales, expect)
    assert _dequant_error_ok(wf, codes, np.broadcast_to(scales[:, None, :].astype(np.float64), wf.shape))
    # every column holds a +-448 code at its absolute maximum
    arg = np.abs(wf).argmax(axis=1)
    picked = np.take_along_axis(codes, arg[:, None, :], axis=1)[:, 0, :]
    assert np.all((picked & 0x7F) == 0x7E)


def test_rows_scaled_folds_rhs_scale_and_zeroes_unrouted_rows():
    inp = synth.small_case(3, 40, 128, 256, seed=7, sizes=[10, 0, 25])  # rows 35..39 unrouted
    _, sr = oracle.quantize_rhs(inp.w)
    codes, scales = oracle.quantize_rows_scaled(inp.dout, sr, inp.group_sizes)
    assert np.all(codes[35:] == 0) and np.all(scales[35:] == 0)
    d = inp.dout.to(torch.float32).numpy()
    g_of = np.repeat([0, 2], [10, 25])
    t = (d[:35] * sr[g_of]).astype(np.float32)  # numpy float32 multiply, IEEE RNE
    tb = np.abs(t).reshape(35, 2, 128).max(axis=2) / np.float32(448.0)
    assert np.array_equal(scales[:35], tb.astype(np.float32))
    s_full = np.repeat(scales[:35].astype(np.float64), 128, axis=1)
    assert _dequant_error_ok(t.astype(np.float64), codes[:35], s_full)


def test_chunks_start_at_each_group():
    sizes = [130, 0, 1, 128, 3]
    M = sum(sizes) + 6  # six unrouted rows at the end
    inp = synth.small_case(5, M, 128, 128, seed=8, sizes=sizes)
    codes, scales = oracle.quantize_chunks(inp.lhs, oracle.Q_DYNAMIC, 0.0, inp.group_sizes)
    assert scales.shape[0] == 2 + 0 + 1 + 1 + 1
    xf = f32(inp.lhs)
    bounds = [(0, 128), (128, 130), (130, 131), (131, 259), (259, 262)]
    for c, (a, b) in enumerate(bounds):
        expect = (np.abs(xf[a:b]).max(axis=0).astype(np.float32) / np.float32(448.0))
        assert np.array_equal(scales[c], expect), c
        sfull = np.broadcast_to(scales[c].astype(np.float64), xf[a:b].shape)
        assert _dequant_error_ok(xf[a:b], codes[a:b], sfull)
    assert np.all(codes[262:] == 0)


def test_chunks_static_rule_matches_row_quantizer():
    inp = synth.small_case(3, 300, 256, 128, seed=9, sizes=[100, 150, 50])
    s = synth.STATIC_SCALE
    c1, sc1 = oracle.quantize_chunks(inp.lhs, oracle.Q_STATIC, s, inp.group_sizes)
    c2, _, _ = oracle.quantize_rows(inp.lhs, oracle.Q_STATIC, s)
    assert np.array_equal(c1, c2)
    assert np.all(sc1 == np.float32(s))


def test_plan_clamps_and_flags():
    offs, flags = oracle.plan([3, 4, 5], 12)
    assert list(offs) == [0, 3, 7, 12] and flags == 0
    offs, flags = oracle.plan([3, -2, 5], 12)
    assert list(offs) == [0, 3, 3, 8] and flags == oracle.FLAG_GROUP_SIZES
    offs, flags = oracle.plan([8, 8, 8], 12)
    assert list(offs) == [0, 8, 12, 12] and flags == oracle.FLAG_GROUP_SIZES
    offs, flags = oracle.plan([0, 0], 5)
    assert list(offs) == [0, 0, 0] and flags == 0


def _codes_division_vs_reciprocal(s: np.float32):
    """Over every finite bf16 value x: the number of inputs whose code differs
    between e4m3(fl32(x / s)) (the LhsRef docstring's clip(lhs / scale)) and
    e4m3(fl32(x * fl32(1 / s))) (the inner_kernel form this oracle follows),
    and the number whose fp32 intermediates differ."""
    bits = np.arange(65536, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    x = x[np.isfinite(x)]
    inv = np.float32(1.0) / s
    with np.errstate(over="ignore"):
        q = (x / s).astype(np.float32)
        p = (x * inv).astype(np.float32)
    d = q != p
    if not d.any():
        return 0, 0
    cq = oracle.e4m3_encode(q[d].astype(np.float64))
    cp = oracle.e4m3_encode(p[d].astype(np.float64))
    return int((cq != cp).sum()), int(d.sum())


def test_static_rule_division_and_reciprocal_give_the_same_codes():
    """Reading of the static rule ("add static LHS scaling support for GMM v2
    FWD", maxtext PR #4735): the LhsRef docstring writes clip(lhs / scale), the
    inner_kernel code multiplies by the inverse scale.  For the static scale of
    every static workload (4/448), exhaustively over all bf16 inputs, the two
    forms give the same E4M3 code although their fp32 intermediates differ on
    about a third of the inputs; the same holds for 40 log-uniform scales in
    [1e-4, 1].  So the choice changes no code on these inputs."""
    diff, fp32_diff = _codes_division_vs_reciprocal(np.float32(4.0) / np.float32(448.0))
    assert diff == 0 and fp32_diff > 20000
    rng = np.random.default_rng(0)
    for s in np.exp(rng.uniform(np.log(1e-4), 0.0, 40)).astype(np.float32):
        assert _codes_division_vs_reciprocal(s)[0] == 0, s
