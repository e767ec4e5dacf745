"""CUDA path vs the CPU oracle on small ragged cases (through the C-ABI).

Codes and scales are compared bit for bit; pass outputs element by element
within 2e-3 * sum|a*b| (plus bf16 output rounding).  Cases span several
tiles, ragged tails, empty groups, unrouted rows, N not a multiple of the
256-wide tile, row tiles short enough for M = 64 MMAs, both rhs layouts and
both output dtypes.  Each pass is run on
its own (the pages' review found a bug where one pass's flag leaked into
another: "Support quantization for tokamax gmm v2", maxtext PR #4451, review
thread on the dlhs selection).
"""
import numpy as np
import pytest
import torch

import moe_fp8_grouped_b200 as gm
import oracle
from moe_fp8_grouped_b200 import synth
from parity import assert_close, assert_within, check_guards, guarded, rule_code, swiglu_bound, untranspose_chunks

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": None,  # the tiny workload: G=8, M=256, K=512, N=512, group 3 empty
    "ragged": (5, 700, 384, 640, [1, 129, 0, 300, 200]),  # 70 unrouted rows, N % 256 = 128
    "g1": (1, 300, 256, 256, [300]),
    "big_group": (2, 1100, 512, 256, [1000, 100]),
    # row tiles of 64, 16, 48, 64 (the tail of 192) and 63 rows run M = 64
    # MMAs in the promoted passes; 65 rows one M = 128 tile; 32 rows unrouted
    "short_tiles": (7, 480, 384, 512, [64, 65, 16, 0, 48, 192, 63]),
}


def case_inputs(name):
    if CASES[name] is None:
        return synth.make_inputs("tiny", seed=0)
    G, M, K, N, sizes = CASES[name]
    return synth.small_case(G, M, K, N, seed=7, sizes=sizes)


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_dev(inp, dev):
    return (inp.lhs.to(dev), inp.w.to(dev), inp.dout.to(dev), inp.group_sizes.to(dev),
            torch.tensor([inp.static_scale], dtype=torch.float32, device=dev))


# ----------------------------------------------------------- quantizers

@pytest.mark.parametrize("transpose", [False, True])
def test_quantize_rhs_bitexact(dev, transpose):
    inp = case_inputs("ragged")
    codes, scales = gm.gmm_quantize_rhs(inp.w.to(dev), transpose_out=transpose)
    qr, sr = oracle.quantize_rhs(inp.w)
    got = codes.cpu().numpy()
    if transpose:
        got = got.transpose(0, 2, 1)
    assert np.array_equal(got, qr)
    assert np.array_equal(scales.cpu().numpy(), sr)


@pytest.mark.parametrize("rule", ["static", "dynamic"])
def test_quantize_rows_bitexact(dev, rule):
    inp = case_inputs("ragged")
    x = inp.lhs.to(dev)
    s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
    codes, scales = gm.gmm_quantize(x, rule, axis=1, static_scale=s if rule == "static" else None)
    qc, qs, _ = oracle.quantize_rows(inp.lhs, rule_code(rule), inp.static_scale)
    assert np.array_equal(codes.cpu().numpy(), qc)
    if rule == "dynamic":
        assert np.array_equal(scales.cpu().numpy().T, qs)


def test_quantize_rows_scaled_bitexact(dev):
    inp = case_inputs("ragged")
    _, sr = oracle.quantize_rhs(inp.w)
    codes, scales = gm.gmm_quantize(inp.dout.to(dev), "dynamic", axis=1, group_sizes=inp.group_sizes.to(dev),
                                    col_scale=torch.from_numpy(sr).to(dev))
    qc, qs = oracle.quantize_rows_scaled(inp.dout, sr, inp.group_sizes)
    assert np.array_equal(codes.cpu().numpy(), qc)
    assert np.array_equal(scales.cpu().numpy().T, qs)


@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("name", ["ragged", "tiny"])
def test_quantize_chunks_bitexact(dev, rule, name):
    inp = case_inputs(name)
    M = inp.lhs.shape[0]
    s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
    codes_t, scales = gm.gmm_quantize(inp.lhs.to(dev), rule, axis=0, static_scale=s if rule == "static" else None,
                                      group_sizes=inp.group_sizes.to(dev))
    offs, _ = oracle.plan(inp.group_sizes, M)
    got_c, got_s = untranspose_chunks(codes_t, scales, offs, M)
    qc, qs = oracle.quantize_chunks(inp.lhs, rule_code(rule), inp.static_scale, inp.group_sizes)
    assert np.array_equal(got_c, qc)
    assert np.array_equal(got_s, qs)


# ---------------------------------------------------------------- passes

@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_fwd(dev, name, rule, transpose, out_dtype):
    inp = case_inputs(name)
    lhs, w, _, gs, s = to_dev(inp, dev)
    M, N = lhs.shape[0], w.shape[2]
    codes, scales = gm.gmm_quantize_rhs(w, transpose_out=transpose)
    raw, out, pad, n = guarded((M, N), out_dtype)
    gm.gmm_fwd(lhs, codes, scales, gs, rule=rule, static_scale=s if rule == "static" else None,
               transpose_rhs=transpose, out=out)
    assert gm.last_launch_count() == 3
    torch.cuda.synchronize()
    check_guards(raw, pad, n)
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, ab = oracle.gmm_fwd(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
    assert_close(out, ref, ab, f"fwd {name} {rule} t={transpose}")


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_dlhs(dev, name, transpose, out_dtype):
    inp = case_inputs(name)
    _, w, dout, gs, _ = to_dev(inp, dev)
    M, K = inp.lhs.shape
    codes, scales = gm.gmm_quantize_rhs(w, transpose_out=transpose)
    raw, out, pad, n = guarded((M, K), out_dtype)
    gm.gmm_dlhs(dout, codes, scales, gs, transpose_rhs=transpose, out=out)
    torch.cuda.synchronize()
    check_guards(raw, pad, n)
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
    assert_close(out, ref, ab, f"dlhs {name} t={transpose}")


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_drhs(dev, name, rule, out_dtype):
    inp = case_inputs(name)
    lhs, w, dout, gs, s = to_dev(inp, dev)
    G, K, N = w.shape
    raw, out, pad, n = guarded((G, K, N), out_dtype)
    gm.tgmm_drhs(lhs, dout, gs, rule=rule, static_scale=s if rule == "static" else None, out=out)
    assert gm.last_launch_count() == 4
    torch.cuda.synchronize()
    check_guards(raw, pad, n)
    ref, ab = oracle.tgmm_drhs(inp.lhs, rule_code(rule), inp.static_scale, inp.dout, inp.group_sizes)
    assert_close(out, ref, ab, f"drhs {name} {rule}")


@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("transpose", [False, True])
def test_fwd_prequantized_lhs(dev, rule, transpose):
    """lhs quantized before the call (for example ahead of an expert-parallel
    all-gather): the forward takes the codes and scales as they are and gives
    the same result as quantizing inside the call."""
    inp = case_inputs("ragged")
    lhs, w, _, gs, s = to_dev(inp, dev)
    codes, scales = gm.gmm_quantize_rhs(w, transpose_out=transpose)
    sarg = s if rule == "static" else None
    ql, sl = gm.gmm_quantize(lhs, rule, axis=1, static_scale=sarg)
    inside = gm.gmm_fwd(lhs, codes, scales, gs, rule=rule, static_scale=sarg, transpose_rhs=transpose,
                        out_dtype=torch.float32)
    outside = gm.gmm_fwd(ql, codes, scales, gs, rule=rule, static_scale=sarg, lhs_scales=sl,
                         transpose_rhs=transpose, out_dtype=torch.float32)
    assert gm.last_launch_count() == 2  # plan + GEMM: no quantize step
    assert torch.equal(inside, outside)
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, ab = oracle.gmm_fwd(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
    assert_close(outside, ref, ab, f"prequantized fwd {rule}")


@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("transpose", [False, True])
def test_fwd_keep_lhs_hands_back_its_codes(dev, rule, transpose):
    """gmm_fwd_keep_lhs gives gmm_fwd's result bit for bit and the codes /
    scales gmm_quantize makes; with the static rule those codes are the
    backward's lhs operand, with the same dW."""
    inp = case_inputs("ragged")
    lhs, w, dout, gs, s = to_dev(inp, dev)
    sarg = s if rule == "static" else None
    codes, scales = gm.gmm_quantize_rhs(w, transpose_out=transpose)
    out, qc, qs = gm.gmm_fwd_keep_lhs(lhs, codes, scales, gs, rule=rule, static_scale=sarg, transpose_rhs=transpose,
                                      out_dtype=torch.float32)
    assert gm.last_launch_count() == 3
    ref = gm.gmm_fwd(lhs, codes, scales, gs, rule=rule, static_scale=sarg, transpose_rhs=transpose,
                     out_dtype=torch.float32)
    assert torch.equal(out, ref)
    c2, s2 = gm.gmm_quantize(lhs, rule, axis=1, static_scale=sarg)
    assert torch.equal(qc, c2)
    if rule == "dynamic":
        assert torch.equal(qs, s2)
    else:
        dl1, dw1 = gm.gmm_backward(qc, dout, codes, scales, gs, rule="static", static_scale=s, transpose_rhs=transpose)
        dl2, dw2 = gm.gmm_backward(lhs, dout, codes, scales, gs, rule="static", static_scale=s,
                                   transpose_rhs=transpose)
        assert torch.equal(dl1, dl2) and torch.equal(dw1, dw2)


@pytest.mark.parametrize("name", ["ragged", "big_group"])
def test_drhs_reuses_static_forward_codes(dev, name):
    """Static rule: the forward's lhs codes (quantized once, as for an
    expert-parallel all-gather in E4M3) feed the tgmm unchanged; the result
    equals quantizing inside the tgmm bit for bit."""
    inp = case_inputs(name)
    lhs, _, dout, gs, s = to_dev(inp, dev)
    ql, _ = gm.gmm_quantize(lhs, "static", axis=1, static_scale=s)
    inside = gm.tgmm_drhs(lhs, dout, gs, rule="static", static_scale=s)
    reused = gm.tgmm_drhs(ql, dout, gs, rule="static", static_scale=s)
    assert gm.last_launch_count() == 4
    assert torch.equal(inside, reused)
    ref, ab = oracle.tgmm_drhs(inp.lhs, oracle.Q_STATIC, inp.static_scale, inp.dout, inp.group_sizes)
    assert_close(reused, ref, ab, f"drhs with forward codes {name}")
    with pytest.raises(gm.GmmError, match="invalid argument"):
        gm.tgmm_drhs(ql, dout, gs, rule="dynamic", static_scale=s)


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_bf16_family(dev, name):
    inp = case_inputs(name)
    lhs, w, dout, gs, _ = to_dev(inp, dev)
    f = gm.gmm_fwd(lhs, w, None, gs, rule="none", out_dtype=torch.float32)
    ref, ab = oracle.gmm_fwd_bf16(inp.lhs, inp.w, inp.group_sizes)
    assert_close(f, ref, ab, "bf16 fwd")
    d = gm.gmm_dlhs(dout, w, None, gs, rule="none", out_dtype=torch.float32)
    ref, ab = oracle.gmm_dlhs_bf16(inp.dout, inp.w, inp.group_sizes)
    assert_close(d, ref, ab, "bf16 dlhs")
    r = gm.tgmm_drhs(lhs, dout, gs, rule="none", out_dtype=torch.float32)
    ref, ab = oracle.tgmm_drhs_bf16(inp.lhs, inp.dout, inp.group_sizes)
    assert_close(r, ref, ab, "bf16 drhs")


# --------------------------------------------------------------- SwiGLU

SWIGLU_CASES = {
    "tiny": None,
    "ragged": (5, 700, 384, 768, [1, 129, 0, 300, 200]),  # F = 384: a tile pair beyond 256
    "g1": (1, 300, 256, 256, [300]),                        # F = 128: one column tile
    "big_group": (2, 1100, 512, 512, [1000, 100]),
}


@pytest.mark.parametrize("name", list(SWIGLU_CASES))
@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_fwd_swiglu(dev, name, rule, transpose, out_dtype):
    """Merged gate|up forward with silu(gate) * up fused into the epilogue,
    against the oracle within the forward's tolerance carried through the
    activation."""
    c = SWIGLU_CASES[name]
    inp = synth.make_inputs("tiny", seed=0) if c is None else synth.small_case(*c[:4], seed=9, sizes=c[4])
    lhs, w, _, gs, s = to_dev(inp, dev)
    M, N = lhs.shape[0], w.shape[2]
    codes, scales = gm.gmm_quantize_rhs(w, transpose_out=transpose)
    raw, out, pad, n = guarded((M, N // 2), out_dtype)
    gm.gmm_fwd_swiglu(lhs, codes, scales, gs, rule=rule, static_scale=s if rule == "static" else None,
                      transpose_rhs=transpose, out=out)
    assert gm.last_launch_count() == 3
    torch.cuda.synchronize()
    check_guards(raw, pad, n)
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, terms = oracle.gmm_fwd_swiglu(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
    assert_within(out, ref, swiglu_bound(out_dtype, terms, ref), f"swiglu {name} {rule} t={transpose}")


def test_fwd_swiglu_bf16_family_and_prequantized(dev):
    inp = synth.small_case(*SWIGLU_CASES["ragged"][:4], seed=10, sizes=SWIGLU_CASES["ragged"][4])
    lhs, w, _, gs, s = to_dev(inp, dev)
    # bf16 family: the same fused epilogue on the kind::f16 path
    out = gm.gmm_fwd_swiglu(lhs, w, None, gs, rule="none", out_dtype=torch.float32)
    h, ab = oracle.gmm_fwd_bf16(inp.lhs, inp.w, inp.group_sizes)
    F = h.shape[1] // 2
    ref = oracle.silu(h[:, :F]) * h[:, F:]
    assert_within(out, ref, swiglu_bound(torch.float32, (h[:, :F], h[:, F:], ab[:, :F], ab[:, F:]), ref),
                  "swiglu bf16 family")
    # pre-quantized lhs gives the same result as quantizing inside the call
    codes, scales = gm.gmm_quantize_rhs(w)
    ql, _ = gm.gmm_quantize(lhs, "static", axis=1, static_scale=s)
    a = gm.gmm_fwd_swiglu(lhs, codes, scales, gs, rule="static", static_scale=s, out_dtype=torch.float32)
    b = gm.gmm_fwd_swiglu(ql, codes, scales, gs, rule="static", static_scale=s, out_dtype=torch.float32)
    assert torch.equal(a, b)


def test_fwd_swiglu_rejects_n_not_two_tiles_of_128(dev):
    inp = synth.small_case(*CASES["ragged"][:4], seed=7, sizes=CASES["ragged"][4])  # N = 640: F = 320
    lhs, w, _, gs, s = to_dev(inp, dev)
    codes, scales = gm.gmm_quantize_rhs(w)
    with pytest.raises(gm.GmmError, match="shape"):
        gm.gmm_fwd_swiglu(lhs, codes, scales, gs, rule="static", static_scale=s)


# ------------------------------------------------------ fused backward

@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("transpose", [False, True])
def test_backward_equals_the_two_calls(dev, name, rule, transpose):
    """gmm_backward quantizes dout once for both passes; its codes are the
    separate calls' codes, so dlhs and dW agree bit for bit, and with the
    oracle within the tolerance."""
    inp = case_inputs(name)
    lhs, w, dout, gs, s = to_dev(inp, dev)
    M, K, N, G = lhs.shape[0], lhs.shape[1], w.shape[2], w.shape[0]
    codes, scales = gm.gmm_quantize_rhs(w, transpose_out=transpose)
    sarg = s if rule == "static" else None
    raw_d, dl, pad_d, n_d = guarded((M, K), torch.float32)
    raw_w, dw, pad_w, n_w = guarded((G, K, N), torch.float32)
    gm.gmm_backward(lhs, dout, codes, scales, gs, rule=rule, static_scale=sarg, transpose_rhs=transpose,
                    dlhs=dl, drhs=dw)
    assert gm.last_launch_count() == 5
    torch.cuda.synchronize()
    check_guards(raw_d, pad_d, n_d)
    check_guards(raw_w, pad_w, n_w)
    d1 = gm.gmm_dlhs(dout, codes, scales, gs, transpose_rhs=transpose, out_dtype=torch.float32)
    w1 = gm.tgmm_drhs(lhs, dout, gs, rule=rule, static_scale=sarg)
    assert torch.equal(dl, d1)
    assert torch.equal(dw, w1)
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
    assert_close(dl, ref, ab, f"backward dlhs {name}")
    ref, ab = oracle.tgmm_drhs(inp.lhs, rule_code(rule), inp.static_scale, inp.dout, inp.group_sizes)
    assert_close(dw, ref, ab, f"backward drhs {name}")


def test_backward_bf16_family_blockwise_and_forward_codes(dev):
    inp = case_inputs("ragged")
    lhs, w, dout, gs, s = to_dev(inp, dev)
    # bf16 family
    dl, dw = gm.gmm_backward(lhs, dout, w, None, gs, rule="none", dlhs_dtype=torch.float32)
    assert torch.equal(dl, gm.gmm_dlhs(dout, w, None, gs, rule="none", out_dtype=torch.float32))
    assert torch.equal(dw, gm.tgmm_drhs(lhs, dout, gs, rule="none"))
    # block-wise weights along N for dlhs (no fold)
    c1, s1 = gm.gmm_quantize_rhs_blocks(w, 1)
    dl, dw = gm.gmm_backward(lhs, dout, c1, s1, gs, rule="dynamic", dlhs_dtype=torch.float32)
    assert torch.equal(dl, gm.gmm_dlhs(dout, c1, s1, gs, out_dtype=torch.float32))
    assert torch.equal(dw, gm.tgmm_drhs(lhs, dout, gs, rule="dynamic"))
    # the forward's static codes as the tgmm lhs
    codes, scales = gm.gmm_quantize_rhs(w)
    ql, _ = gm.gmm_quantize(lhs, "static", axis=1, static_scale=s)
    dl, dw = gm.gmm_backward(ql, dout, codes, scales, gs, rule="static", static_scale=s)
    assert torch.equal(dw, gm.tgmm_drhs(lhs, dout, gs, rule="static", static_scale=s))
    with pytest.raises(gm.GmmError, match="invalid argument"):  # mixed families
        gm.gmm_backward(lhs, dout, codes, scales, gs, rule="none")


# ------------------------------------------------- block-wise rhs scales

@pytest.mark.parametrize("axis", [0, 1])
def test_quantize_rhs_blocks_bitexact(dev, axis):
    inp = case_inputs("ragged")
    w = inp.w.to(dev)
    codes, scales = gm.gmm_quantize_rhs_blocks(w, axis)
    qr, sr = oracle.quantize_rhs_blocks(inp.w, axis)
    assert np.array_equal(codes.cpu().numpy(), qr)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), sr.view(np.uint32))


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_fwd_blockwise(dev, name, rule, out_dtype):
    """Forward with one rhs scale per 128-block of K and column: every
    contraction block is promoted with s_l[m, b] * s_r[g, b, n]."""
    inp = case_inputs(name)
    lhs, w, _, gs, s = to_dev(inp, dev)
    M, N = lhs.shape[0], w.shape[2]
    codes, scales = gm.gmm_quantize_rhs_blocks(w, 0)
    raw, out, pad, n = guarded((M, N), out_dtype)
    gm.gmm_fwd(lhs, codes, scales, gs, rule=rule, static_scale=s if rule == "static" else None, out=out)
    torch.cuda.synchronize()
    check_guards(raw, pad, n)
    qr, sr = oracle.quantize_rhs_blocks(inp.w, 0)
    ref, ab = oracle.gmm_fwd_blockwise(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
    assert_close(out, ref, ab, f"blockwise fwd {name} {rule}")


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_dlhs_blockwise(dev, name, out_dtype):
    inp = case_inputs(name)
    _, w, dout, gs, _ = to_dev(inp, dev)
    M, K = dout.shape[0], w.shape[1]
    codes, scales = gm.gmm_quantize_rhs_blocks(w, 1)
    raw, out, pad, n = guarded((M, K), out_dtype)
    gm.gmm_dlhs(dout, codes, scales, gs, out=out)
    torch.cuda.synchronize()
    check_guards(raw, pad, n)
    qr, sr = oracle.quantize_rhs_blocks(inp.w, 1)
    ref, ab = oracle.gmm_dlhs_blockwise(inp.dout, qr, sr, inp.group_sizes)
    assert_close(out, ref, ab, f"blockwise dlhs {name}")


@pytest.mark.parametrize("rule", ["static", "dynamic"])
def test_fwd_swiglu_blockwise(dev, rule):
    c = SWIGLU_CASES["ragged"]
    inp = synth.small_case(*c[:4], seed=12, sizes=c[4])
    lhs, w, _, gs, s = to_dev(inp, dev)
    codes, scales = gm.gmm_quantize_rhs_blocks(w, 0)
    out = gm.gmm_fwd_swiglu(lhs, codes, scales, gs, rule=rule, static_scale=s if rule == "static" else None,
                            out_dtype=torch.float32)
    qr, sr = oracle.quantize_rhs_blocks(inp.w, 0)
    h, ab = oracle.gmm_fwd_blockwise(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
    F = h.shape[1] // 2
    ref = oracle.silu(h[:, :F]) * h[:, F:]
    assert_within(out, ref, swiglu_bound(torch.float32, (h[:, :F], h[:, F:], ab[:, :F], ab[:, F:]), ref),
                  f"blockwise swiglu {rule}")


def test_blockwise_rejects_transposed_rhs(dev):
    inp = case_inputs("g1")
    lhs, w, dout, gs, s = to_dev(inp, dev)
    codes, scales = gm.gmm_quantize_rhs_blocks(w, 0)
    with pytest.raises(gm.GmmError, match="unsupported"):
        gm.gmm_fwd(lhs, codes, scales, gs, rule="static", static_scale=s, transpose_rhs=True)
    with pytest.raises(gm.GmmError, match="unsupported"):
        gm.gmm_dlhs(dout, codes, scales, gs, transpose_rhs=True)


# ---------------------------------------------------------- limits

@pytest.mark.parametrize("rule", ["static", "dynamic"])
def test_maximum_group_count(dev, rule):
    """G = 1024 (the largest supported), most groups empty, a few large,
    rows left unrouted: all passes and the fused backward against the oracle."""
    G, M, K, N = 1024, 3000, 256, 256
    rng = np.random.default_rng(5)
    sizes = np.zeros(G, np.int64)
    hot = rng.choice(G, 40, replace=False)
    sizes[hot] = rng.multinomial(2900, np.ones(40) / 40)  # 100 of the 3000 rows stay unrouted
    inp = synth.small_case(G, M, K, N, seed=13, sizes=sizes.tolist())
    lhs, w, dout, gs, s = to_dev(inp, dev)
    sarg = s if rule == "static" else None
    codes, scales = gm.gmm_quantize_rhs(w)
    out = gm.gmm_fwd(lhs, codes, scales, gs, rule=rule, static_scale=sarg, out_dtype=torch.float32)
    dl, dw = gm.gmm_backward(lhs, dout, codes, scales, gs, rule=rule, static_scale=sarg, dlhs_dtype=torch.float32)
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, ab = oracle.gmm_fwd(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
    assert_close(out, ref, ab, f"G=1024 fwd {rule}")
    ref, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
    assert_close(dl, ref, ab, f"G=1024 dlhs {rule}")
    sel = np.concatenate([np.arange(0, G * K, K * 7), [hot[0] * K + 3, hot[1] * K + K - 1]])
    ref, ab = oracle.tgmm_drhs(inp.lhs, rule_code(rule), inp.static_scale, inp.dout, inp.group_sizes, sel=sel)
    assert_close(dw.view(G * K, N)[torch.as_tensor(sel, device=dev)], ref, ab, f"G=1024 drhs {rule}")
    empty = np.flatnonzero(sizes == 0)
    assert not dw[torch.as_tensor(empty, device=dev)].any()


@pytest.mark.parametrize("G,M,K,N,sizes", [
    (1, 1, 128, 128, [1]),            # one row, the smallest tile sizes
    (3, 129, 128, 128, [0, 129, 0]),  # a 129-row group: one full and one 1-row tile / chunk
    (4, 200, 256, 384, [0, 0, 0, 0]),  # every group empty: all outputs zero
    (2, 300, 128, 256, [0, 17]),      # 283 unrouted rows
])
def test_degenerate_sizes(dev, G, M, K, N, sizes):
    inp = synth.small_case(G, M, K, N, seed=31, sizes=sizes)
    lhs, w, dout, gs, s = to_dev(inp, dev)
    codes, scales = gm.gmm_quantize_rhs(w)
    for rule in ("static", "dynamic"):
        sarg = s if rule == "static" else None
        out = gm.gmm_fwd(lhs, codes, scales, gs, rule=rule, static_scale=sarg, out_dtype=torch.float32)
        dl, dw = gm.gmm_backward(lhs, dout, codes, scales, gs, rule=rule, static_scale=sarg,
                                 dlhs_dtype=torch.float32)
        qr, sr = oracle.quantize_rhs(inp.w)
        ref, ab = oracle.gmm_fwd(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
        assert_close(out, ref, ab, f"degenerate fwd {sizes} {rule}")
        ref, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
        assert_close(dl, ref, ab, f"degenerate dlhs {sizes}")
        ref, ab = oracle.tgmm_drhs(inp.lhs, rule_code(rule), inp.static_scale, inp.dout, inp.group_sizes)
        assert_close(dw, ref, ab, f"degenerate drhs {sizes} {rule}")
        if sum(sizes) == 0:
            assert not out.any() and not dl.any() and not dw.any()


@pytest.mark.parametrize("seed", range(12))
def test_random_shapes(dev, seed):
    """Random sizes within the supported range (G up to 48, M up to 1600,
    K and N multiples of 128 up to 768, some groups empty, some rows
    unrouted), a random rule, rhs layout and output dtype: forward, fused
    backward and, for even N, the SwiGLU forward against the oracle."""
    rng = np.random.default_rng(1000 + seed)
    G = int(rng.integers(1, 49))
    M = int(rng.integers(1, 1601))
    K = 128 * int(rng.integers(1, 7))
    N = 128 * int(rng.integers(1, 7))
    w = rng.random(G) * (rng.random(G) > 0.3)
    routed = int(rng.integers(0, M + 1))
    sizes = rng.multinomial(routed, w / w.sum()) if w.sum() > 0 else np.zeros(G, np.int64)
    rule = ["static", "dynamic"][seed % 2]
    transpose = bool(rng.integers(0, 2))
    out_dtype = [torch.bfloat16, torch.float32][int(rng.integers(0, 2))]
    inp = synth.small_case(G, M, K, N, seed=seed, sizes=sizes.tolist())
    lhs, wt, dout, gs, s = to_dev(inp, dev)
    sarg = s if rule == "static" else None
    codes, scales = gm.gmm_quantize_rhs(wt, transpose_out=transpose)
    out = gm.gmm_fwd(lhs, codes, scales, gs, rule=rule, static_scale=sarg, transpose_rhs=transpose,
                     out_dtype=out_dtype)
    dl, dw = gm.gmm_backward(lhs, dout, codes, scales, gs, rule=rule, static_scale=sarg, transpose_rhs=transpose,
                             dlhs_dtype=out_dtype)
    qr, sr = oracle.quantize_rhs(inp.w)
    tag = f"seed {seed}: G={G} M={M} K={K} N={N} {rule} t={transpose} {out_dtype}"
    ref, ab = oracle.gmm_fwd(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
    assert_close(out, ref, ab, "fwd " + tag)
    ref, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
    assert_close(dl, ref, ab, "dlhs " + tag)
    ref, ab = oracle.tgmm_drhs(inp.lhs, rule_code(rule), inp.static_scale, inp.dout, inp.group_sizes)
    assert_close(dw, ref, ab, "drhs " + tag)
    if N % 256 == 0:
        sw = gm.gmm_fwd_swiglu(lhs, codes, scales, gs, rule=rule, static_scale=sarg, transpose_rhs=transpose,
                               out_dtype=out_dtype)
        ref, terms = oracle.gmm_fwd_swiglu(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
        assert_within(sw, ref, swiglu_bound(out_dtype, terms, ref), "swiglu " + tag)


# ------------------------------------------------------------ identities

def test_merged_gate_up_identity_gpu(dev):
    """fwd(W0|W1) equals fwd(W0) | fwd(W1) bit for bit (each output column
    sees the same K sequence); drhs likewise; dlhs adds up within tolerance."""
    inp = synth.small_case(4, 600, 512, 512, seed=3, sizes=[200, 0, 250, 150])
    lhs, w, dout, gs, s = to_dev(inp, dev)
    c, sc = gm.gmm_quantize_rhs(w)
    c0, s0 = gm.gmm_quantize_rhs(w[:, :, :256].contiguous())
    c1, s1 = gm.gmm_quantize_rhs(w[:, :, 256:].contiguous())
    for rule in ("static", "dynamic"):
        kw = dict(rule=rule, static_scale=s if rule == "static" else None, out_dtype=torch.float32)
        f = gm.gmm_fwd(lhs, c, sc, gs, **kw)
        f0 = gm.gmm_fwd(lhs, c0, s0, gs, **kw)
        f1 = gm.gmm_fwd(lhs, c1, s1, gs, **kw)
        assert torch.equal(f, torch.cat([f0, f1], dim=1))
        kw.pop("out_dtype")
        r = gm.tgmm_drhs(lhs, dout, gs, **kw)
        r0 = gm.tgmm_drhs(lhs, dout[:, :256].contiguous(), gs, **kw)
        r1 = gm.tgmm_drhs(lhs, dout[:, 256:].contiguous(), gs, **kw)
        assert torch.equal(r, torch.cat([r0, r1], dim=2))
    d = gm.gmm_dlhs(dout, c, sc, gs, out_dtype=torch.float32)
    d0 = gm.gmm_dlhs(dout[:, :256].contiguous(), c0, s0, gs, out_dtype=torch.float32)
    d1 = gm.gmm_dlhs(dout[:, 256:].contiguous(), c1, s1, gs, out_dtype=torch.float32)
    qr, sr = oracle.quantize_rhs(inp.w)
    _, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
    assert np.all(np.abs((d - d0 - d1).cpu().numpy()) <= 2e-3 * ab)


def test_passes_do_not_depend_on_each_other(dev):
    """Each pass reads only its own inputs: a workspace left dirty by another
    pass (or garbage) does not change the result."""
    inp = case_inputs("ragged")
    lhs, w, dout, gs, s = to_dev(inp, dev)
    c, sc = gm.gmm_quantize_rhs(w)
    G, K, N = w.shape
    M = lhs.shape[0]
    nbytes = max(gm.gmm_workspace_bytes(op, M, K, N, G) for op in (0, 1, 2))
    clean = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    dirty = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device=dev)
    a = gm.gmm_dlhs(dout, c, sc, gs, ws=clean, out_dtype=torch.float32)
    b = gm.gmm_dlhs(dout, c, sc, gs, ws=dirty, out_dtype=torch.float32)
    assert torch.equal(a, b)
    a = gm.tgmm_drhs(lhs, dout, gs, rule="static", static_scale=s, ws=clean)
    gm.gmm_fwd(lhs, c, sc, gs, rule="dynamic", ws=dirty)
    b = gm.tgmm_drhs(lhs, dout, gs, rule="static", static_scale=s, ws=dirty)
    assert torch.equal(a, b)


# ------------------------------------------------------- device status

def test_group_sizes_past_M_are_clamped_and_reported(dev):
    inp = synth.small_case(3, 300, 256, 256, seed=4, sizes=[100, 250, 50])
    lhs, w, _, gs, s = to_dev(inp, dev)
    c, sc = gm.gmm_quantize_rhs(w)
    ws = gm.workspace(gm.gmm_workspace_bytes(0, 300, 256, 256, 3), dev)
    out = gm.gmm_fwd(lhs, c, sc, gs, rule="static", static_scale=s, ws=ws, out_dtype=torch.float32)
    st, bits = gm.gmm_read_device_status(ws)
    assert bits & 1 and st == 7  # GMM_ERR_GROUP_SIZES
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, ab = oracle.gmm_fwd(inp.lhs, oracle.Q_STATIC, inp.static_scale, qr, sr, inp.group_sizes)
    assert_close(out, ref, ab, "clamped fwd")
    gs_neg = torch.tensor([100, -5, 50], dtype=torch.int32, device=dev)
    gm.gmm_fwd(lhs, c, sc, gs_neg, rule="static", static_scale=s, ws=ws)
    assert gm.gmm_read_device_status(ws)[0] == 7
    gm.gmm_fwd(lhs, c, sc, torch.tensor([100, 100, 100], dtype=torch.int32, device=dev), rule="static",
               static_scale=s, ws=ws)
    assert gm.gmm_read_device_status(ws) == (0, 0)


@pytest.mark.parametrize("bad", [0.0, float("inf"), float("nan"), -1.0])
def test_unusable_static_scale_reports_and_outputs_zero(dev, bad):
    inp = case_inputs("tiny")
    lhs, w, _, gs, _ = to_dev(inp, dev)
    c, sc = gm.gmm_quantize_rhs(w)
    ws = gm.workspace(gm.gmm_workspace_bytes(0, 256, 512, 512, 8), dev)
    out = gm.gmm_fwd(lhs, c, sc, gs, rule="static", static_scale=torch.tensor([bad], device=dev), ws=ws)
    st, bits = gm.gmm_read_device_status(ws)
    assert st == 4 and bits & 2  # GMM_ERR_SCALE
    assert not out.float().abs().sum().item()
    # codes quantized before the call: the GEMM itself reports the scale
    codes = torch.ones_like(lhs, dtype=torch.uint8)
    out = gm.gmm_fwd(codes, c, sc, gs, rule="static", static_scale=torch.tensor([bad], device=dev), ws=ws)
    st, bits = gm.gmm_read_device_status(ws)
    assert st == 4 and bits & 2
    assert not out.float().abs().sum().item()


def test_bounded_wait_gives_up_and_reports(dev):
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device=dev)
    gm.gmm_selftest_timeout(ws, 50_000_000)  # 50 ms
    st, bits = gm.gmm_read_device_status(ws)
    assert st == 8 and bits & 4  # GMM_ERR_TIMEOUT
    # the context is still usable
    inp = case_inputs("g1")
    lhs, w, _, gs, s = to_dev(inp, dev)
    c, sc = gm.gmm_quantize_rhs(w)
    gm.gmm_fwd(lhs, c, sc, gs, rule="static", static_scale=s)
    torch.cuda.synchronize()


def test_host_errors_return_before_launch(dev):
    inp = case_inputs("tiny")
    lhs, w, _, gs, s = to_dev(inp, dev)
    c, sc = gm.gmm_quantize_rhs(w)
    with pytest.raises(gm.GmmError) as e:
        gm.gmm_fwd(lhs, c, sc, gs, rule="static", static_scale=None)  # a present rule must be applied
    assert e.value.status == 1
    with pytest.raises(gm.GmmError) as e:
        gm.gmm_fwd(lhs, c, sc, gs, rule="static", static_scale=s, ws=torch.empty(16, dtype=torch.uint8,
                                                                                  device=dev))
    assert e.value.status == 9
    with pytest.raises(gm.GmmError) as e:
        gm.gmm_fwd(lhs[:, :500].contiguous(), c[:, :500].contiguous(), sc, gs, rule="static", static_scale=s)
    assert e.value.status == 2


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_output_16_byte_aligned_only(dev, out_dtype):
    """Outputs that are 16- but not 32-byte aligned take the 16-byte store path."""
    inp = case_inputs("ragged")
    lhs, w, dout, gs, s = to_dev(inp, dev)
    G, K, N = w.shape
    M = lhs.shape[0]
    c, sc = gm.gmm_quantize_rhs(w)
    esz = torch.tensor([], dtype=out_dtype).element_size()
    for shape, fn, ref_fn in (
        ((M, N), lambda o: gm.gmm_fwd(lhs, c, sc, gs, rule="static", static_scale=s, out=o),
         lambda: oracle.gmm_fwd(inp.lhs, oracle.Q_STATIC, inp.static_scale, *oracle.quantize_rhs(inp.w),
                                inp.group_sizes)),
        ((G, K, N), lambda o: gm.tgmm_drhs(lhs, dout, gs, rule="dynamic", out=o),
         lambda: oracle.tgmm_drhs(inp.lhs, oracle.Q_DYNAMIC, 0.0, inp.dout, inp.group_sizes)),
    ):
        n = int(np.prod(shape))
        raw = torch.zeros(n * esz + 64, dtype=torch.uint8, device=dev)
        base = raw.data_ptr()
        off = (16 - base % 32) % 32 or 16  # 16 mod 32
        out = raw[off: off + n * esz].view(out_dtype).view(*shape)
        assert out.data_ptr() % 32 == 16
        fn(out)
        ref, ab = ref_fn()
        assert_close(out, ref, ab, f"16B-aligned {shape}")


def test_workspace_16_byte_aligned_only(dev):
    """A workspace that is 16- but not 32-byte aligned puts the quantizers'
    code buffers (forward rows, tgmm chunks, the fused backward's dout) on
    their 16-byte store path: every pass equals its aligned-workspace result
    bit for bit."""
    inp = case_inputs("ragged")
    lhs, w, dout, gs, s = to_dev(inp, dev)
    M, K = lhs.shape
    G, _, N = w.shape
    c, sc = gm.gmm_quantize_rhs(w)
    nbytes = max(gm.gmm_workspace_bytes(op, M, K, N, G) for op in (0, 1, 2, 3))
    raw = torch.zeros(nbytes + 64, dtype=torch.uint8, device=dev)
    off = (16 - raw.data_ptr() % 32) % 32 or 16  # 16 mod 32
    ws16 = raw[off: off + nbytes]
    assert ws16.data_ptr() % 32 == 16
    for rule in ("static", "dynamic"):
        sarg = s if rule == "static" else None
        assert torch.equal(gm.gmm_fwd(lhs, c, sc, gs, rule=rule, static_scale=sarg),
                           gm.gmm_fwd(lhs, c, sc, gs, rule=rule, static_scale=sarg, ws=ws16))
        assert torch.equal(gm.tgmm_drhs(lhs, dout, gs, rule=rule, static_scale=sarg),
                           gm.tgmm_drhs(lhs, dout, gs, rule=rule, static_scale=sarg, ws=ws16))
        dl_a, dw_a = gm.gmm_backward(lhs, dout, c, sc, gs, rule=rule, static_scale=sarg)
        dl_b, dw_b = gm.gmm_backward(lhs, dout, c, sc, gs, rule=rule, static_scale=sarg, ws=ws16)
        assert torch.equal(dl_a, dl_b)
        assert torch.equal(dw_a, dw_b)
