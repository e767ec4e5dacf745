"""The GEMM passes on tiles shared by a pair of CTAs (a two-CTA cluster
issuing M = 256 tensor-core MMAs), 256 columns wide or, in mode
"cta_pairs_narrow", 128 columns wide for the promoted passes with a K-major
B operand, against one-CTA tiles, both forced (the automatic choice takes
pairs for the E4M3 tgmm and for static E4M3 row passes whose groups average
two row tiles or more).  Each pass is checked against the oracle and bit for
bit against the one-CTA 128-row tile (every tile accumulates each output over
the same contraction steps in the same order; static E4M3 row tiles in both
variants sum their even and odd blocks in two accumulators and add the two
at the end).  The cases put the pair tile's
second half past a group's end (odd 128-row tile counts, 1-row and 129-row
groups), leave rows unrouted, leave groups empty and use N not a multiple of
256.
"""
import numpy as np
import pytest
import torch

import moe_fp8_grouped_b200 as gm
import oracle
from moe_fp8_grouped_b200 import synth
from parity import assert_close, assert_within, rule_code, swiglu_bound

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": None,                                          # G=8, M=256, K=512, N=512, group 3 empty
    "ragged": (5, 700, 384, 640, [1, 129, 0, 300, 200]),  # N % 256 = 128: the tgmm keeps one-CTA tiles
    "odd_tiles": (3, 900, 256, 512, [129, 385, 300]),      # 2, 4, 3 row tiles: half-empty pair tiles
    "big_group": (2, 1100, 512, 256, [1000, 100]),
    "unrouted": (4, 1000, 256, 256, [10, 0, 250, 40]),     # 700 rows in no group
    # one-CTA promoted tiles of <= 64 rows run M = 64 MMAs: compared bit for
    # bit with the pair tiles' M = 256 MMAs
    "short_tiles": (7, 480, 384, 512, [64, 65, 16, 0, 48, 192, 63]),
    # K = 128: one contraction block per row tile (static E4M3 tiles fill
    # only the first of their two accumulators)
    "k128": (3, 600, 128, 256, [200, 0, 330]),
}


def case_inputs(name):
    if CASES[name] is None:
        return synth.make_inputs("tiny", seed=0)
    G, M, K, N, sizes = CASES[name]
    return synth.small_case(G, M, K, N, seed=17, sizes=sizes)


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


PAIR_MODES = ["cta_pairs", "cta_pairs_narrow"]


def both_tiles(fn, mode="cta_pairs"):
    """fn() on one-CTA tiles, then on CTA pairs (256-column tiles, or with
    mode "cta_pairs_narrow" 128-column tiles in the promoted passes whose B
    operand is K-major); the auto choice is restored."""
    try:
        gm.gmm_set_tiles("one_cta")
        one = fn()
        gm.gmm_set_tiles(mode)
        pair = fn()
    finally:
        gm.gmm_set_tiles("auto")
    torch.cuda.synchronize()
    return one, pair


def to_dev(inp, dev):
    return (inp.lhs.to(dev), inp.w.to(dev), inp.dout.to(dev), inp.group_sizes.to(dev),
            torch.tensor([inp.static_scale], dtype=torch.float32, device=dev))


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("mode", PAIR_MODES)
def test_fwd_pairs(dev, mode, name, rule, transpose):
    inp = case_inputs(name)
    lhs, w, _, gs, s = to_dev(inp, dev)
    codes, scales = gm.gmm_quantize_rhs(w, transpose_out=transpose)
    sarg = s if rule == "static" else None
    one, pair = both_tiles(lambda: gm.gmm_fwd(lhs, codes, scales, gs, rule=rule, static_scale=sarg,
                                              transpose_rhs=transpose, out_dtype=torch.float32), mode)
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, ab = oracle.gmm_fwd(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
    assert_close(pair, ref, ab, f"pair fwd {name} {rule} t={transpose}")
    assert torch.equal(pair, one), f"pair fwd differs from one-CTA fwd ({name} {rule} t={transpose})"


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("mode", PAIR_MODES)
def test_dlhs_pairs(dev, mode, name, transpose):
    inp = case_inputs(name)
    _, w, dout, gs, _ = to_dev(inp, dev)
    codes, scales = gm.gmm_quantize_rhs(w, transpose_out=transpose)
    one, pair = both_tiles(lambda: gm.gmm_dlhs(dout, codes, scales, gs, transpose_rhs=transpose,
                                               out_dtype=torch.bfloat16), mode)
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, ab = oracle.gmm_dlhs(inp.dout, qr, sr, inp.group_sizes)
    assert_close(pair, ref, ab, f"pair dlhs {name} t={transpose}")
    assert torch.equal(pair, one)


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("mode", PAIR_MODES)
def test_drhs_and_backward_pairs(dev, mode, name, rule):
    inp = case_inputs(name)
    lhs, w, dout, gs, s = to_dev(inp, dev)
    sarg = s if rule == "static" else None
    one, pair = both_tiles(lambda: gm.tgmm_drhs(lhs, dout, gs, rule=rule, static_scale=sarg), mode)
    ref, ab = oracle.tgmm_drhs(inp.lhs, rule_code(rule), inp.static_scale, inp.dout, inp.group_sizes)
    assert_close(pair, ref, ab, f"pair drhs {name} {rule}")
    assert torch.equal(pair, one)
    codes, scales = gm.gmm_quantize_rhs(w)
    (d1, w1), (d2, w2) = both_tiles(lambda: gm.gmm_backward(lhs, dout, codes, scales, gs, rule=rule,
                                                            static_scale=sarg), mode)
    assert torch.equal(d1, d2) and torch.equal(w1, w2)
    assert torch.equal(w2, pair)


@pytest.mark.parametrize("name", ["tiny", "odd_tiles", "unrouted"])
@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("mode", PAIR_MODES)
def test_swiglu_pairs(dev, mode, name, rule, transpose):
    inp = case_inputs(name)
    lhs, w, _, gs, s = to_dev(inp, dev)
    codes, scales = gm.gmm_quantize_rhs(w, transpose_out=transpose)
    one, pair = both_tiles(lambda: gm.gmm_fwd_swiglu(lhs, codes, scales, gs, rule=rule,
                                                     static_scale=s if rule == "static" else None,
                                                     transpose_rhs=transpose, out_dtype=torch.float32), mode)
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, terms = oracle.gmm_fwd_swiglu(inp.lhs, rule_code(rule), inp.static_scale, qr, sr, inp.group_sizes)
    assert_within(pair, ref, swiglu_bound(torch.float32, terms, ref), f"pair swiglu {name}")
    assert torch.equal(pair, one)


@pytest.mark.parametrize("name", ["tiny", "odd_tiles"])
@pytest.mark.parametrize("mode", PAIR_MODES)
def test_bf16_family_pairs(dev, mode, name):
    inp = case_inputs(name)
    lhs, w, dout, gs, _ = to_dev(inp, dev)
    for tr in (False, True):
        wt = w.transpose(1, 2).contiguous() if tr else w
        one, pair = both_tiles(lambda: gm.gmm_fwd(lhs, wt, None, gs, rule="none", transpose_rhs=tr,
                                                  out_dtype=torch.float32), mode)
        ref, ab = oracle.gmm_fwd_bf16(inp.lhs, inp.w, inp.group_sizes)
        assert_close(pair, ref, ab, f"pair bf16 fwd t={tr}")
        assert torch.equal(pair, one)
    one, pair = both_tiles(lambda: gm.gmm_dlhs(dout, w, None, gs, rule="none", out_dtype=torch.float32), mode)
    ref, ab = oracle.gmm_dlhs_bf16(inp.dout, inp.w, inp.group_sizes)
    assert_close(pair, ref, ab, "pair bf16 dlhs")
    assert torch.equal(pair, one)
    one, pair = both_tiles(lambda: gm.tgmm_drhs(lhs, dout, gs, rule="none", out_dtype=torch.float32), mode)
    ref, ab = oracle.tgmm_drhs_bf16(inp.lhs, inp.dout, inp.group_sizes)
    assert_close(pair, ref, ab, "pair bf16 drhs")
    assert torch.equal(pair, one)


@pytest.mark.parametrize("rule", ["static", "dynamic"])
@pytest.mark.parametrize("mode", PAIR_MODES)
def test_blockwise_pairs(dev, mode, rule):
    inp = case_inputs("odd_tiles")
    lhs, w, dout, gs, s = to_dev(inp, dev)
    sarg = s if rule == "static" else None
    c0, s0 = gm.gmm_quantize_rhs_blocks(w, 0)
    c1, s1 = gm.gmm_quantize_rhs_blocks(w, 1)
    one, pair = both_tiles(lambda: gm.gmm_fwd(lhs, c0, s0, gs, rule=rule, static_scale=sarg,
                                              out_dtype=torch.float32), mode)
    qr0, sr0 = oracle.quantize_rhs_blocks(inp.w, 0)
    ref, ab = oracle.gmm_fwd_blockwise(inp.lhs, rule_code(rule), inp.static_scale, qr0, sr0, inp.group_sizes)
    assert_close(pair, ref, ab, f"pair blockwise fwd {rule}")
    assert torch.equal(pair, one)
    one, pair = both_tiles(lambda: gm.gmm_dlhs(dout, c1, s1, gs, out_dtype=torch.float32), mode)
    qr1, sr1 = oracle.quantize_rhs_blocks(inp.w, 1)
    ref, ab = oracle.gmm_dlhs_blockwise(inp.dout, qr1, sr1, inp.group_sizes)
    assert_close(pair, ref, ab, "pair blockwise dlhs")
    assert torch.equal(pair, one)


@pytest.mark.parametrize("mode", PAIR_MODES)
def test_pairs_status_clean_and_max_groups(dev, mode):
    """Many groups, most empty, a few large: pair items span the group
    boundaries the pair prefix is built from (1024 groups, the maximum)."""
    G, M, K, N = 1024, 2000, 256, 256
    sizes = np.zeros(G, np.int32)
    sizes[[3, 500, 1023]] = [700, 513, 600]
    inp = synth.small_case(G, M, K, N, seed=18, sizes=sizes.tolist())
    lhs, w, _, gs, s = to_dev(inp, dev)
    codes, scales = gm.gmm_quantize_rhs(w)
    ws = torch.empty(gm.gmm_workspace_bytes(0, M, K, N, G), dtype=torch.uint8, device=dev)
    one, pair = both_tiles(lambda: gm.gmm_fwd(lhs, codes, scales, gs, rule="static", static_scale=s, ws=ws,
                                              out_dtype=torch.float32), mode)
    st, bits = gm.gmm_read_device_status(ws)
    assert st == 0, (st, bits)
    rows = [0, 3, 699, 700, 1212, 1213, 1812, 1813, 1999]
    qr, sr = oracle.quantize_rhs(inp.w)
    ref, ab = oracle.gmm_fwd(inp.lhs, oracle.Q_STATIC, inp.static_scale, qr, sr, inp.group_sizes, rows=rows)
    assert_close(pair[rows], ref, ab, "pair fwd, 1024 groups")
    assert torch.equal(pair, one)
