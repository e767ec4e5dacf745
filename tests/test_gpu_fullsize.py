"""Full-size workloads on the GPU, checked on sampled outputs.

Each workload runs at its real size through the same calls bench.py times
(gmm_quantize_rhs once, then gmm_fwd, gmm_dlhs, tgmm_drhs with one shared
workspace).  The oracle then recomputes sampled outputs one by one: a forward
or dlhs row depends only on that row and its group's weights, and a drhs row
(g, k) only on group g's rows, so each sample is an exact group-local
sub-problem.  Weight codes and scales of the sampled groups are compared bit
for bit; empty groups must give dW[g] = 0 exactly and unrouted rows 0.
"""
import numpy as np
import pytest
import torch

import moe_fp8_grouped_b200 as gm
import oracle
from moe_fp8_grouped_b200 import synth
from parity import assert_close, assert_within, swiglu_bound

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

WORKLOADS = ["mixtral", "dsv3_up", "dsv3_down", "ep_merged", "ep_separate", "ragged", "ragged_bf16"]


def pick_groups(gs: np.ndarray, rng: np.random.Generator):
    nz = np.flatnonzero(gs > 0)
    picks = {int(nz[np.argmax(gs[nz])]), int(nz[np.argmin(gs[nz])]), int(rng.choice(nz))}
    return sorted(picks)


@pytest.mark.parametrize("name", WORKLOADS)
def test_fullsize_sampled(name):
    dev = torch.device("cuda:0")
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, seed=0, device="cuda")
    gs_h = inp.group_sizes.numpy().astype(np.int64)
    gs = inp.group_sizes.to(dev)
    M, K, N, G = w.M, w.K, w.N, w.G
    bf16 = w.rule == "none"
    rule = w.rule
    s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
    sarg = s if rule == "static" else None
    ws = torch.empty(max(gm.gmm_workspace_bytes(op, M, K, N, G) for op in (0, 1, 2)), dtype=torch.uint8, device=dev)
    if bf16:
        codes, scales = inp.w, None
    else:
        codes, scales = gm.gmm_quantize_rhs(inp.w)
    out = gm.gmm_fwd(inp.lhs, codes, scales, gs, rule=rule, static_scale=sarg, ws=ws)
    dl = gm.gmm_dlhs(inp.dout, codes, scales, gs, ws=ws, rule="none" if bf16 else "dynamic")
    dw = gm.tgmm_drhs(inp.lhs, inp.dout, gs, rule=rule, static_scale=sarg, ws=ws)
    # merged gate|up workloads: the forward with SwiGLU fused, too
    sw = gm.gmm_fwd_swiglu(inp.lhs, codes, scales, gs, rule=rule, static_scale=sarg, ws=ws) if w.merged else None
    st, bits = gm.gmm_read_device_status(ws)
    assert st == 0, (st, bits)

    offs = np.concatenate([[0], np.cumsum(gs_h)])
    rng = np.random.default_rng(0)
    groups = pick_groups(gs_h, rng)
    qrule = {"static": oracle.Q_STATIC, "dynamic": oracle.Q_DYNAMIC, "none": None}[rule]
    for g in groups:
        a, b = int(offs[g]), int(offs[g + 1])
        wg = inp.w[g:g + 1].cpu()
        if not bf16:
            qr, sr = oracle.quantize_rhs(wg)
            assert np.array_equal(codes[g].cpu().numpy(), qr[0]), f"rhs codes of group {g}"
            assert np.array_equal(scales[g].cpu().numpy(), sr[0]), f"rhs scales of group {g}"
        rows = sorted({a, b - 1, int(rng.integers(a, b))})
        one = np.array([len(rows)], np.int32)
        lhs_r = inp.lhs[rows].cpu()
        dout_r = inp.dout[rows].cpu()
        if bf16:
            ref, ab = oracle.gmm_fwd_bf16(lhs_r, wg, one)
            assert_close(out[rows], ref, ab, f"{name} fwd g={g}")
            ref, ab = oracle.gmm_dlhs_bf16(dout_r, wg, one)
            assert_close(dl[rows], ref, ab, f"{name} dlhs g={g}")
        else:
            ref, ab = oracle.gmm_fwd(lhs_r, qrule, inp.static_scale, qr, sr, one)
            assert_close(out[rows], ref, ab, f"{name} fwd g={g}")
            if sw is not None:
                ref, terms = oracle.gmm_fwd_swiglu(lhs_r, qrule, inp.static_scale, qr, sr, one)
                assert_within(sw[rows], ref, swiglu_bound(sw.dtype, terms, ref), f"{name} swiglu g={g}")
            ref, ab = oracle.gmm_dlhs(dout_r, qr, sr, one)
            assert_close(dl[rows], ref, ab, f"{name} dlhs g={g}")
        # drhs rows (g, k): the whole group is the sub-problem
        ks = sorted({0, K - 1, int(rng.integers(0, K))})
        x_g, d_g = inp.lhs[a:b].cpu(), inp.dout[a:b].cpu()
        size = np.array([b - a], np.int32)
        if bf16:
            ref, ab = oracle.tgmm_drhs_bf16(x_g, d_g, size, sel=ks)
        else:
            ref, ab = oracle.tgmm_drhs(x_g, qrule, inp.static_scale, d_g, size, sel=ks)
        assert_close(dw[g, ks], ref, ab, f"{name} drhs g={g}")
    for g in np.flatnonzero(gs_h == 0)[:4]:
        assert not torch.any(dw[int(g)] != 0), f"empty group {g} has nonzero dW"
    tail = int(offs[-1])
    if tail < M:
        assert not torch.any(out[tail:] != 0) and not torch.any(dl[tail:] != 0)
        assert sw is None or not torch.any(sw[tail:] != 0)
    del inp, codes, scales, out, dl, dw, ws, sw
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["dsv3_up", "mixtral"])
def test_fullsize_blockwise_rhs_sampled(name):
    """Block-wise weight scales at full size: gmm_fwd with [G, K/128, N]
    scales and gmm_dlhs with [G, N/128, K] scales, checked on sampled rows
    (each row depends only on itself and its group's weights)."""
    dev = torch.device("cuda:0")
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, seed=0, device="cuda")
    gs_h = inp.group_sizes.numpy().astype(np.int64)
    gs = inp.group_sizes.to(dev)
    M, K, N, G = w.M, w.K, w.N, w.G
    s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
    sarg = s if w.rule == "static" else None
    ws = torch.empty(max(gm.gmm_workspace_bytes(op, M, K, N, G) for op in (0, 1)), dtype=torch.uint8, device=dev)
    c0, s0 = gm.gmm_quantize_rhs_blocks(inp.w, 0)
    out = gm.gmm_fwd(inp.lhs, c0, s0, gs, rule=w.rule, static_scale=sarg, ws=ws)
    del c0
    c1, s1 = gm.gmm_quantize_rhs_blocks(inp.w, 1)
    dl = gm.gmm_dlhs(inp.dout, c1, s1, gs, ws=ws)
    del c1
    st, bits = gm.gmm_read_device_status(ws)
    assert st == 0, (st, bits)
    offs = np.concatenate([[0], np.cumsum(gs_h)])
    rng = np.random.default_rng(1)
    qrule = {"static": oracle.Q_STATIC, "dynamic": oracle.Q_DYNAMIC}[w.rule]
    for g in pick_groups(gs_h, rng):
        a, b = int(offs[g]), int(offs[g + 1])
        wg = inp.w[g:g + 1].cpu()
        qr0, sr0 = oracle.quantize_rhs_blocks(wg, 0)
        qr1, sr1 = oracle.quantize_rhs_blocks(wg, 1)
        assert np.array_equal(s0[g].cpu().numpy(), sr0[0]) and np.array_equal(s1[g].cpu().numpy(), sr1[0])
        rows = sorted({a, b - 1, int(rng.integers(a, b))})
        one = np.array([len(rows)], np.int32)
        ref, ab = oracle.gmm_fwd_blockwise(inp.lhs[rows].cpu(), qrule, inp.static_scale, qr0, sr0, one)
        assert_close(out[rows], ref, ab, f"{name} blockwise fwd g={g}")
        ref, ab = oracle.gmm_dlhs_blockwise(inp.dout[rows].cpu(), qr1, sr1, one)
        assert_close(dl[rows], ref, ab, f"{name} blockwise dlhs g={g}")
    del inp, out, dl, ws, s0, s1
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["mixtral", "dsv3_up", "ragged"])
def test_fullsize_backward_equals_the_two_calls(name):
    """The fused backward at full size: dlhs and dW equal the separate calls
    bit for bit (same codes from one read of dout)."""
    dev = torch.device("cuda:0")
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, seed=0, device="cuda")
    gs = inp.group_sizes.to(dev)
    M, K, N, G = w.M, w.K, w.N, w.G
    s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
    sarg = s if w.rule == "static" else None
    codes, scales = gm.gmm_quantize_rhs(inp.w)
    del inp.w
    ws = torch.empty(gm.gmm_workspace_bytes(3, M, K, N, G), dtype=torch.uint8, device=dev)
    dl, dw = gm.gmm_backward(inp.lhs, inp.dout, codes, scales, gs, rule=w.rule, static_scale=sarg, ws=ws)
    st, bits = gm.gmm_read_device_status(ws)
    assert st == 0, (st, bits)
    assert torch.equal(dl, gm.gmm_dlhs(inp.dout, codes, scales, gs, ws=ws))
    del dl
    dw1 = gm.tgmm_drhs(inp.lhs, inp.dout, gs, rule=w.rule, static_scale=sarg, ws=ws)
    assert torch.equal(dw, dw1)
    del inp, dw, dw1, ws, codes, scales
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["mixtral", "dsv3_up", "ragged"])
def test_fullsize_activation_codes_bit_exact(name):
    """Activation codes and scales at full size, bit for bit against the oracle:
    the lhs along K (the forward's operand, the workload's rule), dout along N
    with the weight column scale folded in (the dlhs operand), and both per
    128-row chunk of each group (the tgmm operands).  Quantization is local to
    a row (axis 1) or to a group's rows (axis 0), so sampled rows and sampled
    groups are exact sub-problems; every group's first and last row is among
    the sampled rows."""
    dev = torch.device("cuda:0")
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, seed=0, device="cuda")
    gs_h = inp.group_sizes.numpy().astype(np.int64)
    gs = inp.group_sizes.to(dev)
    M = w.M
    static = w.rule == "static"
    qrule = oracle.Q_STATIC if static else oracle.Q_DYNAMIC
    s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
    sarg = s if static else None
    offs = np.concatenate([[0], np.cumsum(gs_h)])
    rng = np.random.default_rng(2)
    nz = np.flatnonzero(gs_h > 0)
    rows = sorted(set(offs[nz].tolist()) | set((offs[nz + 1] - 1).tolist())
                  | set(rng.integers(0, M, 256).tolist()))

    # axis 1: lhs rows (the forward's operand)
    codes, scales = gm.gmm_quantize(inp.lhs, w.rule, axis=1, static_scale=sarg)
    qc, qs, _ = oracle.quantize_rows(inp.lhs[rows].cpu(), qrule, inp.static_scale)
    assert np.array_equal(codes[rows].cpu().numpy(), qc), f"{name}: lhs row codes"
    if not static:
        assert np.array_equal(scales[:, rows].cpu().numpy().T, qs), f"{name}: lhs row scales"
    del codes, scales

    # axis 1 with the weight column scale folded in: dout rows (the dlhs operand)
    _, wscales = gm.gmm_quantize_rhs(inp.w)
    inp.w = None
    codes, scales = gm.gmm_quantize(inp.dout, "dynamic", axis=1, group_sizes=gs, col_scale=wscales)
    sr = wscales.cpu().numpy()
    for g in pick_groups(gs_h, rng):
        a, b = int(offs[g]), int(offs[g + 1])
        rg = [r for r in rows if a <= r < b]
        qc, qs = oracle.quantize_rows_scaled(inp.dout[rg].cpu(), sr[g:g + 1], np.array([len(rg)], np.int32))
        assert np.array_equal(codes[rg].cpu().numpy(), qc), f"{name}: dout row codes, group {g}"
        assert np.array_equal(scales[:, rg].cpu().numpy().T, qs), f"{name}: dout row scales, group {g}"
    del codes, scales

    # axis 0: 128-row chunks of each group (the tgmm operands)
    first_chunk = np.concatenate([[0], np.cumsum((gs_h + 127) // 128)])
    for x, rule_x, what in ((inp.lhs, w.rule, "lhs"), (inp.dout, "dynamic", "dout")):
        ct, cs = gm.gmm_quantize(x, rule_x, axis=0, static_scale=sarg if rule_x == "static" else None,
                                 group_sizes=gs)
        for g in pick_groups(gs_h, rng):
            a, b = int(offs[g]), int(offs[g + 1])
            qc, qs = oracle.quantize_chunks(x[a:b].cpu(), oracle.Q_STATIC if rule_x == "static" else oracle.Q_DYNAMIC,
                                            inp.static_scale, np.array([b - a], np.int32))
            j0 = int(first_chunk[g])
            for c in range((b - a + 127) // 128):
                n = min(128, b - a - 128 * c)
                got = ct[j0 + c, :, :n].cpu().numpy().T
                assert np.array_equal(got, qc[128 * c:128 * c + n]), f"{name}: {what} chunk {c} of group {g}"
                assert not ct[j0 + c, :, n:].any(), f"{name}: {what} chunk padding of group {g}"
            assert np.array_equal(cs[j0:j0 + len(qs)].cpu().numpy(), qs), f"{name}: {what} chunk scales, group {g}"
        del ct, cs
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["mixtral", "dsv3_up"])
def test_fullsize_repeatable_and_tile_independent(name):
    """Every output is accumulated in a fixed order (two MMA-issuing threads,
    each unit or half tile owned by one of them), so repeated calls give the
    same bits, and one-CTA tiles give the same bits as the automatic choice
    (CTA pairs for the static forward and the tgmm here).  A race between the
    issuers, the loads and the epilogue would show up as a difference."""
    dev = torch.device("cuda:0")
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, seed=1, device="cuda")
    gs = inp.group_sizes.to(dev)
    s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
    sarg = s if w.rule == "static" else None
    codes, scales = gm.gmm_quantize_rhs(inp.w)

    def run():
        out = gm.gmm_fwd(inp.lhs, codes, scales, gs, rule=w.rule, static_scale=sarg)
        dl, dw = gm.gmm_backward(inp.lhs, inp.dout, codes, scales, gs, rule=w.rule, static_scale=sarg)
        torch.cuda.synchronize()
        return out, dl, dw

    ref = run()
    for label in ("repeat 1", "repeat 2", "one-CTA tiles"):
        try:
            if label == "one-CTA tiles":
                gm.gmm_set_tiles("one_cta")
            got = run()
        finally:
            gm.gmm_set_tiles("auto")
        for what, a, b in zip(("fwd", "dlhs", "drhs"), ref, got):
            assert torch.equal(a, b), f"{name} {what}: {label} differs"
        del got
