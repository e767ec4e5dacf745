"""Pins for the oracle's bf16-family passes (no quantization): the forward
gmm, dlhs gmm and tgmm drhs with bf16 operands and fp64 sums.  They are the
checkers of the same-shape bf16 gmm built on the same kernel family, so they
are pinned here against routes that do not go through their own loops:

- a hand-worked example whose products and sums are small integers;
- numpy fp64 matmul of the exactly widened bf16 operands, group by group
  (a library primitive);
- G = 1 as one ordinary GEMM;
- empty groups give zero dW and unrouted rows give zero rows;
- group sizes past M are clamped;
- dlhs and drhs equal torch.autograd of the fp64 forward (no quantization, so
  only summation order separates them);
- the merged gate|up identity: the forward and drhs split exactly into the
  two separate calls, dlhs is their sum;
- absum is sum_k |a_k b_k|, i.e. |x| @ |w| group by group.

Each pin is written as a function of the oracle library so that it can also
run against builds of the oracle's C source with a plausible mistake planted
(a transposed index, a sum that runs past its group, a dropped row, a missing
absolute value); every such build must fail at least one pin.

Sources: "Support quantization for tokamax gmm v2" (maxtext PR #4451),
Description (fwd gmm, dlhs gmm, drhs tgmm) and review thread on ops.py (dlhs
is the gmm with transpose_rhs flipped); "FP8 Megablox for batch split"
(maxtext PR #3770), Description (W0 | W1 merged along the local N).
"""
import numpy as np
import pytest
import torch

import oracle
from moe_fp8_grouped_b200 import synth

REL = 1e-12  # fp64 sums of exact products: only the summation order differs


def wide(t):
    """bf16 tensor -> float64 numpy (exact)."""
    return t.to(torch.float64).numpy()


def offsets(sizes, M):
    return oracle.plan(sizes, M)[0]


def close(a, b, ab, what):
    scale = max(float(np.max(ab)), 1e-300)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= REL * scale, f"{what}: max error {err} against {REL} * {scale}"


CASES = [
    # G, M, K, N, sizes  (K != N everywhere, so a transposed index cannot pass)
    (4, 200, 256, 384, [60, 0, 100, 40]),
    (3, 300, 384, 128, [1, 129, 150]),  # sums to 280: 20 unrouted rows
    (5, 260, 128, 256, [0, 70, 0, 130, 60]),
]


# ------------------------------------------------------------------ pins

def pin_hand_example(L):
    """lhs rows (1, 2), (3, 4), (5, 6); W0 = I, W1 = [[2, 0], [0, -1]];
    sizes [1, 2]: row 0 uses W0, rows 1-2 use W1."""
    lhs = torch.tensor([[1, 2], [3, 4], [5, 6]], dtype=torch.bfloat16)
    w = torch.tensor([[[1, 0], [0, 1]], [[2, 0], [0, -1]]], dtype=torch.bfloat16)
    dout = torch.tensor([[1, -1], [2, 0], [0, 3]], dtype=torch.bfloat16)
    sizes = np.array([1, 2], np.int32)
    out, ab = oracle.gmm_fwd_bf16(lhs, w, sizes, _L=L)
    assert np.array_equal(out, [[1, 2], [6, -4], [10, -6]]), out
    assert np.array_equal(ab, [[1, 2], [6, 4], [10, 6]]), ab
    # dlhs[m, k] = sum_n dout[m, n] W[g, k, n]
    dl, _ = oracle.gmm_dlhs_bf16(dout, w, sizes, _L=L)
    assert np.array_equal(dl, [[1, -1], [4, 0], [0, -3]]), dl
    # dW[g, k, n] = sum_{m in g} lhs[m, k] dout[m, n]
    dw, dab = oracle.tgmm_drhs_bf16(lhs, dout, sizes, _L=L)
    assert np.array_equal(dw[0], [[1, -1], [2, -2]]), dw[0]
    assert np.array_equal(dw[1], [[6, 15], [8, 18]]), dw[1]
    assert np.array_equal(dab[1], [[6, 15], [8, 18]]), dab[1]


def pin_numpy_matmul(L):
    for G, M, K, N, sizes in CASES:
        inp = synth.small_case(G, M, K, N, seed=61, sizes=sizes)
        x, w, d = wide(inp.lhs), wide(inp.w), wide(inp.dout)
        offs = offsets(inp.group_sizes, M)
        ref_f, ref_fa = np.zeros((M, N)), np.zeros((M, N))
        ref_l, ref_la = np.zeros((M, K)), np.zeros((M, K))
        ref_w, ref_wa = np.zeros((G, K, N)), np.zeros((G, K, N))
        for g in range(G):
            a, b = offs[g], offs[g + 1]
            ref_f[a:b], ref_fa[a:b] = x[a:b] @ w[g], np.abs(x[a:b]) @ np.abs(w[g])
            ref_l[a:b], ref_la[a:b] = d[a:b] @ w[g].T, np.abs(d[a:b]) @ np.abs(w[g]).T
            ref_w[g], ref_wa[g] = x[a:b].T @ d[a:b], np.abs(x[a:b]).T @ np.abs(d[a:b])
        out, ab = oracle.gmm_fwd_bf16(inp.lhs, inp.w, inp.group_sizes, _L=L)
        close(out, ref_f, ref_fa, "fwd vs numpy")
        close(ab, ref_fa, ref_fa, "fwd absum vs |x| @ |w|")
        dl, dab = oracle.gmm_dlhs_bf16(inp.dout, inp.w, inp.group_sizes, _L=L)
        close(dl, ref_l, ref_la, "dlhs vs numpy")
        close(dab, ref_la, ref_la, "dlhs absum")
        dw, wab = oracle.tgmm_drhs_bf16(inp.lhs, inp.dout, inp.group_sizes, _L=L)
        close(dw, ref_w, ref_wa, "drhs vs numpy")
        close(wab, ref_wa, ref_wa, "drhs absum")


def pin_one_group_is_one_gemm(L):
    inp = synth.small_case(1, 96, 256, 128, seed=62, sizes=[96])
    out, ab = oracle.gmm_fwd_bf16(inp.lhs, inp.w, inp.group_sizes, _L=L)
    ref = torch.from_numpy(wide(inp.lhs)) @ torch.from_numpy(wide(inp.w[0]))
    close(out, ref.numpy(), ab, "G=1 fwd vs one GEMM")
    dw, wab = oracle.tgmm_drhs_bf16(inp.lhs, inp.dout, inp.group_sizes, _L=L)
    ref = torch.from_numpy(wide(inp.lhs)).T @ torch.from_numpy(wide(inp.dout))
    close(dw[0], ref.numpy(), wab[0], "G=1 drhs vs one GEMM")


def pin_empty_groups_and_unrouted_rows(L):
    inp = synth.small_case(4, 100, 128, 256, seed=63, sizes=[30, 0, 40, 0])  # rows 70.. unrouted
    out, ab = oracle.gmm_fwd_bf16(inp.lhs, inp.w, inp.group_sizes, _L=L)
    assert np.all(out[70:] == 0) and np.all(ab[70:] == 0)
    assert np.all(np.any(out[:70] != 0, axis=1))
    dl, _ = oracle.gmm_dlhs_bf16(inp.dout, inp.w, inp.group_sizes, _L=L)
    assert np.all(dl[70:] == 0) and np.all(np.any(dl[:70] != 0, axis=1))
    dw, wab = oracle.tgmm_drhs_bf16(inp.lhs, inp.dout, inp.group_sizes, _L=L)
    assert np.all(dw[1] == 0) and np.all(dw[3] == 0) and np.all(wab[1] == 0) and np.all(wab[3] == 0)
    assert np.any(dw[0] != 0) and np.any(dw[2] != 0)


def pin_sizes_past_M_are_clamped(L):
    a = synth.small_case(3, 50, 128, 256, seed=64, sizes=[20, 40, 30])
    b = synth.small_case(3, 50, 128, 256, seed=64, sizes=[20, 30, 0])
    for f in (lambda i: oracle.gmm_fwd_bf16(i.lhs, i.w, i.group_sizes, _L=L)[0],
              lambda i: oracle.gmm_dlhs_bf16(i.dout, i.w, i.group_sizes, _L=L)[0],
              lambda i: oracle.tgmm_drhs_bf16(i.lhs, i.dout, i.group_sizes, _L=L)[0]):
        assert np.array_equal(f(a), f(b))


def pin_gradients_are_autograd_of_forward(L):
    inp = synth.small_case(3, 160, 256, 384, seed=65, sizes=[70, 10, 60])  # 20 unrouted rows
    M = inp.lhs.shape[0]
    x = torch.tensor(wide(inp.lhs), requires_grad=True)
    W = torch.tensor(wide(inp.w), requires_grad=True)
    offs = offsets(inp.group_sizes, M)
    ys = [x[offs[g]:offs[g + 1]] @ W[g] for g in range(3)]
    y = torch.cat(ys + [torch.zeros(M - offs[3], W.shape[2], dtype=torch.float64)])
    y.backward(torch.tensor(wide(inp.dout)))
    dl, dab = oracle.gmm_dlhs_bf16(inp.dout, inp.w, inp.group_sizes, _L=L)
    close(dl, x.grad.numpy(), dab, "dlhs vs autograd")
    dw, wab = oracle.tgmm_drhs_bf16(inp.lhs, inp.dout, inp.group_sizes, _L=L)
    close(dw, W.grad.numpy(), wab, "drhs vs autograd")


def pin_merged_gate_up(L):
    inp = synth.small_case(3, 120, 256, 512, seed=66, sizes=[50, 0, 70])
    w0, w1 = inp.w[:, :, :256].contiguous(), inp.w[:, :, 256:].contiguous()
    d0, d1 = inp.dout[:, :256].contiguous(), inp.dout[:, 256:].contiguous()
    gs = inp.group_sizes
    f, _ = oracle.gmm_fwd_bf16(inp.lhs, inp.w, gs, _L=L)
    f0, _ = oracle.gmm_fwd_bf16(inp.lhs, w0, gs, _L=L)
    f1, _ = oracle.gmm_fwd_bf16(inp.lhs, w1, gs, _L=L)
    assert np.array_equal(f, np.concatenate([f0, f1], axis=1))
    r, _ = oracle.tgmm_drhs_bf16(inp.lhs, inp.dout, gs, _L=L)
    r0, _ = oracle.tgmm_drhs_bf16(inp.lhs, d0, gs, _L=L)
    r1, _ = oracle.tgmm_drhs_bf16(inp.lhs, d1, gs, _L=L)
    assert np.array_equal(r, np.concatenate([r0, r1], axis=2))
    dl, ab = oracle.gmm_dlhs_bf16(inp.dout, inp.w, gs, _L=L)
    dl0, _ = oracle.gmm_dlhs_bf16(d0, w0, gs, _L=L)
    dl1, _ = oracle.gmm_dlhs_bf16(d1, w1, gs, _L=L)
    close(dl, dl0 + dl1, ab, "dlhs merged = sum of the separate calls")


def pin_row_and_entry_selection(L):
    inp = synth.small_case(3, 140, 256, 128, seed=67, sizes=[40, 60, 30])
    full, _ = oracle.gmm_fwd_bf16(inp.lhs, inp.w, inp.group_sizes, _L=L)
    sub, _ = oracle.gmm_fwd_bf16(inp.lhs, inp.w, inp.group_sizes, rows=[139, 3, 41, 100], _L=L)
    assert np.array_equal(sub, full[[139, 3, 41, 100]])
    fd, _ = oracle.gmm_dlhs_bf16(inp.dout, inp.w, inp.group_sizes, _L=L)
    sd, _ = oracle.gmm_dlhs_bf16(inp.dout, inp.w, inp.group_sizes, rows=[0, 99, 130], _L=L)
    assert np.array_equal(sd, fd[[0, 99, 130]])
    dw, _ = oracle.tgmm_drhs_bf16(inp.lhs, inp.dout, inp.group_sizes, _L=L)
    sel = [2 * 256 + 7, 255, 256 + 1]
    sw, _ = oracle.tgmm_drhs_bf16(inp.lhs, inp.dout, inp.group_sizes, sel=sel, _L=L)
    assert np.array_equal(sw, dw.reshape(-1, 128)[sel])


PINS = [pin_hand_example, pin_numpy_matmul, pin_one_group_is_one_gemm, pin_empty_groups_and_unrouted_rows,
        pin_sizes_past_M_are_clamped, pin_gradients_are_autograd_of_forward, pin_merged_gate_up,
        pin_row_and_entry_selection]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin_holds_for_the_oracle(pin):
    pin(oracle.lib())


# --------------------------------------------------------- planted mistakes

# (function, text in its body, replacement): each a plausible slip, each in
# bounds for every case above (no planted read leaves its array)
MUTANTS = {
    "fwd_lhs_read_transposed": ("gmo_gmm_fwd_bf16", "lhs[m * K + k]", "lhs[k * M + m]"),
    "fwd_absum_without_abs": ("gmo_gmm_fwd_bf16", "a[n] += fabs(p);", "a[n] += p;"),
    "dlhs_rhs_index_transposed": ("gmo_gmm_dlhs_bf16", "gmo_bf16_to_f32(wrow[n])",
                                  "gmo_bf16_to_f32(w[(int64_t)g * K * N + n * K + k])"),
    "dlhs_dout_column_reversed": ("gmo_gmm_dlhs_bf16", "dout[m * N + n]", "dout[m * N + (N - 1 - n)]"),
    "drhs_sums_past_its_group": ("gmo_tgmm_drhs_bf16", "m < offs[g + 1]", "m < offs[G]"),
    "drhs_drops_first_row": ("gmo_tgmm_drhs_bf16", "m = offs[g];", "m = offs[g] + 1;"),
    "drhs_dout_row_shifted": ("gmo_tgmm_drhs_bf16", "dout[m * N + n]", "dout[(m > 0 ? m - 1 : m) * N + n]"),
}


def plant(src: str, func: str, old: str, new: str) -> str:
    start = src.index(f"void {func}(")
    end = src.find("\nvoid ", start + 1)
    end = len(src) if end < 0 else end
    body = src[start:end]
    assert body.count(old) == 1, f"{old!r} occurs {body.count(old)} times in {func}"
    return src[:start] + body.replace(old, new) + src[end:]


@pytest.fixture(scope="module")
def mutant_libs(tmp_path_factory):
    d = str(tmp_path_factory.mktemp("oracle_mutants"))
    src = oracle.source_text()
    return {name: oracle.load_variant(oracle.build_variant(plant(src, *m), d, name))
            for name, m in MUTANTS.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_fails_a_pin(name, mutant_libs):
    L = mutant_libs[name]
    failed = []
    for pin in PINS:
        try:
            pin(L)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} passed every pin"
