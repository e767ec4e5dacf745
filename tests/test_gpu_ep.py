"""Expert-parallel forward on one GPU (one rank: the exchange is the
identity), CUDA path vs the oracle: rows gathered by expert (E4M3 codes),
gmm_fwd on the local experts, results returned and summed per token with the
routing weights.  Also the row gather and the combine on their own,
including out-of-range indices and slots.

Tolerance: each term w * h of a token carries the forward's bound
(2e-3 * A, plus 2^-8 |h| for the bf16 gmm output) times |w|; the fp32 sum adds
k * 2^-24 of the magnitudes and a bf16 result its own 2^-8 |y|.
"""
import numpy as np
import pytest
import torch

import moe_fp8_grouped_b200 as gm
import oracle
from moe_fp8_grouped_b200 import ep
from parity import assert_close, assert_within

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available()
    return torch.device("cuda:0")


def test_gather_rows(dev):
    src = torch.arange(5 * 48, dtype=torch.uint8, device=dev).view(5, 48)
    idx = torch.tensor([4, 0, -1, 2, 5, 2], dtype=torch.int32, device=dev)
    out = ep.gather_rows(src, idx)
    want = torch.stack([src[4], src[0], torch.zeros_like(src[0]), src[2], torch.zeros_like(src[0]), src[2]])
    assert torch.equal(out, want)


def test_combine_rows(dev):
    g = torch.Generator().manual_seed(0)
    rows = torch.randn(7, 64, generator=g).bfloat16().to(dev)
    slot = torch.tensor([[0, 3], [6, -1], [2, 2], [9, 1]], dtype=torch.int32, device=dev)
    w = torch.rand(4, 2, generator=g).to(dev)
    y = ep.combine_rows(rows, slot, w, out_dtype=torch.float32)
    r = rows.float()
    want = torch.stack([w[0, 0] * r[0] + w[0, 1] * r[3], w[1, 0] * r[6], w[2, 0] * r[2] + w[2, 1] * r[2],
                        w[3, 1] * r[1]])
    assert torch.allclose(y, want, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("T,E,k,K,N", [(96, 8, 2, 256, 384), (40, 4, 3, 512, 256), (5, 16, 2, 128, 128)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_ep_moe_fwd_single_rank(dev, T, E, k, K, N, out_dtype):
    g = torch.Generator().manual_seed(T + E)
    x = torch.randn(T, K, generator=g).bfloat16()
    w = (torch.randn(E, K, N, generator=g) * 0.02).bfloat16()
    ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)])
    wts = torch.softmax(torch.randn(T, k, generator=g), dim=1)
    s_val = 4.0 / 448.0
    s = torch.tensor([s_val], dtype=torch.float32, device=dev)
    codes, scales = gm.gmm_quantize_rhs(w.to(dev))
    xq, _ = gm.gmm_quantize(x.to(dev), "static", axis=1, static_scale=s)
    y = ep.ep_moe_fwd(xq, s, ids.to(dev), wts.to(dev), codes, scales, out_dtype=out_dtype)
    torch.cuda.synchronize()
    # oracle: every token through every expert it chose, combined in fp64
    qr, sr = oracle.quantize_rhs(w)
    ref = np.zeros((T, N))
    bound = np.zeros((T, N))
    mag = np.zeros((T, N))
    one = np.array([T], np.int32)
    for e in range(E):
        h, ab = oracle.gmm_fwd(x, oracle.Q_STATIC, s_val, qr[e:e + 1], sr[e:e + 1], one)
        for j in range(k):
            sel = (ids[:, j] == e).numpy()
            wj = wts[sel, j].double().numpy()[:, None]
            ref[sel] += wj * h[sel]
            bound[sel] += np.abs(wj) * (2e-3 * ab[sel] + 2.0 ** -8 * np.abs(h[sel]))
            mag[sel] += np.abs(wj * h[sel])
    bound += k * 2.0 ** -23 * mag + (2.0 ** -8 * np.abs(ref) if out_dtype == torch.bfloat16 else 0.0)
    assert_within(y, ref, bound, f"ep_moe_fwd T={T} E={E} k={k}")


def test_ep_forward_graph_replays_the_eager_result(dev):
    g = torch.Generator().manual_seed(5)
    T, E, k, K, N = 64, 8, 2, 256, 256
    x = torch.randn(T, K, generator=g).bfloat16().to(dev)
    w = (torch.randn(E, K, N, generator=g) * 0.02).bfloat16().to(dev)
    ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(dev)
    wts = torch.softmax(torch.randn(T, k, generator=g), dim=1).to(dev)
    s = torch.tensor([4.0 / 448.0], device=dev)
    codes, scales = gm.gmm_quantize_rhs(w)
    xq, _ = gm.gmm_quantize(x, "static", axis=1, static_scale=s)
    eager = ep.ep_moe_fwd(xq, s, ids, wts, codes, scales)
    graph = ep.EPForwardGraph(xq, s, ids, wts, codes, scales)
    assert torch.equal(graph.replay(), eager)
    # new routing weights copied into the captured buffer change the result
    wts.copy_(wts.flip(1))
    assert torch.equal(graph.replay(), ep.ep_moe_fwd(xq, s, ids, wts, codes, scales))


@pytest.mark.parametrize("T,E,k,K,N", [(96, 8, 2, 256, 384), (33, 4, 3, 384, 256)])
def test_ep_moe_bwd_single_rank(dev, T, E, k, K, N):
    """dx and the experts' dW of the one-rank expert-parallel backward against
    the oracle: every routed row's gradient dh = bf16(w * dy) goes through the
    oracle's dlhs and tgmm for its expert; dx sums a token's dlhs rows."""
    g = torch.Generator().manual_seed(100 + T)
    x = torch.randn(T, K, generator=g).bfloat16()
    w = (torch.randn(E, K, N, generator=g) * 0.02).bfloat16()
    dy = torch.randn(T, N, generator=g).bfloat16()
    ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)])
    wts = torch.softmax(torch.randn(T, k, generator=g), dim=1)
    s_val = 4.0 / 448.0
    s = torch.tensor([s_val], dtype=torch.float32, device=dev)
    codes, scales = gm.gmm_quantize_rhs(w.to(dev))
    xq, _ = gm.gmm_quantize(x.to(dev), "static", axis=1, static_scale=s)
    dx, dw = ep.ep_moe_bwd(xq, s, ids.to(dev), wts.to(dev), dy.to(dev), codes, scales, dx_dtype=torch.float32)
    torch.cuda.synchronize()
    qr, sr = oracle.quantize_rhs(w)
    ref_dx = np.zeros((T, K))
    bound_dx = np.zeros((T, K))
    mag = np.zeros((T, K))
    for e in range(E):
        rows = [(t, j) for t in range(T) for j in range(k) if int(ids[t, j]) == e]
        if not rows:
            assert not dw[e].any(), f"expert {e} without rows has nonzero dW"
            continue
        ts = [t for t, _ in rows]
        dh = torch.stack([(dy[t].float() * wts[t, j]).bfloat16() for t, j in rows])
        one = np.array([len(rows)], np.int32)
        dl, ab = oracle.gmm_dlhs(dh, qr[e:e + 1], sr[e:e + 1], one)
        for i, t in enumerate(ts):
            ref_dx[t] += dl[i]
            bound_dx[t] += 2e-3 * ab[i] + 2.0 ** -8 * np.abs(dl[i])
            mag[t] += np.abs(dl[i])
        ref_w, ab_w = oracle.tgmm_drhs(x[ts], oracle.Q_STATIC, s_val, dh, one)
        assert_close(dw[e:e + 1], ref_w, ab_w, f"ep dW expert {e}")
    assert_within(dx, ref_dx, bound_dx + k * 2.0 ** -23 * mag + 1e-30, f"ep dx T={T} E={E} k={k}")


def test_gather_scale_rows(dev):
    src = torch.randn(6, 40).bfloat16().to(dev)
    idx = torch.tensor([5, -1, 0, 2], dtype=torch.int32, device=dev)
    sc = torch.tensor([0.5, 3.0, -1.25, 0.1], device=dev)
    out = ep.gather_scale_rows(src, idx, sc)
    s = src.float()
    want = torch.stack([(s[5] * 0.5), torch.zeros(40, device=dev), (s[0] * -1.25), (s[2] * sc[3])]).bfloat16()
    assert torch.equal(out, want)


@pytest.mark.parametrize("P,El", [(1, 8), (2, 4), (3, 16), (8, 128), (4, 1)])
def test_ep_local_order_kernel_matches_host_indices(dev, P, El):
    """gmm_ep_local_order (the device regrouping of arrived rows) gives the
    same permutation, inverse and group sizes as the host computation, for
    counts with empty blocks, and runs without a host synchronization."""
    g = torch.Generator().manual_seed(P * 100 + El)
    cnt = torch.randint(0, 40, (P, El), generator=g, dtype=torch.int64)
    cnt[torch.rand(P, El, generator=g) < 0.3] = 0
    total = int(cnt.sum())
    perm_h, inv_h, gsz_h = ep.local_order(cnt, total)
    perm_d, inv_d, gsz_d = ep.local_order(cnt.to(dev), total)
    assert perm_d.cpu().tolist() == perm_h.tolist()
    assert inv_d.cpu().tolist() == inv_h.tolist()
    assert gsz_d.cpu().tolist() == gsz_h.tolist()
