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
from parity import assert_within

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
