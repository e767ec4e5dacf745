"""Seeded synthetic inputs for the FP8 grouped matmul workloads.

This module draws random numbers only: group sizes, bf16 activations, bf16
expert weights, bf16 output gradients and the static activation scale.  It
holds none of the method's arithmetic (no quantization, no matmul), so both
the CUDA path and the CPU oracle can take their inputs from it.

Workloads (sizes from the MoE shapes the gmm pages discuss: Mixtral-like,
DeepSeek-V3-shaped, expert-parallel-shrunk and a ragged stress case):

=============  ===  =====  ====  =====  ========  ==========================
name            G     M      K     N     lhs rule  routing
=============  ===  =====  ====  =====  ========  ==========================
tiny             8    256   512    512  static    uniform over 7, group 3 empty
mixtral          8  16384  4096  28672  static    8192 tokens x top-2 distinct
dsv3_up        256  32768  7168   4096  dynamic   Zipf(1.2) over a permutation
dsv3_down      256  32768  2048   7168  dynamic   Zipf(1.2) over a permutation
ep_merged       32   8192  7168    512  static    uniform
ep_separate     32   8192  7168    256  static    uniform (run twice: W0, W1)
ragged         256  65536  2048   7168  dynamic   77 empty, one group 16384
=============  ===  =====  ====  =====  ========  ==========================

Distributions: lhs and dout ~ N(0, 1), weights ~ N(0, 0.02), all drawn in
fp32 and rounded to bf16.  Static per-tensor lhs scale 4/448 (a fixed
calibration range of +-4).  Draw order per workload: group sizes, lhs, rhs,
dout, from one ``torch.Generator`` seeded with ``seed``.
"""
from __future__ import annotations

import dataclasses

import torch

STATIC_SCALE = 4.0 / 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    G: int
    M: int
    K: int
    N: int
    rule: str  # "static" | "dynamic" | "none" (bf16 family)
    routing: str
    tokens: int = 0
    topk: int = 0
    merged: bool = False  # N holds the gate and up projections side by side (N = 2F)

    @property
    def flops_per_pass(self) -> int:
        """Algorithmic FLOPs of one pass when every row is routed: 2*M*K*N."""
        return 2 * self.M * self.K * self.N


WORKLOADS = {
    "tiny": Workload("tiny", 8, 256, 512, 512, "static", "uniform_empty3", merged=True),
    "mixtral": Workload("mixtral", 8, 16384, 4096, 28672, "static", "topk_uniform", tokens=8192, topk=2,
                        merged=True),
    "dsv3_up": Workload("dsv3_up", 256, 32768, 7168, 4096, "dynamic", "zipf", tokens=4096, topk=8, merged=True),
    "dsv3_down": Workload("dsv3_down", 256, 32768, 2048, 7168, "dynamic", "zipf", tokens=4096, topk=8),
    "ep_merged": Workload("ep_merged", 32, 8192, 7168, 512, "static", "uniform", merged=True),
    "ep_separate": Workload("ep_separate", 32, 8192, 7168, 256, "static", "uniform"),
    "ragged": Workload("ragged", 256, 65536, 2048, 7168, "dynamic", "ragged_stress"),
    "ragged_bf16": Workload("ragged_bf16", 256, 65536, 2048, 7168, "none", "ragged_stress"),
}


def with_rows(w: Workload, M: int) -> Workload:
    """The same workload with M rows (tokens scaled alike), e.g. a smaller
    case of the same shape for profiler captures."""
    tokens = M // w.topk if w.topk else 0
    return dataclasses.replace(w, name=f"{w.name}_m{M}", M=M, tokens=tokens)


def with_cols(w: Workload, N: int) -> Workload:
    """The same workload with N output columns."""
    return dataclasses.replace(w, name=f"{w.name}_n{N}", N=N)


def group_sizes(w: Workload, gen: torch.Generator) -> torch.Tensor:
    """int32 [G] row counts per expert, summing to M (CPU)."""
    G, M = w.G, w.M
    if w.routing == "uniform_empty3":
        p = torch.ones(G, dtype=torch.float64)
        p[3] = 0.0
        idx = torch.multinomial(p, M, replacement=True, generator=gen)
        return torch.bincount(idx, minlength=G).to(torch.int32)
    if w.routing == "uniform":
        idx = torch.multinomial(torch.ones(G, dtype=torch.float64), M, replacement=True, generator=gen)
        return torch.bincount(idx, minlength=G).to(torch.int32)
    if w.routing == "topk_uniform":
        # each token picks topk distinct experts uniformly: a random permutation per token
        keys = torch.rand(w.tokens, G, generator=gen)
        picks = keys.argsort(dim=1)[:, : w.topk].reshape(-1)
        return torch.bincount(picks, minlength=G).to(torch.int32)
    if w.routing == "zipf":
        ranks = torch.arange(1, G + 1, dtype=torch.float64)
        p_rank = ranks.pow(-1.2)
        perm = torch.randperm(G, generator=gen)
        p = torch.empty(G, dtype=torch.float64)
        p[perm] = p_rank
        idx = torch.multinomial(p, M, replacement=True, generator=gen)
        return torch.bincount(idx, minlength=G).to(torch.int32)
    if w.routing == "ragged_stress":
        n_empty = round(0.3 * G)
        perm = torch.randperm(G, generator=gen)
        empty, hot, rest = perm[:n_empty], perm[n_empty], perm[n_empty + 1:]
        sizes = torch.zeros(G, dtype=torch.int64)
        sizes[hot] = M // 4
        idx = torch.multinomial(torch.ones(rest.numel(), dtype=torch.float64), M - M // 4, replacement=True,
                                generator=gen)
        sizes[rest] = torch.bincount(idx, minlength=rest.numel())
        del empty
        return sizes.to(torch.int32)
    raise ValueError(f"unknown routing {w.routing}")


def _normal(shape, std, gen, device):
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


@dataclasses.dataclass
class Inputs:
    workload: Workload
    group_sizes: torch.Tensor  # int32 [G], CPU
    lhs: torch.Tensor  # bf16 [M, K]
    w: torch.Tensor  # bf16 [G, K, N]
    dout: torch.Tensor  # bf16 [M, N]
    static_scale: float


def make_inputs(w: Workload | str, seed: int = 0, device: str = "cpu", n_override: int | None = None) -> Inputs:
    """Draw one batch for workload ``w``.  Large tensors are drawn on ``device``
    (a CUDA generator there), group sizes always on the CPU generator."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if n_override is not None:
        w = dataclasses.replace(w, N=n_override)
    gcpu = torch.Generator().manual_seed(seed)
    gs = group_sizes(w, gcpu)
    if device == "cpu":
        gdev = gcpu
    else:
        gdev = torch.Generator(device=device).manual_seed(seed + 1)
    lhs = _normal((w.M, w.K), 1.0, gdev, device)
    wt = _normal((w.G, w.K, w.N), 0.02, gdev, device)
    dout = _normal((w.M, w.N), 1.0, gdev, device)
    return Inputs(w, gs, lhs, wt, dout, STATIC_SCALE)


def small_case(G: int, M: int, K: int, N: int, seed: int = 0, sizes=None, lhs_std: float = 1.0,
               w_std: float = 0.02, dout_std: float = 1.0) -> Inputs:
    """An ad-hoc CPU case for tests: explicit sizes or a uniform multinomial."""
    gen = torch.Generator().manual_seed(seed)
    if sizes is None:
        idx = torch.multinomial(torch.ones(G, dtype=torch.float64), M, replacement=True, generator=gen)
        gs = torch.bincount(idx, minlength=G).to(torch.int32)
    else:
        gs = torch.tensor(sizes, dtype=torch.int32)
    lhs = _normal((M, K), lhs_std, gen, "cpu")
    wt = _normal((G, K, N), w_std, gen, "cpu")
    dout = _normal((M, N), dout_std, gen, "cpu")
    w = Workload("adhoc", G, M, K, N, "static", "explicit")
    return Inputs(w, gs, lhs, wt, dout, STATIC_SCALE)
