"""Expert parallelism around the grouped matmul.

Each of P ranks holds E/P consecutive experts.  A token routed to k experts
sends one row per choice to the rank that holds the expert; the rank runs
gmm_fwd on the rows it received, grouped by its local experts (the
group_offset view of a ragged dot: "FP8 Megablox for batch split", maxtext
PR #3770, Description item 3), and the results travel back to be summed per
token with the routing weights.  Rows are quantized before they move, so
E4M3 codes (one byte per element) cross the links instead of bf16 ("add
static LHS scaling support for GMM v2 FWD", maxtext PR #4735, rebase commit
text: quantize before the expert-parallel exchange and ragged sort).  That
needs a scale that does not depend on the row's position, i.e. the static
rule.

Split of the work:
  - routing metadata (``route``, ``exchange_counts``, ``local_order``): small
    integer tensors and their exchange, on any device (tested on CPU with
    gloo ranks);
  - the row exchange (``exchange_rows``): ``torch.distributed`` all-to-all,
    NCCL on GPUs;
  - row movement and arithmetic (``ep_moe_fwd``, ``ep_moe_bwd``): the
    library's kernels (gmm_gather_rows, gmm_gather_scale_rows, gmm_fwd,
    gmm_backward, gmm_combine_rows), CUDA only.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import _binding as B
from .ops import _check, _dev, _stream, gmm_backward, gmm_fwd


@dataclass
class Route:
    """Where each (token, choice) row goes.  Experts are owned in contiguous
    blocks: rank r holds experts [r * E/P, (r + 1) * E/P)."""
    E: int
    P: int
    k: int
    order: torch.Tensor         # int64 [T*k]: flat positions t*k + j sorted by expert (stable)
    counts: torch.Tensor        # int64 [E]: rows per expert from this rank
    send_splits: list | None    # rows sent to each rank (host ints; None until synchronized)
    bad: torch.Tensor | None = None   # int64 [1] on the device: expert ids out of range


def route(expert_ids: torch.Tensor, E: int, P: int, validate: bool = True, sync: bool = True) -> Route:
    """Sort this rank's routed rows by expert: the send order of the exchange.

    sync=True (the default): one host synchronization reads the range check of
    the ids and, with more than one rank, the send splits.  sync=False: nothing
    is read on the host; ``bad`` stays on the device and ``send_splits`` is
    None (``exchange_counts`` then reads both with the arrival counts, in the
    exchange's one synchronization).  validate=False (one rank only) skips the
    check, for ids already checked (for example in a captured CUDA graph);
    out-of-range ids are then counted against the nearest valid expert."""
    if E % P:
        raise ValueError(f"{E} experts do not split over {P} ranks")
    T, k = expert_ids.shape
    flat = expert_ids.reshape(-1).to(torch.int64)
    bad = ((flat < 0) | (flat >= E)).sum().view(1)
    order = torch.argsort(flat.to(torch.int32), stable=True)  # 32-bit keys: half the radix passes
    counts = torch.zeros(E, dtype=torch.int64, device=flat.device)
    counts.index_add_(0, flat.clamp(0, E - 1), torch.ones_like(flat))
    send = counts.view(P, E // P).sum(dim=1)
    if P == 1 and not validate:
        return Route(E, P, k, order, counts, [T * k])
    if not sync:
        return Route(E, P, k, order, counts, None, bad)
    host = torch.cat([bad, send]).tolist() if P > 1 else bad.tolist()
    if host[0]:
        raise ValueError("expert id out of range")
    return Route(E, P, k, order, counts, host[1:] if P > 1 else [T * k])


def exchange_counts(rt: Route, group=None):
    """One all-to-all of E + P integers: this rank's per-expert counts go to
    the experts' ranks, each with this rank's count of out-of-range ids.
    Returns (recv_counts int64 [P, E/P] on the device: rows each source rank
    sends to each local expert; arrive: host list of rows arriving from each
    rank).  When ``rt`` was routed without synchronizing, this is the
    exchange's one host synchronization: it reads the send splits, the arrival
    counts and every rank's bad-id count at once, and every rank raises when
    any rank routed an id out of range (so that no rank enters the row
    exchange alone)."""
    El = rt.E // rt.P
    if rt.P == 1:
        recv = rt.counts.view(1, El).clone()
        if rt.send_splits is None:
            if int(rt.bad.item()):
                raise ValueError("expert id out of range")
            rt.send_splits = [int(rt.counts.sum().item())]
        return recv, list(rt.send_splits)
    bad = rt.bad if rt.bad is not None else torch.zeros(1, dtype=torch.int64, device=rt.counts.device)
    payload = torch.cat([rt.counts.view(rt.P, El), bad.expand(rt.P).view(rt.P, 1)], dim=1).contiguous()
    recv = torch.empty_like(payload)
    dist.all_to_all_single(recv, payload, group=group)  # E / P counts + 1 flag to each rank
    recv_counts = recv[:, :El].contiguous()
    if rt.send_splits is None:
        send = rt.counts.view(rt.P, El).sum(dim=1)
        host = torch.cat([send, recv_counts.sum(dim=1), recv[:, El]]).tolist()
        P = rt.P
        if any(host[2 * P:]):
            raise ValueError("expert id out of range (on some rank)")
        rt.send_splits = host[:P]
        return recv_counts, host[P:2 * P]
    return recv_counts, [int(v) for v in recv_counts.sum(dim=1).tolist()]


def local_order(recv_counts: torch.Tensor, total: int | None = None):
    """Rows arrive grouped by source rank, then by expert.  Returns (perm, inv,
    group_sizes): perm[i] is the arrival index of the i-th row when the rows
    are grouped by local expert (then by source rank), inv its inverse (the
    grouped position of each arrival row) and group_sizes the rows per local
    expert.  On a CUDA device the library's kernel builds them
    (gmm_ep_local_order, no host synchronization; ``total`` = the arrival
    count, which the caller knows from the exchange); on the CPU (gloo ranks)
    the same indices come from torch."""
    P, El = recv_counts.shape
    if recv_counts.is_cuda:
        if total is None:
            raise ValueError("local_order on the device needs the arrival total")
        cnt = recv_counts.to(torch.int64).contiguous()
        perm = torch.empty(total, dtype=torch.int32, device=cnt.device)
        inv = torch.empty(total, dtype=torch.int32, device=cnt.device)
        gsz = torch.empty(El, dtype=torch.int32, device=cnt.device)
        st = B.lib().gmm_ep_local_order(cnt.data_ptr(), P, El, total, perm.data_ptr() if total else None,
                                        inv.data_ptr() if total else None, gsz.data_ptr(), _stream(cnt))
        _check(st, "gmm_ep_local_order")
        return perm, inv, gsz
    cnt = recv_counts.reshape(-1)
    start = torch.cumsum(cnt, 0) - cnt  # arrival offset of block (p, e)
    by_expert = torch.arange(P * El, device=cnt.device).view(P, El).t().reshape(-1)  # blocks (e, p)
    c = cnt[by_expert]
    if total is None:
        total = int(c.sum())
    first = torch.repeat_interleave(start[by_expert], c, output_size=total)
    within = torch.arange(total, device=cnt.device) - torch.repeat_interleave(torch.cumsum(c, 0) - c, c,
                                                                              output_size=total)
    perm = first + within
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(total, device=cnt.device)
    return perm, inv, recv_counts.sum(dim=0)


def exchange_rows(buf: torch.Tensor, in_splits, out_splits, group=None) -> torch.Tensor:
    """All-to-all of rows: in_splits rows of buf go to each rank; out_splits
    rows arrive from each rank, in rank order."""
    out = torch.empty((sum(out_splits),) + tuple(buf.shape[1:]), dtype=buf.dtype, device=buf.device)
    if len(in_splits) == 1:
        out.copy_(buf)
        return out
    dist.all_to_all_single(out, buf, output_split_sizes=list(out_splits), input_split_sizes=list(in_splits),
                           group=group)
    return out


def gather_rows(src: torch.Tensor, idx: torch.Tensor) -> torch.Tensor:
    """dst[i] = src[idx[i]] with the library's row gather (CUDA)."""
    idx32 = idx.to(device=src.device, dtype=torch.int32).contiguous()
    dst = torch.empty((idx32.numel(),) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] else dst[0].numel() * dst.element_size()
    st = B.lib().gmm_gather_rows(_dev(src, "src"), idx32.data_ptr(), idx32.numel(), row_bytes, src.shape[0],
                                 dst.data_ptr(), _stream(src))
    _check(st, "gmm_gather_rows")
    return dst


def gather_scale_rows(src: torch.Tensor, idx: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """dst[i] = bf16(src[idx[i]] * scale[i]) for bf16 rows (library kernel)."""
    idx32 = idx.to(device=src.device, dtype=torch.int32).contiguous()
    f32 = scale.to(device=src.device, dtype=torch.float32).contiguous()
    dst = torch.empty((idx32.numel(), src.shape[1]), dtype=torch.bfloat16, device=src.device)
    st = B.lib().gmm_gather_scale_rows(_dev(src, "src", torch.bfloat16), idx32.data_ptr(), f32.data_ptr(),
                                       idx32.numel(), src.shape[1], src.shape[0], dst.data_ptr(), _stream(src))
    _check(st, "gmm_gather_scale_rows")
    return dst


def combine_rows(rows: torch.Tensor, slot: torch.Tensor, weight: torch.Tensor, out_dtype=torch.bfloat16):
    """y[t] = sum_j weight[t, j] * rows[slot[t, j]] with the library's kernel."""
    T, k = slot.shape
    N = rows.shape[1]
    y = torch.empty((T, N), dtype=out_dtype, device=rows.device)
    s32 = slot.to(torch.int32).contiguous()
    w32 = weight.to(torch.float32).contiguous()
    st = B.lib().gmm_combine_rows(_dev(rows, "rows", torch.bfloat16), rows.shape[0], _dev(s32, "slot"),
                                  _dev(w32, "weight"), T, k, N, y.data_ptr(),
                                  B.DT_F32 if out_dtype == torch.float32 else B.DT_BF16, _stream(rows))
    _check(st, "gmm_combine_rows")
    return y


def ep_moe_fwd(x_codes: torch.Tensor, static_scale: torch.Tensor, expert_ids: torch.Tensor,
               weights: torch.Tensor, w_codes: torch.Tensor, w_scales: torch.Tensor, group=None,
               out_dtype=torch.bfloat16, validate: bool = True) -> torch.Tensor:
    """One expert-parallel expert projection for this rank's T tokens.

    x_codes: E4M3 codes [T, K] of the tokens (static rule, ``static_scale``
    one float on the device); expert_ids / weights: [T, k] routing; w_codes /
    w_scales: this rank's experts [E/P, K, N] and [E/P, N].  Returns
    y [T, N] = sum_j weights[t, j] * (x[t] @ W[expert_ids[t, j]]).
    On one rank with validate=False nothing synchronizes with the host, so
    the call can be captured in a CUDA graph (see EPForwardGraph).
    """
    P = dist.get_world_size(group) if dist.is_initialized() else 1
    El, K, N = w_codes.shape
    T, k = expert_ids.shape
    # P > 1: one host synchronization per call, in exchange_counts (the
    # splits NCCL needs and the id check of every rank)
    rt = route(expert_ids.to(x_codes.device), El * P, P, validate=validate or P > 1, sync=P == 1)
    order = rt.order
    # permute: this rank's routed rows in expert order, E4M3 codes
    send = gather_rows(x_codes, order // k)
    if P == 1:
        # nothing to exchange: the sorted rows are already grouped by expert
        back_rows, gsz = send, rt.counts
    else:
        recv_counts, arrive = exchange_counts(rt, group)
        recv = exchange_rows(send, rt.send_splits, arrive, group)
        perm, inv, gsz = local_order(recv_counts, sum(arrive))
        back_rows = gather_rows(recv, perm)
    if back_rows.shape[0]:
        h = gmm_fwd(back_rows, w_codes, w_scales, gsz.to(torch.int32), rule="static", static_scale=static_scale,
                    out_dtype=torch.bfloat16)
    else:  # no rows for this rank's experts
        h = torch.empty((0, N), dtype=torch.bfloat16, device=x_codes.device)
    if P > 1:
        # back in arrival order, then to the source ranks
        h = exchange_rows(gather_rows(h, inv), arrive, rt.send_splits, group)
    # h[i] is the result of flat position order[i]; slot of (t, j) = i
    slot = torch.empty_like(order).scatter_(0, order, torch.arange(order.numel(), device=order.device))
    return combine_rows(h, slot.view(T, k), weights, out_dtype)


class EPForwardGraph:
    """ep_moe_fwd on one rank captured once as a CUDA graph over fixed
    buffers: every replay runs the same kernels without their per-call host
    cost.  The routing ids are checked once, when the graph is made; to run
    new inputs, copy them into ``x_codes`` / ``expert_ids`` / ``weights``
    (check new ids first, with ``route(ids, E, 1)``) and call ``replay()``;
    the result is ``out``."""

    def __init__(self, x_codes, static_scale, expert_ids, weights, w_codes, w_scales, out_dtype=torch.bfloat16):
        if dist.is_initialized() and dist.get_world_size() > 1:
            raise ValueError("a captured EP forward covers one rank only (the exchange sizes are data-dependent)")
        self.args = (x_codes, static_scale, expert_ids, weights, w_codes, w_scales)
        ep_moe_fwd(*self.args, out_dtype=out_dtype)  # checks the ids, sets up the workspace
        side = torch.cuda.Stream(device=x_codes.device)
        side.wait_stream(torch.cuda.current_stream(x_codes.device))
        with torch.cuda.stream(side):
            for _ in range(2):
                ep_moe_fwd(*self.args, out_dtype=out_dtype, validate=False)
        torch.cuda.current_stream(x_codes.device).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.out = ep_moe_fwd(*self.args, out_dtype=out_dtype, validate=False)

    def replay(self) -> torch.Tensor:
        self.graph.replay()
        return self.out


def ep_moe_bwd(x_codes: torch.Tensor, static_scale: torch.Tensor, expert_ids: torch.Tensor,
               weights: torch.Tensor, dy: torch.Tensor, w_codes: torch.Tensor, w_scales: torch.Tensor, group=None,
               dx_dtype=torch.bfloat16, dw_dtype=torch.float32):
    """Backward of ep_moe_fwd for the gmm operands: given dy [T, N] (bf16)
    returns dx [T, K] and this rank's expert weight gradient [E/P, K, N].

    Each routed row carries dh = bf16(w[t, j] * dy[t]) to its expert's rank
    together with the forward's E4M3 codes of x[t]; there gmm_backward (dout
    quantized once) gives dlhs rows and dW; the dlhs rows return and are
    summed per token: dx[t] = sum_j dlhs_{t, j}.  The routing weights'
    gradient (dy . h) belongs to the router and is not computed here.
    """
    P = dist.get_world_size(group) if dist.is_initialized() else 1
    El, K, N = w_codes.shape
    T, k = expert_ids.shape
    rt = route(expert_ids.to(x_codes.device), El * P, P, sync=P == 1)
    order = rt.order
    tok = order // k
    send_x = gather_rows(x_codes, tok)
    send_d = gather_scale_rows(dy, tok, weights.reshape(-1)[order])
    if P == 1:
        xr, dr, gsz, perm = send_x, send_d, rt.counts, None
    else:
        recv_counts, arrive = exchange_counts(rt, group)  # the one host synchronization
        perm, inv, gsz = local_order(recv_counts, sum(arrive))
        xr = gather_rows(exchange_rows(send_x, rt.send_splits, arrive, group), perm)
        dr = gather_rows(exchange_rows(send_d, rt.send_splits, arrive, group), perm)
    dw = torch.empty((El, K, N), dtype=dw_dtype, device=x_codes.device)
    if xr.shape[0]:
        dl, dw = gmm_backward(xr, dr, w_codes, w_scales, gsz.to(torch.int32), rule="static",
                              static_scale=static_scale, dlhs_dtype=torch.bfloat16, drhs=dw)
    else:  # no rows for this rank's experts
        dl = torch.empty((0, K), dtype=torch.bfloat16, device=x_codes.device)
        dw.zero_()
    if P > 1:
        dl = exchange_rows(gather_rows(dl, inv), arrive, rt.send_splits, group)
    slot = torch.empty_like(order).scatter_(0, order, torch.arange(order.numel(), device=order.device))
    ones = torch.ones((T, k), dtype=torch.float32, device=x_codes.device)
    return combine_rows(dl, slot.view(T, k), ones, dx_dtype), dw
