"""Expert-parallel routing metadata and row exchange, on CPU gloo ranks.

The rows carried here are integer payloads (rank * 1000 + flat position of
the (token, choice)), so the test sees exactly which row lands where: after
the exchange and the regrouping every rank must hold, for each of its local
experts, the rows routed to that expert by every rank (source rank order,
then position order), and the return exchange must bring every row back to
the position it left from.  The arithmetic around it (gmm_fwd, the combine)
is CUDA only and is checked against the oracle in test_gpu_ep.py.

Source: "FP8 Megablox for batch split" (maxtext PR #3770), Description item
3 (group_offset: a rank's experts as a slice of the ragged dot); "add static
LHS scaling support for GMM v2 FWD" (maxtext PR #4735), rebase commit text
(rows exchanged and sorted by expert after quantization).
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from moe_fp8_grouped_b200 import ep


def test_route_sorts_by_expert_and_counts():
    ids = torch.tensor([[2, 0], [1, 2], [0, 3]])
    rt = ep.route(ids, E=4, P=2)
    flat = ids.reshape(-1)
    assert flat[rt.order].tolist() == [0, 0, 1, 2, 2, 3]
    assert rt.order.tolist() == [1, 4, 2, 0, 3, 5]  # stable within an expert
    assert rt.counts.tolist() == [2, 1, 2, 1]
    assert rt.send_splits == [3, 3]
    with pytest.raises(ValueError):
        ep.route(ids, E=3, P=2)
    with pytest.raises(ValueError):
        ep.route(torch.tensor([[4, 0]]), E=4, P=2)


def test_route_without_sync_defers_the_check():
    ids = torch.tensor([[2, 0], [1, 2], [0, 3]])
    rt = ep.route(ids, E=4, P=2, sync=False)
    assert rt.send_splits is None and int(rt.bad) == 0
    assert rt.counts.tolist() == [2, 1, 2, 1]
    rt = ep.route(torch.tensor([[4, 0]]), E=4, P=2, sync=False)  # no raise yet: the exchange checks
    assert int(rt.bad) == 1


def test_local_order_groups_arrivals_by_expert():
    # from rank 0: 2 rows of expert 0, 1 of expert 1; from rank 1: 0 and 3
    recv = torch.tensor([[2, 1], [0, 3]])
    perm, inv, gsz = ep.local_order(recv)
    # arrival order: [r0e0 r0e0 r0e1 r1e1 r1e1 r1e1]
    assert perm.tolist() == [0, 1, 2, 3, 4, 5]
    assert gsz.tolist() == [2, 4]
    recv = torch.tensor([[1, 2], [3, 0], [0, 1]])
    perm, inv, gsz = ep.local_order(recv, total=7)
    # arrivals: r0e0=0, r0e1=1,2, r1e0=3,4,5, r2e1=6 -> e0: 0,3,4,5; e1: 1,2,6
    assert perm.tolist() == [0, 3, 4, 5, 1, 2, 6]
    assert inv.tolist() == [0, 4, 5, 1, 2, 3, 6]  # grouped position of each arrival
    assert gsz.tolist() == [4, 3]
    perm, inv, gsz = ep.local_order(torch.zeros((2, 3), dtype=torch.int64))
    assert perm.numel() == 0 and inv.numel() == 0 and gsz.tolist() == [0, 0, 0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        E, T, k = 6, 9 + rank, 2
        g = torch.Generator().manual_seed(100 + rank)
        ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)])  # distinct experts per token
        payload = rank * 1000 + torch.arange(T * k)
        rt = ep.route(ids, E, world, sync=False)  # the exchange's one host read happens in exchange_counts
        send = payload[rt.order]
        recv_counts, arrive = ep.exchange_counts(rt)
        assert rt.send_splits == ep.route(ids, E, world).send_splits
        recv = ep.exchange_rows(send, rt.send_splits, arrive)
        perm, inv, gsz = ep.local_order(recv_counts, sum(arrive))
        local = recv[perm]
        back = ep.exchange_rows(local[inv], arrive, rt.send_splits)
        every = [None] * world
        dist.all_gather_object(every, ids.tolist())
        q.put((rank, local.tolist(), gsz.tolist(), torch.equal(back, send), every))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_delivers_rows_to_their_experts_and_back(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    E = 6
    El = E // world
    every = res[0][4]
    for rank, local, gsz, returned, _ in res:
        assert returned, f"rank {rank}: rows did not come back to their positions"
        want = []
        for e in range(rank * El, (rank + 1) * El):
            rows = [src * 1000 + pos for src in range(world)
                    for pos, x in enumerate(v for row in every[src] for v in row) if x == e]
            assert gsz[e - rank * El] == len(rows)
            want += rows
        assert local == want


def _bad_id_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ids = torch.tensor([[0, 1], [2, 3]])
        if rank == world - 1:
            ids[1, 0] = 7  # out of range on one rank only
        rt = ep.route(ids, 4, world, sync=False)
        try:
            ep.exchange_counts(rt)
            q.put((rank, "no error"))
        except ValueError as exc:
            q.put((rank, str(exc)))
    finally:
        dist.destroy_process_group()


def test_an_out_of_range_id_on_one_rank_stops_every_rank():
    """The id check travels with the counts exchange: every rank learns that
    some rank routed an id out of range and raises before the row exchange,
    so no rank waits in a collective the others never enter."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bad_id_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all("out of range" in msg for _, msg in res), res
