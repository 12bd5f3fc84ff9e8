"""The expert-parallel step's collectives on CPU: world-size-2 `gloo` groups.

`moe_forward_ep` runs as two ranks with the library's three compute phases
(dispatch, expert forward, combine) replaced by plain torch stand-ins of the
same contract: rows in expert order, one row per route, y = x * (e + 1) for
global expert e, and the ordered sum of p * y.  What is under test is the part
that needs no GPU: the count exchange, the host split sizes, the row
all-to-alls there and back (bf16 rows as bytes, int32 ids, fp32 weights), and
that every route's y returns to its own send row.  The result must equal the
same stand-in arithmetic done without EP, bit for bit.
"""
from __future__ import annotations

import os
import socket
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
E, K, H = 8, 3, 16
TOKENS = (37, 0)  # rank 1 routes no tokens of its own but still owns experts


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _routes(rank: int, n: int):
    g = torch.Generator().manual_seed(100 + rank)
    x = torch.randn(max(n, 1), H, generator=g).to(torch.bfloat16)
    ids = torch.stack([torch.randperm(E, generator=g)[:K].sort().values for _ in range(max(n, 1))]).to(torch.int32)
    probs = torch.rand(max(n, 1), K, generator=g)
    return x, ids, probs


def _rank_main(rank: int, world: int, port: int, results) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from routed_moe_swiglu_b200 import ep as moe_ep

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n = TOKENS[rank]
        e0, el = moe_ep.expert_range(E, world, rank)

        def fake_dispatch(plan, bufs, x, live_count, logits=None, ids=None, probs=None, stream=None):
            n_live = int(live_count[0])
            order = sorted((int(ids[t, j]), t, j) for t in range(n_live) for j in range(K))
            for row, (e, t, j) in enumerate(order):
                bufs.send_x[row] = x[t]
                bufs.send_ids[row] = e % el
                bufs.send_probs[row] = 1.0
                bufs.route_rows[t, j] = row
                bufs.route_probs[t, j] = probs[t, j]
            for g in range(world):
                bufs.send_counts[g] = sum(1 for e, _, _ in order if e // el == g)

        def fake_expert_forward(shard, bufs, shard_wbuf, n_recv, stream=None):
            for r in range(n_recv):
                e = e0 + int(bufs.recv_ids[r, 0])
                bufs.recv_y[r] = bufs.recv_x[r].float() * float(e + 1) * bufs.recv_probs[r, 0]

        def fake_combine(plan, bufs, live_count, out, stream=None):
            for t in range(int(live_count[0])):
                acc = torch.zeros(H)
                for j in range(K):
                    acc = acc + bufs.route_probs[t, j] * bufs.y_back[bufs.route_rows[t, j]]
                out[t] = acc

        moe_ep.dispatch, moe_ep.expert_forward, moe_ep.combine = fake_dispatch, fake_expert_forward, fake_combine
        x, ids, probs = _routes(rank, n)
        routes_max, recv_max = max(n, 1) * K, sum(TOKENS) * K
        bufs = moe_ep.EpBuffers(
            ep_size=world, workspace=None,
            send_x=torch.full((routes_max, H), float("nan"), dtype=torch.bfloat16),
            send_ids=torch.full((routes_max,), -5, dtype=torch.int32),
            send_probs=torch.zeros(routes_max), send_counts=torch.zeros(world, dtype=torch.int32),
            route_rows=torch.zeros(max(n, 1), K, dtype=torch.int32), route_probs=torch.zeros(max(n, 1), K),
            y_back=torch.full((routes_max, H), float("nan")),
            recv_x=torch.full((recv_max, H), float("nan"), dtype=torch.bfloat16),
            recv_ids=torch.full((recv_max, 1), -5, dtype=torch.int32), recv_probs=torch.zeros(recv_max, 1),
            recv_y=torch.full((recv_max, H), float("nan")), recv_live=torch.zeros(1, dtype=torch.int32),
            shard_workspace=None)
        out = torch.full((max(n, 1), H), float("nan"))
        live = torch.tensor([n], dtype=torch.int32)
        moe_ep.moe_forward_ep(None, None, bufs, x, None, live, out, ids=ids, probs=probs)
        # the same stand-in arithmetic without EP
        want = torch.full((max(n, 1), H), float("nan"))
        for t in range(n):
            acc = torch.zeros(H)
            for j in range(K):
                y = x[t].float() * float(int(ids[t, j]) + 1) * 1.0
                acc = acc + probs[t, j] * y
            want[t] = acc
        results[rank] = (bool(torch.equal(out[:n], want[:n])), bufs.send_counts.tolist())
    finally:
        dist.destroy_process_group()


def _overflow_rank_main(rank: int, world: int, port: int, results) -> None:
    """Rank 1's receive buffer holds one row, and rank 0 sends it more: both
    ranks must raise before any row all-to-all starts."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from routed_moe_swiglu_b200 import MoeError
    from routed_moe_swiglu_b200 import ep as moe_ep

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        row_exchanges = []

        def fake_dispatch(plan, bufs, x, live_count, logits=None, ids=None, probs=None, stream=None):
            bufs.send_counts[:] = torch.tensor([2, 5] if rank == 0 else [0, 0], dtype=torch.int32)

        real_exchange = moe_ep.exchange_rows

        def counting_exchange(*args, **kwargs):
            row_exchanges.append(1)
            return real_exchange(*args, **kwargs)

        moe_ep.dispatch, moe_ep.exchange_rows = fake_dispatch, counting_exchange
        recv = 64 if rank == 0 else 1
        bufs = moe_ep.EpBuffers(
            ep_size=world, workspace=None, send_x=torch.zeros((8, H), dtype=torch.bfloat16),
            send_ids=torch.zeros(8, dtype=torch.int32), send_probs=torch.zeros(8),
            send_counts=torch.zeros(world, dtype=torch.int32), route_rows=torch.zeros(4, K, dtype=torch.int32),
            route_probs=torch.zeros(4, K), y_back=torch.zeros((8, H)),
            recv_x=torch.zeros((recv, H), dtype=torch.bfloat16), recv_ids=torch.zeros((recv, 1), dtype=torch.int32),
            recv_probs=torch.zeros(recv, 1), recv_y=torch.zeros((recv, H)), recv_live=torch.zeros(1, dtype=torch.int32),
            shard_workspace=None)
        live = torch.tensor([2], dtype=torch.int32)
        try:
            moe_ep.moe_forward_ep(None, None, bufs, torch.zeros((4, H), dtype=torch.bfloat16), None, live,
                                  torch.zeros((4, H)), ids=torch.zeros((4, K), dtype=torch.int32),
                                  probs=torch.zeros(4, K))
            results[rank] = ("no error", len(row_exchanges))
        except MoeError as exc:
            results[rank] = (f"MoeError {exc.code}", len(row_exchanges))
        # the group still works: every rank left the step at the same point
        t = torch.tensor([rank + 1])
        dist.all_reduce(t)
        results[f"after{rank}"] = int(t)
    finally:
        dist.destroy_process_group()


def test_receive_overflow_on_one_rank_raises_on_every_rank():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_overflow_rank_main, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(results)
    assert res[0] == ("MoeError 4", 0) and res[1] == ("MoeError 4", 0), res
    assert res["after0"] == 3 and res["after1"] == 3


def test_two_rank_ep_step_exchanges_rows_and_returns_them_in_place():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=240)
            assert p.exitcode == 0
        res = dict(results)
    assert res[0][0] and res[1][0]
    assert sum(res[0][1]) == TOKENS[0] * K and res[1][1] == [0, 0]
    assert res[0][1][1] > 0  # rank 0 really sends rows to rank 1


def test_expert_range_splits_contiguously():
    from routed_moe_swiglu_b200 import ep as moe_ep

    assert [moe_ep.expert_range(128, 4, g) for g in range(4)] == [(0, 32), (32, 32), (64, 32), (96, 32)]
    for bad in ((12, 5, 0), (12, 4, 4), (12, 0, 0)):
        try:
            moe_ep.expert_range(*bad)
        except ValueError:
            continue
        raise AssertionError(f"expert_range{bad} accepted")


def test_shard_plan_carries_the_source_plans_arithmetic():
    """The receiving rank's plan: E/ep experts, top-1, fp32 rows out, and the
    source plan's precision, FC1 flags and clamp (host-only: plans need no GPU)."""
    import routed_moe_swiglu_b200 as rm
    from routed_moe_swiglu_b200 import ep as moe_ep

    src = rm.moe_plan_create(hidden=512, ffn=256, num_experts=16, top_k=4, capacity=100, precision="nvfp4",
                             out_dtype="bf16", probs_in_fc1=True, gate_up_clamp=2.5, squared_relu=True)
    shard = moe_ep.shard_plan_create(src, 4, 1600)
    assert (shard.num_experts, shard.top_k, shard.capacity, shard.hidden, shard.ffn) == (4, 1, 1600, 512, 256)
    assert shard.precision == "nvfp4" and shard.out_dtype == "fp32"
    assert shard.probs_in_fc1 and shard.squared_relu and shard.gate_up_clamp == 2.5
    plain = moe_ep.shard_plan_create(rm.moe_plan_create(hidden=512, ffn=256, num_experts=16, top_k=4,
                                                        capacity=100), 2, 800)
    assert not plain.probs_in_fc1 and not plain.squared_relu and plain.gate_up_clamp == 0.0
    try:
        moe_ep.shard_plan_create(src, 3, 100)
    except ValueError:
        pass
    else:
        raise AssertionError("an EP size that does not divide E was accepted")
