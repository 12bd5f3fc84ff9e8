"""Expert parallelism: one routed-MoE step over ep_size ranks, each holding the
weights of E/ep_size contiguous experts.

The sequence (include/moe.h, "Expert parallelism") is:
  1. ``moe_ep_dispatch`` routes the rank's own tokens and packs one send row per
     route, in expert order, so the rows for rank g are one run;
  2. all-to-alls of the counts and then of the rows (x, local expert ids,
     FC1 weights);
  3. the rank's own experts run ``moe_forward`` over the received rows as top-1
     tokens, whose output rows are the routes' expert outputs y;
  4. the reverse all-to-all brings each y row back to its send row;
  5. ``moe_ep_combine`` adds each token's routes in ascending expert id.

The result is bitwise the one-GPU forward's, for any EP size (Megatron-LM PR
#7798, "What is changed": the expert kernel computes every dispatched row as a
top-1 token with probability 1.0; its "Limitations": generation's combine adds
rank partials and is not EP-invariant, which the ascending-id combine here
is).  cudnn-frontend PR #448 (MoeEp API) names the same parts: a variable-size
all-to-all dispatch, local experts and a top-k combine.

``moe_forward_ep`` does the exchanges with ``torch.distributed`` all-to-alls
(NCCL over NVLink between GPUs), which need the row counts on the host: step 2
reads them back, as an all-to-all dispatcher does.  ``moe_forward_ep_peer``
does them with the library's kernels storing rows into the peers' regions
(``PeerRegions``), flags with bounded waits in place of the host read, so the
whole step can be captured in one CUDA graph.  Every other step is the
library's kernels; this module only sequences them and moves bytes.

The phases (``dispatch``, ``expert_forward``, ``combine``) are separate so that
a driver other than ``moe_forward_ep`` can run the exchange itself.
"""
from __future__ import annotations

import contextlib
from dataclasses import dataclass

from . import (MoeError, Plan, alloc_workspace, moe_ep_combine, moe_ep_dispatch, moe_forward, moe_plan_create)

__all__ = ["expert_range", "shard_plan_create", "EpBuffers", "dispatch", "expert_forward", "combine",
           "exchange_counts", "agree_on_receive_capacity", "exchange_rows", "moe_forward_ep", "PeerRegions",
           "peer_dispatch", "peer_receive", "peer_expert_forward", "peer_return", "peer_combine",
           "moe_forward_ep_peer"]


def expert_range(num_experts: int, ep_size: int, rank: int) -> tuple[int, int]:
    """(first expert, number of experts) owned by EP rank `rank`."""
    if ep_size < 1 or num_experts % ep_size != 0:
        raise ValueError(f"ep_size {ep_size} must divide the {num_experts} experts")
    if not 0 <= rank < ep_size:
        raise ValueError(f"rank {rank} outside [0, {ep_size})")
    per = num_experts // ep_size
    return rank * per, per


def shard_plan_create(plan: Plan, ep_size: int, max_recv_rows: int) -> Plan:
    """The plan of one rank's experts: E/ep_size experts, top-1 routes, fp32
    output, the source plan's precision, FC1 flags and clamp; `max_recv_rows`
    bounds the rows one step may bring to the rank (at most ep_size times the
    source plan's live rows times k)."""
    expert_range(plan.num_experts, ep_size, 0)
    return moe_plan_create(hidden=plan.hidden, ffn=plan.ffn, num_experts=plan.num_experts // ep_size, top_k=1,
                           capacity=max_recv_rows, precision=plan.precision, out_dtype="fp32",
                           probs_in_fc1=plan.probs_in_fc1, gate_up_clamp=plan.gate_up_clamp or None,
                           squared_relu=plan.squared_relu)


@dataclass
class EpBuffers:
    """Device buffers of one rank's EP step (sizes from the two plans)."""
    ep_size: int
    workspace: object      # the source plan's workspace
    send_x: object         # bf16 [max_live * k, H]
    send_ids: object       # int32 [max_live * k]
    send_probs: object     # fp32 [max_live * k]
    send_counts: object    # int32 [ep_size]
    route_rows: object     # int32 [max_live, k]
    route_probs: object    # fp32 [max_live, k]
    y_back: object         # fp32 [max_live * k, H]
    recv_x: object         # bf16 [max_recv, H]
    recv_ids: object       # int32 [max_recv, 1]
    recv_probs: object     # fp32 [max_recv, 1]
    recv_y: object         # fp32 [max_recv, H]
    recv_live: object      # int32 [1]
    shard_workspace: object

    @classmethod
    def allocate(cls, plan: Plan, shard: Plan, ep_size: int, device=None) -> "EpBuffers":
        import torch

        dev = device or "cuda"
        routes = plan.max_live_rows * plan.top_k
        recv = shard.capacity
        H = plan.hidden
        return cls(ep_size=ep_size, workspace=alloc_workspace(plan, dev),
                   send_x=torch.empty(routes, H, dtype=torch.bfloat16, device=dev),
                   send_ids=torch.empty(routes, dtype=torch.int32, device=dev),
                   send_probs=torch.empty(routes, dtype=torch.float32, device=dev),
                   send_counts=torch.empty(ep_size, dtype=torch.int32, device=dev),
                   route_rows=torch.empty(plan.max_live_rows, plan.top_k, dtype=torch.int32, device=dev),
                   route_probs=torch.empty(plan.max_live_rows, plan.top_k, dtype=torch.float32, device=dev),
                   y_back=torch.empty(routes, H, dtype=torch.float32, device=dev),
                   recv_x=torch.empty(recv, H, dtype=torch.bfloat16, device=dev),
                   recv_ids=torch.empty(recv, 1, dtype=torch.int32, device=dev),
                   recv_probs=torch.empty(recv, 1, dtype=torch.float32, device=dev),
                   recv_y=torch.empty(recv, H, dtype=torch.float32, device=dev),
                   recv_live=torch.zeros(1, dtype=torch.int32, device=dev),
                   shard_workspace=alloc_workspace(shard, dev))


def _on(stream):
    """Context that makes `stream` (a torch.cuda.Stream, or None for the
    current one) torch's current stream, so that tensor ops and collectives
    are ordered with the library calls on it."""
    import torch

    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def dispatch(plan: Plan, bufs: EpBuffers, x, live_count, logits=None, ids=None, probs=None, stream=None) -> None:
    """Step 1: fills send_x / send_ids / send_probs / send_counts / route_rows /
    route_probs of `bufs` for the rank's live tokens."""
    moe_ep_dispatch(plan, bufs.ep_size, x, live_count, bufs.send_x, bufs.send_ids, bufs.send_probs, bufs.send_counts,
                    bufs.route_rows, bufs.route_probs, bufs.workspace, logits=logits, ids=ids, probs=probs,
                    stream=stream)


def expert_forward(shard: Plan, bufs: EpBuffers, shard_wbuf, n_recv: int, stream=None) -> None:
    """Step 3: the rank's experts over the first `n_recv` rows of recv_x (their
    local ids and FC1 weights in recv_ids / recv_probs) into recv_y."""
    if n_recv > shard.capacity:
        raise MoeError(4, f"{n_recv} received rows exceed the expert plan's {shard.capacity}")
    with _on(stream):
        bufs.recv_live.fill_(n_recv)
    moe_forward(shard, bufs.recv_x, shard_wbuf, bufs.recv_live, bufs.recv_y, bufs.shard_workspace,
                ids=bufs.recv_ids, probs=bufs.recv_probs, stream=stream)


def combine(plan: Plan, bufs: EpBuffers, live_count, out, stream=None) -> None:
    """Step 5: out rows of the rank's live tokens from the returned y rows."""
    moe_ep_combine(plan, bufs.y_back, bufs.route_rows, bufs.route_probs, live_count, out, stream=stream)


def exchange_counts(send_counts, group=None):
    """All-to-all of one count per rank pair: returns recv_counts, where
    recv_counts[s] is what rank s sends to this rank."""
    import torch
    import torch.distributed as dist

    recv = torch.empty_like(send_counts)
    dist.all_to_all_single(recv, send_counts, group=group)
    return recv


def agree_on_receive_capacity(recv_splits: list[int], capacity: int, device, group=None) -> None:
    """Every rank learns whether any rank would receive more rows than it can
    hold, before any row moves: a MAX all-reduce of one overflow flag.  All
    ranks then raise together (MoeError 4) instead of one rank raising while
    the others wait in the row all-to-all until the group's timeout."""
    import torch
    import torch.distributed as dist

    n_recv = sum(recv_splits)
    flag = torch.tensor([1 if n_recv > capacity else 0], dtype=torch.int32, device=device)
    dist.all_reduce(flag, op=dist.ReduceOp.MAX, group=group)
    if int(flag.item()):
        mine = f"this rank receives {n_recv} rows for {capacity}" if n_recv > capacity else "another rank"
        raise MoeError(4, f"an EP rank's receive buffer is too small ({mine}); no rows were exchanged")


def exchange_rows(send, send_splits: list[int], recv_splits: list[int], recv, group=None):
    """All-to-all of rows: send[:sum(send_splits)] goes out in runs of
    send_splits[g] rows to rank g; the runs from ranks 0, 1, ... land in
    recv[:sum(recv_splits)] in rank order.  bf16 rows move as their bytes
    (uint8), which every backend copies as is.  Returns that view of `recv`."""
    import torch
    import torch.distributed as dist

    n_out = sum(recv_splits)
    if n_out > recv.shape[0]:
        raise MoeError(4, f"{n_out} rows to receive exceed the buffer's {recv.shape[0]}")
    src = send[:sum(send_splits)]
    dst = recv[:n_out]
    if src.dtype == torch.bfloat16:
        src, dst = src.view(torch.uint8), dst.view(torch.uint8)
    dist.all_to_all_single(dst, src, output_split_sizes=list(recv_splits), input_split_sizes=list(send_splits),
                           group=group)
    return recv[:n_out]


def moe_forward_ep(plan: Plan, shard: Plan, bufs: EpBuffers, x, shard_wbuf, live_count, out, group=None,
                   logits=None, ids=None, probs=None, stream=None) -> None:
    """One EP step on this rank (every rank of `group` calls it together):
    `x`, `live_count`, `logits` or `ids` + `probs` and `out` are the rank's own
    tokens as for ``moe_forward`` with `plan`; `shard_wbuf` holds the rank's
    experts, prepared with `shard` (``shard_plan_create``).  `stream`: a
    torch.cuda.Stream for the whole step (default: the current stream)."""
    import torch.distributed as dist

    if dist.get_world_size(group) != bufs.ep_size:
        raise ValueError(f"group has {dist.get_world_size(group)} ranks, buffers are for {bufs.ep_size}")
    with _on(stream):  # every step below on one stream, in order
        dispatch(plan, bufs, x, live_count, logits=logits, ids=ids, probs=probs)
        recv_counts = exchange_counts(bufs.send_counts, group)
        send_splits = bufs.send_counts.tolist()  # the host needs the split sizes
        recv_splits = recv_counts.tolist()
        n_recv = sum(recv_splits)
        capacity = bufs.recv_x.shape[0] if shard is None else min(bufs.recv_x.shape[0], shard.capacity)
        agree_on_receive_capacity(recv_splits, capacity, bufs.send_counts.device, group)
        exchange_rows(bufs.send_x, send_splits, recv_splits, bufs.recv_x, group)
        exchange_rows(bufs.send_ids, send_splits, recv_splits, bufs.recv_ids.view(-1), group)
        exchange_rows(bufs.send_probs, send_splits, recv_splits, bufs.recv_probs.view(-1), group)
        expert_forward(shard, bufs, shard_wbuf, n_recv)
        exchange_rows(bufs.recv_y, recv_splits, send_splits, bufs.y_back, group)
        combine(plan, bufs, live_count, out)


# ---------------------------------------------------------------- the exchange through peer memory


class PeerRegions:
    """One rank's exchange region (include/moe.h, "Expert-parallel exchange
    through peer memory") and the device table of every rank's region as this
    rank addresses it.

    With a process group of ep_size ranks (one GPU each), the region's CUDA IPC
    handle is exchanged through the group once and every peer's region is
    mapped here.  Without one (`addresses` given), the table is taken as is:
    the regions of several ranks in one GPU's memory, or ep_size 1."""

    def __init__(self, plan: Plan, ep_size: int, rank: int, group=None, addresses=None, device=None, region=None):
        import torch

        from . import moe_ep_ipc_handle, moe_ep_ipc_open, moe_ep_region_bytes, moe_ep_region_views

        self.plan, self.ep_size, self.rank = plan, ep_size, rank
        dev = device or "cuda"
        # zero-filled once: flags, counters and the step number start at 0
        if region is None:
            region = torch.zeros(moe_ep_region_bytes(plan, ep_size), dtype=torch.uint8, device=dev)
        elif region.numel() < moe_ep_region_bytes(plan, ep_size):
            raise ValueError("region smaller than moe_ep_region_bytes")
        self.region = region
        self._opened = []
        if addresses is None:
            if ep_size == 1:
                addresses = [self.region.data_ptr()]
            else:
                import torch.distributed as dist

                mine = torch.frombuffer(bytearray(moe_ep_ipc_handle(self.region)), dtype=torch.uint8)
                handles = [torch.empty_like(mine) for _ in range(ep_size)]
                dist.all_gather(handles, mine.to(dev) if dist.get_backend(group) == "nccl" else mine, group=group)
                addresses = []
                for g, h in enumerate(handles):
                    if g == rank:
                        addresses.append(self.region.data_ptr())
                    else:
                        a = moe_ep_ipc_open(bytes(h.cpu().numpy().tobytes()))
                        self._opened.append(a)
                        addresses.append(a)
        self.addresses = list(addresses)
        self.table = torch.tensor(self.addresses, dtype=torch.int64, device=dev)
        self.views = moe_ep_region_views(plan, ep_size, self.region)

    def close(self):
        from . import moe_ep_ipc_close

        for a in self._opened:
            moe_ep_ipc_close(a)
        self._opened = []


def peer_dispatch(plan: Plan, peer: PeerRegions, x, live_count, route_rows, route_probs, workspace, logits=None,
                  ids=None, probs=None, stream=None) -> None:
    from . import moe_ep_peer_dispatch

    moe_ep_peer_dispatch(plan, peer.ep_size, peer.rank, x, live_count, peer.table, route_rows, route_probs, workspace,
                         logits=logits, ids=ids, probs=probs, stream=stream)


def peer_receive(plan: Plan, peer: PeerRegions, wait_limit_ns=None, stream=None) -> None:
    from . import EP_WAIT_LIMIT_NS, moe_ep_peer_receive

    moe_ep_peer_receive(plan, peer.ep_size, peer.region, wait_limit_ns or EP_WAIT_LIMIT_NS, stream=stream)


def peer_expert_forward(shard: Plan, peer: PeerRegions, shard_wbuf, shard_workspace, stream=None) -> None:
    v = peer.views
    moe_forward(shard, v["recv_x"], shard_wbuf, v["recv_live"], v["recv_y"], shard_workspace, ids=v["recv_ids"],
                probs=v["recv_probs"], stream=stream)


def peer_return(plan: Plan, peer: PeerRegions, stream=None) -> None:
    from . import moe_ep_peer_return

    moe_ep_peer_return(plan, peer.ep_size, peer.rank, peer.table, stream=stream)


def peer_combine(plan: Plan, peer: PeerRegions, route_rows, route_probs, live_count, out, wait_limit_ns=None,
                 stream=None) -> None:
    from . import EP_WAIT_LIMIT_NS, moe_ep_peer_combine

    moe_ep_peer_combine(plan, peer.ep_size, peer.region, route_rows, route_probs, live_count, out,
                        wait_limit_ns or EP_WAIT_LIMIT_NS, stream=stream)


def moe_forward_ep_peer(plan: Plan, shard: Plan, peer: PeerRegions, x, shard_wbuf, shard_workspace, live_count, out,
                        route_rows, route_probs, workspace, logits=None, ids=None, probs=None, stream=None) -> None:
    """One EP step on this rank with the exchange through peer memory: no host
    synchronisation, so a CUDA graph can capture it.  `shard` is the rank's
    expert plan (shard_plan_create(plan, ep_size, peer.views["recv_rows"]));
    route_rows [max_live, k] int32 and route_probs [max_live, k] fp32 are the
    step's scratch.  Every rank of the step calls it together."""
    if shard.capacity < peer.views["recv_rows"]:
        raise ValueError(f"the expert plan holds {shard.capacity} rows, the exchange can bring "
                         f"{peer.views['recv_rows']}")
    with _on(stream):
        peer_dispatch(plan, peer, x, live_count, route_rows, route_probs, workspace, logits=logits, ids=ids,
                      probs=probs)
        peer_receive(plan, peer)
        peer_expert_forward(shard, peer, shard_wbuf, shard_workspace)
        peer_return(plan, peer)
        peer_combine(plan, peer, route_rows, route_probs, live_count, out)
