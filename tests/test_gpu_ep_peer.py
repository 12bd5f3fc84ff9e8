"""The expert-parallel step with the exchange through peer memory
(include/moe.h, "Expert-parallel exchange through peer memory"), on one GPU.

Every rank's region lives in this GPU's memory, and each rank's table holds
all regions' addresses, so the same kernels that store rows into a peer's
region over NVLink store them here into another rank's region.  The five
steps of every rank run in turn (all dispatches, then all receives, ...), so
each bounded wait finds its flags already raised by kernels that finished
before it: no kernel waits on another that is still to run.  Each rank's
output must equal, bit for bit, the one-GPU forward of its tokens with all
experts (Megatron-LM PR #7798, "What is changed": every dispatched row
computed as a top-1 token with probability 1.0; its "Limitations": an
EP-invariant combine; Megatron-LM PR #7830: the EP transport inside the
kernels).  Not run across several GPUs here: one GPU per test machine.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import routed_moe_swiglu_b200 as rm
import workloads
from moe_testlib import GpuMoe, assert_close
from routed_moe_swiglu_b200 import ep as moe_ep

pytestmark = pytest.mark.gpu

H, F, E, K = 320, 224, 12, 3


class _PeerRank:
    def __init__(self, g, ep, weights, cap, precision, **variant):
        self.g = g
        self.plan = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=K, capacity=cap, precision=precision,
                                       **variant)
        self.region = torch.zeros(rm.moe_ep_region_bytes(self.plan, ep), dtype=torch.uint8, device="cuda")
        recv_rows = rm.moe_ep_region_views(self.plan, ep, self.region)["recv_rows"]
        self.shard = moe_ep.shard_plan_create(self.plan, ep, recv_rows)
        e0, el = moe_ep.expert_range(E, ep, g)
        self.wbuf = rm.alloc_weight_buffer(self.shard)
        wg, wu, wd = (w[e0:e0 + el].contiguous().cuda() for w in weights)
        rm.moe_prepare_weights(self.shard, wg, wu, wd, self.wbuf)
        self.ws = rm.alloc_workspace(self.plan)
        self.shard_ws = rm.alloc_workspace(self.shard)
        self.route_rows = torch.empty(cap, K, dtype=torch.int32, device="cuda")
        self.route_probs = torch.empty(cap, K, dtype=torch.float32, device="cuda")
        self.cap = cap
        self.live = torch.zeros(1, dtype=torch.int32, device="cuda")
        dt = torch.bfloat16 if self.plan.out_dtype == "bf16" else torch.float32
        self.out = torch.full((cap, H), float("nan"), dtype=dt, device="cuda")

    def load(self, x, logits, t0, t1):
        self.n = t1 - t0
        self.x = torch.full((self.cap, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.x[:self.n] = x[t0:t1].cuda()
        self.logits = torch.full((self.cap, E), float("nan"), dtype=torch.float32, device="cuda")
        self.logits[:self.n] = logits[t0:t1].cuda()
        self.live.fill_(self.n)
        self.out.fill_(float("nan"))


def _ranks(ep, weights, cap, precision, **variant):
    ranks = [_PeerRank(g, ep, weights, cap, precision, **variant) for g in range(ep)]
    addrs = [r.region.data_ptr() for r in ranks]
    for r in ranks:
        r.peer = moe_ep.PeerRegions(r.plan, ep, r.g, addresses=addrs, region=r.region)
    return ranks


def _step(ranks, wait_ns=None):
    """Every rank's five steps, each step for all ranks before the next."""
    for r in ranks:
        moe_ep.peer_dispatch(r.plan, r.peer, r.x, r.live, r.route_rows, r.route_probs, r.ws, logits=r.logits)
    for r in ranks:
        moe_ep.peer_receive(r.plan, r.peer, wait_limit_ns=wait_ns)
    for r in ranks:
        moe_ep.peer_expert_forward(r.shard, r.peer, r.wbuf, r.shard_ws)
    for r in ranks:
        moe_ep.peer_return(r.plan, r.peer)
    for r in ranks:
        moe_ep.peer_combine(r.plan, r.peer, r.route_rows, r.route_probs, r.live, r.out, wait_limit_ns=wait_ns)
    torch.cuda.synchronize()


def _one_gpu(x, logits, weights, t0, t1, precision, **variant):
    n = t1 - t0
    m = GpuMoe(H, F, E, K, max(n, 1), weights, precision=precision, **variant)
    xx = torch.full((max(n, 1), H), float("nan"), dtype=torch.bfloat16)
    ll = torch.full((max(n, 1), E), float("nan"), dtype=torch.float32)
    xx[:n], ll[:n] = x[t0:t1], logits[t0:t1]
    return m.forward(xx.cuda(), n, logits=ll.cuda()).cpu()[:n]


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
@pytest.mark.parametrize("ep", [1, 2, 3, 4])
def test_peer_exchange_is_bitwise_the_one_gpu_forward(precision, ep):
    T = 240
    x, logits, weights = workloads.small_case(H, F, E, K, T, seed=61, zipf=True)
    splits = np.linspace(0, T, ep + 1).astype(int).tolist()
    if ep == 3:
        splits = [0, 150, 150, T]  # ragged, and a rank with no tokens of its own
    cap = max(b - a for a, b in zip(splits, splits[1:]))
    ranks = _ranks(ep, weights, max(cap, 1), precision)
    for g, r in enumerate(ranks):
        r.load(x, logits, splits[g], splits[g + 1])
    _step(ranks)
    for g, r in enumerate(ranks):
        assert int(r.peer.views["status"].item()) == 0
        if r.n == 0:
            continue
        want = _one_gpu(x, logits, weights, splits[g], splits[g + 1], precision)
        got = r.out.cpu()[:r.n]
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), (precision, ep, g)
        assert torch.isnan(r.out.cpu()[r.n:]).all()


def test_peer_exchange_second_step_reuses_the_regions():
    """A second step with other tokens and live counts on the same regions:
    the flags carry the step number, nothing is cleared in between."""
    ep = 2
    x, logits, weights = workloads.small_case(H, F, E, K, 300, seed=62, zipf=True)
    ranks = _ranks(ep, weights, 150, "bf16")
    for t0, t1, s0, s1 in ((0, 150, 150, 300), (10, 90, 200, 297)):
        ranks[0].load(x, logits, t0, t1)
        ranks[1].load(x, logits, s0, s1)
        _step(ranks)
        for r, (a, b) in zip(ranks, ((t0, t1), (s0, s1))):
            want = _one_gpu(x, logits, weights, a, b, "bf16")
            assert torch.equal(r.out.cpu()[:r.n].view(torch.int32), want.view(torch.int32))


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_peer_exchange_tiny_workload_against_the_oracle(precision):
    """The tiny workload at EP 2 against the oracle directly (all 64 tokens)."""
    w = workloads.WORKLOADS["tiny"]
    x, logits = workloads.make_activations(w)
    weights = workloads.make_weights(w)
    global H, F, E, K
    saved = (H, F, E, K)
    H, F, E, K = w.hidden, w.ffn, w.num_experts, w.top_k
    try:
        ranks = _ranks(2, weights, 32, precision)
        ranks[0].load(x, logits, 0, 32)
        ranks[1].load(x, logits, 32, 64)
        _step(ranks)
        got = torch.cat([ranks[0].out.cpu()[:32], ranks[1].out.cpu()[:32]]).numpy()
    finally:
        H, F, E, K = saved
    ids, probs = oracle.route(logits.numpy(), w.top_k)
    if precision == "bf16":
        ref = oracle.forward_bf16(x, ids, probs, *weights)
    elif precision == "mxfp8":
        ref = oracle.forward_mxfp8(x, ids, probs, oracle.quantize_weights_mxfp8(*weights))
    else:
        ref = oracle.forward_nvfp4(x, ids, probs, oracle.quantize_weights_nvfp4(*weights))
    assert_close(got, ref, precision, f"EP 2 peer exchange, tiny, {precision}")


def test_peer_exchange_step_in_one_cuda_graph():
    """EP 1 (the rank its own peer): the whole step captured once, replayed at
    several live counts, bitwise the one-GPU forward (no host read anywhere)."""
    T = 200
    x, logits, weights = workloads.small_case(H, F, E, K, T, seed=63, zipf=True)
    (r,) = _ranks(1, weights, T, "bf16")
    r.load(x, logits, 0, T)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe_ep.moe_forward_ep_peer(r.plan, r.shard, r.peer, r.x, r.wbuf, r.shard_ws, r.live, r.out, r.route_rows,
                                   r.route_probs, r.ws, logits=r.logits)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe_ep.moe_forward_ep_peer(r.plan, r.shard, r.peer, r.x, r.wbuf, r.shard_ws, r.live, r.out, r.route_rows,
                                   r.route_probs, r.ws, logits=r.logits)
    for n in (200, 17, 200, 1):
        r.out.fill_(float("nan"))
        r.live.fill_(n)
        g.replay()
        torch.cuda.synchronize()
        want = _one_gpu(x, logits, weights, 0, n, "bf16")
        assert torch.equal(r.out.cpu()[:n].view(torch.int32), want.view(torch.int32)), n
        assert torch.isnan(r.out.cpu()[n:]).all()
    assert int(r.peer.views["status"].item()) == 0
    del g


def test_peer_exchange_wait_runs_out_when_a_source_never_dispatches():
    """After one step of two ranks, rank 0 starts a second step alone: its
    receive waits for rank 1's flag, which never comes.  The wait gives up at
    its limit, sets MOE_DEV_TIMEOUT, and the rank's later kernels do no work:
    its output rows stay unwritten, its combine's wait runs out as well."""
    ep = 2
    x, logits, weights = workloads.small_case(H, F, E, K, 100, seed=64)
    ranks = _ranks(ep, weights, 50, "bf16")
    ranks[0].load(x, logits, 0, 50)
    ranks[1].load(x, logits, 50, 100)
    _step(ranks)
    r = ranks[0]
    r.out.fill_(-3.0)
    moe_ep.peer_dispatch(r.plan, r.peer, r.x, r.live, r.route_rows, r.route_probs, r.ws, logits=r.logits)
    moe_ep.peer_receive(r.plan, r.peer, wait_limit_ns=5_000_000)
    moe_ep.peer_expert_forward(r.shard, r.peer, r.wbuf, r.shard_ws)
    moe_ep.peer_return(r.plan, r.peer)
    moe_ep.peer_combine(r.plan, r.peer, r.route_rows, r.route_probs, r.live, r.out, wait_limit_ns=5_000_000)
    torch.cuda.synchronize()
    assert int(r.peer.views["status"].item()) & rm.MOE_DEV_TIMEOUT
    assert int(r.peer.views["recv_live"].item()) == 0
    assert torch.all(r.out == -3.0)
    assert int(ranks[1].peer.views["status"].item()) == 0
