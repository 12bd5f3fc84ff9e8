"""Expert parallelism on one GPU: bitwise EP invariance.

Every rank's phases of the EP step (dispatch, the rank's experts over the rows
it receives, combine) run in turn on one GPU; the all-to-alls between them are
plain tensor copies done here, in the collective's row order, so no kernel
waits on another.  Each rank's output must equal, bit for bit, the one-GPU
forward of the same tokens with all experts (Megatron-LM PR #7798, "What is
changed": every dispatched row computed as a top-1 token with probability 1.0;
its "Limitations": an EP-invariant combine; cudnn-frontend PR #448, MoeEp).
The dispatch's integer outputs are checked against the oracle's routes.
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

# H, F not multiples of 128; E = 12 divides into 2, 3, 4 and 6 ranks
H, F, E, K = 320, 224, 12, 3


class _Rank:
    def __init__(self, g, ep, x, logits, weights, t0, t1, precision, max_recv, **variant):
        self.n = t1 - t0
        cap = max(self.n, 1)
        self.plan = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=K, capacity=cap, precision=precision,
                                       **variant)
        self.shard = moe_ep.shard_plan_create(self.plan, ep, max_recv)
        e0, el = moe_ep.expert_range(E, ep, g)
        self.wbuf = rm.alloc_weight_buffer(self.shard)
        wg, wu, wd = (w[e0:e0 + el].contiguous().cuda() for w in weights)
        rm.moe_prepare_weights(self.shard, wg, wu, wd, self.wbuf)
        self.bufs = moe_ep.EpBuffers.allocate(self.plan, self.shard, ep)
        self.x = torch.full((cap, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.x[:self.n] = x[t0:t1].cuda()
        self.logits = torch.full((cap, E), float("nan"), dtype=torch.float32, device="cuda")
        self.logits[:self.n] = logits[t0:t1].cuda()
        self.live = torch.tensor([self.n], dtype=torch.int32, device="cuda")
        dt = torch.bfloat16 if self.plan.out_dtype == "bf16" else torch.float32
        self.out = torch.full((cap, H), float("nan"), dtype=dt, device="cuda")


def _run_ep(precision, ep, x, logits, weights, splits, routes=None, **variant):
    """The EP step for ranks owning tokens [splits[g], splits[g+1]); `routes`
    = (ids, probs) for caller-given routes instead of the logits."""
    T = splits[-1]
    ranks = [_Rank(g, ep, x, logits, weights, splits[g], splits[g + 1], precision, max(T * K, 1), **variant)
             for g in range(ep)]
    for g, r in enumerate(ranks):
        if routes is None:
            moe_ep.dispatch(r.plan, r.bufs, r.x, r.live, logits=r.logits)
        else:
            ids = torch.zeros((max(r.n, 1), K), dtype=torch.int32)
            probs = torch.zeros((max(r.n, 1), K), dtype=torch.float32)
            ids[:r.n] = routes[0][splits[g]:splits[g + 1]]
            probs[:r.n] = routes[1][splits[g]:splits[g + 1]]
            moe_ep.dispatch(r.plan, r.bufs, r.x, r.live, ids=ids.cuda(), probs=probs.cuda())
    torch.cuda.synchronize()
    counts = [r.bufs.send_counts.tolist() for r in ranks]  # counts[s][d]: rows from s to d
    for d, r in enumerate(ranks):
        n_recv = sum(counts[s][d] for s in range(ep))
        for name in ("x", "ids", "probs"):
            if n_recv == 0:
                break
            parts = []
            for s in range(ep):
                off = sum(counts[s][:d])
                parts.append(getattr(ranks[s].bufs, "send_" + name)[off:off + counts[s][d]])
            getattr(r.bufs, "recv_" + name).view(r.shard.capacity, -1)[:n_recv] = torch.cat(parts).view(n_recv, -1)
        moe_ep.expert_forward(r.shard, r.bufs, r.wbuf, n_recv)
    torch.cuda.synchronize()
    for s, r in enumerate(ranks):
        parts = []
        for d in range(ep):
            off = sum(counts[q][d] for q in range(s))
            parts.append(ranks[d].bufs.recv_y[off:off + counts[s][d]])
        r.bufs.y_back[:sum(counts[s])] = torch.cat(parts)
        moe_ep.combine(r.plan, r.bufs, r.live, r.out)
    torch.cuda.synchronize()
    for r in ranks:
        assert rm.moe_get_device_status(r.bufs.shard_workspace) == 0
    return ranks, counts


def _one_gpu(precision, x, logits, weights, T, routes=None, **variant):
    m = GpuMoe(H, F, E, K, T, weights, precision=precision, **variant)
    if routes is None:
        out = m.forward(x[:T].cuda(), T, logits=logits[:T].cuda())
    else:
        out = m.forward(x[:T].cuda(), T, ids=routes[0].cuda(), probs=routes[1].cuda())
    torch.cuda.synchronize()
    return out, m


def _assert_bitwise(ranks, ref, splits):
    for g, r in enumerate(ranks):
        got = r.out[:r.n]
        want = ref[splits[g]:splits[g + 1]]
        assert torch.equal(got.view(torch.int32) if got.dtype == torch.float32 else got.view(torch.int16),
                           want.view(torch.int32) if want.dtype == torch.float32 else want.view(torch.int16)), \
            f"rank {g}: EP output differs from the one-GPU forward"


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
@pytest.mark.parametrize("ep", [2, 4])
def test_ep_output_is_bitwise_the_one_gpu_forward(precision, ep):
    T = 700
    x, logits, weights = workloads.small_case(H, F, E, K, T, seed=31, zipf=True)
    # ragged token shares, one rank with none when ep = 4
    splits = [0, 333, T] if ep == 2 else [0, 250, 250, 611, T]
    ranks, counts = _run_ep(precision, ep, x, logits, weights, splits)
    ref, _ = _one_gpu(precision, x, logits, weights, T)
    _assert_bitwise(ranks, ref, splits)
    assert sum(sum(c) for c in counts) == T * K


def test_ep_dispatch_matches_the_oracle_routes():
    """Send rows in expert order, stable by token; local ids; per-destination
    counts; each route's send row; all integer work, so bit-exact."""
    T, ep = 301, 3
    x, logits, weights = workloads.small_case(H, F, E, K, T, seed=32, zipf=True)
    ranks, counts = _run_ep("bf16", ep, x, logits, weights, [0, T, T, T])
    r = ranks[0]
    ids, probs = oracle.route(logits[:T].numpy(), K)
    order = sorted(((int(ids[t, j]), t, j) for t in range(T) for j in range(K)))
    el = E // ep
    want_counts = [sum(1 for e, _, _ in order if e // el == g) for g in range(ep)]
    assert counts[0] == want_counts
    send_x = r.bufs.send_x[:T * K].cpu()
    send_ids = r.bufs.send_ids[:T * K].cpu().numpy()
    send_probs = r.bufs.send_probs[:T * K].cpu().numpy()
    route_rows = r.bufs.route_rows[:T].cpu().numpy()
    route_probs = r.bufs.route_probs[:T].cpu().numpy()
    for row, (e, t, j) in enumerate(order):
        assert send_ids[row] == e % el
        assert route_rows[t, j] == row
        assert torch.equal(send_x[row].view(torch.int16), x[t].view(torch.int16))
    assert np.all(send_probs == 1.0)
    # the router's own probabilities, passed through unchanged (and within an
    # ulp of the oracle's, as the router's parity test requires)
    gpu_ids = torch.empty((T, K), dtype=torch.int32, device="cuda")
    gpu_probs = torch.empty((T, K), dtype=torch.float32, device="cuda")
    rm.moe_route_topk(r.plan, r.logits, r.live, gpu_ids, gpu_probs)
    np.testing.assert_array_equal(gpu_ids.cpu().numpy(), ids)
    assert np.array_equal(route_probs.view(np.int32), gpu_probs.cpu().numpy().view(np.int32))
    assert np.all(np.abs(route_probs - probs) <= np.spacing(np.abs(probs.astype(np.float32))))
    # the other ranks own no tokens: nothing to send
    assert counts[1] == [0] * ep and counts[2] == [0] * ep


@pytest.mark.parametrize("precision", ["bf16", "nvfp4"])
def test_ep_variants_are_bitwise_the_one_gpu_forward(precision):
    """Probabilities applied in FC1 (sent with the rows), the gate/up clamp, a
    bf16 output, and squared-ReLU experts."""
    T, ep = 400, 2
    x, logits, weights = workloads.small_case(H, F, E, K, T, seed=33, zipf=True)
    splits = [0, 177, T]
    for variant in (dict(probs_in_fc1=True, gate_up_clamp=1.5, out_dtype="bf16"), dict(squared_relu=True)):
        ranks, _ = _run_ep(precision, ep, x, logits, weights, splits, **variant)
        ref, _ = _one_gpu(precision, x, logits, weights, T, **variant)
        _assert_bitwise(ranks, ref, splits)


def test_ep_caller_routes_with_a_dropped_token():
    """Caller-given routes in any order; a token with a repeated id is dropped
    (zero output row, flagged) exactly as in the one-GPU forward."""
    T, ep = 200, 4
    x, logits, weights = workloads.small_case(H, F, E, K, T, seed=34)
    ids, probs = oracle.route(logits[:T].numpy(), K)
    rng = np.random.default_rng(5)
    perm = np.argsort(rng.random((T, K)), axis=1)  # shuffle each token's routes
    ids = np.take_along_axis(ids, perm, axis=1).astype(np.int32)
    probs = np.take_along_axis(probs, perm, axis=1).astype(np.float32)
    ids[17, 1] = ids[17, 0]  # token 17: a repeated expert id
    routes = (torch.from_numpy(ids), torch.from_numpy(probs))
    splits = [0, 60, 60, 150, T]
    ranks, counts = _run_ep("bf16", ep, x, logits, weights, splits, routes=routes)
    ref, m = _one_gpu("bf16", x, logits, weights, T, routes=routes)
    _assert_bitwise(ranks, ref, splits)
    assert torch.all(ranks[0].out[17] == 0)
    assert rm.moe_get_device_status(ranks[0].bufs.workspace) & rm.MOE_DEV_BAD_ROUTE
    assert sum(sum(c) for c in counts) == (T - 1) * K


def test_ep_step_through_nccl_with_one_rank():
    """moe_forward_ep itself over a one-rank NCCL group (each all-to-all is a
    copy to itself): the NCCL calls on device buffers, the host split sizes and
    the phases in sequence give the one-GPU forward's output bit for bit."""
    import socket

    import torch.distributed as dist

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1)
    try:
        T = 500
        x, logits, weights = workloads.small_case(H, F, E, K, T, seed=35, zipf=True)
        for precision in ("bf16", "mxfp8"):
            plan = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=K, capacity=T, precision=precision)
            shard = moe_ep.shard_plan_create(plan, 1, T * K)
            wbuf = rm.alloc_weight_buffer(shard)
            rm.moe_prepare_weights(shard, *(w.cuda() for w in weights), wbuf)
            bufs = moe_ep.EpBuffers.allocate(plan, shard, 1)
            out = torch.full((T, H), float("nan"), device="cuda")
            live = torch.tensor([T], dtype=torch.int32, device="cuda")
            moe_ep.moe_forward_ep(plan, shard, bufs, x.cuda(), wbuf, live, out, logits=logits.cuda())
            torch.cuda.synchronize()
            ref, _ = _one_gpu(precision, x, logits, weights, T)
            assert torch.equal(out.view(torch.int32), ref.view(torch.int32)), precision
            assert bufs.send_counts.tolist() == [T * K]
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_ep_output_against_the_oracle(precision):
    """The EP step at EP 2 against the oracle directly, every token."""
    T = 120
    x, logits, weights = workloads.small_case(H, F, E, K, T, seed=33, zipf=True)
    ranks, _ = _run_ep(precision, 2, x, logits, weights, [0, 70, T])
    got = torch.cat([ranks[0].out[:70], ranks[1].out[:T - 70]]).float().cpu().numpy()
    ids, probs = oracle.route(logits[:T].numpy(), K)
    if precision == "bf16":
        ref = oracle.forward_bf16(x[:T], ids, probs, *weights)
    elif precision == "mxfp8":
        ref = oracle.forward_mxfp8(x[:T], ids, probs, oracle.quantize_weights_mxfp8(*weights))
    else:
        ref = oracle.forward_nvfp4(x[:T], ids, probs, oracle.quantize_weights_nvfp4(*weights))
    assert_close(got, ref, precision, f"EP 2 ({precision}) against the oracle")
