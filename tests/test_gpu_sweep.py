"""The live-count sweep workload at its stated size: H=2688, F=1856, E=128,
top-6, bf16, a 262,144-row buffer, one CUDA graph captured once and replayed
with device live counts 1, 64, 1,024, 8,192, then 64 and 1 again.

Megatron-LM PR #8367, "Problem" and its decode-step table: the live token
count is known only on the device, inside buffers of up to 262,144 rows, and
the expert kernels must do work in proportion to it.  Checked here:

  - every live token's output is bitwise the same at every live count and in
    every replay (the tokens shared by two counts, and a count replayed twice);
  - rows at or past the live count are never written (a NaN fill survives);
  - routes, offsets and the permutation at 8,192 live rows are the oracle's,
    bit for bit (8,192 > 1,024 rows: the three-pass permute);
  - a seeded subset of 48 tokens at 8,192 live rows matches the oracle within
    the bf16 tolerance.

Two plans: the one bench.py times (workspace sized for the whole buffer) and
one sized for the sweep's largest live count (8,192 rows)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import routed_moe_swiglu_b200 as rm
import workloads
from moe_testlib import GpuMoe, assert_close

pytestmark = pytest.mark.gpu

LIVE_ORDER = (1, 64, 1024, 8192, 64, 1)


@pytest.fixture(scope="module")
def sweep_problem():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rm.load_library()
    w = workloads.WORKLOADS["sweep"]
    x, logits = workloads.make_activations(w)  # NaN at and past row 8,192
    weights = workloads.make_weights(w)
    return w, x, logits, weights


def _check_permutation_8192(m: GpuMoe, ref_ids, E):
    v = m.views()
    live, k = ref_ids.shape
    assert np.array_equal(m.read_i32(v["route_ids"], live * k).reshape(live, k), ref_ids)
    offsets, perm, _ = oracle.permute(ref_ids, E)
    assert np.array_equal(m.read_i32(v["offsets"], E + 1), offsets.astype(np.int32))
    assert np.array_equal(m.read_i32(v["perm"], live * k), perm)


@pytest.mark.parametrize("max_live", [0, 8192], ids=["plan_for_whole_buffer", "plan_for_8192_rows"])
def test_sweep_one_graph_bitwise_across_live_counts(sweep_problem, max_live):
    w, x, logits, weights = sweep_problem
    H, E, k, cap = w.hidden, w.num_experts, w.top_k, w.capacity
    m = GpuMoe(H, w.ffn, E, k, cap, weights, max_live=max_live)
    m.clear_status()
    xd, ld = x.cuda(), logits.cuda()
    out = torch.full((cap, H), float("nan"), device="cuda")
    live = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        live.fill_(16)
        rm.moe_forward(m.plan, xd, m.wbuf, live, out, m.ws, logits=ld)  # first call outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        rm.moe_forward(m.plan, xd, m.wbuf, live, out, m.ws, logits=ld)
    res = {}
    for n in LIVE_ORDER:
        out.fill_(float("nan"))
        live.fill_(n)
        g.replay()
        torch.cuda.synchronize()
        assert not torch.isnan(out[:n]).any(), n
        assert torch.isnan(out[n:]).all(), f"rows at or past live count {n} were written"
        o = out[:n].clone()
        if n in res:  # a replay at the same count: the same bits
            assert torch.equal(o.view(torch.int32), res[n].view(torch.int32)), n
        else:
            res[n] = o
        if n == 8192:
            ref_ids, ref_probs = oracle.route(logits[:n].numpy(), k)
            _check_permutation_8192(m, ref_ids, E)
    # tokens shared by two live counts: the same bits
    counts = sorted(res)
    for a, b in zip(counts, counts[1:]):
        assert torch.equal(res[b][:a].view(torch.int32), res[a].view(torch.int32)), (a, b)
    toks = workloads.sample_tokens(8192, 48, w.seed).numpy()
    ref = oracle.forward_bf16(x[:8192], ref_ids, ref_probs, *weights, tokens=toks)
    assert_close(res[8192].cpu().numpy()[toks], ref, "bf16", "sweep at 8,192 live rows")
    assert m.status() == 0
    del g
