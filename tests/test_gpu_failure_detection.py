"""Device-side failure detection without a GPU fault.

Every pipeline wait of the forward's kernels is bounded; a wait that runs out
sets MOE_DEV_TIMEOUT in the status word, stops the other roles of its CTA
through an abort flag and lets the kernel exit normally.
`moe_check_bounded_wait` runs that mechanism on waits that nothing
satisfies; the test reads the status the device reported, the waits'
durations, and then uses the same context for a forward checked against the
oracle.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import routed_moe_swiglu_b200 as rm
import workloads
from moe_testlib import GpuMoe, assert_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_reports_timeout_and_context_stays_usable():
    limit_ns = 20_000_000  # 20 ms
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    rm.moe_check_bounded_wait(limit_ns, status, elapsed)
    torch.cuda.synchronize()
    assert status.item() == rm.MOE_DEV_TIMEOUT
    waited, stopped = elapsed.cpu().tolist()
    assert limit_ns <= waited < 10 * limit_ns, waited       # the wait ran out at its limit
    assert waited <= stopped < waited + 100_000_000, stopped  # the other left through the abort flag

    # a second call ORs into the caller's word; a fresh word gets the bit again
    rm.moe_check_bounded_wait(1_000, status)
    torch.cuda.synchronize()
    assert status.item() == rm.MOE_DEV_TIMEOUT

    # the context is intact: a forward on the same device matches the oracle
    w = workloads.WORKLOADS["tiny"]
    x, logits = workloads.make_activations(w)
    weights = workloads.make_weights(w)
    m = GpuMoe(w.hidden, w.ffn, w.num_experts, w.top_k, w.capacity, weights)
    m.clear_status()
    out = m.forward(x.cuda(), w.max_live, logits=logits.cuda())
    torch.cuda.synchronize()
    ids, probs = oracle.route(logits.numpy(), w.top_k)
    ref = oracle.forward_bf16(x, ids, probs, *weights)
    assert_close(out.cpu().numpy(), ref, "bf16", "forward after a timed-out wait")
    assert m.status() == 0


def test_bounded_wait_rejects_bad_arguments():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in (0, 10_000_000_001):
        with pytest.raises(rm.MoeError) as ei:
            rm.moe_check_bounded_wait(bad, status)
        assert ei.value.code == rm.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert status.item() == 0


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_forward_does_no_work_while_a_timeout_is_flagged(precision):
    """A forward whose workspace carries MOE_DEV_TIMEOUT (set here on the host,
    as a wait that ran out would set it) writes no output rows and reads no
    permutation: every kernel after the router sees the bit and does nothing.
    Cleared, the same workspace serves a correct forward again.  Shapes past
    1,024 live rows, so the permute runs its multi-block form."""
    H, F, E, k, T = 256, 256, 16, 4, 1500
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=77)
    m = GpuMoe(H, F, E, k, T, weights, precision=precision)
    m.clear_status()
    good = m.forward(x.cuda(), T, logits=logits.cuda()).cpu()
    assert m.status() == 0
    ws_status = m.ws[:4].view(torch.int32)
    ws_status.fill_(rm.MOE_DEV_TIMEOUT)
    out = m.forward(x.cuda(), T, logits=logits.cuda(), sentinel=-5.0)
    torch.cuda.synchronize()
    assert torch.all(out == -5.0)
    assert m.status() & rm.MOE_DEV_TIMEOUT
    m.clear_status()
    again = m.forward(x.cuda(), T, logits=logits.cuda()).cpu()
    assert m.status() == 0
    assert torch.equal(again.view(torch.int32), good.view(torch.int32))
