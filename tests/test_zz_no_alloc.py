"""moe_forward_noalloc: the forward for callers that cannot allocate device
memory (a plug-in handed only its input and output pointers, code that must
not call cudaMalloc inside someone else's stream capture).  Its scratch is
the library's fixed device array instead of a caller workspace; these tests
check it through the C ABI against moe_forward with a caller workspace, on
consecutive calls, bit for bit (the same kernels on the same inputs: a
leftover of an earlier call in the shared array would show as changed bits),
and that plans too large for the array are refused.

The file name sorts last so that a run stopping at its first failure has
already run every other test."""
from __future__ import annotations

import pytest
import torch

import routed_moe_swiglu_b200 as rm
import workloads

pytestmark = pytest.mark.gpu


def _setup(H, F, E, k, T, cap, seed, precision="bf16"):
    x, logits, (wg, wu, wd) = workloads.small_case(H, F, E, k, T, seed=seed, capacity=cap)
    plan = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=k, capacity=cap, precision=precision)
    assert rm.moe_workspace_bytes(plan) <= rm.MOE_NOALLOC_SCRATCH_BYTES
    wbuf = rm.alloc_weight_buffer(plan)
    rm.moe_prepare_weights(plan, wg.cuda(), wu.cuda(), wd.cuda(), wbuf)
    return plan, wbuf, x.cuda(), logits.cuda()


def _reference(plan, wbuf, x, logits, live, cap, H):
    ws = rm.alloc_workspace(plan)
    out = torch.full((cap, H), float("nan"), device="cuda")
    rm.moe_forward(plan, x, wbuf, live, out, ws, logits=logits)
    torch.cuda.synchronize()
    return out.cpu()


def _noalloc(plan, wbuf, x, logits, live, cap, H):
    out = torch.full((cap, H), float("nan"), device="cuda")
    rm.moe_forward_noalloc(plan, x, wbuf, live, out, logits=logits)
    torch.cuda.synchronize()
    return out.cpu()


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_noalloc_matches_workspace_forward_on_consecutive_calls(precision):
    H, F, E, k, T, cap = 256, 512, 8, 2, 64, 80
    plan, wbuf, x, logits = _setup(H, F, E, k, T, cap, seed=101, precision=precision)
    live = torch.tensor([T], dtype=torch.int32, device="cuda")
    ref = _reference(plan, wbuf, x, logits, live, cap, H)
    for _ in range(2):  # the shared scratch keeps the previous call's contents
        got = _noalloc(plan, wbuf, x, logits, live, cap, H)
        assert torch.equal(got[:T].view(torch.int32), ref[:T].view(torch.int32)), precision
        assert torch.isnan(got[T:]).all()


def test_noalloc_follows_a_different_problem():
    """A call after a call on other shapes and live counts sees none of its leftovers."""
    a = _setup(320, 224, 6, 3, 150, 160, seed=102)
    b = _setup(256, 256, 16, 4, 40, 48, seed=103)
    for (plan, wbuf, x, logits), (T, cap, H) in ((a, (150, 160, 320)), (b, (40, 48, 256)), (a, (97, 160, 320))):
        live = torch.tensor([T], dtype=torch.int32, device="cuda")
        ref = _reference(plan, wbuf, x, logits, live, cap, H)
        got = _noalloc(plan, wbuf, x, logits, live, cap, H)
        assert torch.equal(got[:T].view(torch.int32), ref[:T].view(torch.int32)), (T, cap, H)
        assert torch.isnan(got[T:]).all()


def test_noalloc_refuses_plans_larger_than_its_scratch():
    plan = rm.moe_plan_create(hidden=2048, ffn=1024, num_experts=128, top_k=8, capacity=65536)
    assert rm.moe_workspace_bytes(plan) > rm.MOE_NOALLOC_SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    live = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(rm.MoeError) as ei:
        rm.moe_forward_noalloc(plan, dummy, dummy, live, dummy.view(torch.float32), logits=dummy.view(torch.float32))
    assert ei.value.code == 4  # MOE_ERR_WORKSPACE_TOO_SMALL, nothing launched
