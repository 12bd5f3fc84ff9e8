"""Robustness checks the pages' test designs ask for, on the GPU.

- Kernel determinism under contention: the forward's bits do not change
  while another stream keeps the GPU busy (a replay under a racing stream).
- The bf16 weight packer byte for byte against a second implementation (a
  numpy unpacking of the blocked layout).
- Out-of-range writes: canary bytes around every buffer the library writes
  (the workspace, the weight buffer, the output) survive a refit and a forward.
- Outlier tokens (a few tokens scaled by 30), in bf16 and MXFP8, against the
  oracle.
- Two layers (plans, weight buffers, workspaces) used in turn stay
  independent.
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


def test_bitwise_identical_under_a_racing_stream():
    w = workloads.WORKLOADS["decode"]
    x, logits = workloads.make_activations(w)
    weights = workloads.make_weights(w)
    m = GpuMoe(w.hidden, w.ffn, w.num_experts, w.top_k, w.capacity, weights, max_live=1024)
    xd, ld = x.cuda(), logits.cuda()
    quiet = m.forward(xd, w.max_live, logits=ld).clone()
    torch.cuda.synchronize()
    a = torch.randn(8192, 8192, device="cuda", dtype=torch.bfloat16)
    other = torch.cuda.Stream()
    outs = []
    for _ in range(3):
        with torch.cuda.stream(other):  # contention: large GEMMs on another stream
            for _ in range(4):
                a = torch.nn.functional.normalize(a @ a, dim=1).to(torch.bfloat16)
        outs.append(m.forward(xd, w.max_live, logits=ld).clone())
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(o[:w.max_live], quiet[:w.max_live])
    assert m.status() == 0


def _unpack_bf16_w1(buf: np.ndarray, E, F, H, hp, fp, relu2=False):
    """Second implementation of the bf16 FC1 layout: blocks [E][row block][K block]
    of [2 atoms][128 rows][64], rows interleaved (16 gate, 16 up) per 16 f."""
    rows = (fp + 255) // 256 * 256 if relu2 else 2 * fp
    blk = buf.reshape(E, rows // 128, hp // 128, 2, 128, 64)
    full = blk.transpose(0, 1, 4, 2, 3, 5).reshape(E, rows, hp)  # [E][row][k]
    if relu2:
        return full[:, :F, :]
    r = np.arange(rows)
    g = (r >> 4) & 1
    f = (r >> 7) * 64 + ((r >> 5) & 3) * 16 + (r & 15)
    gate = np.zeros((E, fp, hp), buf.dtype)
    up = np.zeros((E, fp, hp), buf.dtype)
    gate[:, f[g == 0], :] = full[:, r[g == 0], :]
    up[:, f[g == 1], :] = full[:, r[g == 1], :]
    return gate, up


@pytest.mark.parametrize("H,F", [(256, 200), (320, 512)])
def test_bf16_weight_packer_byte_for_byte(H, F):
    E = 3
    gen = torch.Generator().manual_seed(51)
    wg = torch.randn((E, F, H), generator=gen).bfloat16()
    wu = torch.randn((E, F, H), generator=gen).bfloat16()
    wd = torch.randn((E, H, F), generator=gen).bfloat16()
    plan = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=2, capacity=16)
    buf = rm.alloc_weight_buffer(plan)
    buf.fill_(0x5A)  # stale contents: every byte of the layout must be rewritten
    rm.moe_prepare_weights(plan, wg.cuda(), wu.cuda(), wd.cuda(), buf)
    torch.cuda.synchronize()
    b = buf.cpu().view(torch.int16).numpy()
    hp, fp, hr = (H + 127) // 128 * 128, (F + 127) // 128 * 128, (H + 127) // 128 * 128
    n1 = E * 2 * fp * hp
    gate, up = _unpack_bf16_w1(b[:n1], E, F, H, hp, fp)
    src_g = wg.view(torch.int16).numpy()
    src_u = wu.view(torch.int16).numpy()
    assert np.array_equal(gate[:, :F, :H], src_g) and np.array_equal(up[:, :F, :H], src_u)
    assert np.all(gate[:, :, H:] == 0) and np.all(gate[:, F:, :] == 0) and np.all(up[:, F:, :] == 0)
    off2 = (n1 * 2 + 255) // 256 * 256 // 2
    blk = b[off2:off2 + E * hr * fp].reshape(E, hr // 128, fp // 128, 2, 128, 64)
    w2 = blk.transpose(0, 1, 4, 2, 3, 5).reshape(E, hr, fp)
    assert np.array_equal(w2[:, :H, :F], wd.view(torch.int16).numpy())
    assert np.all(w2[:, :, F:] == 0) and np.all(w2[:, H:, :] == 0)


def _with_canaries(n_bytes: int, pad: int = 4096):
    """A device buffer of n_bytes with `pad` canary bytes on each side (the
    middle starts 256-byte aligned)."""
    full = torch.full((n_bytes + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    return full, full[pad:pad + n_bytes]


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_canaries_around_every_written_buffer_survive(precision):
    H, F, E, k, T, cap = 320, 224, 12, 3, 300, 400
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=52, capacity=cap, zipf=True)
    plan = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=k, capacity=cap, precision=precision)
    wfull, wbuf = _with_canaries(rm.moe_weight_buffer_bytes(plan))
    sfull, ws = _with_canaries(rm.moe_workspace_bytes(plan))
    ofull, obytes = _with_canaries(cap * H * 4)
    out = obytes.view(torch.float32).view(cap, H)
    out.fill_(float("nan"))
    rm.moe_clear_device_status(ws)
    rm.moe_prepare_weights(plan, *(w.cuda() for w in weights), wbuf)
    live = torch.tensor([T], dtype=torch.int32, device="cuda")
    rm.moe_forward(plan, x.cuda(), wbuf, live, out, ws, logits=logits.cuda())
    torch.cuda.synchronize()
    for full, mid in ((wfull, wbuf), (sfull, ws), (ofull, obytes)):
        pad = (full.numel() - mid.numel()) // 2
        assert torch.all(full[:pad] == 0xA5) and torch.all(full[pad + mid.numel():] == 0xA5)
    assert torch.isnan(out[T:]).all() and not torch.isnan(out[:T]).any()
    assert rm.moe_get_device_status(ws) == 0


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_outlier_tokens_match_the_oracle(precision):
    # the pages' second input distribution: 5% of the tokens scaled by 30 (NVFP4's scale per
    # token row keeps the other tokens' resolution)
    H, F, E, k, T = 256, 512, 16, 4, 400
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=53)
    rng = np.random.default_rng(53)
    hot = rng.choice(T, size=T // 20, replace=False)
    x = x.float()
    x[torch.from_numpy(hot)] *= 30.0
    x = x.bfloat16()
    m = GpuMoe(H, F, E, k, T, weights, precision=precision)
    out = m.forward(x.cuda(), T, logits=logits.cuda())
    torch.cuda.synchronize()
    ids, probs = oracle.route(logits.numpy(), k)
    if precision == "bf16":
        ref = oracle.forward_bf16(x, ids, probs, *weights)
    elif precision == "nvfp4":
        ref = oracle.forward_nvfp4(x, ids, probs, oracle.quantize_weights_nvfp4(*weights))
    else:
        ref = oracle.forward_mxfp8(x, ids, probs, oracle.quantize_weights_mxfp8(*weights))
    got = out.cpu().numpy()
    # the tolerance holds for the outlier tokens and for the others separately
    cold = np.setdiff1d(np.arange(T), hot)
    assert_close(got[hot], ref[hot], precision, f"outlier tokens ({precision})")
    assert_close(got[cold], ref[cold], precision, f"other tokens ({precision})")


def test_two_layers_used_in_turn_stay_independent():
    H, F, E, k, T = 256, 256, 8, 2, 128
    xa, la, wa = workloads.small_case(H, F, E, k, T, seed=54)
    xb, lb, wb = workloads.small_case(H, F, E, k, T, seed=55)
    ma = GpuMoe(H, F, E, k, T, wa)
    mb = GpuMoe(H, F, E, k, T, wb, precision="mxfp8")
    outs = []
    for _ in range(2):
        outs.append((ma.forward(xa.cuda(), T, logits=la.cuda()).clone(), mb.forward(xb.cuda(), T, logits=lb.cuda()).clone()))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    ida, pa = oracle.route(la.numpy(), k)
    assert_close(outs[0][0].cpu().numpy(), oracle.forward_bf16(xa, ida, pa, *wa), "bf16", "layer a")
    idb, pb = oracle.route(lb.numpy(), k)
    assert_close(outs[0][1].cpu().numpy(),
                 oracle.forward_mxfp8(xb, idb, pb, oracle.quantize_weights_mxfp8(*wb)), "mxfp8", "layer b")
