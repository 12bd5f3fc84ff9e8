"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: routed expert ids, the permutation (offsets, perm), MXFP8 codes
and scales.  Floating point: the tolerance of tests/moe_testlib.py.
Each test fails (never skips) when the library is missing on a machine with a GPU."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import routed_moe_swiglu_b200 as rm
import workloads
from moe_testlib import GpuMoe, assert_close, oracle_forward, workload_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rm.load_library()  # raises when the CUDA library is missing
    torch.cuda.init()


# ---------------------------------------------------------------- route


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "sweep"])
def test_route_ids_bit_exact(name):
    w = workloads.WORKLOADS[name]
    _, logits = workloads.make_activations(w)
    live = w.max_live
    plan = rm.moe_plan_create(hidden=w.hidden, ffn=w.ffn, num_experts=w.num_experts, top_k=w.top_k,
                              capacity=w.capacity, max_live_rows=w.max_live)
    lg = logits.cuda()
    ids = torch.full((w.capacity, w.top_k), -7, dtype=torch.int32, device="cuda")
    probs = torch.full((w.capacity, w.top_k), -7.0, dtype=torch.float32, device="cuda")
    lv = torch.tensor([live], dtype=torch.int32, device="cuda")
    rm.moe_route_topk(plan, lg, lv, ids, probs)
    torch.cuda.synchronize()
    ids_h, probs_h = ids.cpu().numpy(), probs.cpu().numpy()
    ref_ids, ref_probs = oracle.route(logits[:live].numpy(), w.top_k)
    assert np.array_equal(ids_h[:live], ref_ids)
    ulp = np.spacing(np.abs(ref_probs))
    assert np.all(np.abs(probs_h[:live] - ref_probs) <= ulp)
    if live < w.capacity:  # rows past the live count untouched
        assert np.all(ids_h[live:live + 64] == -7) and np.all(probs_h[live:live + 64] == -7.0)


# ---------------------------------------------------------------- quantize


@pytest.mark.parametrize("anchor", [0.0, 1.0, 2.0 ** 20, 2.0 ** -20, 3.0])
def test_mxfp8_quantize_exhaustive_bf16(anchor):
    bits = np.arange(65536, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals)]
    blocks = np.zeros((vals.size, 32), np.float32)
    blocks[:, 0] = vals
    blocks[:, 1] = anchor
    blocks[:, 7] = -vals * 0.5
    x = torch.from_numpy(blocks).to(torch.bfloat16)
    blocks = x.float().numpy()  # the bf16 values both sides quantise
    q = torch.empty((vals.size, 32), dtype=torch.uint8, device="cuda")
    s = torch.empty((vals.size, 1), dtype=torch.uint8, device="cuda")
    rm.mxfp8_quantize_block32(x.cuda(), q, s)
    torch.cuda.synchronize()
    rq, rs = oracle.mxfp8_quantize(blocks)
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(q.cpu().numpy(), rq)


def test_mxfp8_quantize_strided_and_live_bound():
    gen = torch.Generator().manual_seed(3)
    full = (torch.randn((300, 512), generator=gen) * torch.exp(torch.randn((300, 1), generator=gen) * 4))
    full = full.to(torch.bfloat16)
    x = full.cuda()[:, :384]  # row stride 512, 384 columns
    q = torch.full((300, 384), 0xAB, dtype=torch.uint8, device="cuda")
    s = torch.full((300, 12), 0xAB, dtype=torch.uint8, device="cuda")
    live = torch.tensor([257], dtype=torch.int32, device="cuda")
    rm.mxfp8_quantize_block32(x, q, s, live_rows=live)
    torch.cuda.synchronize()
    rq, rs = oracle.mxfp8_quantize_bf16(full[:, :384].contiguous())
    assert np.array_equal(q.cpu().numpy()[:257], rq[:257])
    assert np.array_equal(s.cpu().numpy()[:257], rs[:257])
    assert np.all(q.cpu().numpy()[257:] == 0xAB) and np.all(s.cpu().numpy()[257:] == 0xAB)


# ---------------------------------------------------------------- forward, bf16


PRECISIONS = ("bf16", "mxfp8", "nvfp4")


def _oracle_tokens(precision, x, ids, probs, weights):
    """The oracle's output for caller routes in the given precision."""
    if precision == "mxfp8":
        return oracle.forward_mxfp8(x, ids, probs, oracle.quantize_weights_mxfp8(*weights))
    if precision == "nvfp4":
        return oracle.forward_nvfp4(x, ids, probs, oracle.quantize_weights_nvfp4(*weights))
    return oracle.forward_bf16(x, ids, probs, *weights)


def _check_permutation(m: GpuMoe, ref_ids, E, align=32):
    v = m.views()
    live, k = ref_ids.shape
    ids_gpu = m.read_i32(v["route_ids"], live * k).reshape(live, k)
    assert np.array_equal(ids_gpu, ref_ids)
    offsets, perm, inv = oracle.permute(ref_ids, E)
    off_gpu = m.read_i32(v["offsets"], E + 1)
    assert np.array_equal(off_gpu, offsets.astype(np.int32))
    perm_gpu = m.read_i32(v["perm"], live * k)
    assert np.array_equal(perm_gpu, perm)
    # padded rows: every expert segment starts on a 32-row (bf16) / 128-row (MXFP8) boundary, order kept
    pad = m.read_i32(v["pad_offsets"], E + 1)
    inv_gpu = m.read_i32(v["inv"], live * k).reshape(live, k)
    e_of = ref_ids
    rank = inv.astype(np.int64) - offsets[e_of]
    assert np.array_equal(inv_gpu, (pad[e_of] + rank).astype(np.int32))
    assert np.all(pad % align == 0)


def test_forward_tiny_all_tokens():
    w, x, logits, weights = workload_problem("tiny")
    m = GpuMoe(w.hidden, w.ffn, w.num_experts, w.top_k, w.capacity, weights)
    out = m.forward(x.cuda(), w.max_live, logits=logits.cuda())
    torch.cuda.synchronize()
    ref_ids, _, ref = oracle_forward(x, logits, weights, w.top_k, w.max_live)
    assert_close(out.cpu().numpy(), ref, "bf16", "tiny")
    _check_permutation(m, ref_ids, w.num_experts)
    assert m.status() == 0


@pytest.mark.parametrize("H,F,E,k,T,cap", [
    (264, 200, 5, 3, 300, 320),     # K tail (264 = 4*64 + 8), N tail, ragged M tiles
    (512, 384, 16, 4, 1000, 1000),  # several M tiles per expert
    (128, 136, 1, 1, 130, 256),     # one expert: a dense SwiGLU MLP, 2 M tiles
    (256, 512, 64, 8, 17, 64),      # more experts than routes: many empty experts
])
def test_forward_ragged_shapes(H, F, E, k, T, cap):
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=H + F + E, capacity=cap)
    m = GpuMoe(H, F, E, k, cap, weights)
    out = m.forward(x.cuda(), T, logits=logits.cuda())
    torch.cuda.synchronize()
    ref_ids, _, ref = oracle_forward(x, logits, weights, k, T)
    o = out.cpu().numpy()
    assert_close(o[:T], ref, "bf16", f"ragged {H},{F},{E},{k},{T}")
    assert np.all(np.isnan(o[T:]))  # rows past the live count never written
    _check_permutation(m, ref_ids, E)


@pytest.mark.parametrize("precision", ["bf16", "mxfp8"])
def test_small_plan_permute_matches_three_pass_permute(precision):
    """Plans of at most 1,024 live rows permute in one block; larger plans in
    three passes (per-block histogram, scan, per-block scatter).  Both forms
    give the oracle's permutation, and the same tokens the same output bit for
    bit, on a skewed load with a ragged last chunk; the three-pass plan keeps
    the shared tokens' outputs bit for bit across live counts 1,000..1,100."""
    H, F, E, k, T = 256, 192, 24, 4, 1000
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=2024, capacity=4096, zipf=True)
    small = GpuMoe(H, F, E, k, 4096, weights, precision=precision, max_live=1024)
    large = GpuMoe(H, F, E, k, 4096, weights, precision=precision, max_live=4096)
    outs = []
    for m in (small, large):
        outs.append(m.forward(x.cuda(), T, logits=logits.cuda()).cpu().numpy())
        assert m.status() == 0
    torch.cuda.synchronize()
    assert np.array_equal(outs[0][:T], outs[1][:T])
    vs, vl = small.views(), large.views()
    for name, count in (("route_ids", T * k), ("offsets", E + 1), ("pad_offsets", E + 1), ("perm", T * k),
                        ("inv", T * k)):
        assert np.array_equal(small.read_i32(vs[name], count), large.read_i32(vl[name], count)), name
    ref_ids, _ = oracle.route(logits[:T].numpy(), k)
    _check_permutation(small, ref_ids, E, align=32 if precision == "bf16" else 128)
    # the three-pass plan across live counts around the one-block plans' limit: the shared
    # tokens' outputs agree bit for bit and every permutation is the oracle's
    x2, logits2, _ = workloads.small_case(H, F, E, k, 1100, seed=2024, capacity=4096, zipf=True)
    outs = {}
    for n in (1000, 1024, 1025, 1100):
        outs[n] = large.forward(x2.cuda(), n, logits=logits2.cuda()).cpu().numpy()
        assert large.status() == 0
        ids_n, _ = oracle.route(logits2[:n].numpy(), k)
        _check_permutation(large, ids_n, E, align=32 if precision == "bf16" else 128)
    for n in (1024, 1025, 1100):
        assert np.array_equal(outs[n][:1000], outs[1000][:1000]), n


@pytest.fixture(scope="module")
def decode_problem():
    w, x, logits, weights = workload_problem("decode")
    m = GpuMoe(w.hidden, w.ffn, w.num_experts, w.top_k, w.capacity, weights)
    return w, x, logits, weights, m


def test_forward_decode_all_live_tokens(decode_problem):
    w, x, logits, weights, m = decode_problem
    live = w.max_live
    out = m.forward(x.cuda(), live, logits=logits.cuda(), sentinel=-12345.0)
    torch.cuda.synchronize()
    ref_ids, _, ref = oracle_forward(x, logits, weights, w.top_k, live)
    o = out.cpu().numpy()
    assert_close(o[:live], ref, "bf16", "decode")
    assert np.all(o[live:] == -12345.0)
    _check_permutation(m, ref_ids, w.num_experts)
    assert m.status() == 0


def test_forward_prefill_subset_and_full_permutation():
    w, x, logits, weights = workload_problem("prefill")
    m = GpuMoe(w.hidden, w.ffn, w.num_experts, w.top_k, w.capacity, weights)
    live = w.max_live
    out = m.forward(x.cuda(), live, logits=logits.cuda())
    torch.cuda.synchronize()
    toks = workloads.sample_tokens(live, 512, w.seed).numpy()
    ref_ids, _, ref = oracle_forward(x, logits, weights, w.top_k, live, tokens=toks)
    assert_close(out.cpu().numpy()[toks], ref, "bf16", "prefill subset")
    _check_permutation(m, ref_ids, w.num_experts)
    counts = np.bincount(ref_ids.reshape(-1), minlength=w.num_experts)
    assert counts.max() > 8 * np.median(counts)  # the Zipf bias really skews the loads


def test_every_tile_width():
    """Caller routes that give experts 1..513 routes: every route-tile width
    (N = 32..256 in steps of 32), full tiles followed by a tail of 1, 31, 32
    or 33 rows, and K and output-column tails (H = 320, F = 200)."""
    H, F, E, k = 320, 200, 20, 2
    counts = np.array([1, 15, 16, 17, 31, 32, 33, 63, 64, 65, 100, 127, 128, 129, 200, 255, 256, 257, 300, 513])
    T = int(counts.sum()) // k
    x, _, weights = workloads.small_case(H, F, E, k, T, seed=77)
    gen = np.random.default_rng(77)
    experts = np.repeat(np.arange(E), counts)  # route list by expert; token t gets entries t and t + T
    ids = np.stack([experts[:T], experts[T:]], axis=1)
    ids = ids[gen.permutation(T)].astype(np.int32)
    assert np.all(ids[:, 0] != ids[:, 1])
    p = gen.uniform(0.1, 1.0, size=(T, k))
    probs = (p / p.sum(axis=1, keepdims=True)).astype(np.float32)
    m = GpuMoe(H, F, E, k, T, weights)
    out = m.forward(x.cuda(), T, ids=torch.from_numpy(ids).cuda(), probs=torch.from_numpy(probs).cuda())
    torch.cuda.synchronize()
    ref = oracle.forward_bf16(x, ids, probs, *weights)
    assert_close(out.cpu().numpy(), ref, "bf16", "every tile width")
    assert m.status() == 0


# ---------------------------------------------------------------- invariance and edge cases


def test_batch_invariance_across_live_counts_and_replays(decode_problem):
    """A token's output is bitwise identical whatever the live count and on
    every repeat (the live count is only read on the device)."""
    w, x, logits, weights, m = decode_problem
    xd, ld = x.cuda(), logits.cuda()
    outs = {}
    for live in (1, 7, 64, 200, 256):
        outs[live] = m.forward(xd, live, logits=ld).cpu()
    for live in (7, 64, 200, 256):
        n = min(live, 1)
        assert torch.equal(outs[live][:n], outs[1][:n])
    for a, b in ((7, 64), (64, 200), (200, 256)):
        assert torch.equal(outs[a][:a], outs[b][:a])
    again = m.forward(xd, 256, logits=ld).cpu()
    assert torch.equal(again[:256], outs[256][:256])


def test_token_order_invariance():
    H, F, E, k, T = 256, 256, 16, 4, 200
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=77)
    m = GpuMoe(H, F, E, k, T, weights)
    base = m.forward(x.cuda(), T, logits=logits.cuda()).cpu()
    p = torch.randperm(T, generator=torch.Generator().manual_seed(1))
    perm_out = m.forward(x[p].contiguous().cuda(), T, logits=logits[p].contiguous().cuda()).cpu()
    assert torch.equal(perm_out, base[p])


def test_caller_routes_match_router_and_are_canonicalised():
    H, F, E, k, T = 256, 256, 16, 4, 100
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=5)
    m = GpuMoe(H, F, E, k, T, weights)
    a = m.forward(x.cuda(), T, logits=logits.cuda()).cpu()
    ids, probs = oracle.route(logits.numpy(), k)
    # hand them over reversed: the library must sort them back
    ids_r = torch.from_numpy(ids[:, ::-1].copy()).cuda()
    probs_r = torch.from_numpy(probs[:, ::-1].copy()).cuda()
    b = m.forward(x.cuda(), T, ids=ids_r, probs=probs_r).cpu()
    assert torch.equal(a, b)
    assert m.status() == 0


@pytest.mark.parametrize("precision", PRECISIONS)
def test_bad_routes_are_flagged_and_zeroed(precision):
    H, F, E, k, T = 256, 256, 8, 2, 10
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=6)
    m = GpuMoe(H, F, E, k, T, weights, precision=precision)
    ids, probs = oracle.route(logits.numpy(), k)
    ids[3] = [4, 4]      # repeated expert
    ids[5, 1] = E + 3    # out of range
    m.clear_status()
    out = m.forward(x.cuda(), T, ids=torch.from_numpy(ids).cuda(), probs=torch.from_numpy(probs).cuda()).cpu()
    assert m.status() & rm.MOE_DEV_BAD_ROUTE
    assert torch.all(out[3] == 0) and torch.all(out[5] == 0)
    good = [t for t in range(T) if t not in (3, 5)]
    ref = _oracle_tokens(precision, x[good], ids[good], probs[good], weights)
    assert_close(out.numpy()[good], ref, precision, "good tokens next to bad ones")


@pytest.mark.parametrize("precision", PRECISIONS)
def test_live_count_out_of_range_is_clamped_and_flagged(precision):
    H, F, E, k, cap = 128, 128, 8, 2, 40
    x, logits, weights = workloads.small_case(H, F, E, k, 32, seed=8, capacity=cap)
    x[32:] = 0.5  # finite rows past 32 so that a clamp to 40 stays checkable
    logits[32:] = torch.randn((cap - 32, E), generator=torch.Generator().manual_seed(9))
    m = GpuMoe(H, F, E, k, cap, weights, precision=precision, max_live=36)
    m.clear_status()
    out = m.forward(x.cuda(), -5, logits=logits.cuda())
    torch.cuda.synchronize()
    assert m.status() & rm.MOE_DEV_LIVE_CLAMPED
    assert torch.all(torch.isnan(out))  # clamped to zero rows: nothing written
    m.clear_status()
    assert m.status() == 0
    out = m.forward(x.cuda(), 1000, logits=logits.cuda()).cpu()
    assert m.status() & rm.MOE_DEV_LIVE_CLAMPED
    assert not torch.isnan(out[:36]).any() and torch.isnan(out[36:]).all()
    _, _, ref = oracle_forward(x, logits, weights, k, 36, precision=precision)
    assert_close(out.numpy()[:36], ref, precision, "clamped")


@pytest.mark.parametrize("precision", PRECISIONS)
def test_zero_live_rows_writes_nothing(precision):
    H, F, E, k, cap = 128, 128, 8, 2, 64
    x, logits, weights = workloads.small_case(H, F, E, k, 0, seed=10, capacity=cap)
    m = GpuMoe(H, F, E, k, cap, weights, precision=precision)
    out = m.forward(x.cuda(), 0, logits=logits.cuda(), sentinel=3.0)
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)
    assert m.status() == 0


def test_refit_negative_control():
    """A refit without moe_prepare_weights keeps serving the old weights; with
    it, the result equals a freshly built plan on the new weights."""
    H, F, E, k, T = 256, 256, 8, 2, 64
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=11)
    _, _, weights_b = workloads.small_case(H, F, E, k, T, seed=12)
    m = GpuMoe(H, F, E, k, T, weights)
    wg, wu, wd = (w.cuda() for w in weights)
    rm.moe_prepare_weights(m.plan, wg, wu, wd, m.wbuf)
    a = m.forward(x.cuda(), T, logits=logits.cuda()).cpu()
    for dst, src in zip((wg, wu, wd), weights_b):  # in-place update of the sources only
        dst.copy_(src.cuda())
    stale = m.forward(x.cuda(), T, logits=logits.cuda()).cpu()
    assert torch.equal(stale, a)
    rm.moe_prepare_weights(m.plan, wg, wu, wd, m.wbuf)
    refit = m.forward(x.cuda(), T, logits=logits.cuda()).cpu()
    fresh = GpuMoe(H, F, E, k, T, weights_b).forward(x.cuda(), T, logits=logits.cuda()).cpu()
    assert torch.equal(refit, fresh) and not torch.equal(refit, a)


@pytest.mark.parametrize("precision", PRECISIONS)
def test_graph_capture_replay_with_device_live_counts(precision):
    """One capture serves every live count: the sweep workload's shapes at a
    reduced buffer, replayed with live counts written between replays."""
    w = workloads.WORKLOADS["sweep"]
    H, F, E, k = w.hidden, w.ffn, w.num_experts, w.top_k
    if precision != "bf16":  # smaller shapes: the block-scaled oracles decode every weight element per route
        H, F, E, k = 512, 512, 32, 4
    cap = 8192
    x, logits, weights = workloads.small_case(H, F, E, k, 1024, seed=4, capacity=cap)
    m = GpuMoe(H, F, E, k, cap, weights, precision=precision, max_live=1024)
    xd, ld = x.cuda(), logits.cuda()
    out = torch.full((cap, H), float("nan"), device="cuda")
    live = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        live.fill_(16)
        rm.moe_forward(m.plan, xd, m.wbuf, live, out, m.ws, logits=ld)  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        rm.moe_forward(m.plan, xd, m.wbuf, live, out, m.ws, logits=ld)
    res = {}
    for n in (1, 64, 1024, 64):
        out.fill_(float("nan"))
        live.fill_(n)
        g.replay()
        torch.cuda.synchronize()
        o = out.cpu()
        assert not torch.isnan(o[:n]).any() and torch.isnan(o[n:]).all()
        if n in res:
            assert torch.equal(o[:n], res[n])
        res[n] = o[:n].clone()
    assert torch.equal(res[64][:1], res[1]) and torch.equal(res[1024][:64], res[64])
    toks = workloads.sample_tokens(1024, 48, 4).numpy()
    _, _, ref = oracle_forward(x, logits, weights, k, 1024, tokens=toks, precision=precision)
    assert_close(res[1024].numpy()[toks], ref, precision, "graph replay")
    del g


def test_stage_events_eager_and_same_result():
    """moe_forward_with_events works outside graph capture, records ordered
    events and gives the same bits as moe_forward."""
    H, F, E, k, T = 256, 256, 8, 2, 50
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=21)
    m = GpuMoe(H, F, E, k, T, weights)
    a = m.forward(x.cuda(), T, logits=logits.cuda()).cpu()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(rm.MOE_NUM_STAGES + 1)]
    for e in evs:
        e.record()
    out = torch.full((T, H), float("nan"), device="cuda")
    m.live.fill_(T)
    rm.moe_forward_with_events(m.plan, x.cuda(), m.wbuf, m.live, out, m.ws, evs, logits=logits.cuda())
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), a)
    times = [evs[i].elapsed_time(evs[i + 1]) for i in range(rm.MOE_NUM_STAGES)]
    assert all(t >= 0.0 for t in times)
