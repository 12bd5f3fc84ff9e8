"""MXFP8 path vs the oracle: weight and activation quantisation inside
prepare/forward bit-exact; the SwiGLU intermediate's codes and scales equal,
bit for bit, the oracle quantiser applied to the GPU's own fp32 h (kept by
MOE_FLAG_KEEP_H_FP32), and equal the oracle's own codes up to last-bit
accumulation-order effects; outputs within the MXFP8 tolerance
(max |d| <= 5e-2 * RMS).

The fused FC1-epilogue quantisation is Megatron-LM PR #7798, "Background";
the 32-element block rule is Megatron-LM PR #7830, "1. Mega backend for
generation" (mxfp8_quantize_per_block_32) and cudnn-frontend PR #448."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import routed_moe_swiglu_b200 as rm
import workloads
from moe_testlib import GpuMoe, assert_close, oracle_forward, workload_problem

pytestmark = pytest.mark.gpu

SF_BLOCK = 512


def sf_offset(row, g):
    row = np.asarray(row)
    return (row % 32) * 16 + ((row // 32) % 4) * 4 + g


def decode_scales(blob: np.ndarray, rows: np.ndarray, K: int) -> np.ndarray:
    """Scale bytes [len(rows), K/32] of padded rows from the [tile][stage][512] layout."""
    ks = (K + 127) // 128
    out = np.empty((rows.size, K // 32), np.uint8)
    for g in range(K // 32):
        idx = ((rows // 128) * ks + g // 4) * SF_BLOCK + sf_offset(rows % 128, g % 4)
        out[:, g] = blob[idx]
    return out


def _ws_bytes(m: GpuMoe, ptr, nbytes):
    off = ptr - m.ws.data_ptr()
    return m.ws[off:off + nbytes].cpu().numpy()


@pytest.mark.parametrize("F", [192, 160])  # 160: a partial 64-f weight tile (zero rows) and K stage
def test_prepare_weights_bit_exact(F):
    H, E = 256, 3
    gen = torch.Generator().manual_seed(31)
    wg = (torch.randn((E, F, H), generator=gen) * torch.exp(torch.randn((E, F, 1), generator=gen))).bfloat16()
    wu = (torch.randn((E, F, H), generator=gen) * 0.1).bfloat16()
    wd = (torch.randn((E, H, F), generator=gen) * torch.exp(torch.randn((E, H, 1), generator=gen) * 3)).bfloat16()
    plan = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=2, capacity=16, precision="mxfp8")
    buf = rm.alloc_weight_buffer(plan)
    buf.fill_(0x5A)  # stale contents: padding rows and scale slots must be rewritten
    rm.moe_prepare_weights(plan, wg.cuda(), wu.cuda(), wd.cuda(), buf)
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    gq, gs, uq, us, dq, ds = oracle.quantize_weights_mxfp8(wg, wu, wd)
    # W1 codes: per 64-f tile, per 16 f, the 16 gate rows then the 16 up rows; K pitches
    # padded to 128 with zeros, rows of f >= F zero
    hp, fp = (H + 127) // 128 * 128, (F + 127) // 128 * 128
    n1 = E * 2 * fp * hp
    w1 = b[:n1].reshape(E, fp // 64, 4, 2, 16, hp)
    f = np.arange(F)
    assert np.array_equal(w1[:, f // 64, (f % 64) // 16, 0, f % 16, :H], gq)
    assert np.array_equal(w1[:, f // 64, (f % 64) // 16, 1, f % 16, :H], uq)
    assert np.all(w1[..., H:] == 0)
    fpad = np.arange(F, fp)
    assert np.all(w1[:, fpad // 64, (fpad % 64) // 16, :, fpad % 16] == 0)
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    nt1, ks1 = fp // 64, (H + 127) // 128
    off_w1s = al(n1)
    w1s = b[off_w1s:off_w1s + E * nt1 * ks1 * SF_BLOCK]
    for e in range(E):
        for gu, ref in ((0, gs), (1, us)):
            trow = ((f % 64) // 16) * 32 + gu * 16 + f % 16
            for g in range(H // 32):
                idx = ((e * nt1 + f // 64) * ks1 + g // 4) * SF_BLOCK + sf_offset(trow, g % 4)
                assert np.array_equal(w1s[idx], ref[e, :, g]), (e, gu, g)
    off_w2 = off_w1s + al(E * nt1 * ks1 * SF_BLOCK)
    w2 = b[off_w2:off_w2 + E * H * fp].reshape(E, H, fp)
    assert np.array_equal(w2[..., :F], dq)
    assert np.all(w2[..., F:] == 0)
    nt2, ks2 = (H + 127) // 128, (F + 127) // 128
    off_w2s = off_w2 + al(E * H * fp)
    w2s = b[off_w2s:off_w2s + E * nt2 * ks2 * SF_BLOCK]
    c = np.arange(H)
    for e in range(E):
        for g in range(F // 32):
            idx = ((e * nt2 + c // 128) * ks2 + g // 4) * SF_BLOCK + sf_offset(c % 128, g % 4)
            assert np.array_equal(w2s[idx], ds[e, :, g]), (e, g)
        # k-group slots past F/32 in the last stage are scale byte 0
        for g in range(F // 32, 4 * ks2):
            idx = ((e * nt2 + c // 128) * ks2 + g // 4) * SF_BLOCK + sf_offset(c % 128, g % 4)
            assert np.all(w2s[idx] == 0)


def _read_rows_f32(m: GpuMoe, ptr, rows_total, pitch, rows):
    """fp32 rows `rows` of a [rows_total, pitch] workspace buffer (read on the device)."""
    off = ptr - m.ws.data_ptr()
    t = m.ws[off:off + rows_total * pitch * 4].view(torch.float32).view(rows_total, pitch)
    return t[torch.from_numpy(np.asarray(rows, np.int64)).cuda()].cpu().numpy()


def _check_h_own_quantisation(m: GpuMoe, F, rows, hf_ref=None):
    """The fused epilogue's E4M3 codes and E8M0 scales of h are exactly the
    oracle quantiser applied to the epilogue's own fp32 h (rows: padded route rows)."""
    v = m.views()
    assert v["h_fp32"], "the plan keeps no fp32 h (MOE_FLAG_KEEP_H_FP32)"
    R = v["rows_padded"]
    fp = (F + 127) // 128 * 128
    hf = _read_rows_f32(m, v["h_fp32"], R, fp, rows)
    assert np.all(hf[:, F:] == 0), "padding columns of h must be exact zeros"
    own_q, own_s = oracle.mxfp8_quantize(np.ascontiguousarray(hf[:, :F]))
    hq = _ws_bytes(m, v["h"], R * fp).reshape(R, fp)[rows][:, :F]
    hs = decode_scales(_ws_bytes(m, v["h_scales"], (R // 128) * (fp // 128) * SF_BLOCK), rows, F)
    bad_q = np.argwhere(hq != own_q)
    assert bad_q.size == 0, f"{len(bad_q)} h codes differ from the oracle quantiser, first {bad_q[:4]}"
    assert np.array_equal(hs, own_s), np.argwhere(hs != own_s)[:4]
    if hf_ref is not None:
        # and the fp32 values are the oracle's up to accumulation order
        got = hf[:, :F].reshape(hf_ref.shape)
        scale = np.abs(hf_ref).max(axis=-1, keepdims=True) + 1e-30
        assert np.max(np.abs(got - hf_ref) / scale) < 1e-4
    return hq.size


def _check_intermediates(m: GpuMoe, x, ids, H, F, toks, h_ref):
    v = m.views()
    live, k = ids.shape
    inv = m.read_i32(v["inv"], live * k).reshape(live, k)
    rows = inv[toks].reshape(-1).astype(np.int64)
    R = v["rows_padded"]
    hp, fp = (H + 127) // 128 * 128, (F + 127) // 128 * 128  # row pitches (zero padding)
    # x codes and scales of every sampled route row equal the oracle's quantisation of x[t]
    xq_all = _ws_bytes(m, v["xq"], R * hp).reshape(R, hp)
    assert np.all(xq_all[rows][:, H:] == 0)
    xq_all = xq_all[:, :H]
    xs_blob = _ws_bytes(m, v["xq_scales"], (R // 128) * ((H + 127) // 128) * SF_BLOCK)
    ref_q, ref_s = oracle.mxfp8_quantize_bf16(x[torch.from_numpy(np.repeat(toks, k))].contiguous())
    assert np.array_equal(xq_all[rows], ref_q)
    assert np.array_equal(decode_scales(xs_blob, rows, H), ref_s)
    # h: codes/scales equal the oracle's wherever the fp32 pre-quantisation value agrees
    hq_all = _ws_bytes(m, v["h"], R * fp).reshape(R, fp)
    assert np.all(hq_all[rows][:, F:] == 0)
    hq_all = hq_all[:, :F]
    hs_blob = _ws_bytes(m, v["h_scales"], (R // 128) * ((F + 127) // 128) * SF_BLOCK)
    hq_ref, hs_ref, _ = h_ref
    got_q = hq_all[rows].reshape(len(toks), k, F)
    got_s = decode_scales(hs_blob, rows, F).reshape(len(toks), k, F // 32)
    frac_s = np.mean(got_s == hs_ref)
    frac_q = np.mean(got_q == hq_ref)
    assert frac_s > 0.995 and frac_q > 0.995, (frac_s, frac_q)
    # where a code differs with the same scale it is a neighbouring grid point
    same_s = np.repeat(got_s == hs_ref, 32, axis=2)
    diff = (got_q != hq_ref) & same_s
    a = got_q[diff].astype(np.int32)
    b = hq_ref[diff].astype(np.int32)
    mag = lambda c: np.where(c & 0x80, -(c & 0x7F), c & 0x7F)  # noqa: E731
    assert np.all(np.abs(mag(a) - mag(b)) <= 1), np.stack([a, b])[:, :10]
    if m.plan.keep_h_fp32:
        _check_h_own_quantisation(m, F, rows, h_ref[2])


@pytest.mark.parametrize("H,F,E,k,T", [(256, 256, 8, 2, 64), (320, 224, 6, 3, 200), (512, 1024, 16, 4, 300)])
def test_forward_mxfp8_small(H, F, E, k, T):
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=H + F, capacity=T + 16)
    m = GpuMoe(H, F, E, k, T + 16, weights, precision="mxfp8", keep_h_fp32=True)
    out = m.forward(x.cuda(), T, logits=logits.cuda())
    torch.cuda.synchronize()
    ids, probs = oracle.route(logits[:T].numpy(), k)
    wq = oracle.quantize_weights_mxfp8(*weights)
    ref, h_ref = oracle.forward_mxfp8(x[:T], ids, probs, wq, want_h=True)
    o = out.cpu().numpy()
    assert_close(o[:T], ref, "mxfp8", f"mxfp8 {H},{F},{E},{k},{T}")
    assert np.all(np.isnan(o[T:]))
    _check_intermediates(m, x, ids, H, F, np.arange(T), h_ref)
    assert m.status() == 0


def test_mxfp8_every_tile_width():
    """Caller routes that give experts 1..257 routes: every route-tile width
    (N = 32..128 in steps of 32), full tiles followed by tails of 1, 31, 32 or
    33 rows, a K tail (H = 320) and a partial 64-f weight tile (F = 224)."""
    H, F, E, k = 320, 224, 17, 2
    counts = np.array([1, 31, 32, 33, 63, 64, 65, 95, 96, 97, 127, 128, 129, 201, 255, 256, 257])
    T = int(counts.sum()) // k
    x, _, weights = workloads.small_case(H, F, E, k, T, seed=78)
    gen = np.random.default_rng(78)
    experts = np.repeat(np.arange(E), counts)
    ids = np.stack([experts[:T], experts[T:]], axis=1)
    ids = ids[gen.permutation(T)].astype(np.int32)
    assert np.all(ids[:, 0] != ids[:, 1])
    p = gen.uniform(0.1, 1.0, size=(T, k))
    probs = (p / p.sum(axis=1, keepdims=True)).astype(np.float32)
    m = GpuMoe(H, F, E, k, T, weights, precision="mxfp8", keep_h_fp32=True)
    out = m.forward(x.cuda(), T, ids=torch.from_numpy(ids).cuda(), probs=torch.from_numpy(probs).cuda())
    torch.cuda.synchronize()
    ids_c = np.sort(ids, axis=1)
    order = np.argsort(ids, axis=1)
    probs_c = np.take_along_axis(probs, order, axis=1)
    wq = oracle.quantize_weights_mxfp8(*weights)
    ref, h_ref = oracle.forward_mxfp8(x, ids_c, probs_c, wq, want_h=True)
    assert_close(out.cpu().numpy(), ref, "mxfp8", "mxfp8 every tile width")
    _check_intermediates(m, x, ids_c, H, F, np.arange(T), h_ref)
    assert m.status() == 0


def test_forward_mxfp8_workload_subset():
    w, x, logits, weights = workload_problem("mxfp8")
    m = GpuMoe(w.hidden, w.ffn, w.num_experts, w.top_k, w.capacity, weights, precision="mxfp8", keep_h_fp32=True)
    live = w.max_live
    out = m.forward(x.cuda(), live, logits=logits.cuda())
    torch.cuda.synchronize()
    toks = workloads.sample_tokens(live, 256, w.seed).numpy()
    ids, probs = oracle.route(logits[:live].numpy(), w.top_k)
    wq = oracle.quantize_weights_mxfp8(*weights)
    ref, h_ref = oracle.forward_mxfp8(x[:live], ids, probs, wq, tokens=toks, want_h=True)
    assert_close(out.cpu().numpy()[toks], ref, "mxfp8", "mxfp8 workload subset")
    _check_intermediates(m, x, ids, w.hidden, w.ffn, toks, h_ref)
    # the MXFP8 result stays a few percent from the bf16 oracle (the pages report ~4%)
    ref_bf16 = oracle.forward_bf16(x[:live], ids, probs, *weights, tokens=toks)
    d = np.linalg.norm(out.cpu().numpy()[toks] - ref_bf16) / np.linalg.norm(ref_bf16)
    assert 0.01 < d < 0.08, d


def test_mxfp8_batch_invariance():
    H, F, E, k = 512, 512, 16, 4
    x, logits, weights = workloads.small_case(H, F, E, k, 600, seed=41)
    m = GpuMoe(H, F, E, k, 600, weights, precision="mxfp8")
    xd, ld = x.cuda(), logits.cuda()
    a = m.forward(xd, 600, logits=ld).cpu()
    for n in (1, 33, 300):
        b = m.forward(xd, n, logits=ld).cpu()
        assert torch.equal(b[:n], a[:n])
    assert torch.equal(m.forward(xd, 600, logits=ld).cpu(), a)


@pytest.mark.parametrize("variant", [dict(), dict(squared_relu=True), dict(probs_in_fc1=True),
                                     dict(gate_up_clamp=1.0), dict(squared_relu=True, probs_in_fc1=True,
                                                                   gate_up_clamp=0.75)])
def test_fused_h_quantiser_bit_exact_every_epilogue(variant):
    """Every MXFP8 gate/up epilogue (SwiGLU, squared ReLU, probability in FC1,
    clamp) quantises h exactly as the oracle quantiser does on the same fp32
    values: every live route row, every block, bit for bit.  H, F not
    multiples of 128 and enough tokens for every route-tile width."""
    H, F, E, k, T = 320, 224, 12, 3, 700
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=91, zipf=True)
    wg, wu, wd = weights
    relu2 = variant.get("squared_relu", False)
    m = GpuMoe(H, F, E, k, T, (wg, wg if relu2 else wu, wd), precision="mxfp8", keep_h_fp32=True, **variant)
    out = m.forward(x.cuda(), T, logits=logits.cuda())
    torch.cuda.synchronize()
    assert m.status() == 0
    ids, probs = oracle.route(logits.numpy(), k)
    wq = oracle.quantize_weights_mxfp8(wg, wg if relu2 else wu, wd)
    ref, h_ref = oracle.forward_mxfp8(x, ids, probs, wq, want_h=True, **variant)
    assert_close(out.cpu().numpy(), ref, "mxfp8", f"mxfp8 {variant}")
    inv = m.read_i32(m.views()["inv"], T * k).reshape(T, k)
    n = _check_h_own_quantisation(m, F, inv.reshape(-1).astype(np.int64), h_ref[2])
    assert n == T * k * F


def test_keep_h_fp32_changes_no_result():
    """The debug flag adds stores only: outputs and h bytes are bitwise those of a plain plan."""
    H, F, E, k, T = 512, 256, 16, 4, 300
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=92)
    a = GpuMoe(H, F, E, k, T, weights, precision="mxfp8")
    b = GpuMoe(H, F, E, k, T, weights, precision="mxfp8", keep_h_fp32=True)
    assert a.views()["h_fp32"] is None and b.views()["h_fp32"]
    oa = a.forward(x.cuda(), T, logits=logits.cuda())
    ob = b.forward(x.cuda(), T, logits=logits.cuda())
    torch.cuda.synchronize()
    assert torch.equal(oa.view(torch.int32), ob.view(torch.int32))
    va, vb = a.views(), b.views()
    R = va["rows_padded"]
    # the route rows (padding rows between experts are never written)
    rows = a.read_i32(va["inv"], T * k).astype(np.int64)
    assert np.array_equal(rows, b.read_i32(vb["inv"], T * k))
    ha = _ws_bytes(a, va["h"], R * 256).reshape(R, 256)[rows]
    hb = _ws_bytes(b, vb["h"], R * 256).reshape(R, 256)[rows]
    assert np.array_equal(ha, hb)
