"""NVFP4 path (the per-token recipe) vs the oracle: the public quantiser, the
weights' and x rows' codes, block scales and second-level scales bit-exact;
the gate/up GEMM's fp32 h close to the oracle's and its h codes exactly the
oracle's quantisation of that fp32 h; outputs within the block-scaled
tolerance (max |d| <= 5e-2 * RMS)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import routed_moe_swiglu_b200 as rm
import workloads
from moe_testlib import GpuMoe, assert_close, workload_problem

pytestmark = pytest.mark.gpu

SF_BLOCK = 512


def sf_offset(row, b):
    row = np.asarray(row)
    return (row % 32) * 16 + ((row // 32) % 4) * 4 + b


def sf_index(rows, blk, K):
    """Byte index of the block scale of (padded row, 16-element block) in the
    [tile][K block of 256][4 MMA steps][512] layout."""
    ks = (K + 255) // 256
    return ((((rows // 128) * ks + blk // 16) * 4 + (blk % 16) // 4) * SF_BLOCK + sf_offset(rows % 128, blk % 4))


def decode_scales(blob: np.ndarray, rows: np.ndarray, K: int) -> np.ndarray:
    out = np.empty((rows.size, K // 16), np.uint8)
    for b in range(K // 16):
        out[:, b] = blob[sf_index(rows, b, K)]
    return out


def _ws(m: GpuMoe, ptr, nbytes):
    off = ptr - m.ws.data_ptr()
    return m.ws[off:off + nbytes].cpu().numpy()


def _pad256(n):
    return (n + 255) // 256 * 256


def test_nvfp4_quantize_block16_bit_exact():
    gen = torch.Generator().manual_seed(50)
    rows, cols = 96, 384
    x = torch.randn((rows, cols), generator=gen) * torch.exp(torch.randn((rows, 1), generator=gen) * 4)
    x[5] = 0.0
    x[7, 3:40] = 0.0
    x[9, ::11] *= 500.0
    x = x.bfloat16()
    q = torch.full((rows, cols // 2), 0xAB, dtype=torch.uint8, device="cuda")
    s = torch.full((rows, cols // 16), 0xAB, dtype=torch.uint8, device="cuda")
    g = torch.full((rows,), -1.0, dtype=torch.float32, device="cuda")
    live = torch.tensor([rows - 10], dtype=torch.int32, device="cuda")
    rm.nvfp4_quantize_block16(x.cuda(), q, s, g, live_rows=live)
    torch.cuda.synchronize()
    rq, rs, rg = oracle.nvfp4_quantize(x)
    n = rows - 10
    assert np.array_equal(q.cpu().numpy()[:n], rq[:n])
    assert np.array_equal(s.cpu().numpy()[:n], rs[:n])
    assert np.array_equal(g.cpu().numpy()[:n], rg[:n])
    assert np.all(q.cpu().numpy()[n:] == 0xAB) and np.all(g.cpu().numpy()[n:] == -1.0)  # rows past the live count


@pytest.mark.parametrize("F,relu2", [(192, False), (160, False), (160, True)])
def test_prepare_weights_nvfp4_bit_exact(F, relu2):
    H, E = 288, 3
    gen = torch.Generator().manual_seed(51)
    wg = (torch.randn((E, F, H), generator=gen) * torch.exp(torch.randn((E, F, 1), generator=gen))).bfloat16()
    wu = (torch.randn((E, F, H), generator=gen) * 0.1).bfloat16()
    wd = (torch.randn((E, H, F), generator=gen) * torch.exp(torch.randn((E, H, 1), generator=gen) * 3)).bfloat16()
    plan = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=2, capacity=16, precision="nvfp4",
                              squared_relu=relu2)
    buf = rm.alloc_weight_buffer(plan)
    buf.fill_(0x5A)  # stale contents: padding must be rewritten
    rm.moe_prepare_weights(plan, wg.cuda(), None if relu2 else wu.cuda(), wd.cuda(), buf)
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    w1_q, w1_s, g1, wd_q, wd_s, g2 = oracle.quantize_weights_nvfp4(wg, None if relu2 else wu, wd)
    hp, fp = _pad256(H), _pad256(F)
    w1r = fp if relu2 else 2 * fp
    nt1, ks1, nt2, ks2 = w1r // 128, hp // 256, (H + 127) // 128, fp // 256
    al = lambda n: (n + 255) // 256 * 256  # noqa: E731
    n1 = E * w1r * hp // 2
    w1 = b[:n1].reshape(E, w1r, hp // 2)
    f = np.arange(F)
    for gu in ((0,) if relu2 else (0, 1)):
        trow = f if relu2 else (f // 64) * 128 + ((f % 64) // 16) * 32 + gu * 16 + f % 16
        assert np.array_equal(w1[:, trow, :H // 2], w1_q[:, gu * F + f]), gu
        assert np.all(w1[:, trow, H // 2:] == 0)
    off_w1s = al(n1)
    w1s = b[off_w1s:off_w1s + E * nt1 * ks1 * 4 * SF_BLOCK]
    for e in range(E):
        for gu in ((0,) if relu2 else (0, 1)):
            trow = f if relu2 else (f // 64) * 128 + ((f % 64) // 16) * 32 + gu * 16 + f % 16
            srow = e * nt1 * 128 + trow
            for blk in range(H // 16):
                assert np.array_equal(w1s[sf_index(srow, blk, hp)], w1_s[e, gu * F + f, blk]), (e, gu, blk)
    off_w2 = off_w1s + al(E * nt1 * ks1 * 4 * SF_BLOCK)
    w2 = b[off_w2:off_w2 + E * H * fp // 2].reshape(E, H, fp // 2)
    assert np.array_equal(w2[..., :F // 2], wd_q)
    assert np.all(w2[..., F // 2:] == 0)
    off_w2s = off_w2 + al(E * H * fp // 2)
    w2s = b[off_w2s:off_w2s + E * nt2 * ks2 * 4 * SF_BLOCK]
    c = np.arange(H)
    for e in range(E):
        srow = (e * nt2 + c // 128) * 128 + c % 128
        for blk in range(F // 16):
            assert np.array_equal(w2s[sf_index(srow, blk, fp)], wd_s[e, :, blk]), (e, blk)
        for blk in range(F // 16, fp // 16):  # K padding: scale byte 0
            assert np.all(w2s[sf_index(srow, blk, fp)] == 0)
    off_wg = off_w2s + al(E * nt2 * ks2 * 4 * SF_BLOCK)
    gg = b[off_wg:off_wg + E * 8].view(np.float32).reshape(E, 2)
    assert np.array_equal(gg[:, 0], g1) and np.array_equal(gg[:, 1], g2)


def _check_intermediates(m: GpuMoe, x, ids, H, F, toks, h_ref):
    v = m.views()
    live, k = ids.shape
    inv = m.read_i32(v["inv"], live * k).reshape(live, k)
    rows = inv[toks].reshape(-1).astype(np.int64)
    R = v["rows_padded"]
    hp, fp = _pad256(H), _pad256(F)
    # x: codes, block scales and row scales of every sampled route row equal the oracle's
    # quantisation of x[t] with the token's own scale
    xq_all = _ws(m, v["xq"], R * hp // 2).reshape(R, hp // 2)
    assert np.all(xq_all[rows][:, H // 2:] == 0)
    xs_blob = _ws(m, v["xq_scales"], (R // 128) * (hp // 256) * 4 * SF_BLOCK)
    xg = m.read_f32(v["xq_row_scales"], R)
    ref_q, ref_s, ref_g = oracle.nvfp4_quantize(x[torch.from_numpy(np.repeat(toks, k))].contiguous())
    assert np.array_equal(xq_all[rows][:, :H // 2], ref_q)
    assert np.array_equal(decode_scales(xs_blob, rows, H), ref_s)
    assert np.array_equal(xg[rows], ref_g)
    # h: the GEMM's fp32 rows agree with the oracle's to accumulation order, and the
    # quantisation pass turns them into exactly the oracle quantiser's codes
    hq_ref, hs_ref, hg_ref, hf_ref = h_ref
    hf = m.read_f32(v["h_fp32"], R * fp).reshape(R, fp)
    got_f = hf[rows][:, :F].reshape(len(toks), k, F)
    assert np.all(hf[rows][:, F:] == 0)
    scale = np.abs(hf_ref).max(axis=2, keepdims=True) + 1e-30
    assert np.max(np.abs(got_f - hf_ref) / scale) < 1e-4
    hq_all = _ws(m, v["h"], R * fp // 2).reshape(R, fp // 2)
    hs_blob = _ws(m, v["h_scales"], (R // 128) * (fp // 256) * 4 * SF_BLOCK)
    hg = m.read_f32(v["h_row_scales"], R)
    own_q, own_s, own_g = oracle.nvfp4_quantize(np.ascontiguousarray(hf[rows][:, :F]))
    assert np.array_equal(hq_all[rows][:, :F // 2], own_q)
    assert np.array_equal(decode_scales(hs_blob, rows, F), own_s)
    assert np.array_equal(hg[rows], own_g)
    # and those codes are the oracle's own almost everywhere
    assert np.mean(own_q.reshape(len(toks), k, F // 2) == hq_ref) > 0.99


def _forward_case(H, F, E, k, T, seed, **variant):
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=seed, capacity=T + 16)
    relu2 = variant.get("squared_relu", False)
    # squared-ReLU experts have one FC1 projection: the library ignores w_up, the oracle gets None
    oracle_weights = (weights[0], None, weights[2]) if relu2 else weights
    m = GpuMoe(H, F, E, k, T + 16, weights, precision="nvfp4", **variant)
    out = m.forward(x.cuda(), T, logits=logits.cuda())
    torch.cuda.synchronize()
    ids, probs = oracle.route(logits[:T].numpy(), k)
    wq = oracle.quantize_weights_nvfp4(*oracle_weights)
    ref, h_ref = oracle.forward_nvfp4(x[:T], ids, probs, wq, want_h=True, **variant)
    o = out.cpu().numpy()
    assert_close(o[:T], ref, "nvfp4", f"nvfp4 {H},{F},{E},{k},{T} {variant}")
    assert np.all(np.isnan(o[T:]))
    _check_intermediates(m, x, ids, H, F, np.arange(T), h_ref)
    assert m.status() == 0


@pytest.mark.parametrize("H,F,E,k,T", [(256, 256, 8, 2, 64), (320, 224, 6, 3, 200), (512, 1024, 16, 4, 300)])
def test_forward_nvfp4_small(H, F, E, k, T):
    _forward_case(H, F, E, k, T, seed=H + F + 1)


@pytest.mark.parametrize("variant", [dict(squared_relu=True), dict(probs_in_fc1=True, gate_up_clamp=3.0)])
def test_forward_nvfp4_variants(variant):
    _forward_case(320, 224, 6, 3, 150, seed=77, **variant)


def test_nvfp4_every_tile_width():
    """Caller routes that give experts 1..257 routes: every route-tile width
    (N = 32..128), tails of 1, 31, 32 or 33 rows, a K tail (H = 320: 64
    padding elements of the last 256-element block) and a partial weight tile."""
    H, F, E, k = 320, 224, 17, 2
    counts = np.array([1, 31, 32, 33, 63, 64, 65, 95, 96, 97, 127, 128, 129, 201, 255, 256, 257])
    T = int(counts.sum()) // k
    x, _, weights = workloads.small_case(H, F, E, k, T, seed=79)
    gen = np.random.default_rng(79)
    experts = np.repeat(np.arange(E), counts)
    ids = np.stack([experts[:T], experts[T:]], axis=1)
    ids = ids[gen.permutation(T)].astype(np.int32)
    assert np.all(ids[:, 0] != ids[:, 1])
    p = gen.uniform(0.1, 1.0, size=(T, k))
    probs = (p / p.sum(axis=1, keepdims=True)).astype(np.float32)
    m = GpuMoe(H, F, E, k, T, weights, precision="nvfp4")
    out = m.forward(x.cuda(), T, ids=torch.from_numpy(ids).cuda(), probs=torch.from_numpy(probs).cuda())
    torch.cuda.synchronize()
    order = np.argsort(ids, axis=1)
    ids_c = np.take_along_axis(ids, order, axis=1)
    probs_c = np.take_along_axis(probs, order, axis=1)
    wq = oracle.quantize_weights_nvfp4(*weights)
    ref, h_ref = oracle.forward_nvfp4(x, ids_c, probs_c, wq, want_h=True)
    assert_close(out.cpu().numpy(), ref, "nvfp4", "nvfp4 every tile width")
    _check_intermediates(m, x, ids_c, H, F, np.arange(T), h_ref)
    assert m.status() == 0


def test_forward_nvfp4_workload_subset():
    w, x, logits, weights = workload_problem("nvfp4")
    m = GpuMoe(w.hidden, w.ffn, w.num_experts, w.top_k, w.capacity, weights, precision="nvfp4")
    live = w.max_live
    out = m.forward(x.cuda(), live, logits=logits.cuda())
    torch.cuda.synchronize()
    toks = workloads.sample_tokens(live, 128, w.seed).numpy()
    ids, probs = oracle.route(logits[:live].numpy(), w.top_k)
    wq = oracle.quantize_weights_nvfp4(*weights)
    ref, h_ref = oracle.forward_nvfp4(x[:live], ids, probs, wq, tokens=toks, want_h=True)
    assert_close(out.cpu().numpy()[toks], ref, "nvfp4", "nvfp4 workload subset")
    _check_intermediates(m, x, ids, w.hidden, w.ffn, toks, h_ref)
    # NVFP4 stays some percent from the bf16 oracle, further than MXFP8
    ref_bf16 = oracle.forward_bf16(x[:live], ids, probs, *weights, tokens=toks)
    d = np.linalg.norm(out.cpu().numpy()[toks] - ref_bf16) / np.linalg.norm(ref_bf16)
    assert 0.03 < d < 0.3, d


def test_forward_nvfp4_decode_workload():
    w, x, logits, weights = workload_problem("decode_nvfp4")
    m = GpuMoe(w.hidden, w.ffn, w.num_experts, w.top_k, w.capacity, weights, precision="nvfp4")
    live = w.max_live
    out = m.forward(x.cuda(), live, logits=logits.cuda(), sentinel=-7.0)
    torch.cuda.synchronize()
    ids, probs = oracle.route(logits[:live].numpy(), w.top_k)
    ref = oracle.forward_nvfp4(x[:live], ids, probs, oracle.quantize_weights_nvfp4(*weights))
    o = out.cpu().numpy()
    assert_close(o[:live], ref, "nvfp4", "nvfp4 decode")
    assert np.all(o[live:] == -7.0)
    assert m.status() == 0


def test_nvfp4_batch_invariance():
    H, F, E, k = 512, 512, 16, 4
    x, logits, weights = workloads.small_case(H, F, E, k, 600, seed=42)
    m = GpuMoe(H, F, E, k, 600, weights, precision="nvfp4")
    xd, ld = x.cuda(), logits.cuda()
    a = m.forward(xd, 600, logits=ld).cpu()
    for n in (1, 33, 300):
        b = m.forward(xd, n, logits=ld).cpu()
        assert torch.equal(b[:n], a[:n])
    assert torch.equal(m.forward(xd, 600, logits=ld).cpu(), a)
