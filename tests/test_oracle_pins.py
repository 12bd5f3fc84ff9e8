"""Pins of the CPU oracle to things other than itself (no GPU needed).

Which plausible mistake each pin catches:
  route      brute-force ranking (wrong comparison, wrong tie rule, wrong
             output order); k=1 gives p=1 exactly; k=E equals the library
             softmax (dropped exp, wrong max shift); k=2 equals the logistic
             closed form (wrong sign in the exponent).
  permute    a stable library argsort of (expert, token) (wrong rank, not
             stable, off-by-one offsets); bijection invariants.
  mxfp8      the E4M3 code table equals torch's float8_e4m3fn decode; every
             finite bf16 value in blocks of four different amax binades
             equals an independent quantiser (numpy log2 scale + torch's RNE
             cast with a clamp to +-448); closed forms: scale rule, grid
             round-trips, ties to even, saturation, sign of zero.
  forward    E=1, k=1, p=1 equals a dense SwiGLU MLP from torch float64
             matmuls (transposed operand, swapped gate/up, wrong silu);
             zero gate or zero up weights give exact zeros; doubling p
             doubles the output exactly; the combine is the fp32 FMA chain
             in ascending expert id (checked against exact rational
             arithmetic); token order and duplication invariance;
             MXFP8 E=1 dense check with the independent quantiser.
  nvfp4      a worked row fixes the E2M1 grid, every tie, saturation and the
             sign of zero; random rows over many binades (fp32 and bf16,
             scale per row and per matrix) equal an independent quantiser
             (numpy fp32 divisions, torch's E4M3 cast, E2M1 by distance to
             all eight values); closed forms: g = amax / 2688, all-zero rows,
             power-of-two invariance, the error bound; E=1 dense check.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import workloads

# ---------------------------------------------------------------- helpers


def f32_round_exact(q: Fraction) -> np.float32:
    """Round an exact rational to the nearest float32 (ties to even)."""
    approx = np.float32(float(q))
    best = None
    for cand in (np.nextafter(approx, np.float32(-np.inf)), approx, np.nextafter(approx, np.float32(np.inf))):
        d = abs(Fraction(float(cand)) - q)
        if best is None or d < best[0] or (d == best[0] and (int(np.float32(cand).view(np.uint32)) & 1) == 0):
            best = (d, cand)
    return np.float32(best[1])


def fmaf_exact(a, b, c) -> np.float32:
    return f32_round_exact(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def indep_mxfp8(v: np.ndarray):
    """Independent MXFP8 quantiser: numpy for the shared exponent, torch's
    float8_e4m3fn cast (round-to-nearest-even) after a clamp to +-448.
    v: float64 [rows, cols], cols % 32 == 0.  Returns codes, scale bytes."""
    rows, cols = v.shape
    blocks = v.reshape(rows, cols // 32, 32)
    amax = np.abs(blocks).max(axis=2)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(amax > 0, amax, 1.0)))
    s = np.where(amax > 0, np.clip(e - 8, -127, 127), -127).astype(np.int64)
    scaled = blocks * np.exp2(-s.astype(np.float64))[:, :, None]
    scaled32 = torch.from_numpy(np.clip(scaled, -448.0, 448.0).astype(np.float32))
    codes = scaled32.to(torch.float8_e4m3fn).view(torch.uint8).numpy().reshape(rows, cols)
    return codes, (s + 127).astype(np.uint8)


def torch_e4m3_table() -> np.ndarray:
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def indep_dequant(codes: np.ndarray, sbytes: np.ndarray) -> np.ndarray:
    tab = torch_e4m3_table()
    rows, cols = codes.shape
    return (tab[codes].reshape(rows, cols // 32, 32) * np.exp2(sbytes.astype(np.float64) - 127)[:, :, None]
            ).reshape(rows, cols)


def bf16_round(a64: np.ndarray) -> np.ndarray:
    return torch.from_numpy(a64.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def rand_bf16(gen, shape, std=1.0):
    return (torch.randn(shape, generator=gen) * std).to(torch.bfloat16)


# ---------------------------------------------------------------- route


def _brute_topk(row: np.ndarray, k: int) -> np.ndarray:
    order = np.lexsort((np.arange(row.size), -row.astype(np.float64)))
    return np.sort(order[:k])


def test_route_ids_match_brute_force_tiny():
    w = workloads.WORKLOADS["tiny"]
    _, logits = workloads.make_activations(w)
    lg = logits.numpy()
    ids, probs = oracle.route(lg, w.top_k)
    for t in range(lg.shape[0]):
        assert np.array_equal(ids[t], _brute_topk(lg[t], w.top_k))
    assert np.all(np.diff(ids, axis=1) > 0)


def test_route_ties_go_to_lower_id():
    rng = np.random.default_rng(5)
    lg = rng.integers(-3, 3, size=(200, 16)).astype(np.float32)  # many exact ties
    for k in (1, 3, 8, 16):
        ids, _ = oracle.route(lg, k)
        for t in range(lg.shape[0]):
            assert np.array_equal(ids[t], _brute_topk(lg[t], k))


def test_route_k1_prob_is_one():
    rng = np.random.default_rng(1)
    lg = rng.standard_normal((300, 128)).astype(np.float32)
    ids, probs = oracle.route(lg, 1)
    assert np.all(probs == 1.0)
    assert np.array_equal(ids[:, 0], np.argmax(lg, axis=1))


def test_route_k_equals_e_is_softmax():
    rng = np.random.default_rng(2)
    lg = (rng.standard_normal((100, 8)) * 3).astype(np.float32)
    ids, probs = oracle.route(lg, 8)
    ref = scipy.special.softmax(lg.astype(np.float64), axis=1).astype(np.float32)
    assert np.array_equal(ids, np.tile(np.arange(8), (100, 1)))
    ulp = np.spacing(np.abs(ref))
    assert np.all(np.abs(probs - ref) <= ulp)


def test_route_k2_is_logistic():
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((200, 32)).astype(np.float32)
    ids, probs = oracle.route(lg, 2)
    for t in range(200):
        a, b = ids[t]
        pa = scipy.special.expit(float(lg[t, a]) - float(lg[t, b]))
        assert abs(probs[t, 0] - np.float32(pa)) <= np.spacing(np.float32(pa))
        assert abs(probs[t, 1] - np.float32(1 - pa)) <= np.spacing(np.float32(1 - pa))


def test_route_probs_sum_to_one():
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((500, 128)).astype(np.float32)
    _, probs = oracle.route(lg, 8)
    assert np.all(np.abs(probs.astype(np.float64).sum(1) - 1.0) <= 8 * 2.0 ** -24)


# ---------------------------------------------------------------- permute


@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (1000, 128, 8), (7, 4, 4), (1, 128, 6)])
def test_permute_matches_stable_argsort(T, E, k):
    rng = np.random.default_rng(T + E + k)
    ids = np.stack([np.sort(rng.choice(E, size=k, replace=False)) for _ in range(T)]).astype(np.int32)
    offsets, perm, inv = oracle.permute(ids, E)
    flat_e = ids.reshape(-1).astype(np.int64)
    tok = np.repeat(np.arange(T), k)
    order = np.argsort(flat_e * T + tok, kind="stable")
    assert np.array_equal(perm, order.astype(np.int32))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat_e, minlength=E))]))
    assert offsets[-1] == T * k
    assert np.array_equal(np.sort(perm), np.arange(T * k))
    assert np.array_equal(inv.reshape(-1)[perm], np.arange(T * k))


def test_permute_empty_experts():
    ids = np.array([[0, 3], [0, 3], [3, 5]], np.int32)
    offsets, perm, inv = oracle.permute(ids, 8)
    assert offsets.tolist() == [0, 2, 2, 2, 5, 5, 6, 6, 6]
    assert perm.tolist() == [0, 2, 1, 3, 4, 5]


# ---------------------------------------------------------------- mxfp8


def test_e4m3_table_matches_torch_decode():
    tab = torch_e4m3_table()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if math.isnan(tab[c]):
            assert math.isnan(v), c
        else:
            assert v == tab[c], c
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9


def _all_finite_bf16() -> np.ndarray:
    bits = np.arange(65536, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    return vals[np.isfinite(vals)]


@pytest.mark.parametrize("anchor", [0.0, 1.0, 2.0 ** 20, 2.0 ** -20, 3.0])
def test_mxfp8_exhaustive_bf16_sweep(anchor):
    vals = _all_finite_bf16().astype(np.float32)
    blocks = np.zeros((vals.size, 32), np.float32)
    blocks[:, 0] = vals
    blocks[:, 1] = anchor
    blocks[:, 7] = -vals * 0.5  # a second in-block value, exactly representable
    q, s = oracle.mxfp8_quantize(blocks)
    q2, s2 = indep_mxfp8(blocks.astype(np.float64))
    assert np.array_equal(s[:, 0], s2[:, 0])
    assert np.array_equal(q, q2)


def test_mxfp8_closed_forms():
    # scale = 2^(floor(log2 amax) - 8): amax 1.0 -> s=-8; amax 3.0 -> s=-7; amax 0.5 -> -9
    for amax, s_exp in [(1.0, -8), (3.0, -7), (0.5, -9), (448.0, 0), (2.0 ** 100, 92), (1.5 * 2.0 ** -130, -127)]:
        blk = np.zeros((1, 32), np.float32)
        blk[0, 3] = amax
        q, s = oracle.mxfp8_quantize(blk)
        assert int(s[0, 0]) - 127 == s_exp, (amax, s)
    # all-zero block -> byte 0, codes 0
    q, s = oracle.mxfp8_quantize(np.zeros((1, 32), np.float32))
    assert s[0, 0] == 0 and np.all(q == 0)
    # grid values k * 2^s round-trip exactly
    s_val = -4
    grid = np.array([oracle.e4m3_value(c) for c in range(127)])
    blk = np.zeros((4, 32), np.float32)
    chosen = np.concatenate([[448.0], grid[[1, 2, 9, 40, 77, 100, 120]]])
    for r in range(4):
        blk[r, :8] = chosen * 2.0 ** s_val * (1 if r % 2 == 0 else -1)
    q, s = oracle.mxfp8_quantize(blk)
    deq = oracle.mxfp8_dequantize(q, s)
    assert np.array_equal(deq, blk)
    # a scaled value of 500 saturates to 448 when amax already fixes the scale (amax scaled = 500)
    blk = np.zeros((1, 32), np.float32)
    blk[0, 0] = 500.0
    blk[0, 1] = -500.0
    q, s = oracle.mxfp8_quantize(blk)
    assert s[0, 0] == 127 and q[0, 0] == 0x7E and q[0, 1] == 0xFE
    # midpoint between 1.0 (0x38) and 1.125 (0x39) -> even code 0x38; 1.1875 -> 0x3A (1.25 even)
    blk = np.zeros((1, 32), np.float32)
    blk[0, 0] = 256.0  # fixes s = 0
    blk[0, 1] = 1.0625
    blk[0, 2] = 1.1875
    blk[0, 3] = -1e-30  # rounds to zero, keeps its sign
    q, s = oracle.mxfp8_quantize(blk)
    assert s[0, 0] == 127
    assert q[0, 1] == 0x38 and q[0, 2] == 0x3A and q[0, 3] == 0x80


def test_mxfp8_bf16_entry_matches_float_entry():
    gen = torch.Generator().manual_seed(9)
    x = rand_bf16(gen, (33, 256), 3.0)
    q1, s1 = oracle.mxfp8_quantize_bf16(x)
    q2, s2 = oracle.mxfp8_quantize(x.float().numpy())
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


# ---------------------------------------------------------------- forward (bf16)


def _dense_swiglu_ref(x, wg, wu, wd):
    """torch float64 dense SwiGLU MLP with the intermediate rounded to fp32 then bf16."""
    x64 = x.to(torch.float64)
    g = x64 @ wg.to(torch.float64).T
    u = x64 @ wu.to(torch.float64).T
    h = (torch.nn.functional.silu(g) * u).to(torch.float32).to(torch.bfloat16).to(torch.float64)
    return (h @ wd.to(torch.float64).T).to(torch.float32), h


def test_forward_k1_single_expert_is_dense_mlp():
    gen = torch.Generator().manual_seed(11)
    T, H, F = 24, 96, 160  # H != F: a transposed operand cannot pass
    x = rand_bf16(gen, (T, H))
    wg = rand_bf16(gen, (1, F, H), H ** -0.5)
    wu = rand_bf16(gen, (1, F, H), H ** -0.5)
    wd = rand_bf16(gen, (1, H, F), F ** -0.5)
    ids = np.zeros((T, 1), np.int32)
    probs = np.ones((T, 1), np.float32)
    out, h = oracle.forward_bf16(x, ids, probs, wg, wu, wd, want_h=True)
    ref, href = _dense_swiglu_ref(x, wg[0], wu[0], wd[0])
    # h may differ by a bf16 rounding flip where the double sums differ in the last bit
    hflip = np.mean(h[:, 0, :] != href.numpy().astype(np.float32))
    assert hflip < 1e-3
    rms = float(np.sqrt(np.mean(ref.numpy().astype(np.float64) ** 2)))
    assert np.max(np.abs(out - ref.numpy())) <= 1e-3 * rms
    if hflip == 0:
        assert np.max(np.abs(out - ref.numpy())) <= 1e-6 * rms


def test_forward_zero_gate_or_up_gives_zero():
    gen = torch.Generator().manual_seed(12)
    T, H, F, E, k = 10, 64, 64, 4, 2
    x = rand_bf16(gen, (T, H))
    wg = rand_bf16(gen, (E, F, H), 0.1)
    wu = rand_bf16(gen, (E, F, H), 0.1)
    wd = rand_bf16(gen, (E, H, F), 0.1)
    ids, probs = oracle.route(np.random.default_rng(0).standard_normal((T, E)).astype(np.float32), k)
    out = oracle.forward_bf16(x, ids, probs, torch.zeros_like(wg), wu, wd)
    assert np.all(out == 0.0)
    out = oracle.forward_bf16(x, ids, probs, wg, torch.zeros_like(wu), wd)
    assert np.all(out == 0.0)


def _small_problem(seed, T=12, H=64, F=96, E=6, k=3):
    gen = torch.Generator().manual_seed(seed)
    x = rand_bf16(gen, (T, H))
    wg = rand_bf16(gen, (E, F, H), H ** -0.5)
    wu = rand_bf16(gen, (E, F, H), H ** -0.5)
    wd = rand_bf16(gen, (E, H, F), F ** -0.5)
    ids, probs = oracle.route(np.random.default_rng(seed).standard_normal((T, E)).astype(np.float32), k)
    return x, wg, wu, wd, ids, probs


def test_forward_doubling_probs_doubles_output():
    x, wg, wu, wd, ids, probs = _small_problem(13)
    a = oracle.forward_bf16(x, ids, probs, wg, wu, wd)
    b = oracle.forward_bf16(x, ids, probs * 2, wg, wu, wd)
    assert np.array_equal(b, a * 2)


def test_forward_combine_is_ascending_fma_chain():
    x, wg, wu, wd, ids, probs = _small_problem(14, T=5, k=3)
    T, k = ids.shape
    # per-route expert rows y_e(t) via k=1, p=1 calls
    ys = {}
    for j in range(k):
        ys[j] = oracle.forward_bf16(x, ids[:, j:j + 1].copy(), np.ones((T, 1), np.float32), wg, wu, wd)
    # hand the routes over in a scrambled order: the oracle must sort them
    scr = ids[:, ::-1].copy()
    pscr = probs[:, ::-1].copy()
    out = oracle.forward_bf16(x, scr, pscr, wg, wu, wd)
    for t in range(T):
        for c in range(0, out.shape[1], 7):
            acc = np.float32(0.0)
            for j in range(k):  # ids are ascending along j
                acc = fmaf_exact(probs[t, j], ys[j][t, c], acc)
            assert out[t, c] == acc


def test_forward_identical_experts_half_probs_is_identity():
    x, wg, wu, wd, ids, probs = _small_problem(15, E=2, k=2)
    wg = torch.stack([wg[0], wg[0]])
    wu = torch.stack([wu[0], wu[0]])
    wd = torch.stack([wd[0], wd[0]])
    T = ids.shape[0]
    ids = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    half = np.full((T, 2), 0.5, np.float32)
    out = oracle.forward_bf16(x, ids, half, wg, wu, wd)
    one = oracle.forward_bf16(x, ids[:, :1].copy(), np.ones((T, 1), np.float32), wg, wu, wd)
    assert np.array_equal(out, one)


def test_forward_token_order_and_duplication_invariance():
    x, wg, wu, wd, ids, probs = _small_problem(16, T=9)
    out = oracle.forward_bf16(x, ids, probs, wg, wu, wd)
    p = np.random.default_rng(0).permutation(9)
    out_p = oracle.forward_bf16(x[torch.from_numpy(p)], ids[p].copy(), probs[p].copy(), wg, wu, wd)
    assert np.array_equal(out_p, out[p])
    dup = np.concatenate([np.arange(9), np.arange(9)])
    out_d = oracle.forward_bf16(x, ids, probs, wg, wu, wd, tokens=dup)
    assert np.array_equal(out_d[:9], out_d[9:]) and np.array_equal(out_d[:9], out)


# ---------------------------------------------------------------- forward (mxfp8)


def test_forward_mxfp8_k1_single_expert_is_dense_mlp():
    gen = torch.Generator().manual_seed(21)
    T, H, F = 16, 128, 96
    x = rand_bf16(gen, (T, H))
    wg = rand_bf16(gen, (1, F, H), H ** -0.5)
    wu = rand_bf16(gen, (1, F, H), H ** -0.5)
    wd = rand_bf16(gen, (1, H, F), F ** -0.5)
    wq = oracle.quantize_weights_mxfp8(wg, wu, wd)
    ids = np.zeros((T, 1), np.int32)
    probs = np.ones((T, 1), np.float32)
    out, (hq, hs, hf) = oracle.forward_mxfp8(x, ids, probs, wq, want_h=True)
    # independent pipeline: numpy scales + torch e4m3 cast
    xq = indep_dequant(*indep_mxfp8(x.double().numpy()))
    g_w = indep_dequant(*indep_mxfp8(wg[0].double().numpy()))
    u_w = indep_dequant(*indep_mxfp8(wu[0].double().numpy()))
    d_w = indep_dequant(*indep_mxfp8(wd[0].double().numpy()))
    g = xq @ g_w.T
    u = xq @ u_w.T
    h32 = (scipy.special.expit(g) * g * u).astype(np.float32)
    assert np.mean(h32 != hf[:, 0, :]) < 2e-2  # double-sum order may flip a last fp32 bit
    hc, hsc = indep_mxfp8(hf[:, 0, :].astype(np.float64))  # quantiser consistency on the oracle's own h
    assert np.array_equal(hc, hq[:, 0, :]) and np.array_equal(hsc, hs[:, 0, :])
    ref = (indep_dequant(*indep_mxfp8(h32.astype(np.float64))) @ d_w.T).astype(np.float32)
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
    assert np.max(np.abs(out - ref)) <= 5e-2 * rms
    assert np.mean(np.abs(out - ref)) <= 2e-3 * np.mean(np.abs(ref))


def test_forward_mxfp8_zero_gate_gives_zero():
    x, wg, wu, wd, ids, probs = _small_problem(22, H=64, F=64)
    wq = oracle.quantize_weights_mxfp8(torch.zeros_like(wg), wu, wd)
    out = oracle.forward_mxfp8(x, ids, probs, wq)
    assert np.all(out == 0.0)


def test_forward_mxfp8_close_to_bf16():
    """MXFP8 and bf16 forwards of the same problem differ by a few percent
    (the pages report ~4% relative distance for MXFP8 MoE layers)."""
    x, wg, wu, wd, ids, probs = _small_problem(23, T=32, H=256, F=128, E=4, k=2)
    a = oracle.forward_bf16(x, ids, probs, wg, wu, wd).astype(np.float64)
    b = oracle.forward_mxfp8(x, ids, probs, oracle.quantize_weights_mxfp8(wg, wu, wd)).astype(np.float64)
    d = np.linalg.norm(b - a) / np.linalg.norm(a)
    assert 0.005 < d < 0.12


# ---------------------------------------------------------------- variants (apply_topk_in_fc1, clamp, bf16 out)


def _pow2_probs(ids, seed):
    """Per-route probabilities that are powers of two (1/2, 1/4, 1/8)."""
    rng = np.random.default_rng(seed)
    return (2.0 ** -rng.integers(1, 4, size=ids.shape)).astype(np.float32)


def test_variant_probs_in_fc1_pow2_probs_equal_plain_forward():
    # scaling the SwiGLU row by a power of two commutes with the fp32 and bf16
    # roundings and scales y exactly, and acc + p*y is then the plain fmaf(p, y, acc):
    # both variants must agree bit for bit (a dropped or doubled probability fails)
    x, wg, wu, wd, ids, _ = _small_problem(21, T=10, k=3)
    probs = _pow2_probs(ids, 21)
    plain = oracle.forward_bf16(x, ids, probs, wg, wu, wd)
    fc1 = oracle.forward_bf16(x, ids, probs, wg, wu, wd, probs_in_fc1=True)
    assert np.array_equal(plain, fc1)
    wq = oracle.quantize_weights_mxfp8(wg, wu, wd)
    plain8 = oracle.forward_mxfp8(x, ids, probs, wq)
    fc18 = oracle.forward_mxfp8(x, ids, probs, wq, probs_in_fc1=True)
    assert np.array_equal(plain8, fc18)


def _dense_variant_ref(x, wg, wu, wd, p=None, clamp=None):
    """torch float64 dense SwiGLU MLP: pre-activations clamped to [-clamp, clamp],
    the row scaled by p, rounded to fp32 then bf16; y in fp32."""
    x64 = x.to(torch.float64)
    g = x64 @ wg.to(torch.float64).T
    u = x64 @ wu.to(torch.float64).T
    if clamp is not None:
        g, u = g.clamp(-clamp, clamp), u.clamp(-clamp, clamp)
    h = torch.nn.functional.silu(g) * u
    if p is not None:
        h = h * p
    h = h.to(torch.float32).to(torch.bfloat16).to(torch.float64)
    return (h @ wd.to(torch.float64).T).to(torch.float32)


def _single_expert(seed, T=20, H=96, F=160):
    gen = torch.Generator().manual_seed(seed)
    x = rand_bf16(gen, (T, H))
    wg = rand_bf16(gen, (1, F, H), H ** -0.5)
    wu = rand_bf16(gen, (1, F, H), H ** -0.5)
    wd = rand_bf16(gen, (1, H, F), F ** -0.5)
    return x, wg, wu, wd, np.zeros((T, 1), np.int32)


def _close_to_dense(out, ref):
    rms = float(np.sqrt(np.mean(ref.numpy().astype(np.float64) ** 2)))
    # rare bf16 rounding flips of h where the two double sums differ in the last bit
    assert np.max(np.abs(out - ref.numpy())) <= 1e-3 * rms
    assert np.mean(np.abs(out - ref.numpy())) <= 1e-6 * rms


def test_variant_probs_in_fc1_is_dense_mlp_times_p_before_rounding():
    x, wg, wu, wd, ids = _single_expert(22)
    p = np.full(ids.shape, 0.3, np.float32)
    out = oracle.forward_bf16(x, ids, p, wg, wu, wd, probs_in_fc1=True)
    ref = _dense_variant_ref(x, wg[0], wu[0], wd[0], p=float(np.float32(0.3)))
    _close_to_dense(out, ref)
    # and not the plain forward (p applied once, after FC2)
    plain = oracle.forward_bf16(x, ids, p, wg, wu, wd)
    assert not np.array_equal(out, plain)


def test_variant_clamp_matches_dense_reference_and_is_inert_when_wide():
    x, wg, wu, wd, ids = _single_expert(23)
    one = np.ones(ids.shape, np.float32)
    c = 0.25  # |g|, |u| ~ N(0, 1): most pre-activations are clamped
    out = oracle.forward_bf16(x, ids, one, wg, wu, wd, gate_up_clamp=c)
    _close_to_dense(out, _dense_variant_ref(x, wg[0], wu[0], wd[0], clamp=c))
    plain = oracle.forward_bf16(x, ids, one, wg, wu, wd)
    assert not np.array_equal(out, plain)
    wide = oracle.forward_bf16(x, ids, one, wg, wu, wd, gate_up_clamp=1e6)
    assert np.array_equal(wide, plain)


def test_round_bf16_matches_torch_cast_including_ties():
    rng = np.random.default_rng(24)
    a = (rng.standard_normal(4096) * np.exp(rng.standard_normal(4096) * 4)).astype(np.float32)
    # exact ties: low 16 bits 0x8000, with even and odd kept halves
    ties = (rng.integers(0x3F000000, 0x43000000, size=512, dtype=np.uint32) & 0xFFFF0000) | 0x8000
    a = np.concatenate([a, ties.view(np.float32), -ties.view(np.float32), np.float32([0.0, -0.0])])
    got = oracle.round_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    # ties go to the even kept half
    t = ties.view(np.float32)
    kept = oracle.round_bf16(t)
    assert np.all(kept & 1 == 0)


# ---------------------------------------------------------------- squared-ReLU experts


def _dense_relu2_ref(x, w1, wd, p=None, clamp=None):
    """torch float64 dense squared-ReLU MLP: relu(W1 x)^2 (pre-activation clamped,
    row scaled by p), rounded to fp32 then bf16; y in fp32."""
    g = x.to(torch.float64) @ w1.to(torch.float64).T
    if clamp is not None:
        g = g.clamp(-clamp, clamp)
    h = torch.relu(g) ** 2
    if p is not None:
        h = h * p
    h = h.to(torch.float32).to(torch.bfloat16).to(torch.float64)
    return (h @ wd.to(torch.float64).T).to(torch.float32)


def test_squared_relu_single_expert_is_dense_relu2_mlp():
    x, wg, _, wd, ids = _single_expert(41)
    one = np.ones(ids.shape, np.float32)
    out = oracle.forward_bf16(x, ids, one, wg, None, wd, squared_relu=True)
    _close_to_dense(out, _dense_relu2_ref(x, wg[0], wd[0]))
    # with the variants: probability in FC1 and a clamp on the one pre-activation
    p = np.full(ids.shape, 0.3, np.float32)
    out = oracle.forward_bf16(x, ids, p, wg, None, wd, squared_relu=True, probs_in_fc1=True, gate_up_clamp=0.5)
    _close_to_dense(out, _dense_relu2_ref(x, wg[0], wd[0], p=float(np.float32(0.3)), clamp=0.5))


def test_squared_relu_negative_preactivations_give_zero():
    gen = torch.Generator().manual_seed(42)
    T, H, F, E, k = 8, 64, 96, 4, 2
    x = rand_bf16(gen, (T, H)).abs()
    w1 = -rand_bf16(gen, (E, F, H), 0.1).abs()  # x >= 0, W1 <= 0: every pre-activation <= 0
    wd = rand_bf16(gen, (E, H, F), 0.1)
    ids, probs = oracle.route(np.random.default_rng(42).standard_normal((T, E)).astype(np.float32), k)
    out = oracle.forward_bf16(x, ids, probs, w1, None, wd, squared_relu=True)
    assert np.all(out == 0.0)
    # the same weights as SwiGLU gate and up give a nonzero output: the flag selects the activation
    out_swiglu = oracle.forward_bf16(x, ids, probs, w1, w1, wd)
    assert np.any(out_swiglu != 0.0)


def test_squared_relu_ignores_probs_scaling_by_pow2_like_plain():
    # the combine rules do not depend on the activation: power-of-two probabilities give the
    # same bits with the probability applied in FC1 or in the combine
    x, wg, _, wd, ids, _ = _small_problem(43, T=10, k=3)
    probs = _pow2_probs(ids, 43)
    a = oracle.forward_bf16(x, ids, probs, wg, None, wd, squared_relu=True)
    b = oracle.forward_bf16(x, ids, probs, wg, None, wd, squared_relu=True, probs_in_fc1=True)
    assert np.array_equal(a, b)


def test_squared_relu_mxfp8_single_expert_is_dense_relu2_mlp():
    gen = torch.Generator().manual_seed(44)
    T, H, F = 16, 128, 96
    x = rand_bf16(gen, (T, H))
    w1 = rand_bf16(gen, (1, F, H), H ** -0.5)
    wd = rand_bf16(gen, (1, H, F), F ** -0.5)
    wq = oracle.quantize_weights_mxfp8(w1, w1, wd)
    # the up codes are not read: poison them, the result must not change
    gq, gs, uq, us, dq, ds = wq
    poisoned = (gq, gs, np.full_like(uq, 0x7F), np.full_like(us, 0xFE), dq, ds)
    ids = np.zeros((T, 1), np.int32)
    probs = np.ones((T, 1), np.float32)
    out, (hq, hs, hf) = oracle.forward_mxfp8(x, ids, probs, poisoned, want_h=True, squared_relu=True)
    # independent pipeline: numpy scales + torch e4m3 cast
    xq = indep_dequant(*indep_mxfp8(x.double().numpy()))
    g = xq @ indep_dequant(*indep_mxfp8(w1[0].double().numpy())).T
    h32 = (np.maximum(g, 0.0) ** 2).astype(np.float32)
    assert np.mean(h32 != hf[:, 0, :]) < 2e-2
    ref = (indep_dequant(*indep_mxfp8(h32.astype(np.float64))) @ indep_dequant(*indep_mxfp8(wd[0].double().numpy())).T)
    ref = ref.astype(np.float32)
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
    assert np.max(np.abs(out - ref)) <= 5e-2 * rms
    assert np.mean(np.abs(out - ref)) <= 2e-3 * np.mean(np.abs(ref))


# ---------------------------------------------------------------- nvfp4 (per-token recipe)

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def indep_e2m1(x64: np.ndarray) -> np.ndarray:
    """E2M1 codes by distance to all eight magnitudes, ties to the even code."""
    d = np.abs(np.abs(x64)[..., None] - E2M1_GRID) + 1e-12 * (np.arange(8) & 1)
    return (np.argmin(d, axis=-1) | (np.signbit(x64).astype(np.int64) << 3)).astype(np.uint8)


def indep_nvfp4(v, per_row=True):
    """Independent NVFP4 quantiser of fp32 rows [rows, cols]: numpy float32
    arithmetic for the scales and quotients, torch's float8_e4m3fn cast for
    the block scales.  Returns packed codes, scale bytes, second-level scales."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows, cols = v.shape
    amax = np.abs(v).max(axis=1) if per_row else np.full(rows, np.abs(v).max(), np.float32)
    with np.errstate(divide="ignore", invalid="ignore", under="ignore"):
        g = (amax / np.float32(2688.0)).astype(np.float32)
        g = np.where((amax > 0) & (g > 0), g, np.float32(1.0)).astype(np.float32)
        blocks = v.reshape(rows, cols // 16, 16)
        amax_b = np.abs(blocks).max(axis=2)
        sf = ((amax_b / g[:, None]).astype(np.float32) / np.float32(6.0)).astype(np.float32)
        sbytes = torch.from_numpy(np.minimum(sf, np.float32(448.0))).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        sval = torch_e4m3_table()[sbytes].astype(np.float32)
        d = (sval * g[:, None]).astype(np.float32)
        quot = (blocks / d[:, :, None]).astype(np.float32)
    codes = np.where(d[:, :, None] != 0, indep_e2m1(quot.astype(np.float64)),
                     (np.signbit(blocks).astype(np.uint8) << 3)).reshape(rows, cols).astype(np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, sbytes.astype(np.uint8), (g if per_row else g[:1])


def indep_nvfp4_dequant(q, s, g, per_row=True) -> np.ndarray:
    rows, half = q.shape
    codes = np.empty((rows, 2 * half), np.int64)
    codes[:, 0::2] = q & 15
    codes[:, 1::2] = q >> 4
    mag = E2M1_GRID[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    gg = g.astype(np.float64) if per_row else np.full(rows, float(g[0]))
    return (mag.reshape(rows, -1, 16) * torch_e4m3_table()[s][:, :, None] * gg[:, None, None]).reshape(rows, -1)


def test_nvfp4_grid_ties_saturation_and_sign():
    # amax 2688 fixes g = 1; a block with amax 6 has scale 1.0 (E4M3 0x38), so its codes are E2M1(v)
    row = np.zeros((1, 48), np.float32)
    row[0, 0] = 2688.0
    row[0, 16:32] = [0, 0.25, 0.5, 0.75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, -0.1]
    row[0, 32:48] = [6, -6, 0.2499, 0.2501, 5.01, -4.99, 2.51, -2.49, 0, 0, 0, 0, 0, 0, 0, -0.0]
    q, s, g = oracle.nvfp4_quantize(row)
    assert g[0] == 1.0 and s[0, 0] == 0x7E and s[0, 1] == 0x38 and s[0, 2] == 0x38
    codes = np.empty(48, np.int64)
    codes[0::2], codes[1::2] = q[0] & 15, q[0] >> 4
    # ties to even: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4; -0.1 -> -0
    assert list(codes[16:32]) == [0, 0, 1, 2, 2, 2, 3, 4, 4, 4, 5, 6, 6, 6, 7, 8]
    assert list(codes[32:40]) == [7, 15, 0, 1, 7, 14, 5, 12]
    assert codes[47] == 8 and codes[0] == 7  # -0.0 keeps its sign; 2688 / 448 = 6
    # beyond 6 saturates: a block whose scale is capped at 448 by the row's g
    row = np.zeros((1, 16), np.float32)
    row[0, :2] = [2688.0, -2688.0]
    q, s, g = oracle.nvfp4_quantize(row)
    assert (q[0, 0] & 15) == 7 and (q[0, 0] >> 4) == 15


@pytest.mark.parametrize("per_row", [True, False])
def test_nvfp4_matches_independent_quantiser(per_row):
    gen = np.random.default_rng(17)
    rows = []
    for mag in (1e-30, 1e-6, 1e-2, 1.0, 37.0, 1e4, 1e30):
        rows.append(gen.standard_normal((6, 64)) * mag)
    v = np.concatenate(rows).astype(np.float32)
    v[3, 5:21] = 0.0          # a whole block of zeros next to live ones
    v[10] = 0.0               # an all-zero row
    v[20, ::7] *= 1000.0      # a few outliers
    q, s, g = oracle.nvfp4_quantize(v, per_row=per_row)
    q2, s2, g2 = indep_nvfp4(v, per_row=per_row)
    assert np.array_equal(g, g2) and np.array_equal(s, s2) and np.array_equal(q, q2)
    # bf16 entry equals the fp32 entry on the same values
    xb = torch.from_numpy(v).to(torch.bfloat16)
    qa, sa, ga = oracle.nvfp4_quantize(xb, per_row=per_row)
    qb, sb, gb = oracle.nvfp4_quantize(xb.float().numpy(), per_row=per_row)
    assert np.array_equal(qa, qb) and np.array_equal(sa, sb) and np.array_equal(ga, gb)
    assert np.array_equal(oracle.nvfp4_dequantize(q, s, g, per_row), indep_nvfp4_dequant(q2, s2, g2, per_row))


def test_nvfp4_closed_forms():
    gen = np.random.default_rng(5)
    v = gen.standard_normal((8, 128)).astype(np.float32)
    q, s, g = oracle.nvfp4_quantize(v)
    amax = np.abs(v).max(axis=1)
    assert np.array_equal(g, (amax / np.float32(2688.0)).astype(np.float32))
    # all-zero row: g = 1, scale bytes 0, codes 0
    qz, sz, gz = oracle.nvfp4_quantize(np.zeros((1, 32), np.float32))
    assert gz[0] == 1.0 and np.all(sz == 0) and np.all(qz == 0)
    # scaling a row by 2^j scales g by 2^j exactly and leaves codes and block scales unchanged
    for j in (-20, -3, 5, 40):
        qj, sj, gj = oracle.nvfp4_quantize(v * np.float32(2.0 ** j))
        assert np.array_equal(qj, q) and np.array_equal(sj, s) and np.array_equal(gj, g * np.float32(2.0 ** j))
    # error bound: every element is within one block divisor value(s) * g of its value
    deq = oracle.nvfp4_dequantize(q, s, g)
    div = (torch_e4m3_table()[s] * g[:, None].astype(np.float64))
    assert np.all(np.abs(deq - v).reshape(8, 8, 16) <= div[:, :, None] * (1 + 1e-12))
    # and the block amax is reproduced within a quarter of itself (E2M1 step at 4..6, E4M3 rounding)
    amax_b = np.abs(v).reshape(8, 8, 16).max(axis=2)
    amax_dq = np.abs(deq).reshape(8, 8, 16).max(axis=2)
    assert np.all(np.abs(amax_dq - amax_b) <= 0.25 * amax_b)


def _nvfp4_dense_ref(x, wg, wu, wd):
    """Independent NVFP4 pipeline for one expert (E=1, k=1, p=1): independent
    quantisers, float64 matmuls, fp32 h quantised per row."""
    xq = indep_nvfp4_dequant(*indep_nvfp4(x.float().numpy()))
    w1 = np.concatenate([wg[0].float().numpy(), wu[0].float().numpy()])
    w1d = indep_nvfp4_dequant(*indep_nvfp4(w1, per_row=False), per_row=False)
    wdd = indep_nvfp4_dequant(*indep_nvfp4(wd[0].float().numpy(), per_row=False), per_row=False)
    F = wg.shape[1]
    g = xq @ w1d[:F].T
    u = xq @ w1d[F:].T
    h32 = (scipy.special.expit(g) * g * u).astype(np.float32)
    return h32, (indep_nvfp4_dequant(*indep_nvfp4(h32)) @ wdd.T).astype(np.float32)


def test_forward_nvfp4_k1_single_expert_is_dense_mlp():
    gen = torch.Generator().manual_seed(31)
    T, H, F = 16, 128, 96
    x = rand_bf16(gen, (T, H))
    wg = rand_bf16(gen, (1, F, H), H ** -0.5)
    wu = rand_bf16(gen, (1, F, H), H ** -0.5)
    wd = rand_bf16(gen, (1, H, F), F ** -0.5)
    wq = oracle.quantize_weights_nvfp4(wg, wu, wd)
    ids = np.zeros((T, 1), np.int32)
    probs = np.ones((T, 1), np.float32)
    out, (hq, hs, hg, hf) = oracle.forward_nvfp4(x, ids, probs, wq, want_h=True)
    h32, ref = _nvfp4_dense_ref(x, wg, wu, wd)
    assert np.mean(h32 != hf[:, 0, :]) < 2e-2  # double-sum order may flip a last fp32 bit
    q2, s2, g2 = indep_nvfp4(hf[:, 0, :])    # quantiser consistency on the oracle's own h
    assert np.array_equal(q2, hq[:, 0, :]) and np.array_equal(s2, hs[:, 0, :]) and np.array_equal(g2, hg[:, 0])
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
    assert np.max(np.abs(out - ref)) <= 5e-2 * rms
    assert np.mean(np.abs(out - ref)) <= 5e-3 * np.mean(np.abs(ref))


def test_forward_nvfp4_weight_scales_are_per_expert_matrix():
    x, wg, wu, wd, ids, probs = _small_problem(33, H=64, F=32, E=3)
    w1_q, w1_s, g1, wd_q, wd_s, g2 = oracle.quantize_weights_nvfp4(wg, wu, wd)
    for e in range(3):
        a1 = max(float(wg[e].float().abs().max()), float(wu[e].float().abs().max()))
        assert g1[e] == np.float32(np.float32(a1) / np.float32(2688.0))
        assert g2[e] == np.float32(np.float32(float(wd[e].float().abs().max())) / np.float32(2688.0))


def test_forward_nvfp4_zero_gate_gives_zero():
    x, wg, wu, wd, ids, probs = _small_problem(34, H=64, F=64)
    out = oracle.forward_nvfp4(x, ids, probs, oracle.quantize_weights_nvfp4(torch.zeros_like(wg), wu, wd))
    assert np.all(out == 0.0)


def test_forward_nvfp4_close_to_bf16():
    """NVFP4 and bf16 forwards of the same problem differ by some percent: more
    than MXFP8 (3 bits of element precision instead of 4, scales to 1/16)."""
    x, wg, wu, wd, ids, probs = _small_problem(35, T=32, H=256, F=128, E=4, k=2)
    a = oracle.forward_bf16(x, ids, probs, wg, wu, wd).astype(np.float64)
    b = oracle.forward_nvfp4(x, ids, probs, oracle.quantize_weights_nvfp4(wg, wu, wd)).astype(np.float64)
    c = oracle.forward_mxfp8(x, ids, probs, oracle.quantize_weights_mxfp8(wg, wu, wd)).astype(np.float64)
    d4 = np.linalg.norm(b - a) / np.linalg.norm(a)
    d8 = np.linalg.norm(c - a) / np.linalg.norm(a)
    assert 0.02 < d4 < 0.3 and d8 < d4
