"""GPU parity of the forward's variants (cudnn-frontend PR #448, the MoeEp
options; Megatron-LM PR #8367, the output type): the router probability
applied to the SwiGLU row (`apply_topk_in_fc1`), the gate/up clamp, and the
bf16 finalize output, in bf16, MXFP8 and NVFP4, against the oracle's variants on
the same inputs, with the tolerances of the plain forward.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from moe_testlib import GpuMoe, assert_close, assert_close_bf16_out

pytestmark = pytest.mark.gpu

# H, F not multiples of 128 (K and output-column tails); enough tokens for
# route tiles of every width and both x-row dispatch kinds
SHAPE = dict(H=320, F=224, E=12, k=3, T=700)


def _case(seed, zipf=True):
    H, F, E, k, T = (SHAPE[c] for c in "HFEkT")
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=seed, zipf=zipf)
    ids, probs = oracle.route(logits.numpy(), k)
    return x, logits, weights, ids, probs


def _run(precision, weights, x, logits, **variant):
    H, F, E, k, T = (SHAPE[c] for c in "HFEkT")
    m = GpuMoe(H, F, E, k, T, weights, precision=precision, **variant)
    out = m.forward(x.cuda(), T, logits=logits.cuda())
    torch.cuda.synchronize()
    assert m.status() == 0
    return out


def _oracle(precision, x, ids, probs, weights, **variant):
    if precision == "bf16":
        return oracle.forward_bf16(x, ids, probs, *weights, **variant)
    if precision == "nvfp4":
        return oracle.forward_nvfp4(x, ids, probs, oracle.quantize_weights_nvfp4(*weights), **variant)
    return oracle.forward_mxfp8(x, ids, probs, oracle.quantize_weights_mxfp8(*weights), **variant)


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_probs_in_fc1_matches_oracle(precision):
    x, logits, weights, ids, probs = _case(31)
    out = _run(precision, weights, x, logits, probs_in_fc1=True)
    ref = _oracle(precision, x, ids, probs, weights, probs_in_fc1=True)
    assert_close(out.float().cpu().numpy(), ref, precision, f"probs in fc1 ({precision})")
    # applied once: not the plain forward's result
    plain = _oracle(precision, x, ids, probs, weights)
    assert np.max(np.abs(ref - plain)) > 0


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_probs_in_fc1_with_power_of_two_probs_is_bitwise_the_plain_forward(precision):
    # scaling h by 2^-n commutes with its rounding / quantisation (NVFP4: the row's
    # scale takes the factor exactly, codes and block scales stay) and scales the
    # down GEMM's fp32 sums exactly, and acc + p*y is fmaf(p, y, acc)
    H, F, E, k, T = (SHAPE[c] for c in "HFEkT")
    x, _, weights, ids, _ = _case(32)
    p = (2.0 ** -np.random.default_rng(32).integers(1, 4, size=ids.shape)).astype(np.float32)
    outs = []
    for fc1 in (False, True):
        m = GpuMoe(H, F, E, k, T, weights, precision=precision, probs_in_fc1=fc1)
        outs.append(m.forward(x.cuda(), T, ids=torch.from_numpy(ids).cuda(), probs=torch.from_numpy(p).cuda()))
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_gate_up_clamp_matches_oracle(precision):
    x, logits, weights, ids, probs = _case(33)
    c = 0.5
    out = _run(precision, weights, x, logits, gate_up_clamp=c)
    ref = _oracle(precision, x, ids, probs, weights, gate_up_clamp=c)
    assert_close(out.cpu().numpy(), ref, precision, f"clamp ({precision})")
    plain = _oracle(precision, x, ids, probs, weights)
    assert np.max(np.abs(ref - plain)) > 1e-3 * np.sqrt(np.mean(plain.astype(np.float64) ** 2))


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_bf16_output_is_the_fp32_output_rounded(precision):
    x, logits, weights, ids, probs = _case(34)
    out32 = _run(precision, weights, x, logits)
    out16 = _run(precision, weights, x, logits, out_dtype="bf16")
    assert out16.dtype == torch.bfloat16
    # the same fp32 sums, rounded to nearest even: bit for bit
    rounded = oracle.round_bf16(out32.cpu().numpy())
    assert np.array_equal(out16.view(torch.int16).cpu().numpy().view(np.uint16), rounded)
    assert_close_bf16_out(out16.float().cpu().numpy(), _oracle(precision, x, ids, probs, weights), precision,
                          f"bf16 out ({precision})")


def test_all_variants_together_on_the_decode_workload():
    w = workloads.WORKLOADS["decode"]
    x, logits = workloads.make_activations(w)
    weights = workloads.make_weights(w)
    m = GpuMoe(w.hidden, w.ffn, w.num_experts, w.top_k, w.capacity, weights, probs_in_fc1=True,
               gate_up_clamp=2.0, out_dtype="bf16")
    out = m.forward(x.cuda(), w.max_live, logits=logits.cuda())
    torch.cuda.synchronize()
    assert m.status() == 0
    live = w.max_live
    ids, probs = oracle.route(logits[:live].numpy(), w.top_k)
    toks = np.arange(0, live, 7)
    ref = oracle.forward_bf16(x[:live], ids, probs, *weights, tokens=toks, probs_in_fc1=True, gate_up_clamp=2.0)
    assert_close_bf16_out(out[toks].float().cpu().numpy(), ref, "bf16", "decode, all variants")
    # rows past the live count are untouched (NaN sentinel)
    assert torch.isnan(out[live:].float()).all()



# ---------------------------------------------------------------- squared-ReLU experts (bf16)


@pytest.mark.parametrize("precision", ["bf16", "mxfp8", "nvfp4"])
def test_squared_relu_matches_oracle(precision):
    x, logits, weights, ids, probs = _case(35)
    wg, _, wd = weights
    H, F, E, k, T = (SHAPE[c] for c in "HFEkT")
    m = GpuMoe(H, F, E, k, T, (wg, wg, wd), precision=precision, squared_relu=True)
    out = m.forward(x.cuda(), T, logits=logits.cuda())
    torch.cuda.synchronize()
    assert m.status() == 0
    if precision == "bf16":
        ref = oracle.forward_bf16(x, ids, probs, wg, None, wd, squared_relu=True)
    elif precision == "nvfp4":
        # one FC1 matrix (the gate rows) with its own second-level scale
        ref = oracle.forward_nvfp4(x, ids, probs, oracle.quantize_weights_nvfp4(wg, None, wd), squared_relu=True)
    else:
        # the oracle's MXFP8 path quantises W1 as its gate rows; the up rows are not used
        ref = oracle.forward_mxfp8(x, ids, probs, oracle.quantize_weights_mxfp8(wg, wg, wd), squared_relu=True)
    assert_close(out.cpu().numpy(), ref, precision, f"squared ReLU ({precision})")


def test_squared_relu_with_variants_on_nano_shapes():
    # H = 2688, F = 1856: F pads to 1920 columns of h and to 2048 FC1 rows, so the last pair
    # tile's second CTA holds only padding rows and must store nothing
    H, F, E, k, T = 2688, 1856, 128, 6, 600
    x, logits, weights = workloads.small_case(H, F, E, k, T, seed=36)
    wg, _, wd = weights
    import routed_moe_swiglu_b200 as rm
    m = GpuMoe(H, F, E, k, T, weights, squared_relu=True, probs_in_fc1=True, gate_up_clamp=1.5,
               out_dtype="bf16")
    rm.moe_prepare_weights(m.plan, wg.cuda(), None, wd.cuda(), m.wbuf)  # w_up is not read
    out = m.forward(x.cuda(), T, logits=logits.cuda())
    torch.cuda.synchronize()
    assert m.status() == 0
    ids, probs = oracle.route(logits.numpy(), k)
    toks = np.arange(0, T, 5)
    ref = oracle.forward_bf16(x, ids, probs, wg, None, wd, tokens=toks, squared_relu=True, probs_in_fc1=True,
                              gate_up_clamp=1.5)
    assert_close_bf16_out(out[toks].float().cpu().numpy(), ref, "bf16", "squared ReLU, Nano shapes, all variants")
