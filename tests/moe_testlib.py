"""Shared helpers of the GPU tests: build a problem from the seeded
workloads, run the CUDA path through the C ABI, run the oracle on the same
inputs, and the tolerance check stated for the method:

  bf16:  max|gpu - oracle| <= 2e-2 * RMS(oracle) and
         mean|gpu - oracle| / mean|oracle| <= 2e-3
  MXFP8: max|gpu - oracle| <= 5e-2 * RMS(oracle)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import routed_moe_swiglu_b200 as rm
import workloads

TOL = {"bf16": dict(max_rms=2e-2, mean_rel=2e-3), "mxfp8": dict(max_rms=5e-2, mean_rel=None),
       "nvfp4": dict(max_rms=5e-2, mean_rel=None)}


def assert_close(gpu: np.ndarray, ref: np.ndarray, precision: str, what: str = "") -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    d = np.abs(gpu - ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    stats = dict(max_abs=float(d.max()) if d.size else 0.0, rms=rms,
                 mean_rel=float(d.mean() / max(np.abs(ref).mean(), 1e-30)) if d.size else 0.0)
    t = TOL[precision]
    assert stats["max_abs"] <= t["max_rms"] * rms, f"{what}: {stats}"
    if t["mean_rel"] is not None:
        assert stats["mean_rel"] <= t["mean_rel"], f"{what}: {stats}"
    return stats


def assert_close_bf16_out(gpu16: np.ndarray, ref32: np.ndarray, precision: str, what: str = "") -> dict:
    """A bf16 output against the oracle's fp32 output: the fp32 tolerance above
    plus half a bf16 ulp of each reference value (2^-8 relative), the rounding
    the output itself adds."""
    gpu = np.asarray(gpu16, dtype=np.float64)
    ref = np.asarray(ref32, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    d = np.abs(gpu - ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    t = TOL[precision]
    excess = d - (t["max_rms"] * rms + 2.0 ** -8 * np.abs(ref))
    stats = dict(max_abs=float(d.max()) if d.size else 0.0, rms=rms, max_excess=float(excess.max()) if d.size else 0.0,
                 mean_rel=float(d.mean() / max(np.abs(ref).mean(), 1e-30)) if d.size else 0.0)
    assert stats["max_excess"] <= 0.0, f"{what}: {stats}"
    if t["mean_rel"] is not None:
        assert stats["mean_rel"] <= t["mean_rel"] + 2.0 ** -9, f"{what}: {stats}"
    return stats


class GpuMoe:
    """A plan + prepared weight buffer + workspace on cuda:0."""

    def __init__(self, hidden, ffn, experts, top_k, capacity, weights, precision="bf16", max_live=0, **variant):
        self.plan = rm.moe_plan_create(hidden=hidden, ffn=ffn, num_experts=experts, top_k=top_k,
                                       capacity=capacity, precision=precision, max_live_rows=max_live, **variant)
        self.H, self.F, self.E, self.k, self.cap = hidden, ffn, experts, top_k, capacity
        self.precision = precision
        self.wbuf = rm.alloc_weight_buffer(self.plan)
        self.ws = rm.alloc_workspace(self.plan)
        self.live = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.prepare(weights)

    def prepare(self, weights):
        wg, wu, wd = (w.to("cuda") for w in weights)
        rm.moe_prepare_weights(self.plan, wg, wu, wd, self.wbuf)
        torch.cuda.synchronize()

    def forward(self, x, live, logits=None, ids=None, probs=None, out=None, sentinel=float("nan")):
        if out is None:
            dt = torch.bfloat16 if self.plan.out_dtype == "bf16" else torch.float32
            out = torch.full((self.cap, self.H), sentinel, dtype=dt, device="cuda")
        self.live.fill_(int(live))
        rm.moe_forward(self.plan, x, self.wbuf, self.live, out, self.ws, logits=logits, ids=ids, probs=probs)
        return out

    def views(self):
        return rm.moe_get_workspace_views(self.plan, self.ws)

    def read_i32(self, ptr, n):
        """Copy n int32 from a device pointer inside the workspace."""
        off = ptr - self.ws.data_ptr()
        return self.ws[off:off + 4 * n].view(torch.int32).cpu().numpy().copy()

    def read_f32(self, ptr, n):
        off = ptr - self.ws.data_ptr()
        return self.ws[off:off + 4 * n].view(torch.float32).cpu().numpy().copy()

    def status(self):
        return rm.moe_get_device_status(self.ws)

    def clear_status(self):
        rm.moe_clear_device_status(self.ws)


def oracle_forward(x_cpu, logits_cpu, weights, k, live, tokens=None, precision="bf16", wq=None):
    """Oracle routes for all live rows and outputs for `tokens` (default all)."""
    ids, probs = oracle.route(logits_cpu[:live].numpy(), k)
    toks = np.arange(live) if tokens is None else np.asarray(tokens)
    if precision == "bf16":
        out = oracle.forward_bf16(x_cpu[:live], ids, probs, *weights, tokens=toks)
    elif precision == "nvfp4":
        if wq is None:
            wq = oracle.quantize_weights_nvfp4(*weights)
        out = oracle.forward_nvfp4(x_cpu[:live], ids, probs, wq, tokens=toks)
    else:
        if wq is None:
            wq = oracle.quantize_weights_mxfp8(*weights)
        out = oracle.forward_mxfp8(x_cpu[:live], ids, probs, wq, tokens=toks)
    return ids, probs, out


def workload_problem(name):
    w = workloads.WORKLOADS[name]
    x, logits = workloads.make_activations(w)
    weights = workloads.make_weights(w)
    return w, x, logits, weights
