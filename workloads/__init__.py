"""Seeded synthetic inputs for the routed-MoE SwiGLU forward.

This module only draws random numbers: it holds none of the method's
arithmetic (no routing, no softmax, no GEMM), so both the CUDA path's tests
and the CPU oracle may take their inputs from it.  Every tensor is drawn on
the CPU from a ``torch.Generator`` seeded per workload, in a fixed order, so
the same seed gives the same bits on any machine.

Workloads (shapes and value distributions as the method's evaluation
describes them; weights are random-init, there are no trained checkpoints):

  tiny      T=64, H=256, F=512, E=8, top-2, seed 0.  Router logits N(0,1),
            each row redrawn until every pair of its logits differs by at
            least 1e-3 (so the top-2 is unambiguous).
  decode    H=2048, F=1024, E=128, top-8, a 65,536-row buffer with 256 live
            rows, seed 1.  Rows past the live count hold NaN in x and in the
            logits: they must never be read into a result.
  prefill   T=16,384 live rows (= buffer), H=2048, F=1024, E=128, top-8,
            seed 2.  Logits N(0,1) plus a per-expert bias -1.1*ln(rank), the
            ranks a seeded permutation of 1..E (a Zipf(s=1.1) popularity), so
            expert loads are heavily skewed.
  mxfp8     T=4,096, same shapes and routing distribution as prefill, seed 3,
            run in MXFP8.
  nvfp4     T=4,096, same shapes and routing distribution as prefill, seed 5,
            run in NVFP4 (the per-token recipe).
  decode_nvfp4  the decode workload's shapes and buffer, seed 6, in NVFP4.
  sweep     H=2688, F=1856, E=128, top-6, a 262,144-row buffer, seed 4; live
            counts {1, 64, 1024, 8192} are written on the device between
            replays of one captured graph.  Rows at or past the largest live
            count hold NaN.

Weights: w_gate, w_up [E, F, H] ~ N(0, 1/H); w_down [E, H, F] ~ N(0, 1/F)
(variance 1/fan_in), bf16.  Activations x ~ N(0, 1), bf16.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    hidden: int
    ffn: int
    num_experts: int
    top_k: int
    capacity: int  # rows in the preallocated buffer
    live: tuple  # live row counts this workload runs with
    seed: int
    precision: str  # "bf16", "mxfp8" or "nvfp4"
    zipf_bias: bool = False
    distinct_logits_gap: float = 0.0
    nan_past_live: bool = False

    @property
    def max_live(self) -> int:
        return max(self.live)

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "hidden": self.hidden,
            "ffn": self.ffn,
            "experts": self.num_experts,
            "top_k": self.top_k,
            "capacity": self.capacity,
            "live": list(self.live),
            "precision": self.precision,
            "seed": self.seed,
        }


WORKLOADS = {
    "tiny": Workload("tiny", 256, 512, 8, 2, 64, (64,), 0, "bf16", distinct_logits_gap=1e-3),
    "decode": Workload("decode", 2048, 1024, 128, 8, 65536, (256,), 1, "bf16", nan_past_live=True),
    "prefill": Workload("prefill", 2048, 1024, 128, 8, 16384, (16384,), 2, "bf16", zipf_bias=True),
    "mxfp8": Workload("mxfp8", 2048, 1024, 128, 8, 4096, (4096,), 3, "mxfp8", zipf_bias=True),
    "nvfp4": Workload("nvfp4", 2048, 1024, 128, 8, 4096, (4096,), 5, "nvfp4", zipf_bias=True),
    "decode_nvfp4": Workload("decode_nvfp4", 2048, 1024, 128, 8, 65536, (256,), 6, "nvfp4", nan_past_live=True),
    "sweep": Workload("sweep", 2688, 1856, 128, 6, 262144, (1, 64, 1024, 8192), 4, "bf16",
                      nan_past_live=True),
}


def _randn(gen: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    t = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def make_weights(w: Workload, gen: torch.Generator | None = None):
    """(w_gate [E,F,H], w_up [E,F,H], w_down [E,H,F]) bf16 on the CPU, drawn
    expert by expert so the float32 staging stays small."""
    if gen is None:
        gen = torch.Generator().manual_seed(w.seed * 1000 + 7)
    E, F, H = w.num_experts, w.ffn, w.hidden
    wg = torch.empty((E, F, H), dtype=torch.bfloat16)
    wu = torch.empty((E, F, H), dtype=torch.bfloat16)
    wd = torch.empty((E, H, F), dtype=torch.bfloat16)
    sg = 1.0 / math.sqrt(H)
    sd = 1.0 / math.sqrt(F)
    for e in range(E):
        wg[e] = _randn(gen, (F, H), sg).to(torch.bfloat16)
        wu[e] = _randn(gen, (F, H), sg).to(torch.bfloat16)
        wd[e] = _randn(gen, (H, F), sd).to(torch.bfloat16)
    return wg, wu, wd


def zipf_bias(w: Workload, gen: torch.Generator) -> torch.Tensor:
    """Per-expert bias -s*ln(rank), ranks a seeded permutation of 1..E, s=1.1."""
    ranks = torch.randperm(w.num_experts, generator=gen).to(torch.float64) + 1.0
    return (-1.1 * torch.log(ranks)).to(torch.float32)


def make_activations(w: Workload):
    """(x bf16 [cap, H], logits fp32 [cap, E]).  Rows below the largest live
    count are drawn; the rest are NaN when the workload says so (else drawn
    too, which only happens when the buffer equals the live count)."""
    gen = torch.Generator().manual_seed(w.seed)
    n = w.max_live
    E, H, cap = w.num_experts, w.hidden, w.capacity
    logits = torch.full((cap, E), float("nan"), dtype=torch.float32)
    live_logits = _randn(gen, (n, E))
    if w.distinct_logits_gap > 0.0:
        for r in range(n):
            row = live_logits[r]
            while True:
                s = torch.sort(row).values
                if float((s[1:] - s[:-1]).min()) >= w.distinct_logits_gap:
                    break
                row = _randn(gen, (E,))
            live_logits[r] = row
    if w.zipf_bias:
        live_logits += zipf_bias(w, gen)
    logits[:n] = live_logits
    x = torch.full((cap, H), float("nan"), dtype=torch.bfloat16)
    x[:n] = _randn(gen, (n, H)).to(torch.bfloat16)
    if not w.nan_past_live and n < cap:
        raise ValueError("workload without NaN padding must have capacity == live")
    return x, logits


def sample_tokens(n_live: int, count: int, seed: int) -> torch.Tensor:
    """A seeded sorted subset of token indices in [0, n_live) (all when count >= n_live)."""
    if count >= n_live:
        return torch.arange(n_live, dtype=torch.int64)
    gen = torch.Generator().manual_seed(seed + 12345)
    return torch.sort(torch.randperm(n_live, generator=gen)[:count]).values


def small_case(hidden: int, ffn: int, experts: int, top_k: int, tokens: int, seed: int,
               capacity: int | None = None, zipf: bool = False):
    """Arbitrary small shapes for parity edge cases: returns
    (x [cap,H] bf16, logits [cap,E] fp32, (wg, wu, wd)).  Rows past `tokens`
    are NaN when capacity > tokens."""
    cap = tokens if capacity is None else capacity
    w = Workload("small", hidden, ffn, experts, top_k, cap, (tokens,), seed, "bf16", zipf_bias=zipf,
                 nan_past_live=cap > tokens)
    x, logits = make_activations(w) if tokens > 0 else (
        torch.full((cap, hidden), float("nan"), dtype=torch.bfloat16),
        torch.full((cap, experts), float("nan"), dtype=torch.float32))
    return x, logits, make_weights(w)
