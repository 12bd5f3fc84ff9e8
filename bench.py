#!/usr/bin/env python
"""Benchmark of the routed-MoE SwiGLU forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole path (route, permute, gather, gate/up GEMM
+ SwiGLU, down GEMM, combine; NVFP4 also quantises h between the GEMMs, timed
with the gate/up stage) over one batch of seeded synthetic inputs that
are already resident in HBM.  The K timed steps are K replays of a captured
one-forward CUDA graph (the granularity of the end-to-end loop), bracketed
by a barrier and a device synchronise; the time is the max over ranks.  The
stage split comes from a second graph with events between the stages.  Every
step re-reads all expert weights (1.6-3.8 GB), more than the 126 MB L2, so
no L2 flush is needed between steps.

The default run (decode headline, one GPU) also measures the other
configurations in the same process and reports each under `configs`: the
16,384-token bf16 prefill (tensor-bound), the 4,096-token MXFP8 prefill and
the live-count sweep (with its bitwise invariance across counts and
replays).

Metric: routed tokens/s = live tokens processed per second (whole job).
Extra keys: `roofline` for the dominant kernel (algorithmic bytes or FLOPs
per launch / its CUDA-event duration, against MEASURED_PEAKS.json), `e2e`
(same metric through the C ABI with pinned host buffers, copies inside the
timed region), `cpu_baseline` (the CPU oracle on a bounded sample, rank 0,
N=1), `clocks` (NVML samples during the timed region), `gpu_launches`.

With --gpus N > 1 (launched by torch.distributed.run) every rank runs an
independent replica of the workload on its own GPU (tokens are independent,
so the path shards by token with no data-path collective): weak scaling.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

def kernels_per_forward(precision: str, max_live: int) -> int:
    """Library kernels one forward launches: route, permute, the x gather (MXFP8, NVFP4:
    bf16 copies the rows inside its gate/up GEMM), gate/up GEMM, NVFP4's h quantisation,
    down GEMM, combine."""
    return 1 + 1 + (precision != "bf16") + 1 + (precision == "nvfp4") + 1 + 1
STAGES = ("route", "permute", "gather", "gemm_gate_up", "gemm_down", "combine")
# measured after the headline (decode) in the default run: the tensor-bound prefill,
# the MXFP8 prefill and the live-count sweep
EXTRA_CONFIGS = ("prefill", "mxfp8", "sweep")
DEFAULT_STEPS = {"tiny": 200, "decode": 200, "prefill": 30, "mxfp8": 50, "nvfp4": 50, "decode_nvfp4": 200,
                 "sweep": 20}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None,
                    help="untimed warm-up steps (default: as many as the timed steps, at least 3)")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=tuple(workloads.WORKLOADS), default="decode")
    ap.add_argument("--live", type=int, default=None, help="live rows (default: the workload's largest)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other configurations' records (prefill, mxfp8, sweep) after the decode line")
    ap.add_argument("--probs-in-fc1", action="store_true",
                    help="variant: router probabilities applied to the SwiGLU row (apply_topk_in_fc1)")
    ap.add_argument("--gate-up-clamp", type=float, default=None, help="variant: clamp of the gate/up pre-activations")
    ap.add_argument("--out-bf16", action="store_true", help="variant: bf16 finalize output")
    ap.add_argument("--squared-relu", action="store_true", help="variant: squared-ReLU experts (bf16 only)")
    ap.add_argument("--capacity", type=int, default=None,
                    help="override the buffer rows (profiling captures only; not a benchmark configuration)")
    a = ap.parse_args()
    if a.steps is None:
        a.steps = DEFAULT_STEPS[a.workload]
    if a.warmup is None:
        a.warmup = a.steps
    if a.warmup < 3:
        a.warmup = 3
    return a


# ---------------------------------------------------------------- distributed plumbing


class Dist:
    """One process per GPU (RANK / LOCAL_RANK / WORLD_SIZE from the launcher).
    The path shards by token with replicated weights, so the only collectives
    are the barrier around the timed region and the max over ranks of its
    time.  backend: "nccl" on GPUs; "gloo" runs the same steps on CPU (tests)."""

    def __init__(self, n_gpus, backend: str | None = None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        self.pg = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            if self.backend == "nccl":
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                        device_id=torch.device("cuda", self.local))
            else:
                dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=60))
            self.pg = dist
        elif torch.cuda.is_available():
            torch.cuda.set_device(0)

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if self.pg is None:
            return v
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """Polls NVML (SM clock, max clock, clock-event reasons) on a thread."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:  # map the CUDA device to NVML by PCI bus id (CUDA_VISIBLE_DEVICES may renumber)
                pr = torch.cuda.get_device_properties(device_index)
                bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:  # no NVML: report that, keep going
            self.err = str(exc)
        self._stop = threading.Event()
        self._t = None
        self.window = (0.0, 0.0)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(0.001)  # several samples even in a timed region of a few ms

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
            time.sleep(0.01)

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        t0, t1 = self.window
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside and self.samples:  # very short region: nearest samples
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:2]
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= int(s[2])
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if bits & b], "samples": len(inside)}


# ---------------------------------------------------------------- peaks / traffic


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


_CSRC = "routed_moe_swiglu_b200/csrc/"
KERNEL_SOURCES = {
    ("gemm_gate_up", "bf16"): [_CSRC + "gemm_bf16_pair.cu", _CSRC + "ptx.cuh", _CSRC + "moe_internal.cuh"],
    ("gemm_down", "bf16"): [_CSRC + "gemm_bf16_pair.cu", _CSRC + "ptx.cuh", _CSRC + "moe_internal.cuh"],
    ("gemm_gate_up", "mxfp8"): [_CSRC + "gemm_mxfp8.cu", _CSRC + "mxfp8.cuh", _CSRC + "ptx.cuh",
                                _CSRC + "moe_internal.cuh"],
    ("gemm_down", "mxfp8"): [_CSRC + "gemm_mxfp8.cu", _CSRC + "mxfp8.cuh", _CSRC + "ptx.cuh",
                             _CSRC + "moe_internal.cuh"],
    ("combine", "bf16"): [_CSRC + "permute.cu", _CSRC + "moe_internal.cuh"],
    ("combine", "mxfp8"): [_CSRC + "permute.cu", _CSRC + "moe_internal.cuh"],
    ("gemm_gate_up", "nvfp4"): [_CSRC + "gemm_mxfp8.cu", _CSRC + "mxfp8.cuh", _CSRC + "nvfp4.cuh", _CSRC + "nvfp4.cu",
                                _CSRC + "ptx.cuh", _CSRC + "moe_internal.cuh"],
    ("gemm_down", "nvfp4"): [_CSRC + "gemm_mxfp8.cu", _CSRC + "mxfp8.cuh", _CSRC + "nvfp4.cuh", _CSRC + "ptx.cuh",
                             _CSRC + "moe_internal.cuh"],
    ("combine", "nvfp4"): [_CSRC + "permute.cu", _CSRC + "moe_internal.cuh"],
}


def source_hash(stage, precision):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES.get((stage, precision), []):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(stage, workload, precision):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's
    sources are unchanged since it was taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(f"{stage}@{workload}")
    if not rec or rec.get("source_sha") != source_hash(stage, precision):
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- the CUDA arm


def _workload(a, name):
    w = workloads.WORKLOADS[name]
    if a.capacity is not None and name == a.workload:
        import dataclasses

        w = dataclasses.replace(w, capacity=a.capacity, live=tuple(min(v, a.capacity) for v in w.live),
                                nan_past_live=True)
    return w


def measure(a, dist: Dist, w, live, K, W, want_e2e=False, want_sweep=False):
    """One workload on this rank's GPU: K timed forwards (replays of a one-step
    CUDA graph, the granularity of the end-to-end loop too), their stage split
    from a second graph with events between the stages, the live-count sweep
    (when the workload has several live counts) and the end-to-end loop."""
    import routed_moe_swiglu_b200 as rm

    x, logits = workloads.make_activations(w)
    wg, wu, wd = workloads.make_weights(w)
    dev = torch.device("cuda", torch.cuda.current_device())
    plan = rm.moe_plan_create(hidden=w.hidden, ffn=w.ffn, num_experts=w.num_experts, top_k=w.top_k,
                              capacity=w.capacity, precision=w.precision, probs_in_fc1=a.probs_in_fc1,
                              gate_up_clamp=a.gate_up_clamp, out_dtype="bf16" if a.out_bf16 else "fp32",
                              squared_relu=a.squared_relu)
    wbuf = rm.alloc_weight_buffer(plan, dev)
    wgd, wud, wdd = wg.to(dev), wu.to(dev), wd.to(dev)
    rm.moe_prepare_weights(plan, wgd, wud, wdd, wbuf)
    # the kernel-layout rebuild a refit runs (moe_prepare_weights), timed warm
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record()
    for _ in range(3):
        rm.moe_prepare_weights(plan, wgd, wud, wdd, wbuf)
    p1.record()
    torch.cuda.synchronize()
    prepare_ms = p0.elapsed_time(p1) / 3
    del wgd, wud, wdd
    ws = rm.alloc_workspace(plan, dev)
    xd, ld = x.to(dev), logits.to(dev)
    out_dt = torch.bfloat16 if a.out_bf16 else torch.float32
    out = torch.zeros((w.capacity, w.hidden), dtype=out_dt, device=dev)
    live_d = torch.tensor([live], dtype=torch.int32, device=dev)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        rm.moe_forward(plan, xd, wbuf, live_d, out, ws, logits=ld)  # first call outside capture
    stream.synchronize()
    g1 = torch.cuda.CUDAGraph()  # one forward: the timed step, the warm-up, the sweep and e2e
    with torch.cuda.graph(g1, stream=stream):
        rm.moe_forward(plan, xd, wbuf, live_d, out, ws, logits=ld)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)] for _ in range(K)]
    with torch.cuda.stream(stream):  # torch creates the CUDA event on its first record
        for ev in events:
            for e in ev:
                e.record(stream)
    stream.synchronize()
    # the stage split: K forwards with an event between every two stages (which
    # serialises the kernels fully), replayed after the timed region
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge, stream=stream):
        for i in range(K):
            rm.moe_forward_with_events(plan, xd, wbuf, live_d, out, ws, events[i], logits=ld)

    with torch.cuda.stream(stream):
        for _ in range(W):
            g1.replay()
    stream.synchronize()

    clocks = ClockSampler(dev.index)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for _ in range(K):
            g1.replay()
        t_end.record(stream)
    torch.cuda.synchronize()
    h1 = time.perf_counter()
    dist.barrier()
    clocks.window = (h0, h1)
    clocks.stop()
    ms_total = dist.max(t_start.elapsed_time(t_end))
    ms_step = ms_total / K
    with torch.cuda.stream(stream):
        ge.replay()
    stream.synchronize()

    stage_ms = {s: [] for s in STAGES}
    for ev in events:
        for j, s in enumerate(STAGES):
            stage_ms[s].append(ev[j].elapsed_time(ev[j + 1]))
    stage_avg = {s: sum(v) / len(v) for s, v in stage_ms.items()}
    ms_step_events = events[0][0].elapsed_time(events[-1][-1]) / K  # the instrumented graph, same K forwards
    status = rm.moe_get_device_status(ws)

    # routing statistics of this batch, read from the library's own workspace
    views = rm.moe_get_workspace_views(plan, ws)
    off = views["offsets"] - views["base"]
    offsets = ws[off:off + 4 * (w.num_experts + 1)].view(torch.int32).cpu()
    counts = (offsets[1:] - offsets[:-1]).tolist()

    res = {
        "ms_per_step": ms_step,
        "value": dist.world * live / (ms_step / 1e3),
        "stage_ms": stage_avg,
        "prepare_ms": prepare_ms,
        "fc1_projections": 1 if a.squared_relu else 2,
        "ms_per_step_with_stage_events": ms_step_events,
        "clocks": clocks.summary(),
        "timed_s": ms_total / 1e3,
        "touched": sum(1 for c in counts if c > 0),
        "routes": int(offsets[-1]),
        "status": status,
        "max_rows_per_expert": max(counts),
        "live": live,
    }

    # ---------------- live-count sweep: the same one-step graph, device live counts;
    # each token's output must be bitwise the same at every count and in every replay
    if want_sweep and len(w.live) > 1:
        sweep, kept = [], {}
        reps = max(3, min(20, K))
        invariant = True
        for n in w.live:
            live_d.fill_(n)
            with torch.cuda.stream(stream):
                g1.replay()
            stream.synchronize()
            first = out[:n].clone()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g1.replay()
                e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            same_replays = bool(torch.equal(first.view(torch.int32), out[:n].view(torch.int32)))
            kept[n] = first
            o_n = ws[off:off + 4 * (w.num_experts + 1)].view(torch.int32).cpu()
            c_n = o_n[1:] - o_n[:-1]
            sweep.append({"live": n, "ms_per_step": ms, "tokens_per_s": n / (ms / 1e3),
                          "routes": int(o_n[-1]), "touched": int((c_n > 0).sum()),
                          "bitwise_equal_across_replays": same_replays})
            invariant = invariant and same_replays
        ns = sorted(kept)
        for lo, hi in zip(ns, ns[1:]):
            invariant = invariant and bool(torch.equal(kept[hi][:lo].view(torch.int32), kept[lo].view(torch.int32)))
        del kept
        live_d.fill_(live)
        torch.cuda.synchronize()
        res["sweep"] = sweep
        res["sweep_bitwise_invariant"] = invariant

    # ---------------- end to end through the C ABI with pinned host buffers
    # Every step copies its inputs (x, logits, live count) in from pinned host
    # memory and its output back.  Two device buffer sets, each with its own
    # one-step graph, let step i+1's input copy and step i's output copy run on
    # the copy engines while a forward runs: inputs on s_in, outputs on s_out,
    # forwards in order on `stream`; events keep each set's reuse ordered (a
    # set's inputs are rewritten once its last forward is done, its output
    # once it has been read back).
    if want_e2e:
        x_pin = x[:live].contiguous().pin_memory()
        l_pin = logits[:live].contiguous().pin_memory()
        n_pin = torch.tensor([live], dtype=torch.int32).pin_memory()
        o_pins = [torch.empty((live, w.hidden), dtype=out_dt).pin_memory() for _ in range(2)]
        xd2, ld2, out2, live_d2 = xd.clone(), ld.clone(), torch.zeros_like(out), live_d.clone()
        g1b = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1b, stream=stream):
            rm.moe_forward(plan, xd2, wbuf, live_d2, out2, ws, logits=ld2)
        sets = [(xd, ld, live_d, out, g1), (xd2, ld2, live_d2, out2, g1b)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in, ev_fwd, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
        with torch.cuda.stream(stream):
            for e in ev_in + ev_fwd + ev_out:
                e.record(stream)
        stream.synchronize()

        def e2e_step(i):
            b = i & 1
            xb, lb, nb, ob, gb = sets[b]
            s_in.wait_event(ev_fwd[b])
            with torch.cuda.stream(s_in):
                xb[:live].copy_(x_pin, non_blocking=True)
                lb[:live].copy_(l_pin, non_blocking=True)
                nb.copy_(n_pin, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])
            with torch.cuda.stream(stream):
                gb.replay()
                ev_fwd[b].record(stream)
            s_out.wait_event(ev_fwd[b])
            with torch.cuda.stream(s_out):
                o_pins[b].copy_(ob[:live], non_blocking=True)
                ev_out[b].record(s_out)

        def e2e_run(steps, e_start=None, e_stop=None):
            if e_start is not None:
                e_start.record(stream)
            s_in.wait_stream(stream)
            for i in range(steps):
                e2e_step(i)
            stream.wait_event(ev_out[0])
            stream.wait_event(ev_out[1])
            if e_stop is not None:
                e_stop.record(stream)

        e2e_run(W)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        e2e_run(K, e0, e1)
        torch.cuda.synchronize()
        dist.barrier()
        e_ms = dist.max(e0.elapsed_time(e1)) / K
        assert torch.equal(o_pins[(K - 1) & 1], out[:live].cpu() if (K - 1) & 1 == 0 else out2[:live].cpu())
        res["e2e"] = {"value": dist.world * live / (e_ms / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": x_pin.numel() * 2 + l_pin.numel() * 4 + 4,
                      "d2h_bytes_per_step": o_pins[0].numel() * o_pins[0].element_size(), "ms_per_step": e_ms,
                      "copies": "overlapped with the neighbouring steps' forwards (two buffer sets)"}
        del g1b
    del ge, g1
    return res


def run_ours(a, dist: Dist):
    w = _workload(a, a.workload)
    live = min(a.live or w.max_live, w.capacity)
    res = measure(a, dist, w, live, a.steps, a.warmup, want_e2e=not a.no_e2e, want_sweep=a.live is None)
    return w, live, res


def _bpe(precision):
    """Bytes per operand element with its block scales: E4M3 + an E8M0 per 32,
    E2M1 + an E4M3 per 16, bf16."""
    return {"mxfp8": 1 + 1 / 32, "nvfp4": 0.5 + 1 / 16}.get(precision, 2)


def _tc_ratio(precision):
    return {"mxfp8": 2.0, "nvfp4": 4.0}.get(precision, 1.0)  # nominal dense peak over bf16


def roofline(w, res, peaks):
    """Roofline of the dominant kernel (largest share of the step).  The
    algorithmic work counts only what the method must do (routes * 6 * H * F
    FLOPs; the touched experts' weights once, x in once per token, out once
    per token) and not the padded work or the h / y round trips."""
    st = res["stage_ms"]
    dom = max(st, key=lambda s: st[s])
    ms = st[dom]
    H, F, E = w.hidden, w.ffn, w.num_experts
    R, n = res["routes"], res["live"]
    bpe = _bpe(w.precision)
    tc_ratio = _tc_ratio(w.precision)
    sustained = res["timed_s"] > 1.0
    tflops_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    out = {"kernel": dom}
    if dom in ("gemm_gate_up", "gemm_down"):
        if dom == "gemm_gate_up":
            nproj = res.get("fc1_projections", 2)  # gate and up, or the one squared-ReLU projection
            flops = 2.0 * nproj * R * H * F
            bytes_ = res["touched"] * nproj * F * H * bpe + n * H * bpe  # weights + x, once
        else:
            flops = 2.0 * R * H * F
            bytes_ = res["touched"] * H * F * bpe  # weights, once
        t_hbm = bytes_ / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (tflops_peak * 1e12 * tc_ratio)
        if t_hbm >= t_tc:
            ach = bytes_ / (ms / 1e3) / 1e9
            out.update(bound="hbm", achieved=ach, peak=peaks["hbm_gbs"], unit="GB/s",
                       algorithmic_per_launch=bytes_)
        else:
            ach = flops / (ms / 1e3) / 1e12
            pk = tflops_peak * tc_ratio
            out.update(bound="tensor", achieved=ach, peak=pk, unit="TFLOP/s", algorithmic_per_launch=flops,
                       peak_kind=("sustained" if sustained else "burst")
                       + {"mxfp8": " bf16 x2 (fp8 nominal ratio)", "nvfp4": " bf16 x4 (fp4 nominal ratio)"}.get(
                           w.precision, " bf16"))
    else:
        # memory-bound helper kernels: bytes they must move
        if dom == "combine":
            bytes_ = R * H * 4 + n * H * 4 + R * 8
        elif dom == "gather":
            bytes_ = n * H * 2 + R * H * bpe
        else:
            bytes_ = n * E * 4
        out.update(bound="hbm", achieved=bytes_ / (ms / 1e3) / 1e9, peak=peaks["hbm_gbs"], unit="GB/s",
                   algorithmic_per_launch=bytes_)
    out["frac"] = out["achieved"] / out["peak"]
    out["peak_source"] = peaks["source"]
    out["kernel_ms"] = ms
    out["traffic"] = recorded_traffic(dom, w.name, w.precision)
    return out


def step_roofline(w, res, peaks, point=None):
    """The whole step against the roofline of the method's algorithmic work:
    bytes = the touched experts' weights once + x, logits in and out out per
    live token; FLOPs = routes * 6 * H * F (squared-ReLU: 4).  frac = the
    roofline time (the larger of bytes / HBM and FLOPs / tensor peak) over
    the measured step time.  `point`: a sweep entry (live, routes, touched,
    ms_per_step) instead of the timed step."""
    H, F, E = w.hidden, w.ffn, w.num_experts
    src = res if point is None else point
    n, R, touched, ms = src["live"], src["routes"], src["touched"], src["ms_per_step"]
    nproj = res.get("fc1_projections", 2)
    bpe = _bpe(w.precision)
    bytes_ = touched * (nproj + 1) * H * F * bpe + n * (H * 2 + E * 4 + H * 4)
    flops = 2.0 * (nproj + 1) * R * H * F
    out = {}
    for kind, tf in (("burst", peaks["bf16_tflops"]), ("sustained", peaks["bf16_tflops_sustained"])):
        t_b = bytes_ / (peaks["hbm_gbs"] * 1e9)
        t_f = flops / (tf * 1e12 * _tc_ratio(w.precision))
        t = max(t_b, t_f)
        out[f"frac_{kind}"] = t / (ms / 1e3)
        if kind == "burst":
            out.update(bound="hbm" if t_b >= t_f else "tensor", bytes=bytes_, flops=flops,
                       roofline_ms=t * 1e3, hbm_frac=t_b / (ms / 1e3), tensor_frac=t_f / (ms / 1e3))
    out["peak_source"] = peaks["source"]
    return out


def sub_record(a, dist, name, peaks):
    """A spec configuration measured in the same process as the headline."""
    w = _workload(a, name)
    K = DEFAULT_STEPS[name]
    res = measure(a, dist, w, w.max_live, K, K, want_e2e=False, want_sweep=True)
    rec = {"workload": workload_config(w, w.max_live, a)["workload"], "steps": K, "warmup": K,
           "ms_per_step": res["ms_per_step"], "tokens_per_s": res["value"],
           "stage_ms": {k: round(v, 5) for k, v in res["stage_ms"].items()},
           "roofline": roofline(w, res, peaks), "step_roofline": step_roofline(w, res, peaks),
           "clocks": res["clocks"], "device_status": res["status"],
           "gpu_launches": kernels_per_forward(w.precision, w.capacity) * K}
    if "sweep" in res:
        for e in res["sweep"]:
            e["step_roofline_frac"] = step_roofline(w, res, peaks, point=e)["frac_burst"]
        rec["sweep"] = res["sweep"]
        rec["bitwise_invariant"] = res["sweep_bitwise_invariant"]
    del res
    torch.cuda.empty_cache()
    return rec


# ---------------------------------------------------------------- the oracle (CPU) arm


def oracle_variant(a):
    """The oracle's options for the variant the CUDA arm runs (the bf16
    output rounding costs nothing next to the expert forward)."""
    v = {"probs_in_fc1": bool(a.probs_in_fc1), "gate_up_clamp": a.gate_up_clamp}
    if a.squared_relu:
        v["squared_relu"] = True
    return v


def oracle_weights(w, weights, variant):
    """The oracle's quantised weights for a block-scaled workload (None for bf16)."""
    import oracle

    if w.precision == "mxfp8":
        return oracle.quantize_weights_mxfp8(*weights)
    if w.precision == "nvfp4":
        relu2 = bool((variant or {}).get("squared_relu"))
        return oracle.quantize_weights_nvfp4(weights[0], None if relu2 else weights[1], weights[2])
    return None


def oracle_forward_tokens(w, x, ids, probs, weights, wq, sel, variant):
    import oracle

    if w.precision == "mxfp8":
        return oracle.forward_mxfp8(x, ids, probs, wq, tokens=sel, **(variant or {}))
    if w.precision == "nvfp4":
        return oracle.forward_nvfp4(x, ids, probs, wq, tokens=sel, **(variant or {}))
    return oracle.forward_bf16(x, ids, probs, *weights, tokens=sel, **(variant or {}))


def oracle_tokens_per_s(w, x, logits, weights, live, budget_s, min_tokens=8, variant=None):
    """Time the oracle (as it stands) on the host cores over a bounded sample
    of the live tokens: route all live rows, then the expert forward of a
    growing prefix of a seeded token sample until ~budget_s of work."""
    import numpy as np

    import oracle

    wq = oracle_weights(w, weights, variant)
    toks = workloads.sample_tokens(live, live, w.seed).numpy()
    t0 = time.perf_counter()
    ids, probs = oracle.route(logits[:live].numpy(), w.top_k)
    route_s = time.perf_counter() - t0
    done, spent, n = 0, 0.0, min_tokens
    while spent < budget_s:
        sel = toks[(done + np.arange(n)) % live]
        t0 = time.perf_counter()
        oracle_forward_tokens(w, x[:live], ids, probs, weights, wq, sel, variant)
        dt = time.perf_counter() - t0
        spent += dt
        done += n
        per_tok = dt / n
        n = max(1, min(4 * n, int((budget_s - spent) / max(per_tok, 1e-9)) + 1))
    per_token = spent / done + route_s / live
    return 1.0 / per_token, done, oracle.threads()


def run_reference(a, dist: Dist):
    """The oracle as the reference arm: K timed steps, each the oracle's
    forward over a bounded token sample of the same workload."""
    w = workloads.WORKLOADS[a.workload]
    live = a.live or w.max_live
    if dist.rank != 0:
        return None
    import numpy as np

    import oracle

    x, logits = workloads.make_activations(w)
    weights = workloads.make_weights(w)
    variant = oracle_variant(a)
    wq = oracle_weights(w, weights, variant)
    ids, probs = oracle.route(logits[:live].numpy(), w.top_k)
    toks = workloads.sample_tokens(live, live, w.seed).numpy()

    def step(n, start):
        sel = toks[(start + np.arange(n)) % live]
        oracle_forward_tokens(w, x[:live], ids, probs, weights, wq, sel, variant)

    t0 = time.perf_counter()
    step(4, 0)
    per_tok = (time.perf_counter() - t0) / 4
    budget = 150.0  # whole run
    n = max(1, int(budget / (a.steps + a.warmup) / max(per_tok, 1e-9)))
    n = min(n, live)
    for i in range(a.warmup):
        step(n, i * n)
    t0 = time.perf_counter()
    for i in range(a.steps):
        step(n, (a.warmup + i) * n)
    el = time.perf_counter() - t0
    value = n * a.steps / el
    return w, live, {"value": value, "ms_per_step": el / a.steps * 1e3, "sample": n}


# ---------------------------------------------------------------- main


def workload_config(w, live, a=None):
    variant = []
    if a is not None and a.probs_in_fc1:
        variant.append("probs applied in FC1")
    if a is not None and a.gate_up_clamp:
        variant.append(f"gate/up clamp {a.gate_up_clamp:g}")
    if a is not None and a.out_bf16:
        variant.append("bf16 output")
    if a is not None and a.squared_relu:
        variant.append("squared-ReLU experts")
    return {
        "variant": ", ".join(variant) if variant else "plain (fp32 output, probabilities in the combine)",
        "workload": f"{w.name}: {w.precision} H={w.hidden} F={w.ffn} E={w.num_experts} top-{w.top_k}, "
                    f"{live} live rows of a {w.capacity}-row buffer",
        "hidden": w.hidden, "ffn": w.ffn, "experts": w.num_experts, "top_k": w.top_k,
        "capacity": w.capacity, "live_rows": live, "seed": w.seed,
        "l2": "no flush: every step re-reads all expert weights (> 126 MB L2)",
        "graph": "one CUDA graph of K forwards; live count read on the device",
    }


def main():
    a = parse_args()
    dist = Dist(a.gpus)
    if a.impl == "reference":
        r = run_reference(a, dist)
        if dist.rank == 0 and r is not None:
            w, live, res = r
            import oracle

            line = {
                "impl": "reference", "metric": "routed tokens/s", "value": res["value"], "unit": "tokens/s",
                "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup, "ms_per_step": res["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": w.precision, "data": "synthetic",
                "config": workload_config(w, live, a),
                "cpu_baseline": {"value": res["value"], "unit": "tokens/s", "cores": oracle.threads(),
                                 "kind": "oracle",
                                 "sample": f"{res['sample']} tokens per step of the {w.name} workload"},
                "e2e": {"value": res["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
            }
            print(json.dumps(line), flush=True)
        dist.close()
        return

    w, live, res = run_ours(a, dist)
    peaks = measured_peaks()
    line = {
        "metric": "routed tokens/s", "value": res["value"], "unit": "tokens/s", "n_gpus": dist.world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.precision, "data": "synthetic",
        "config": workload_config(w, live, a),
        "roofline": roofline(w, res, peaks),
        "step_roofline": step_roofline(w, res, peaks),
        "stage_ms": {k: round(v, 5) for k, v in res["stage_ms"].items()},
        "ms_per_step_with_stage_events": round(res["ms_per_step_with_stage_events"], 5),
        "prepare_weights_ms": round(res["prepare_ms"], 4),
        "clocks": res["clocks"],
        "gpu_launches": kernels_per_forward(w.precision, w.capacity) * a.steps,
        "device_status": res["status"],
        "routing": {"routes": res["routes"], "experts_touched": res["touched"],
                    "max_rows_per_expert": res["max_rows_per_expert"]},
    }
    if "e2e" in res:
        line["e2e"] = res["e2e"]
    if "sweep" in res:
        line["sweep"] = res["sweep"]
        line["sweep_bitwise_invariant"] = res["sweep_bitwise_invariant"]
    if dist.world == 1 and not a.no_extra and a.workload == "decode" and a.live is None and a.capacity is None:
        # the other spec configurations, each timed alone in this process
        line["configs"] = {name: sub_record(a, dist, name, peaks) for name in EXTRA_CONFIGS}
    if dist.rank == 0 and dist.world == 1 and not a.no_cpu_baseline:
        x, logits = workloads.make_activations(w)
        weights = workloads.make_weights(w)
        v, n, cores = oracle_tokens_per_s(w, x, logits, weights, live, a.cpu_seconds, variant=oracle_variant(a))
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"{n} tokens of the {w.name} workload (route of all {live} live rows "
                                          f"+ expert forward of the sample), ~{a.cpu_seconds:.0f} s"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
