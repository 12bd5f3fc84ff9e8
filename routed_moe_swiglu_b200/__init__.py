"""routed_moe_swiglu_b200 -- B200 (sm_100a) routed-MoE SwiGLU expert forward.

A thin ctypes binding over the C ABI of ``libroutedmoe.so`` (declared in
``include/moe.h``).  Every function here only marshals arguments: torch
tensors become device pointers, the current torch CUDA stream becomes the
``stream`` argument.  All computation runs in the library's CUDA kernels;
there is no CPU path, and calling any entry point without the built library
raises.

Typical use::

    import routed_moe_swiglu_b200 as rm
    plan = rm.moe_plan_create(hidden=2048, ffn=1024, num_experts=128, top_k=8,
                              capacity=65536, precision="bf16")
    wbuf = rm.alloc_weight_buffer(plan)
    rm.moe_prepare_weights(plan, w_gate, w_up, w_down, wbuf)
    ws = rm.alloc_workspace(plan)
    rm.moe_forward(plan, x, wbuf, live_count, out, ws, logits=logits)
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "MoeError", "Plan", "load_library", "library_path", "moe_version", "moe_plan_create", "moe_plan_destroy",
    "moe_weight_buffer_bytes", "moe_workspace_bytes", "alloc_weight_buffer", "alloc_workspace",
    "moe_prepare_weights", "mxfp8_quantize_block32", "nvfp4_quantize_block16", "moe_route_topk", "moe_forward",
    "moe_forward_with_events",
    "moe_forward_noalloc", "MOE_NOALLOC_SCRATCH_BYTES", "moe_ep_dispatch", "moe_ep_combine",
    "MOE_NUM_STAGES", "STAGE_NAMES",
    "moe_get_workspace_views", "moe_get_device_status", "moe_clear_device_status",
    "MOE_DEV_LIVE_CLAMPED", "MOE_DEV_BAD_ROUTE", "MOE_DEV_TIMEOUT",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libroutedmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_DEV_LIVE_CLAMPED = 0x1
MOE_DEV_BAD_ROUTE = 0x2
MOE_DEV_TIMEOUT = 0x4
MOE_FLAG_PROBS_IN_FC1 = 0x1
MOE_FLAG_OUT_BF16 = 0x2
MOE_FLAG_SQUARED_RELU = 0x4
MOE_FLAG_KEEP_H_FP32 = 0x8
_PRECISION = {"bf16": 0, "mxfp8": 1, "nvfp4": 2}


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_status_string(code)} (status {code})")


class _EpViews(ctypes.Structure):
    _fields_ = [("status", ctypes.c_void_p), ("recv_live", ctypes.c_void_p), ("recv_x", ctypes.c_void_p),
                ("recv_ids", ctypes.c_void_p), ("recv_probs", ctypes.c_void_p), ("recv_y", ctypes.c_void_p),
                ("y_back", ctypes.c_void_p), ("recv_rows", ctypes.c_longlong)]


class _Desc(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("ffn", ctypes.c_int), ("num_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("capacity", ctypes.c_longlong), ("max_live_rows", ctypes.c_longlong),
                ("precision", ctypes.c_int), ("flags", ctypes.c_uint), ("gate_up_clamp", ctypes.c_float)]


class _Views(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("route_ids", "route_probs", "offsets", "perm", "inv", "pad_offsets",
                                                 "h", "h_scales", "xq", "xq_scales")] + [
        ("rows_padded", ctypes.c_longlong), ("status", ctypes.c_void_p), ("xq_row_scales", ctypes.c_void_p),
        ("h_row_scales", ctypes.c_void_p), ("h_fp32", ctypes.c_void_p)]


_lib = None


def load_library():
    """Load libroutedmoe.so (built by ``python -m routed_moe_swiglu_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(f"routed_moe_swiglu_b200: CUDA library not built ({library_path} missing); "
                           "run `python -m routed_moe_swiglu_b200.build`")
    lib = ctypes.CDLL(library_path)
    P, I, LL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
    sig = {
        "moe_plan_create": ([ctypes.POINTER(_Desc), ctypes.POINTER(P)], I),
        "moe_plan_destroy": ([P], None),
        "moe_plan_get_desc": ([P, ctypes.POINTER(_Desc)], I),
        "moe_weight_buffer_bytes": ([P], SZ),
        "moe_workspace_bytes": ([P], SZ),
        "moe_prepare_weights": ([P, P, P, P, P, SZ, P], I),
        "mxfp8_quantize_block32": ([P, LL, I, LL, P, P, P, P], I),
        "nvfp4_quantize_block16": ([P, LL, I, LL, P, P, P, P, P], I),
        "moe_route_topk": ([P, P, P, P, P, P], I),
        "moe_forward": ([P, P, P, P, P, P, P, P, P, SZ, P], I),
        "moe_forward_with_events": ([P, P, P, P, P, P, P, P, P, SZ, P, ctypes.POINTER(P)], I),
        "moe_forward_noalloc": ([P, P, P, P, P, P, P, P, P], I),
        "moe_ep_dispatch": ([P, I, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P], I),
        "moe_ep_combine": ([P, P, P, P, P, P, P], I),
        "moe_ep_region_bytes": ([P, I], SZ),
        "moe_ep_region_views_get": ([P, I, P, ctypes.POINTER(_EpViews)], I),
        "moe_ep_peer_dispatch": ([P, I, I, P, P, P, P, P, P, P, P, P, SZ, P], I),
        "moe_ep_peer_receive": ([P, I, P, ctypes.c_ulonglong, P], I),
        "moe_ep_peer_return": ([P, I, I, P, P], I),
        "moe_ep_peer_combine": ([P, I, P, P, P, P, P, ctypes.c_ulonglong, P], I),
        "moe_ep_ipc_handle": ([P, P], I),
        "moe_ep_ipc_open": ([P, ctypes.POINTER(P)], I),
        "moe_ep_ipc_close": ([P], I),
        "moe_get_workspace_views": ([P, P, ctypes.POINTER(_Views)], I),
        "moe_get_device_status": ([P, ctypes.POINTER(ctypes.c_uint), P], I),
        "moe_clear_device_status": ([P, P], I),
        "moe_check_bounded_wait": ([ctypes.c_ulonglong, P, P, P], I),
        "moe_status_string": ([I], ctypes.c_char_p),
        "moe_version": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _status_string(code: int) -> str:
    try:
        return load_library().moe_status_string(code).decode()
    except Exception:  # the library itself failed to load
        return "unknown"


def _check(code: int, what: str) -> None:
    if code != MOE_OK:
        raise MoeError(code, what)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("routed_moe_swiglu_b200 takes device tensors only")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def moe_version() -> str:
    return load_library().moe_version().decode()


class Plan:
    """Owns a host-side moe_plan handle (immutable once created)."""

    def __init__(self, handle, desc: _Desc):
        self._h = handle
        self.hidden = desc.hidden
        self.ffn = desc.ffn
        self.num_experts = desc.num_experts
        self.top_k = desc.top_k
        self.capacity = desc.capacity
        self.max_live_rows = desc.max_live_rows
        self.precision = {v: k for k, v in _PRECISION.items()}[desc.precision]
        self.probs_in_fc1 = bool(desc.flags & MOE_FLAG_PROBS_IN_FC1)
        self.out_dtype = "bf16" if desc.flags & MOE_FLAG_OUT_BF16 else "fp32"
        self.gate_up_clamp = float(desc.gate_up_clamp)
        self.squared_relu = bool(desc.flags & MOE_FLAG_SQUARED_RELU)
        self.keep_h_fp32 = bool(desc.flags & MOE_FLAG_KEEP_H_FP32)

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h is not None and _lib is not None:
            _lib.moe_plan_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_plan_create(hidden: int, ffn: int, num_experts: int, top_k: int, capacity: int,
                    precision: str = "bf16", max_live_rows: int = 0, out_dtype: str = "fp32",
                    probs_in_fc1: bool = False, gate_up_clamp: float | None = None,
                    squared_relu: bool = False, keep_h_fp32: bool = False) -> Plan:
    """out_dtype "fp32" or "bf16" (MOE_FLAG_OUT_BF16); probs_in_fc1 applies each
    route's probability to its SwiGLU row (MOE_FLAG_PROBS_IN_FC1); gate_up_clamp
    clamps the gate and up pre-activations (None: no clamp); squared_relu makes
    the experts relu(W1 x)^2 MLPs (MOE_FLAG_SQUARED_RELU; w_up unused);
    keep_h_fp32 (MXFP8) also stores the fp32 h the gate/up epilogue quantises,
    read through the h_fp32 workspace view (MOE_FLAG_KEEP_H_FP32)."""
    lib = load_library()
    if out_dtype not in ("fp32", "bf16"):
        raise ValueError(f"out_dtype must be 'fp32' or 'bf16', not {out_dtype!r}")
    flags = (MOE_FLAG_OUT_BF16 if out_dtype == "bf16" else 0) | (MOE_FLAG_PROBS_IN_FC1 if probs_in_fc1 else 0) | (
        MOE_FLAG_SQUARED_RELU if squared_relu else 0) | (MOE_FLAG_KEEP_H_FP32 if keep_h_fp32 else 0)
    d = _Desc(hidden, ffn, num_experts, top_k, capacity, max_live_rows, _PRECISION[precision], flags,
              float(gate_up_clamp) if gate_up_clamp else 0.0)
    h = ctypes.c_void_p()
    _check(lib.moe_plan_create(ctypes.byref(d), ctypes.byref(h)), "moe_plan_create")
    out = _Desc()
    _check(lib.moe_plan_get_desc(h, ctypes.byref(out)), "moe_plan_get_desc")
    return Plan(h, out)


def moe_plan_destroy(plan: Plan) -> None:
    plan.close()


def moe_weight_buffer_bytes(plan: Plan) -> int:
    return int(load_library().moe_weight_buffer_bytes(plan.handle))


def moe_workspace_bytes(plan: Plan) -> int:
    return int(load_library().moe_workspace_bytes(plan.handle))


def alloc_weight_buffer(plan: Plan, device=None):
    import torch

    return torch.empty(moe_weight_buffer_bytes(plan), dtype=torch.uint8, device=device or "cuda")


def alloc_workspace(plan: Plan, device=None):
    """A workspace for one stream, with its device status word cleared."""
    import torch

    ws = torch.empty(moe_workspace_bytes(plan), dtype=torch.uint8, device=device or "cuda")
    moe_clear_device_status(ws)
    return ws


def moe_prepare_weights(plan: Plan, w_gate, w_up, w_down, kernel_buf, stream=None) -> None:
    _check(load_library().moe_prepare_weights(plan.handle, _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(kernel_buf),
                                              kernel_buf.numel() * kernel_buf.element_size(), _stream(stream)),
           "moe_prepare_weights")


def mxfp8_quantize_block32(x, q, scales, live_rows=None, stream=None) -> None:
    rows, cols = x.shape
    _check(load_library().mxfp8_quantize_block32(_ptr(x), rows, cols, x.stride(0), _ptr(q), _ptr(scales),
                                                 _ptr(live_rows), _stream(stream)), "mxfp8_quantize_block32")


def nvfp4_quantize_block16(x, q, scales, row_scales, live_rows=None, stream=None) -> None:
    """x bf16 [rows, cols] (row stride in elements a multiple of 8) -> q uint8 [rows, cols/2],
    scales uint8 [rows, cols/16], row_scales fp32 [rows] (the per-token NVFP4 recipe)."""
    rows, cols = x.shape
    _check(load_library().nvfp4_quantize_block16(_ptr(x), rows, cols, x.stride(0), _ptr(q), _ptr(scales),
                                                 _ptr(row_scales), _ptr(live_rows), _stream(stream)),
           "nvfp4_quantize_block16")


def moe_route_topk(plan: Plan, logits, live_count, ids, probs, stream=None) -> None:
    _check(load_library().moe_route_topk(plan.handle, _ptr(logits), _ptr(live_count), _ptr(ids), _ptr(probs),
                                         _stream(stream)), "moe_route_topk")


def _check_out(plan: Plan, out) -> None:
    import torch

    want = torch.bfloat16 if plan.out_dtype == "bf16" else torch.float32
    if out.dtype != want:
        raise ValueError(f"out must be {want} for this plan, not {out.dtype}")


def moe_forward(plan: Plan, x, kernel_buf, live_count, out, workspace, logits=None, ids=None, probs=None,
                stream=None) -> None:
    _check_out(plan, out)
    _check(load_library().moe_forward(plan.handle, _ptr(x), _ptr(logits), _ptr(ids), _ptr(probs), _ptr(kernel_buf),
                                      _ptr(live_count), _ptr(out), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)), "moe_forward")


MOE_NOALLOC_SCRATCH_BYTES = 64 << 20


def moe_forward_noalloc(plan: Plan, x, kernel_buf, live_count, out, logits=None, ids=None, probs=None,
                        stream=None) -> None:
    """moe_forward without a workspace, for callers that cannot allocate device
    memory: the library's own fixed scratch array (MOE_NOALLOC_SCRATCH_BYTES)
    serves every call, so calls must not overlap on the GPU.  Make the first
    call on a device outside any stream capture."""
    _check_out(plan, out)
    _check(load_library().moe_forward_noalloc(plan.handle, _ptr(x), _ptr(logits), _ptr(ids), _ptr(probs),
                                              _ptr(kernel_buf), _ptr(live_count), _ptr(out), _stream(stream)),
           "moe_forward_noalloc")


def moe_ep_dispatch(plan: Plan, ep_size: int, x, live_count, send_x, send_ids, send_probs, send_counts, route_rows,
                    route_probs, workspace, logits=None, ids=None, probs=None, stream=None) -> None:
    """Expert-parallel send side (include/moe.h): route, order by expert, pack one
    send row per live route.  `ep.py` composes it into a whole step."""
    _check(load_library().moe_ep_dispatch(plan.handle, int(ep_size), _ptr(x), _ptr(logits), _ptr(ids), _ptr(probs),
                                          _ptr(live_count), _ptr(send_x), _ptr(send_ids), _ptr(send_probs),
                                          _ptr(send_counts), _ptr(route_rows), _ptr(route_probs), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_ep_dispatch")


def moe_ep_combine(plan: Plan, y_rows, route_rows, route_probs, live_count, out, stream=None) -> None:
    """Expert-parallel combine: out[t] = sum over j (ascending expert id) of
    route_probs[t, j] * y_rows[route_rows[t, j]] as fp32 FMAs from zero."""
    _check_out(plan, out)
    _check(load_library().moe_ep_combine(plan.handle, _ptr(y_rows), _ptr(route_rows), _ptr(route_probs),
                                         _ptr(live_count), _ptr(out), _stream(stream)), "moe_ep_combine")


# ---------------------------------------------------------------- peer-memory EP exchange

MOE_EP_IPC_HANDLE_BYTES = 64
EP_WAIT_LIMIT_NS = 4_000_000_000


def moe_ep_region_bytes(plan: Plan, ep_size: int) -> int:
    return int(load_library().moe_ep_region_bytes(plan.handle, int(ep_size)))


def moe_ep_region_views(plan: Plan, ep_size: int, region) -> dict:
    """Device tensors (views of `region`) of one rank's exchange state: status,
    recv_live, recv_x, recv_ids, recv_probs, recv_y, y_back."""
    import torch

    v = _EpViews()
    _check(load_library().moe_ep_region_views_get(plan.handle, int(ep_size), _ptr(region), ctypes.byref(v)),
           "moe_ep_region_views_get")
    base = region.data_ptr()
    rows, H = int(v.recv_rows), plan.hidden

    def view(ptr, n, dtype, shape):
        off = ptr - base
        return region[off:off + n * torch.empty((), dtype=dtype).element_size()].view(dtype).view(shape)

    return {"status": view(v.status, 1, torch.int32, (1,)), "recv_live": view(v.recv_live, 1, torch.int32, (1,)),
            "recv_x": view(v.recv_x, rows * H, torch.bfloat16, (rows, H)),
            "recv_ids": view(v.recv_ids, rows, torch.int32, (rows, 1)),
            "recv_probs": view(v.recv_probs, rows, torch.float32, (rows, 1)),
            "recv_y": view(v.recv_y, rows * H, torch.float32, (rows, H)),
            "y_back": view(v.y_back, plan.max_live_rows * plan.top_k * H, torch.float32,
                           (plan.max_live_rows * plan.top_k, H)),
            "recv_rows": rows}


def moe_ep_peer_dispatch(plan: Plan, ep_size: int, rank: int, x, live_count, regions, route_rows, route_probs,
                         workspace, logits=None, ids=None, probs=None, stream=None) -> None:
    """Step 1 of the peer-memory EP step (include/moe.h): `regions` is a device
    int64 tensor of the ep_size region addresses as this rank sees them."""
    _check(load_library().moe_ep_peer_dispatch(plan.handle, int(ep_size), int(rank), _ptr(x), _ptr(logits), _ptr(ids),
                                               _ptr(probs), _ptr(live_count), _ptr(regions), _ptr(route_rows),
                                               _ptr(route_probs), _ptr(workspace),
                                               workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_ep_peer_dispatch")


def moe_ep_peer_receive(plan: Plan, ep_size: int, region, wait_limit_ns: int = EP_WAIT_LIMIT_NS, stream=None):
    _check(load_library().moe_ep_peer_receive(plan.handle, int(ep_size), _ptr(region), int(wait_limit_ns),
                                              _stream(stream)), "moe_ep_peer_receive")


def moe_ep_peer_return(plan: Plan, ep_size: int, rank: int, regions, stream=None) -> None:
    _check(load_library().moe_ep_peer_return(plan.handle, int(ep_size), int(rank), _ptr(regions), _stream(stream)),
           "moe_ep_peer_return")


def moe_ep_peer_combine(plan: Plan, ep_size: int, region, route_rows, route_probs, live_count, out,
                        wait_limit_ns: int = EP_WAIT_LIMIT_NS, stream=None) -> None:
    _check_out(plan, out)
    _check(load_library().moe_ep_peer_combine(plan.handle, int(ep_size), _ptr(region), _ptr(route_rows),
                                              _ptr(route_probs), _ptr(live_count), _ptr(out), int(wait_limit_ns),
                                              _stream(stream)), "moe_ep_peer_combine")


def moe_ep_ipc_handle(region) -> bytes:
    buf = ctypes.create_string_buffer(MOE_EP_IPC_HANDLE_BYTES)
    _check(load_library().moe_ep_ipc_handle(_ptr(region), buf), "moe_ep_ipc_handle")
    return buf.raw


def moe_ep_ipc_open(handle: bytes) -> int:
    out = ctypes.c_void_p()
    _check(load_library().moe_ep_ipc_open(ctypes.create_string_buffer(bytes(handle), MOE_EP_IPC_HANDLE_BYTES),
                                          ctypes.byref(out)), "moe_ep_ipc_open")
    return int(out.value)


def moe_ep_ipc_close(addr: int) -> None:
    _check(load_library().moe_ep_ipc_close(ctypes.c_void_p(addr)), "moe_ep_ipc_close")


MOE_NUM_STAGES = 6
STAGE_NAMES = ("route", "permute", "gather", "gemm_gate_up", "gemm_down", "combine")


def moe_forward_with_events(plan: Plan, x, kernel_buf, live_count, out, workspace, events, logits=None, ids=None,
                            probs=None, stream=None) -> None:
    """moe_forward recording torch.cuda.Event objects `events` (MOE_NUM_STAGES + 1,
    enable_timing=True) around each stage."""
    _check_out(plan, out)
    if len(events) != MOE_NUM_STAGES + 1:
        raise ValueError("need MOE_NUM_STAGES + 1 events")
    if any(e.cuda_event == 0 for e in events):
        raise ValueError("events must exist on the device (record each once before use)")
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(load_library().moe_forward_with_events(plan.handle, _ptr(x), _ptr(logits), _ptr(ids), _ptr(probs),
                                                  _ptr(kernel_buf), _ptr(live_count), _ptr(out), _ptr(workspace),
                                                  workspace.numel() * workspace.element_size(), _stream(stream),
                                                  arr), "moe_forward_with_events")


def moe_get_workspace_views(plan: Plan, workspace) -> dict:
    v = _Views()
    _check(load_library().moe_get_workspace_views(plan.handle, _ptr(workspace), ctypes.byref(v)),
           "moe_get_workspace_views")
    d = {n: getattr(v, n) for n, _ in _Views._fields_}
    d["base"] = workspace.data_ptr()
    return d


def moe_get_device_status(workspace, stream=None) -> int:
    flags = ctypes.c_uint(0)
    _check(load_library().moe_get_device_status(_ptr(workspace), ctypes.byref(flags), _stream(stream)),
           "moe_get_device_status")
    return int(flags.value)


def moe_clear_device_status(workspace, stream=None) -> None:
    _check(load_library().moe_clear_device_status(_ptr(workspace), _stream(stream)), "moe_clear_device_status")


def moe_check_bounded_wait(limit_ns: int, status, elapsed_ns=None, stream=None) -> None:
    """Run the device's bounded-wait check (see include/moe.h): `status` is a
    device int32 tensor of one element the MOE_DEV_* bits are OR-ed into,
    `elapsed_ns` an optional device int64 tensor of two elements."""
    _check(load_library().moe_check_bounded_wait(int(limit_ns), _ptr(status),
                                                 _ptr(elapsed_ns) if elapsed_ns is not None else None,
                                                 _stream(stream)), "moe_check_bounded_wait")
