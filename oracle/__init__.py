"""CPU oracle for the routed-MoE SwiGLU expert forward (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``moe_oracle.c`` (plain C,
fp64 sums, one token at a time) through ctypes and numpy; it shares no code
with the CUDA library and never imports it.  Each function cites the page
and section it follows in ``moe_oracle.c``.

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against closed forms, library special cases or brute force (see the header
of that file for which pin covers which mistake).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into oracle/libmoe_oracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-shared", "-fPIC", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I = ctypes.c_int
    lib.oracle_threads.restype = I
    lib.oracle_e4m3_value.restype = ctypes.c_double
    lib.oracle_e4m3_value.argtypes = [I]
    lib.oracle_mxfp8_quantize.argtypes = [P, I64, I64, P, P]
    lib.oracle_mxfp8_quantize_bf16.argtypes = [P, I64, I64, P, P]
    lib.oracle_mxfp8_dequantize.argtypes = [P, P, I64, I64, P]
    lib.oracle_route.argtypes = [P, I64, I, I, P, P]
    lib.oracle_permute.argtypes = [P, I64, I, I, P, P, P]
    D = ctypes.c_double
    lib.oracle_forward_bf16.argtypes = [P, P, P, P, P, P, I64, I, I, I, I, P, I64, P, P, I, D]
    lib.oracle_forward_mxfp8.argtypes = [P, P, P, P, P, P, P, P, P, I64, I, I, I, I, P, I64, P, P, P, P, I, D]
    lib.oracle_round_bf16.argtypes = [P, I64, P]
    lib.oracle_nvfp4_quantize.argtypes = [P, I64, I64, I, P, P, P]
    lib.oracle_nvfp4_quantize_bf16.argtypes = [P, I64, I64, I, P, P, P]
    lib.oracle_nvfp4_dequantize.argtypes = [P, P, P, I64, I64, I, P]
    lib.oracle_forward_nvfp4.argtypes = [P, P, P, P, P, P, P, P, P, I64, I, I, I, I, P, I64, P, P, P, P, P, I, D]
    for name in ("oracle_mxfp8_quantize", "oracle_mxfp8_quantize_bf16", "oracle_mxfp8_dequantize",
                 "oracle_route", "oracle_permute", "oracle_forward_bf16", "oracle_forward_mxfp8",
                 "oracle_round_bf16", "oracle_nvfp4_quantize", "oracle_nvfp4_quantize_bf16",
                 "oracle_nvfp4_dequantize", "oracle_forward_nvfp4"):
        getattr(lib, name).restype = I
    _lib = lib
    return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle buffers must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def _bf16_bits(a) -> np.ndarray:
    """Accept a torch bf16 tensor or a uint16 numpy array of bf16 bit patterns."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16
        return np.ascontiguousarray(a)
    import torch  # plain CPU tensor handling only

    assert a.dtype == torch.bfloat16
    return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def threads() -> int:
    return int(_load().oracle_threads())


def e4m3_value(code: int) -> float:
    return float(_load().oracle_e4m3_value(int(code)))


def route(logits: np.ndarray, k: int):
    """Top-k routing of fp32 logits [T, E] -> (ids int32 [T,k] ascending, probs fp32 [T,k])."""
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), np.int32)
    probs = np.empty((T, k), np.float32)
    _check(_load().oracle_route(_ptr(lg), T, E, k, _ptr(ids), _ptr(probs)), "route")
    return ids, probs


def permute(ids: np.ndarray, num_experts: int):
    """Stable expert permutation -> (offsets int64 [E+1], perm int32 [R], inv int32 [T,k])."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    offsets = np.empty(num_experts + 1, np.int64)
    perm = np.empty(T * k, np.int32)
    inv = np.empty((T, k), np.int32)
    _check(_load().oracle_permute(_ptr(ids), T, num_experts, k, _ptr(offsets), _ptr(perm), _ptr(inv)),
           "permute")
    return offsets, perm, inv


def mxfp8_quantize(values: np.ndarray):
    """fp32 [rows, cols] (cols % 32 == 0) -> (codes uint8 [rows, cols], scales uint8 [rows, cols/32])."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    rows, cols = v.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, cols // 32), np.uint8)
    _check(_load().oracle_mxfp8_quantize(_ptr(v), rows, cols, _ptr(q), _ptr(s)), "mxfp8_quantize")
    return q, s


def mxfp8_quantize_bf16(bits) -> tuple[np.ndarray, np.ndarray]:
    """bf16 (torch tensor or uint16 bits) [..., cols] -> codes [..., cols], scales [..., cols/32]."""
    b = _bf16_bits(bits)
    shape = b.shape
    cols = shape[-1]
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    q = np.empty(shape, np.uint8)
    s = np.empty(shape[:-1] + (cols // 32,), np.uint8)
    _check(_load().oracle_mxfp8_quantize_bf16(_ptr(b), rows, cols, _ptr(q), _ptr(s)), "mxfp8_quantize_bf16")
    return q, s


def mxfp8_dequantize(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    cols = q.shape[-1]
    rows = int(np.prod(q.shape[:-1])) if q.ndim > 1 else 1
    out = np.empty(q.shape, np.float32)
    _check(_load().oracle_mxfp8_dequantize(_ptr(q), _ptr(s), rows, cols, _ptr(out)), "mxfp8_dequantize")
    return out


PROBS_IN_FC1 = 1
SQUARED_RELU = 2


def _variant(probs_in_fc1, gate_up_clamp, squared_relu=False):
    flags = (PROBS_IN_FC1 if probs_in_fc1 else 0) | (SQUARED_RELU if squared_relu else 0)
    clamp = float(gate_up_clamp) if gate_up_clamp else 0.0
    return flags, clamp


def round_bf16(out):
    """The bf16 finalize: fp32 values rounded to bf16 (nearest even); returns
    the bf16 bit patterns as uint16."""
    a = np.ascontiguousarray(out, dtype=np.float32)
    r = np.empty(a.shape, np.uint16)
    _check(_load().oracle_round_bf16(_ptr(a), a.size, _ptr(r)), "round_bf16")
    return r


def forward_bf16(x, ids, probs, w_gate, w_up, w_down, tokens=None, want_h=False, probs_in_fc1=False,
                 gate_up_clamp=None, squared_relu=False):
    """bf16 routed SwiGLU forward for `tokens` (default: all rows of ids).

    x [T,H] bf16, ids/probs [T,k], w_gate/w_up [E,F,H] bf16, w_down [E,H,F] bf16.
    Returns out fp32 [ntok, H] (and h fp32 [ntok, k, F] when want_h).
    probs_in_fc1 / gate_up_clamp select the variants described in
    moe_oracle.c (probability applied to the SwiGLU row; clamp of the gate
    and up pre-activations); squared_relu: experts h = relu(w_gate . x)^2,
    w_up unused (None)."""
    flags, clamp = _variant(probs_in_fc1, gate_up_clamp, squared_relu)
    xb = _bf16_bits(x)
    gb, db = _bf16_bits(w_gate), _bf16_bits(w_down)
    ub = None if squared_relu else _bf16_bits(w_up)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    probs = np.ascontiguousarray(probs, dtype=np.float32)
    T, k = ids.shape
    E, F, H = gb.shape
    assert xb.shape[1] == H and db.shape == (E, H, F)
    toks = np.arange(T, dtype=np.int64) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    out = np.empty((toks.size, H), np.float32)
    h = np.empty((toks.size, k, F), np.float32) if want_h else None
    _check(_load().oracle_forward_bf16(_ptr(xb), _ptr(ids), _ptr(probs), _ptr(gb), _ptr(ub), _ptr(db),
                                       xb.shape[0], H, F, E, k, _ptr(toks), toks.size, _ptr(out), _ptr(h),
                                       flags, clamp),
           "forward_bf16")
    return (out, h) if want_h else out


def quantize_weights_mxfp8(w_gate, w_up, w_down):
    """Quantise the bf16 expert weights with the oracle's MXFP8 rule:
    gate/up in blocks along H (their last axis), down in blocks along F."""
    gq, gs = mxfp8_quantize_bf16(w_gate)
    uq, us = mxfp8_quantize_bf16(w_up)
    dq, ds = mxfp8_quantize_bf16(w_down)
    return gq, gs, uq, us, dq, ds


def forward_mxfp8(x, ids, probs, wq, tokens=None, want_h=False, probs_in_fc1=False, gate_up_clamp=None,
                  squared_relu=False):
    """MXFP8 routed SwiGLU forward; `wq` = quantize_weights_mxfp8(...) output.

    Returns out fp32 [ntok, H] and, when want_h, (h codes [ntok,k,F],
    h scales [ntok,k,F/32], h pre-quantisation fp32 [ntok,k,F]).  Variants
    as in forward_bf16 (squared_relu: the gate codes are the one FC1
    projection, the up codes are not read)."""
    flags, clamp = _variant(probs_in_fc1, gate_up_clamp, squared_relu)
    xb = _bf16_bits(x)
    gq, gs, uq, us, dq, ds = wq
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    probs = np.ascontiguousarray(probs, dtype=np.float32)
    T, k = ids.shape
    E, F, H = gq.shape
    toks = np.arange(T, dtype=np.int64) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    out = np.empty((toks.size, H), np.float32)
    hq = hs = hf = None
    if want_h:
        hq = np.empty((toks.size, k, F), np.uint8)
        hs = np.empty((toks.size, k, F // 32), np.uint8)
        hf = np.empty((toks.size, k, F), np.float32)
    _check(_load().oracle_forward_mxfp8(_ptr(xb), _ptr(ids), _ptr(probs), _ptr(gq), _ptr(gs), _ptr(uq),
                                        _ptr(us), _ptr(dq), _ptr(ds), xb.shape[0], H, F, E, k, _ptr(toks),
                                        toks.size, _ptr(out), _ptr(hq), _ptr(hs), _ptr(hf), flags, clamp),
           "forward_mxfp8")
    return (out, (hq, hs, hf)) if want_h else out


def nvfp4_quantize(values, per_row: bool = True):
    """NVFP4 (the per-token recipe) of an fp32 [rows, cols] matrix (cols % 16 == 0), or of a
    bf16 tensor / uint16 bit array.  Returns (codes uint8 [rows, cols/2], element 2i in the
    low nibble; E4M3 block scales uint8 [rows, cols/16]; second-level scales fp32 [rows]
    when per_row, else [1] for the whole matrix)."""
    bf16 = not (isinstance(values, np.ndarray) and values.dtype != np.uint16)
    v = _bf16_bits(values) if bf16 else np.ascontiguousarray(values, dtype=np.float32)
    rows, cols = v.shape
    q = np.empty((rows, cols // 2), np.uint8)
    s = np.empty((rows, cols // 16), np.uint8)
    g = np.empty(rows if per_row else 1, np.float32)
    fn = _load().oracle_nvfp4_quantize_bf16 if bf16 else _load().oracle_nvfp4_quantize
    _check(fn(_ptr(v), rows, cols, 1 if per_row else 0, _ptr(q), _ptr(s), _ptr(g)), "nvfp4_quantize")
    return q, s, g


def nvfp4_dequantize(q, s, g, per_row: bool = True) -> np.ndarray:
    """float64 [rows, cols] values of NVFP4 codes, block scales and second-level scales."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    g = np.ascontiguousarray(g, dtype=np.float32)
    rows, half = q.shape
    out = np.empty((rows, 2 * half), np.float64)
    _check(_load().oracle_nvfp4_dequantize(_ptr(q), _ptr(s), _ptr(g), rows, 2 * half, 1 if per_row else 0,
                                           _ptr(out)), "nvfp4_dequantize")
    return out


def quantize_weights_nvfp4(w_gate, w_up, w_down):
    """NVFP4 expert weights with one second-level scale per expert matrix: W1[e] = the gate
    rows then the up rows (w_up None: squared-ReLU experts, gate rows only), blocks along
    H; W_down[e] blocks along F.  Returns (w1_q [E,R1,H/2], w1_s [E,R1,H/16], g1 [E],
    wd_q [E,H,F/2], wd_s [E,H,F/16], g2 [E])."""
    import torch  # plain CPU tensor handling only

    gb = _bf16_bits(w_gate)
    E, F, H = gb.shape
    w1 = gb if w_up is None else np.concatenate([gb, _bf16_bits(w_up)], axis=1)
    db = _bf16_bits(w_down)
    R1 = w1.shape[1]
    w1_q = np.empty((E, R1, H // 2), np.uint8)
    w1_s = np.empty((E, R1, H // 16), np.uint8)
    wd_q = np.empty((E, H, F // 2), np.uint8)
    wd_s = np.empty((E, H, F // 16), np.uint8)
    g1 = np.empty(E, np.float32)
    g2 = np.empty(E, np.float32)
    for e in range(E):
        w1_q[e], w1_s[e], g = nvfp4_quantize(np.ascontiguousarray(w1[e]), per_row=False)
        g1[e] = g[0]
        wd_q[e], wd_s[e], g = nvfp4_quantize(np.ascontiguousarray(db[e]), per_row=False)
        g2[e] = g[0]
    del torch
    return w1_q, w1_s, g1, wd_q, wd_s, g2


def forward_nvfp4(x, ids, probs, wq, tokens=None, want_h=False, probs_in_fc1=False, gate_up_clamp=None,
                  squared_relu=False):
    """NVFP4 routed SwiGLU forward (per-token recipe); `wq` = quantize_weights_nvfp4(...).

    Returns out fp32 [ntok, H] and, when want_h, (h codes [ntok,k,F/2], h block scales
    [ntok,k,F/16], h second-level scales [ntok,k], h pre-quantisation fp32 [ntok,k,F])."""
    flags, clamp = _variant(probs_in_fc1, gate_up_clamp, squared_relu)
    xb = _bf16_bits(x)
    w1_q, w1_s, g1, wd_q, wd_s, g2 = wq
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    probs = np.ascontiguousarray(probs, dtype=np.float32)
    T, k = ids.shape
    E, H, half_f = wd_q.shape
    F = 2 * half_f
    toks = np.arange(T, dtype=np.int64) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    out = np.empty((toks.size, H), np.float32)
    hq = hs = hg = hf = None
    if want_h:
        hq = np.empty((toks.size, k, F // 2), np.uint8)
        hs = np.empty((toks.size, k, F // 16), np.uint8)
        hg = np.empty((toks.size, k), np.float32)
        hf = np.empty((toks.size, k, F), np.float32)
    _check(_load().oracle_forward_nvfp4(_ptr(xb), _ptr(ids), _ptr(probs), _ptr(w1_q), _ptr(w1_s), _ptr(g1),
                                        _ptr(wd_q), _ptr(wd_s), _ptr(g2), xb.shape[0], H, F, E, k, _ptr(toks),
                                        toks.size, _ptr(out), _ptr(hq), _ptr(hs), _ptr(hg), _ptr(hf), flags,
                                        clamp),
           "forward_nvfp4")
    return (out, (hq, hs, hg, hf)) if want_h else out
