"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point include/moe.h declares, and rejects bad arguments before
launching anything."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import routed_moe_swiglu_b200 as rm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    txt = open(os.path.join(ROOT, "include", "moe.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*([a-z][a-z0-9_]*)\s*\(", txt, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = rm.load_library()
    names = _declared_functions()
    assert len(names) >= 14, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/moe.h but not exported"


def test_version_and_status_strings():
    assert rm.moe_version().count(".") == 2
    lib = rm.load_library()
    for code in range(7):
        assert lib.moe_status_string(code).decode() not in ("", "unknown status")


@pytest.mark.parametrize("kw,code", [
    (dict(hidden=2050), 2),                # not a multiple of 8
    (dict(ffn=0), 2),
    (dict(top_k=17), 2),                   # k > 16
    (dict(num_experts=4, top_k=5), 2),     # k > E
    (dict(num_experts=1025), 2),
    (dict(capacity=0), 2),
    (dict(max_live_rows=10 ** 9), 2),      # above capacity
    (dict(hidden=2056, precision="mxfp8"), 2),  # MXFP8 needs multiples of 32
    (dict(ffn=1040, precision="nvfp4"), 2),     # so does NVFP4
])
def test_plan_rejects_unsupported(kw, code):
    args = dict(hidden=2048, ffn=1024, num_experts=128, top_k=8, capacity=1024, precision="bf16")
    args.update(kw)
    with pytest.raises(rm.MoeError) as ei:
        rm.moe_plan_create(**args)
    assert ei.value.code == code


def test_plan_sizes():
    p = rm.moe_plan_create(hidden=2048, ffn=1024, num_experts=128, top_k=8, capacity=65536, max_live_rows=256)
    assert p.max_live_rows == 256
    # weight buffer: gate+up+down bf16, each 256-byte aligned region
    assert rm.moe_weight_buffer_bytes(p) >= 3 * 128 * 2048 * 1024 * 2
    ws = rm.moe_workspace_bytes(p)
    rows_pad = 256 * 8 + 128 * 32  # routes + experts x the 32-row segment alignment
    assert ws >= rows_pad * (2048 * 2 + 1024 * 2 + 2048 * 4)
    q = rm.moe_plan_create(hidden=2048, ffn=1024, num_experts=128, top_k=8, capacity=65536)
    assert q.max_live_rows == 65536 and rm.moe_workspace_bytes(q) > ws


def test_forward_rejects_bad_arguments_before_launch():
    lib = rm.load_library()
    p = rm.moe_plan_create(hidden=256, ffn=512, num_experts=8, top_k=2, capacity=64)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    ws = rm.moe_workspace_bytes(p)
    null = None
    # no routing input at all
    assert lib.moe_forward(p.handle, fake, null, null, null, fake, fake, fake, fake, ws, null) == 1
    # both logits and ids/probs
    assert lib.moe_forward(p.handle, fake, fake, fake, fake, fake, fake, fake, fake, ws, null) == 1
    # ids without probs
    assert lib.moe_forward(p.handle, fake, null, fake, null, fake, fake, fake, fake, ws, null) == 1
    # workspace too small
    assert lib.moe_forward(p.handle, fake, fake, null, null, fake, fake, fake, fake, ws - 1, null) == 4
    # misaligned x
    bad = ctypes.c_void_p((1 << 20) + 8)
    assert lib.moe_forward(p.handle, bad, fake, null, null, fake, fake, fake, fake, ws, null) == 3
    # null plan / null out
    assert lib.moe_forward(None, fake, fake, null, null, fake, fake, fake, fake, ws, null) == 1
    assert lib.moe_forward(p.handle, fake, fake, null, null, fake, fake, null, fake, ws, null) == 1


def test_prepare_and_quantize_reject_bad_arguments():
    lib = rm.load_library()
    p = rm.moe_plan_create(hidden=256, ffn=512, num_experts=8, top_k=2, capacity=64)
    fake = ctypes.c_void_p(1 << 20)
    nb = rm.moe_weight_buffer_bytes(p)
    assert lib.moe_prepare_weights(p.handle, fake, fake, fake, fake, nb - 1, None) == 4
    assert lib.moe_prepare_weights(p.handle, None, fake, fake, fake, nb, None) == 1
    assert lib.moe_prepare_weights(p.handle, fake, fake, fake, ctypes.c_void_p((1 << 20) + 16), nb, None) == 3
    # cols not a multiple of 32
    assert lib.mxfp8_quantize_block32(fake, 4, 48, 48, fake, fake, None, None) == 2
    # ld_in < cols
    assert lib.mxfp8_quantize_block32(fake, 4, 64, 32, fake, fake, None, None) == 1
    # zero rows is a no-op success
    assert lib.mxfp8_quantize_block32(fake, 0, 64, 64, fake, fake, None, None) == 0


def test_product_path_does_not_touch_the_oracle():
    """The package must not import, load or reference the oracle."""
    pkg = os.path.join(ROOT, "routed_moe_swiglu_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "moe_oracle" not in txt and "from oracle" not in txt, f


def test_bounded_wait_check_rejects_bad_arguments_before_launch():
    lib = rm.load_library()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    assert lib.moe_check_bounded_wait(0, fake, None, None) == 1
    assert lib.moe_check_bounded_wait(10_000_000_001, fake, None, None) == 1
    assert lib.moe_check_bounded_wait(1000, None, None, None) == 1


def test_plan_rejects_unknown_flags_and_bad_clamp():
    lib = rm.load_library()
    base = dict(hidden=256, ffn=512, num_experts=8, top_k=2, capacity=64, max_live_rows=0, precision=0)
    for flags, clamp in ((0x8, 0.0), (0x80000000, 0.0), (0, -1.0), (0, float("nan")), (0, float("inf"))):
        d = rm._Desc(*base.values(), flags, clamp)
        h = ctypes.c_void_p()
        assert lib.moe_plan_create(ctypes.byref(d), ctypes.byref(h)) == 1, (flags, clamp)
    p = rm.moe_plan_create(hidden=256, ffn=512, num_experts=8, top_k=2, capacity=64, out_dtype="bf16",
                           probs_in_fc1=True, gate_up_clamp=3.5)
    assert p.out_dtype == "bf16" and p.probs_in_fc1 and p.gate_up_clamp == 3.5



def test_squared_relu_plans():
    lib = rm.load_library()
    m = rm.moe_plan_create(hidden=256, ffn=512, num_experts=8, top_k=2, capacity=64, precision="mxfp8",
                           squared_relu=True)
    # MXFP8: one projection of F rows per expert (codes) instead of gate and up
    assert rm.moe_weight_buffer_bytes(m) < rm.moe_weight_buffer_bytes(
        rm.moe_plan_create(hidden=256, ffn=512, num_experts=8, top_k=2, capacity=64, precision="mxfp8"))
    p = rm.moe_plan_create(hidden=256, ffn=200, num_experts=8, top_k=2, capacity=64, squared_relu=True)
    assert p.squared_relu
    # one FC1 projection: rows padded to 256 per expert, K padded to 256
    assert rm.moe_weight_buffer_bytes(p) >= 8 * 256 * 256 * 2 + 8 * 256 * 256 * 2
    fake = ctypes.c_void_p(1 << 20)
    nb = rm.moe_weight_buffer_bytes(p)
    # w_up may be NULL for squared-ReLU plans (validation then proceeds to the buffer size)
    assert lib.moe_prepare_weights(p.handle, fake, None, fake, fake, nb - 1, None) == 4
    q = rm.moe_plan_create(hidden=256, ffn=200, num_experts=8, top_k=2, capacity=64)
    assert lib.moe_prepare_weights(q.handle, fake, None, fake, fake, rm.moe_weight_buffer_bytes(q), None) == 1


def test_nvfp4_plans_and_quantizer_arguments():
    lib = rm.load_library()
    E, H, F = 128, 2048, 1024
    p4 = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=8, capacity=4096, precision="nvfp4")
    p8 = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=8, capacity=4096, precision="mxfp8")
    assert p4.precision == "nvfp4"
    # weights: E2M1 codes (half a byte per element) + an E4M3 scale per 16 + fp32 scales [E][2]
    w4 = rm.moe_weight_buffer_bytes(p4)
    assert 3 * E * H * F * (0.5 + 1 / 16) <= w4 < 0.6 * rm.moe_weight_buffer_bytes(p8)
    # workspace: NVFP4 adds the fp32 h rows and per-row scales to MXFP8's buffers
    assert rm.moe_workspace_bytes(p4) > rm.moe_workspace_bytes(p8)
    # squared-ReLU NVFP4 plans hold one FC1 projection
    r4 = rm.moe_plan_create(hidden=H, ffn=F, num_experts=E, top_k=8, capacity=4096, precision="nvfp4",
                            squared_relu=True)
    assert rm.moe_weight_buffer_bytes(r4) < w4
    fake = ctypes.c_void_p(1 << 20)
    # nvfp4_quantize_block16(in, rows, cols, ld_in, q, scales, row_scales, live, stream)
    assert lib.nvfp4_quantize_block16(fake, 4, 48, 48, fake, fake, fake, None, None) == 2   # cols % 32
    assert lib.nvfp4_quantize_block16(fake, 4, 64, 32, fake, fake, fake, None, None) == 1   # ld_in < cols
    assert lib.nvfp4_quantize_block16(fake, 4, 64, 64, fake, fake, None, None, None) == 1   # no row scales
    assert lib.nvfp4_quantize_block16(ctypes.c_void_p((1 << 20) + 8), 4, 64, 64, fake, fake, fake, None,
                                      None) == 3                                             # misaligned in
    assert lib.nvfp4_quantize_block16(fake, 0, 64, 64, fake, fake, fake, None, None) == 0   # no rows: no-op


def test_ep_entries_reject_bad_arguments_before_launch():
    lib = rm.load_library()
    p = rm.moe_plan_create(hidden=256, ffn=512, num_experts=8, top_k=2, capacity=64)
    f = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    ws = rm.moe_workspace_bytes(p)
    null = None

    def dispatch(ep=2, x=f, logits=f, ids=null, probs=null, send_x=f, counts=f, wsb=ws):
        return lib.moe_ep_dispatch(p.handle, ep, x, logits, ids, probs, f, send_x, f, f, counts, f, f, f, wsb, null)

    assert dispatch(ep=3) == 2            # 3 does not divide the 8 experts
    assert dispatch(ep=0) == 2
    assert dispatch(ep=16) == 2           # more ranks than experts
    assert dispatch(logits=null) == 1     # no routing input
    assert dispatch(ids=f) == 1           # ids without probs, and logits too
    assert dispatch(counts=null) == 1
    assert dispatch(wsb=ws - 1) == 4
    assert dispatch(send_x=ctypes.c_void_p((1 << 20) + 8)) == 3
    assert dispatch(x=ctypes.c_void_p((1 << 20) + 2)) == 3
    assert lib.moe_ep_combine(p.handle, f, f, f, f, null, null) == 1
    assert lib.moe_ep_combine(None, f, f, f, f, f, null) == 1
    assert lib.moe_ep_combine(p.handle, ctypes.c_void_p((1 << 20) + 4), f, f, f, f, null) == 3


def test_ep_peer_region_size_and_argument_checks():
    """The peer-memory exchange's region: a header, one receive slot per source
    of max_live * k rows (x, id, weight), the returned y rows, the compacted
    received rows; host-side checks before any launch."""
    lib = rm.load_library()
    H, k, cap = 256, 2, 64
    p = rm.moe_plan_create(hidden=H, ffn=512, num_experts=8, top_k=k, capacity=cap)
    send = cap * k
    sizes = {ep: rm.moe_ep_region_bytes(p, ep) for ep in (1, 2, 4, 8)}
    for ep, b in sizes.items():
        # slots ep * send * (2H + 8) + y_back send * 4H + received ep * send * (2H + 8 + 4H + 8)
        floor = ep * send * (2 * H + 8) + send * 4 * H + ep * send * (2 * H + 4 * H + 16)
        assert floor <= b <= floor + 4096 + 16 * 256, (ep, b, floor)
    assert sizes[2] > sizes[1] and sizes[4] > sizes[2]
    assert rm.moe_ep_region_bytes(p, 0) == 0 and rm.moe_ep_region_bytes(p, 129) == 0
    f = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    null = None
    ws = rm.moe_workspace_bytes(p)

    def dispatch(ep=2, rank=0, logits=f, table=f, wsb=ws):
        return lib.moe_ep_peer_dispatch(p.handle, ep, rank, f, logits, null, null, f, table, f, f, f, wsb, null)

    assert dispatch(ep=3) == 2       # 3 does not divide the 8 experts
    assert dispatch(rank=2) == 1     # rank outside [0, ep)
    assert dispatch(rank=-1) == 1
    assert dispatch(logits=null) == 1
    assert dispatch(table=null) == 1
    assert dispatch(wsb=ws - 1) == 4
    assert lib.moe_ep_peer_receive(p.handle, 2, f, 0, null) == 1                          # no wait limit
    assert lib.moe_ep_peer_receive(p.handle, 2, ctypes.c_void_p((1 << 20) + 64), 1000, null) == 3
    assert lib.moe_ep_peer_return(p.handle, 2, 2, f, null) == 1
    assert lib.moe_ep_peer_combine(p.handle, 2, f, f, f, f, null, 1000, null) == 1
    assert lib.moe_ep_peer_combine(p.handle, 5, f, f, f, f, f, 1000, null) == 2
