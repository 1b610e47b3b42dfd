"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry
point include/ssd.h declares, and rejects bad arguments with the documented status
before anything is enqueued.  Pointers here are fake but 16-byte aligned addresses; a
validation failure must return before they are ever dereferenced or passed to CUDA."""
import ctypes
import os
import re

import pytest

import state_space_model_04_b200 as ssd
from state_space_model_04_b200 import ssd as binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUP, CUDA, TIMEOUT, WS, INTERNAL = range(7)

pytestmark = pytest.mark.skipif(not os.path.exists(binding.LIB_PATH), reason="library not built")


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"SSD_API\s+[\w\s\*]+?\b(ssd_\w+)\s*\(", txt)
    return names


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 10
    L = ssd.lib()
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings():
    L = ssd.lib()
    assert L.ssd_version() >= 100
    for s in range(7):
        assert ssd.status_string(s).startswith("SSD_")
    assert "unknown" in ssd.status_string(99)


# fake, aligned, distinct device addresses (never dereferenced: validation fails first)
def _fake(n):
    return [ctypes.c_void_p(0x10000000 + 0x1000000 * i) for i in range(n)]


def _prefill(b=1, T=512, H=4, P=64, N=64, G=1, chunk=256, io=1, ptrs=None, ws_bytes=1 << 30,
             h0=None, hf=None):
    L = ssd.lib()
    x, dt, A, B, C, D, y, ws = ptrs or _fake(8)
    return L.ssd_prefill(b, T, H, P, N, G, chunk, io, x, dt, A, B, C, D, h0, y, hf, ws,
                         ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(chunk=100), INVALID), (dict(chunk=32), INVALID), (dict(io=7), INVALID),
    (dict(H=6, G=4), INVALID), (dict(b=-1), INVALID), (dict(T=-5), INVALID), (dict(N=0), INVALID),
    (dict(P=32), UNSUP), (dict(N=96), UNSUP), (dict(b=70000), UNSUP),
    (dict(ws_bytes=16), WS),
])
def test_prefill_rejects(kw, status):
    assert _prefill(**kw) == status
    assert ssd.last_error() != ""


def test_prefill_null_and_misaligned_pointers():
    for i in range(7):  # x, dt, A, B, C, D, y
        p = _fake(8)
        p[i] = None
        assert _prefill(ptrs=p) == INVALID, i
        p = _fake(8)
        p[i] = ctypes.c_void_p(p[i].value + 4)
        assert _prefill(ptrs=p) == INVALID, i
    p = _fake(8)
    p[7] = None
    assert _prefill(ptrs=p) == WS


def test_prefill_rejects_aliasing():
    p = _fake(8)
    p[6] = p[0]  # y == x
    assert _prefill(ptrs=p) == INVALID
    p = _fake(8)
    hf = ctypes.c_void_p(p[0].value)  # h_final overlaps x
    assert _prefill(ptrs=p, hf=hf) == INVALID
    h0 = ctypes.c_void_p(0x7000000000)
    hf = ctypes.c_void_p(0x7000000000 + 4096)  # partial overlap of h0 / h_final
    assert _prefill(ptrs=_fake(8), h0=h0, hf=hf) == INVALID
    for io, N in [(0, 64), (1, 128)]:  # fp32 path, tensor-core path with a split workspace
        p = _fake(8)
        hf = ctypes.c_void_p(p[7].value + 256)  # h_final inside the workspace
        assert _prefill(N=N, io=io, ptrs=p, hf=hf) == INVALID, io
        assert "h_final" in ssd.last_error()


def test_prefill_empty_batch_is_noop():
    assert _prefill(b=0) == OK
    assert _prefill(T=0) == OK  # no h_final requested: nothing to do, no CUDA call


def test_workspace_queries():
    assert ssd.prefill_workspace_size(1, 512, 4, 64, 64, 1, 256, 0) > 0
    assert ssd.prefill_workspace_size(8, 4096, 80, 64, 128, 1, 256, 1) > 0
    assert ssd.prefill_workspace_size(1, 512, 4, 64, 64, 1, 100, 0) == 0  # invalid chunk
    assert ssd.prefill_workspace_size(0, 512, 4, 64, 64, 1, 256, 0) == 0
    assert ssd.decode_workspace_size(64, 32, 1) >= 64 * 32 * 4
    assert ssd.decode_workspace_size(0, 1, 1) == 0


def _decode(layers=2, b=1, H=4, P=64, N=128, G=1, k=4, act=1, io=1, ptrs=None, ws_bytes=1 << 20):
    L = ssd.lib()
    h, cs, xbc, dt, A, D, w, bb, y, ws = ptrs or _fake(10)
    return L.ssd_decode_step(layers, b, H, P, N, G, k, act, io, h, cs, xbc, dt, A, D, w, bb, y, ws,
                             ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(act=3), INVALID), (dict(io=2), INVALID), (dict(H=5, G=2), INVALID), (dict(k=0), INVALID),
    (dict(k=3), UNSUP), (dict(P=128), UNSUP), (dict(N=32), UNSUP), (dict(layers=-1), INVALID),
    (dict(ws_bytes=0), WS),
])
def test_decode_rejects(kw, status):
    assert _decode(**kw) == status


def test_decode_null_aliasing_and_empty():
    for i in range(10):
        p = _fake(10)
        p[i] = None
        assert _decode(ptrs=p) in (INVALID, WS), i
    p = _fake(10)
    p[8] = p[0]  # y aliases h
    assert _decode(ptrs=p) == INVALID
    # a written buffer (h 0, conv_state 1, y 8, workspace 9) overlapping anything else
    for w, other in [(9, 0), (9, 1), (9, 2), (9, 4), (0, 4), (1, 6), (8, 7), (8, 3)]:
        p = _fake(10)
        p[w] = ctypes.c_void_p(p[other].value + 16)  # inside even the 32-byte A, D and dt
        assert _decode(ptrs=p) == INVALID, (w, other)
        assert "overlaps" in ssd.last_error()
    assert _decode(b=0) == OK
    assert _decode(layers=0) == OK


def test_decode_plan_rejects():
    L = ssd.lib()
    handle = ctypes.c_void_p()
    f = _fake(10)
    # ring = 0
    st = L.ssd_decode_plan_create(ctypes.byref(handle), 1, 1, 4, 64, 128, 1, 4, 1, 1, f[0], f[1], f[2],
                                  f[3], 0, f[4], f[5], f[6], f[7], f[8], 8, f[9], 1 << 20)
    assert st == INVALID and not handle.value
    st = L.ssd_decode_plan_create(ctypes.byref(handle), 1, 1, 4, 64, 128, 1, 4, 1, 1, f[0], f[1], f[2],
                                  f[3], 2, f[4], f[5], f[6], f[7], f[8], -1, f[9], 1 << 20)
    assert st == INVALID
    assert L.ssd_decode_plan_create(None, 1, 1, 4, 64, 128, 1, 4, 1, 1, f[0], f[1], f[2], f[3], 2,
                                    f[4], f[5], f[6], f[7], f[8], 8, f[9], 1 << 20) == INVALID
    # a written buffer overlapping a ring or the weights: y_ring inside xbc_ring's second
    # step, the workspace inside conv_w
    g = _fake(10)
    y_in_ring = ctypes.c_void_p(g[2].value + 1 * 4 * 64 * 2 + 2 * 128 * 2 * 2)
    assert L.ssd_decode_plan_create(ctypes.byref(handle), 1, 1, 4, 64, 128, 1, 4, 1, 1, g[0], g[1], g[2], g[3], 2,
                                    g[4], g[5], g[6], g[7], y_in_ring, 8, g[9], 1 << 20) == INVALID
    assert L.ssd_decode_plan_create(ctypes.byref(handle), 1, 1, 4, 64, 128, 1, 4, 1, 1, g[0], g[1], g[2], g[3], 2,
                                    g[4], g[5], g[6], g[7], g[8], 8, g[6], 1 << 20) == INVALID
    assert not handle.value
    assert L.ssd_decode_plan_launch(None, None) == INVALID
    assert L.ssd_decode_plan_destroy(None) == OK
    # the one-call loop runs the same checks before anything is built or enqueued
    assert L.ssd_decode_loop(1, 1, 4, 64, 128, 1, 4, 1, 1, f[0], f[1], f[2], f[3], 0, f[4], f[5], f[6], f[7],
                             f[8], 8, f[9], 1 << 20, None) == INVALID          # ring = 0
    assert L.ssd_decode_loop(1, 1, 4, 64, 128, 1, 4, 1, 1, f[0], f[1], f[2], f[3], 2, f[4], f[5], f[6], f[7],
                             f[8], -1, f[9], 1 << 20, None) == INVALID         # n_steps < 0
    assert L.ssd_decode_loop(1, 1, 4, 64, 128, 1, 4, 1, 1, f[0], f[1], f[2], f[3], 2, f[4], f[5], f[6], f[7],
                             f[8], 8, f[9], 16, None) == WS                    # workspace too small


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 64, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ssd.prefill(x, torch.zeros(1, 64, 4), torch.zeros(4), torch.zeros(1, 64, 1, 64, dtype=torch.bfloat16),
                    torch.zeros(1, 64, 1, 64, dtype=torch.bfloat16), torch.zeros(4))


def test_binding_refuses_tensors_on_another_device():
    """Every tensor of a call must sit on the device of its first operand (the kernels read
    the pointers directly; a tensor on another GPU would be a peer address).  The check runs
    before the library is called; None operands are skipped."""
    import torch
    from state_space_model_04_b200.ssd import _check_device
    a = torch.zeros(4)
    _check_device(a.device, b=torch.zeros(2), c=None)
    with pytest.raises(ValueError, match="c is on meta"):
        _check_device(a.device, b=torch.zeros(2), c=torch.empty(2, device="meta"))


def test_segment_hook_and_workspace():
    """The split of a sequence into segments sizes the workspace: one fp32 state and one
    log decay per (sequence, head) for every segment but the last."""
    args = (1, 4096, 24, 64, 128, 1, 256, 1)
    assert ssd.lib().ssd_debug_force_prefill_segments(-1) == 1  # SSD_ERR_INVALID_ARG
    try:
        assert ssd.prefill_segments(*args) >= 1
        assert ssd.prefill_whole_units(*args) == 0                            # every pair split
        assert ssd.prefill_segments(16, 4096, 80, 64, 128, 1, 256, 1) == 1  # enough sequence-heads
        assert ssd.prefill_whole_units(16, 4096, 80, 64, 128, 1, 256, 1) == 16 * 80
        # 640 pairs on 148 SMs: the 48 pairs of the ragged last wave are split, the rest run whole
        assert ssd.prefill_segments(8, 4096, 80, 64, 128, 1, 256, 1) > 1
        assert ssd.prefill_whole_units(8, 4096, 80, 64, 128, 1, 256, 1) in (0, 592)
        assert ssd.prefill_segments(1, 4096, 24, 64, 64, 1, 256, 1) == 1    # N = 64: the SIMT path
        assert ssd.prefill_whole_units(1, 4096, 24, 64, 64, 1, 256, 1) == 24
        assert ssd.prefill_segments(1, 512, 4, 64, 64, 1, 100, 0) == 0      # invalid chunk
        assert ssd.prefill_whole_units(1, 512, 4, 64, 64, 1, 100, 0) == -1
        ssd.debug_force_prefill_segments(1)
        assert ssd.prefill_segments(*args) == 1
        one = ssd.prefill_workspace_size(*args)
        ssd.debug_force_prefill_segments(4)
        assert ssd.prefill_segments(*args) == 4
        four = ssd.prefill_workspace_size(*args)
        assert four - one >= 3 * 24 * (64 * 128 * 4 + 4)
        ssd.debug_force_prefill_segments(1000)  # clamped to one block per segment
        assert ssd.prefill_workspace_size(*args) - one >= 31 * 24 * 64 * 128 * 4
    finally:
        ssd.debug_force_prefill_segments(0)


def test_fma_prefill_hook_routes_tensor_core_shapes_to_the_literal_chunk_path():
    """With the hook on, a tensor-core shape is sized (and run) by the fp32-FMA path, whose
    workspace depends on the chunk length; off, the tensor-core sizing ignores it."""
    L = ssd.lib()
    assert L.ssd_debug_force_fma_prefill(2) == INVALID and L.ssd_debug_force_fma_prefill(-1) == INVALID
    shape = (2, 1024, 8, 64, 128, 1)
    tc = {c: ssd.prefill_workspace_size(*shape, c, ssd.SSD_BF16) for c in (64, 128, 256)}
    assert len(set(tc.values())) == 1
    try:
        ssd.debug_force_fma_prefill(True)
        fma = {c: ssd.prefill_workspace_size(*shape, c, ssd.SSD_BF16) for c in (64, 128, 256)}
        assert len(set(fma.values())) == 3
        assert ssd.prefill_segments(*shape, 256, ssd.SSD_BF16) == 1
        assert ssd.prefill_whole_units(*shape, 256, ssd.SSD_BF16) == 2 * 8
    finally:
        ssd.debug_force_fma_prefill(False)
    assert ssd.prefill_workspace_size(*shape, 64, ssd.SSD_BF16) == tc[64]


def test_split_planner_decisions_on_148_sms():
    """The split planner's choices at the configurations' shapes (148 SMs, the count used
    when no device is visible): the 130M-layer shape in 6 segments, the long-context shape
    in 11, the 2.7B-layer shape with the 48 pairs of its ragged last wave in 3 segments, and
    a shape whose pairs fill whole waves unsplit."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("decisions depend on the device's SM count")
    bf16 = ssd.SSD_BF16
    assert ssd.prefill_segments(1, 4096, 24, 64, 128, 1, 256, bf16) == 6
    assert ssd.prefill_whole_units(1, 4096, 24, 64, 128, 1, 256, bf16) == 0
    assert ssd.prefill_segments(1, 65536, 80, 64, 128, 8, 256, bf16) == 11
    assert ssd.prefill_whole_units(1, 65536, 80, 64, 128, 8, 256, bf16) == 0
    assert ssd.prefill_segments(8, 4096, 80, 64, 128, 1, 256, bf16) == 3
    assert ssd.prefill_whole_units(8, 4096, 80, 64, 128, 1, 256, bf16) == 592
    assert ssd.prefill_segments(74, 4096, 4, 64, 128, 1, 256, bf16) == 1   # 296 pairs: two whole waves
    assert ssd.prefill_whole_units(74, 4096, 4, 64, 128, 1, 256, bf16) == 296


def _split_workspace_floor(units, n_full, nseg, P=64, N=128):
    """Bytes a split tensor-core prefill touches in its workspace: the 512-byte header, one
    fp32 state and one log decay per split unit and segment but the last, and the in-place
    copy of h0, which the fused kernel reads at the same unit offsets as h0 itself (units
    n_full .. units - 1), so it reaches units * P * N floats past its start."""
    seg = (units - n_full) * (nseg - 1)
    return 512 + seg * P * N * 4 + seg * 4 + units * P * N * 4


def test_workspace_holds_the_in_place_h0_copy_when_some_units_run_whole():
    """h_final aliasing h0 with only the ragged last wave split (the 2.7B-layer shape: 592
    pairs whole, 48 in 3 segments) and with a forced partial split: the workspace the query
    returns covers the h0 copy at the split units' own offsets."""
    bf16 = ssd.SSD_BF16
    assert ssd.prefill_whole_units(8, 4096, 80, 64, 128, 1, 256, bf16) == 592
    assert ssd.prefill_segments(8, 4096, 80, 64, 128, 1, 256, bf16) == 3
    assert ssd.prefill_workspace_size(8, 4096, 80, 64, 128, 1, 256, bf16) >= _split_workspace_floor(640, 592, 3)
    ssd.debug_force_prefill_split(100, 4)
    try:
        assert ssd.prefill_whole_units(2, 1024, 80, 64, 128, 1, 256, bf16) == 100
        assert ssd.prefill_segments(2, 1024, 80, 64, 128, 1, 256, bf16) == 4
        assert ssd.prefill_workspace_size(2, 1024, 80, 64, 128, 1, 256, bf16) >= _split_workspace_floor(160, 100, 4)
    finally:
        ssd.debug_force_prefill_split(0, 0)


def test_decay_precision_hook_rejects_unknown_modes():
    L = ssd.lib()
    assert L.ssd_debug_decay_precision(3) == INVALID and L.ssd_debug_decay_precision(-1) == INVALID
    assert L.ssd_debug_decay_precision(0) == OK


def test_starve_hook_rejects_out_of_range_limits():
    import state_space_model_04_b200 as ssd
    L = ssd.lib()
    assert L.ssd_debug_starve_next_prefill(999_999) == 1
    assert L.ssd_debug_starve_next_prefill(10_000_000_001) == 1


def test_prefill_dt_raw_rejects_bad_clamp_and_bias():
    """ssd_prefill_dt_raw validates its clamp range and dt_bias before anything else runs."""
    L = ssd.lib()
    x, dt, A, B, C, D, y, ws = _fake(8)
    bias = ctypes.c_void_p(0x20000000)

    def call(lo, hi, bias_ptr=bias, H=4):
        return L.ssd_prefill_dt_raw(1, 512, H, 64, 64, 1, 256, 1, x, dt, bias_ptr, lo, hi, A, B, C, D, None, y,
                                    None, ws, 1 << 30, None)
    inf, nan = float("inf"), float("nan")
    for lo, hi in [(-1e-3, 1.0), (0.5, 0.5), (0.5, 0.1), (nan, 1.0), (0.0, nan), (inf, inf)]:
        assert call(lo, hi) == INVALID, (lo, hi)
        assert ssd.last_error() != ""
    assert call(0.0, inf, ctypes.c_void_p(0x20000004)) == INVALID      # misaligned dt_bias
    # a bad shape is reported as for ssd_prefill
    assert L.ssd_prefill_dt_raw(1, 512, 6, 64, 64, 4, 256, 1, x, dt, None, 0.0, inf, A, B, C, D, None, y, None, ws,
                                1 << 30, None) == INVALID


def test_context_parallel_entry_points_reject():
    L = ssd.lib()
    p = _fake(4)
    # context scan: rank outside [0, world), shapes it does not take
    assert L.ssd_prefill_context_scan(2, 2, 1, 4, 64, 128, None, p[0], p[1], p[2], None) == INVALID
    assert L.ssd_prefill_context_scan(2, -1, 1, 4, 64, 128, None, p[0], p[1], p[2], None) == INVALID
    assert L.ssd_prefill_context_scan(0, 0, 1, 4, 64, 128, None, p[0], p[1], p[2], None) == INVALID
    assert L.ssd_prefill_context_scan(2, 1, 1, 4, 64, 64, None, p[0], p[1], p[2], None) == UNSUP
    assert L.ssd_prefill_context_scan(2, 1, 1, 4, 64, 128, None, None, p[1], p[2], None) == INVALID
    assert L.ssd_prefill_context_scan(2, 1, 1, 4, 64, 128, None, p[0], p[1], None, None) == INVALID
    # local state: tensor-core shapes only, outputs required, workspace sized
    x, dt, A, B, hl, ld, ws = _fake(7)
    assert L.ssd_prefill_local_state(1, 512, 4, 64, 64, 1, 1, x, dt, A, B, hl, ld, ws, 1 << 30, None) == UNSUP
    assert L.ssd_prefill_local_state(1, 512, 4, 64, 128, 1, 0, x, dt, A, B, hl, ld, ws, 1 << 30, None) == UNSUP
    assert L.ssd_prefill_local_state(1, 512, 4, 64, 128, 1, 1, x, dt, A, B, None, ld, ws, 1 << 30, None) == INVALID
    assert L.ssd_prefill_local_state(1, 512, 4, 64, 128, 1, 1, x, dt, A, B, hl, ld, ws, 16, None) == WS
    for inp in (x, dt, A, B):  # the workspace, written while the inputs are read, overlaps one
        assert L.ssd_prefill_local_state(1, 512, 4, 64, 128, 1, 1, x, dt, A, B, hl, ld, inp, 1 << 30, None) == INVALID
    assert ssd.lib().ssd_prefill_local_state_workspace_size(1, 512, 4, 64, 128, 1, 1) > 0
    assert ssd.lib().ssd_prefill_local_state_workspace_size(1, 512, 4, 64, 64, 1, 1) == 0
