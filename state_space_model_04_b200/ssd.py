"""Python binding of libssd_b200.so (argument marshalling only).

Every step of the SSD prefill and decode runs in the library's sm_100a kernels; this
module checks tensor dtypes/devices/shapes, allocates outputs and workspaces with torch
(device memory and streams are the only things torch provides) and forwards raw
pointers to the C ABI declared in include/ssd.h.  There is no CPU fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd_b200.so")

SSD_OK = 0
SSD_F32, SSD_BF16 = 0, 1
SSD_ACT_NONE, SSD_ACT_SILU = 0, 1

_i = ctypes.c_int
_sz = ctypes.c_size_t
_vp = ctypes.c_void_p


class SSDError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__("%s failed: status %d (%s) %s" % (where, status, status_string(status), detail))
        self.status = status


class _KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libssd_b200.so; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libssd_b200.so is not built: run `python -m state_space_model_04_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.ssd_version.restype = _i
        L.ssd_status_string.argtypes = [_i]
        L.ssd_status_string.restype = ctypes.c_char_p
        L.ssd_last_error.restype = ctypes.c_char_p
        L.ssd_prefill_workspace_size.argtypes = [_i] * 8
        L.ssd_prefill_workspace_size.restype = _sz
        L.ssd_prefill.argtypes = [_i] * 8 + [_vp] * 10 + [_sz, _vp]
        L.ssd_prefill.restype = _i
        L.ssd_prefill_dt_raw.argtypes = [_i] * 8 + [_vp] * 3 + [ctypes.c_float] * 2 + [_vp] * 8 + [_sz, _vp]
        L.ssd_prefill_dt_raw.restype = _i
        L.ssd_prefill_check.argtypes = [_vp, _vp]
        L.ssd_prefill_check.restype = _i
        L.ssd_debug_starve_next_prefill.argtypes = [ctypes.c_ulonglong]
        L.ssd_debug_starve_next_prefill.restype = _i
        L.ssd_prefill_local_state_workspace_size.argtypes = [_i] * 7
        L.ssd_prefill_local_state_workspace_size.restype = _sz
        L.ssd_prefill_local_state.argtypes = [_i] * 7 + [_vp] * 7 + [_sz, _vp]
        L.ssd_prefill_local_state.restype = _i
        L.ssd_prefill_context_scan.argtypes = [_i] * 6 + [_vp] * 5
        L.ssd_prefill_context_scan.restype = _i
        L.ssd_prefill_segments.argtypes = [_i] * 8
        L.ssd_prefill_segments.restype = _i
        L.ssd_prefill_whole_units.argtypes = [_i] * 8
        L.ssd_prefill_whole_units.restype = _i
        L.ssd_debug_decay_precision.argtypes = [_i]
        L.ssd_debug_decay_precision.restype = _i
        L.ssd_debug_force_prefill_split.argtypes = [_i, _i]
        L.ssd_debug_force_prefill_split.restype = _i
        L.ssd_debug_force_prefill_segments.argtypes = [_i]
        L.ssd_debug_force_prefill_segments.restype = _i
        L.ssd_debug_force_fma_prefill.argtypes = [_i]
        L.ssd_debug_force_fma_prefill.restype = _i
        L.ssd_decode_workspace_size.argtypes = [_i] * 3
        L.ssd_decode_workspace_size.restype = _sz
        L.ssd_decode_step.argtypes = [_i] * 9 + [_vp] * 10 + [_sz, _vp]
        L.ssd_decode_step.restype = _i
        L.ssd_decode_plan_create.argtypes = [ctypes.POINTER(_vp)] + [_i] * 9 + [_vp] * 4 + [_i] + [_vp] * 5 + [_i, _vp, _sz]
        L.ssd_decode_plan_create.restype = _i
        L.ssd_decode_plan_launch.argtypes = [_vp, _vp]
        L.ssd_decode_plan_launch.restype = _i
        L.ssd_decode_plan_destroy.argtypes = [_vp]
        L.ssd_decode_plan_destroy.restype = _i
        L.ssd_decode_loop.argtypes = [_i] * 9 + [_vp] * 4 + [_i] + [_vp] * 5 + [_i, _vp, _sz, _vp]
        L.ssd_decode_loop.restype = _i
        L.ssd_decode_step_noalloc.argtypes = [_i] * 9 + [_vp] * 10
        L.ssd_decode_step_noalloc.restype = _i
        L.ssd_launch_count.restype = ctypes.c_uint64
        L.ssd_profile_begin.restype = _i
        L.ssd_profile_end.argtypes = [ctypes.POINTER(_KernelTime), _i]
        L.ssd_profile_end.restype = _i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().ssd_status_string(int(status)).decode()


def last_error() -> str:
    return lib().ssd_last_error().decode()


def launch_count() -> int:
    """Kernels the library has enqueued in this process (decode plans count their steps)."""
    return int(lib().ssd_launch_count())


def profile_begin():
    """Start bracketing every library kernel launch with CUDA events on its stream."""
    _check(lib().ssd_profile_begin(), "ssd_profile_begin")


def profile_end(max_entries=64):
    """Stop and return {kernel name: (launches, summed event milliseconds)}."""
    buf = (_KernelTime * max_entries)()
    n = lib().ssd_profile_end(buf, max_entries)
    if n < 0:
        _check(-n, "ssd_profile_end")
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(n)}


def _check_device(device, **tensors):
    """Every tensor of one call must sit on the GPU of its first operand, and that GPU must be
    the current device: the library launches there and its kernels read these pointers
    directly (a tensor on another GPU would be a peer address)."""
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError("%s is on %s, the call's other tensors on %s" % (name, t.device, device))
    if device.type == "cuda" and device.index is not None and device.index != torch.cuda.current_device():
        raise ValueError("the tensors are on %s but the current device is cuda:%d (call under "
                         "torch.cuda.device(...))" % (device, torch.cuda.current_device()))


def _check(status: int, where: str):
    if status != SSD_OK:
        raise SSDError(status, where, last_error())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _io(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    if t.dtype == torch.float32:
        return SSD_F32
    raise TypeError("io tensors must be bfloat16 or float32, got %s" % t.dtype)


def _need(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (no CPU path exists)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    return t


def prefill_workspace_size(b, T, H, P, N, G, chunk, io_dtype) -> int:
    return int(lib().ssd_prefill_workspace_size(b, T, H, P, N, G, chunk, io_dtype))


def prefill(x, dt, A, B, C, D, chunk=256, h0=None, y=None, h_final=None, workspace=None,
            want_final=True, stream=None, check=False, dt_raw=False, dt_bias=None, dt_min=0.0,
            dt_max=float("inf")):
    """Chunked SSD prefill.  Shapes: x [b,T,H,P], dt [b,T,H] f32, A [H] f32,
    B/C [b,T,G,N], D [H] f32, h0 [b,H,P,N] f32 or None.  Returns (y, h_final).
    dt_raw=True passes dt as the raw step (ssd_prefill_dt_raw): the kernels form
    clamp(softplus(dt + dt_bias[h]), dt_min, dt_max) themselves; dt_bias [H] f32 or None.
    check=True synchronises and raises if a device-side wait recorded an error."""
    _need(x, "x")
    io = _io(x)
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _need(dt, "dt", torch.float32, (b, T, H))
    _need(A, "A", torch.float32, (H,))
    _need(D, "D", torch.float32, (H,))
    _need(B, "B", x.dtype, (b, T, G, N))
    _need(C, "C", x.dtype, (b, T, G, N))
    if h0 is not None:
        _need(h0, "h0", torch.float32, (b, H, P, N))
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", x.dtype, x.shape)
    if h_final is None and want_final:
        h_final = torch.empty((b, H, P, N), dtype=torch.float32, device=x.device)
    if h_final is not None:
        _need(h_final, "h_final", torch.float32, (b, H, P, N))
    if dt_bias is not None:
        _need(dt_bias, "dt_bias", torch.float32, (H,))
    need = prefill_workspace_size(b, T, H, P, N, G, chunk, io)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check_device(x.device, dt=dt, A=A, B=B, C=C, D=D, h0=h0, y=y, h_final=h_final, dt_bias=dt_bias,
                  workspace=workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if dt_raw:
        st = lib().ssd_prefill_dt_raw(b, T, H, P, N, G, int(chunk), io, _ptr(x), _ptr(dt), _ptr(dt_bias),
                                      float(dt_min), float(dt_max), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                      _ptr(h0), _ptr(y), _ptr(h_final), _ptr(workspace), ws_bytes,
                                      _stream(stream))
        _check(st, "ssd_prefill_dt_raw")
    else:
        if dt_bias is not None:
            raise ValueError("dt_bias applies to the raw step only (pass dt_raw=True)")
        st = lib().ssd_prefill(b, T, H, P, N, G, int(chunk), io, _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                               _ptr(C), _ptr(D), _ptr(h0), _ptr(y), _ptr(h_final), _ptr(workspace),
                               ws_bytes, _stream(stream))
        _check(st, "ssd_prefill")
    if check and workspace is not None:
        prefill_check(workspace, stream)
    return y, h_final


def prefill_check(workspace, stream=None):
    """Synchronise and raise if the last prefill on `workspace` recorded a device-side error."""
    _check(lib().ssd_prefill_check(_ptr(workspace), _stream(stream)), "ssd_prefill_check")


def debug_starve_next_prefill(wait_limit_s=0.1):
    """Failure-detection test hook: the next tensor-core prefill issues no loads, so its
    bounded waits expire after `wait_limit_s` and prefill_check raises SSD_ERR_TIMEOUT."""
    _check(lib().ssd_debug_starve_next_prefill(int(wait_limit_s * 1e9)), "ssd_debug_starve_next_prefill")


def prefill_local_state(x, dt, A, B, h_local=None, log_decay=None, workspace=None, stream=None):
    """The state these tokens leave when started from zero, and their total log decay
    sum(dt * A), per (sequence, head): returns (h_local [b,H,P,N] f32, log_decay [b,H] f32).
    x [b,T,H,P] bf16, dt [b,T,H] f32, A [H] f32, B [b,T,G,N] bf16 (ssd_prefill_local_state)."""
    _need(x, "x", torch.bfloat16)
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _need(dt, "dt", torch.float32, (b, T, H))
    _need(A, "A", torch.float32, (H,))
    _need(B, "B", x.dtype, (b, T, G, N))
    if h_local is None:
        h_local = torch.empty((b, H, P, N), dtype=torch.float32, device=x.device)
    if log_decay is None:
        log_decay = torch.empty((b, H), dtype=torch.float32, device=x.device)
    _need(h_local, "h_local", torch.float32, (b, H, P, N))
    _need(log_decay, "log_decay", torch.float32, (b, H))
    need = int(lib().ssd_prefill_local_state_workspace_size(b, T, H, P, N, G, SSD_BF16))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check_device(x.device, dt=dt, A=A, B=B, h_local=h_local, log_decay=log_decay, workspace=workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().ssd_prefill_local_state(b, T, H, P, N, G, SSD_BF16, _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                       _ptr(h_local), _ptr(log_decay), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "ssd_prefill_local_state")
    return h_local, log_decay


def prefill_context_scan(rank, h_local_all, log_decay_all, h0=None, h_in=None, stream=None):
    """State entering context shard `rank` from the rank-major gathered local states
    [world,b,H,P,N] and log decays [world,b,H] (ssd_prefill_context_scan)."""
    world, b, H, P, N = h_local_all.shape
    _need(h_local_all, "h_local_all", torch.float32)
    _need(log_decay_all, "log_decay_all", torch.float32, (world, b, H))
    if h0 is not None:
        _need(h0, "h0", torch.float32, (b, H, P, N))
    if h_in is None:
        h_in = torch.empty((b, H, P, N), dtype=torch.float32, device=h_local_all.device)
    _need(h_in, "h_in", torch.float32, (b, H, P, N))
    _check_device(h_local_all.device, log_decay_all=log_decay_all, h0=h0, h_in=h_in)
    st = lib().ssd_prefill_context_scan(world, int(rank), b, H, P, N, _ptr(h0), _ptr(h_local_all),
                                        _ptr(log_decay_all), _ptr(h_in), _stream(stream))
    _check(st, "ssd_prefill_context_scan")
    return h_in


def prefill_segments(b, T, H, P, N, G, chunk, io_dtype) -> int:
    """Segments per sequence ssd_prefill uses for this shape (1 = one pass; 0 = invalid)."""
    return int(lib().ssd_prefill_segments(b, T, H, P, N, G, chunk, io_dtype))


def prefill_whole_units(b, T, H, P, N, G, chunk, io_dtype) -> int:
    """(Sequence, head) pairs ssd_prefill runs whole for this shape (-1 = invalid); the rest
    are split into prefill_segments(...) segments each."""
    return int(lib().ssd_prefill_whole_units(b, T, H, P, N, G, chunk, io_dtype))


def debug_decay_precision(mode=0):
    """Decay-precision ablation of the tensor-core prefill: 0 fp32 (default), 1 exponentiated
    decay factors rounded to bf16, 2 log-space prefix sums rounded to bf16 before exp."""
    _check(lib().ssd_debug_decay_precision(int(mode)), "ssd_debug_decay_precision")


def debug_force_prefill_split(n_full, nseg):
    """Test hook: the first n_full (sequence, head) units run whole, the rest are split into
    nseg segments (nseg = 0: the cost model)."""
    _check(lib().ssd_debug_force_prefill_split(int(n_full), int(nseg)), "ssd_debug_force_prefill_split")


def debug_force_fma_prefill(on=False):
    """Measurement hook: route every following prefill through the fp32-FMA path, which uses
    the chunk length as given (the tensor-core kernel always evaluates 128-token chunks)."""
    _check(lib().ssd_debug_force_fma_prefill(1 if on else 0), "ssd_debug_force_fma_prefill")


def debug_force_prefill_segments(nseg=0):
    """Test hook: split every following tensor-core prefill into `nseg` sequence segments
    (0 = let the cost model choose)."""
    _check(lib().ssd_debug_force_prefill_segments(int(nseg)), "ssd_debug_force_prefill_segments")


def decode_workspace_size(layers, b, G) -> int:
    return int(lib().ssd_decode_workspace_size(layers, b, G))


def _decode_shapes(h, conv_state, A, D, conv_w, conv_b, G):
    _need(h, "h", torch.float32)
    layers, b, H, P, N = h.shape
    k = conv_w.shape[-1]
    Dc = H * P + 2 * G * N
    _need(conv_state, "conv_state", torch.float32, (layers, b, Dc, k - 1))
    _need(A, "A", torch.float32, (layers, H))
    _need(D, "D", torch.float32, (layers, H))
    _need(conv_w, "conv_w", torch.float32, (layers, Dc, k))
    _need(conv_b, "conv_b", torch.float32, (layers, Dc))
    return layers, b, H, P, N, k, Dc


def decode_step(h, conv_state, xbc, dt, A, D, conv_w, conv_b, G=1, act=SSD_ACT_SILU, y=None,
                workspace=None, stream=None):
    """One decode step for all layers; h and conv_state are updated in place.  Returns y."""
    layers, b, H, P, N, k, Dc = _decode_shapes(h, conv_state, A, D, conv_w, conv_b, G)
    _need(xbc, "xbc", None, (layers, b, Dc))
    io = _io(xbc)
    _need(dt, "dt", torch.float32, (layers, b, H))
    if y is None:
        y = torch.empty((layers, b, H, P), dtype=xbc.dtype, device=h.device)
    _need(y, "y", xbc.dtype, (layers, b, H, P))
    if workspace is None:
        workspace = torch.empty(decode_workspace_size(layers, b, G), dtype=torch.uint8, device=h.device)
    _check_device(h.device, conv_state=conv_state, xbc=xbc, dt=dt, A=A, D=D, conv_w=conv_w, conv_b=conv_b, y=y,
                  workspace=workspace)
    st = lib().ssd_decode_step(layers, b, H, P, N, G, k, act, io, _ptr(h), _ptr(conv_state), _ptr(xbc),
                               _ptr(dt), _ptr(A), _ptr(D), _ptr(conv_w), _ptr(conv_b), _ptr(y),
                               _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "ssd_decode_step")
    return y


def decode_step_noalloc(h, conv_state, xbc, dt, A, D, conv_w, conv_b, y, G=1, act=SSD_ACT_SILU,
                        stream=None):
    """decode_step through ssd_decode_step_noalloc: no workspace, and the caller passes
    the output y, so nothing is allocated on this path (for callers that cannot allocate
    device memory).  Calls that overlap on the GPU race on the library's shared scratch."""
    layers, b, H, P, N, k, Dc = _decode_shapes(h, conv_state, A, D, conv_w, conv_b, G)
    _need(xbc, "xbc", None, (layers, b, Dc))
    io = _io(xbc)
    _need(dt, "dt", torch.float32, (layers, b, H))
    _need(y, "y", xbc.dtype, (layers, b, H, P))
    _check_device(h.device, conv_state=conv_state, xbc=xbc, dt=dt, A=A, D=D, conv_w=conv_w, conv_b=conv_b, y=y)
    st = lib().ssd_decode_step_noalloc(layers, b, H, P, N, G, k, act, io, _ptr(h), _ptr(conv_state),
                                       _ptr(xbc), _ptr(dt), _ptr(A), _ptr(D), _ptr(conv_w), _ptr(conv_b),
                                       _ptr(y), _stream(stream))
    _check(st, "ssd_decode_step_noalloc")
    return y


class DecodePlan:
    """n_steps decode steps recorded once as a CUDA graph; launch() runs them all on the
    device with no host round trip.  Step t reads xbc_ring[t % ring], dt_ring[t % ring]
    and writes y_ring[t % ring].  The plan holds references to every tensor it uses."""

    def __init__(self, h, conv_state, xbc_ring, dt_ring, A, D, conv_w, conv_b, n_steps, G=1,
                 act=SSD_ACT_SILU, y_ring=None):
        layers, b, H, P, N, k, Dc = _decode_shapes(h, conv_state, A, D, conv_w, conv_b, G)
        ring = xbc_ring.shape[0]
        _need(xbc_ring, "xbc_ring", None, (ring, layers, b, Dc))
        io = _io(xbc_ring)
        _need(dt_ring, "dt_ring", torch.float32, (ring, layers, b, H))
        if y_ring is None:
            y_ring = torch.empty((ring, layers, b, H, P), dtype=xbc_ring.dtype, device=h.device)
        _need(y_ring, "y_ring", xbc_ring.dtype, (ring, layers, b, H, P))
        _check_device(h.device, conv_state=conv_state, xbc_ring=xbc_ring, dt_ring=dt_ring, A=A, D=D,
                      conv_w=conv_w, conv_b=conv_b, y_ring=y_ring)
        self.workspace = torch.empty(decode_workspace_size(layers, b, G), dtype=torch.uint8, device=h.device)
        self._keep = (h, conv_state, xbc_ring, dt_ring, A, D, conv_w, conv_b, y_ring)
        self.y_ring = y_ring
        self.n_steps = n_steps
        handle = ctypes.c_void_p()
        st = lib().ssd_decode_plan_create(ctypes.byref(handle), layers, b, H, P, N, G, k, act, io,
                                          _ptr(h), _ptr(conv_state), _ptr(xbc_ring), _ptr(dt_ring), ring,
                                          _ptr(A), _ptr(D), _ptr(conv_w), _ptr(conv_b), _ptr(y_ring),
                                          int(n_steps), _ptr(self.workspace), self.workspace.numel())
        _check(st, "ssd_decode_plan_create")
        self._h = handle

    def launch(self, stream=None):
        if self._h is None:
            raise RuntimeError("plan destroyed")
        _check(lib().ssd_decode_plan_launch(self._h, _stream(stream)), "ssd_decode_plan_launch")
        return self.y_ring

    def close(self):
        if getattr(self, "_h", None) is not None:
            _check(lib().ssd_decode_plan_destroy(self._h), "ssd_decode_plan_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def decode_loop(h, conv_state, xbc_ring, dt_ring, A, D, conv_w, conv_b, n_steps, G=1,
                act=SSD_ACT_SILU, stream=None):
    """Run n_steps decode steps as one graph launch (ssd_decode_loop: plan built, launched,
    released, no host synchronisation inside).  Returns y_ring [ring, layers, b, H, P]; the
    call waits for the launch before returning because its workspace is a temporary."""
    layers, b, H, P, N, k, Dc = _decode_shapes(h, conv_state, A, D, conv_w, conv_b, G)
    ring = xbc_ring.shape[0]
    _need(xbc_ring, "xbc_ring", None, (ring, layers, b, Dc))
    io = _io(xbc_ring)
    _need(dt_ring, "dt_ring", torch.float32, (ring, layers, b, H))
    _check_device(h.device, conv_state=conv_state, xbc_ring=xbc_ring, dt_ring=dt_ring, A=A, D=D,
                  conv_w=conv_w, conv_b=conv_b)
    y_ring = torch.empty((ring, layers, b, H, P), dtype=xbc_ring.dtype, device=h.device)
    ws = torch.empty(decode_workspace_size(layers, b, G), dtype=torch.uint8, device=h.device)
    st = lib().ssd_decode_loop(layers, b, H, P, N, G, k, act, io, _ptr(h), _ptr(conv_state), _ptr(xbc_ring),
                               _ptr(dt_ring), ring, _ptr(A), _ptr(D), _ptr(conv_w), _ptr(conv_b), _ptr(y_ring),
                               int(n_steps), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "ssd_decode_loop")
    torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
    return y_ring
