"""fp64 CPU oracle for the Mamba-2 SSD hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product (``state_space_model_04_b200`` and its sm_100a kernels)
never imports it, shares no code with it and has no CPU fallback.

The arithmetic lives in ``ssd_oracle.c`` (plain C, double precision, OpenMP over
independent (batch, head) or (layer, batch) pairs); this module only marshals numpy
arrays into it.  Every function follows "Compiler-First State Space Duality and Portable
O(1) Autoregressive Caching" (arXiv 2603.09555): the discretised recurrence (Eq. 2), the
chunked dual form (Eq. 3 and the "Chunked recurrence" property) and the O(1) cache
section (depthwise conv over k-1 cached inputs plus one recurrence step).

Pins (tests/test_oracle_pins.py) tie it to closed forms, hand-derived worked examples
(tests/golden/), brute force on tiny inputs and the invariants the pages state; the only
function without an outside pin is the full-size prefill, which is pinned by the same
code on small sizes plus those invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile ssd_oracle.c into libssd_oracle.so with gcc (-O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i = ctypes.c_int
        lib.oracle_ssd_recurrence.argtypes = [i] * 6 + [_dp] * 9 + [i]
        lib.oracle_ssd_chunked.argtypes = [i] * 7 + [_dp] * 9 + [i]
        lib.oracle_ssd_quadratic.argtypes = [i] * 6 + [_dp] * 9 + [i]
        lib.oracle_decode_step.argtypes = [i] * 8 + [_dp] * 9 + [i]
        lib.oracle_decode_step_mag.argtypes = [i] * 8 + [_dp] * 9 + [i]
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_dt_from_raw.argtypes = [ctypes.c_size_t, i, _dp, _dp, ctypes.c_double, ctypes.c_double, _dp]
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _c(a):
    """Contiguous float64 copy (the oracle reads the exact values the GPU sees)."""
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    return a.ctypes.data_as(_dp) if a is not None else None


def _prefill(fn, x, dt, A, B, C, D, h0, L=None, nthreads=0):
    x, dt, A, B, C, D = map(_c, (x, dt, A, B, C, D))
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (b, T, H) and A.shape == (H,) and D.shape == (H,)
    assert B.shape == (b, T, G, N) and C.shape == (b, T, G, N) and H % G == 0
    h0c = _c(h0) if h0 is not None else None
    if h0c is not None:
        assert h0c.shape == (b, H, P, N)
    y = np.zeros((b, T, H, P), np.float64)
    hf = np.zeros((b, H, P, N), np.float64)
    args = [b, T, H, P, N, G] + ([L] if L is not None else [])
    args += [_p(x), _p(dt), _p(A), _p(B), _p(C), _p(D), _p(h0c), _p(y), _p(hf), int(nthreads)]
    fn(*args)
    return y, hf


def ssd_recurrence(x, dt, A, B, C, D, h0=None, nthreads=0):
    """Token-by-token recurrence (the definition).  Returns (y, h_final) in float64."""
    return _prefill(_load().oracle_ssd_recurrence, x, dt, A, B, C, D, h0, None, nthreads)


def ssd_chunked(x, dt, A, B, C, D, L, h0=None, nthreads=0):
    """Naive chunked dual form with chunk length L (L must divide T)."""
    assert x.shape[1] % L == 0
    return _prefill(_load().oracle_ssd_chunked, x, dt, A, B, C, D, h0, int(L), nthreads)


def ssd_quadratic(x, dt, A, B, C, D, h0=None, nthreads=0):
    """Whole-sequence quadratic form (one chunk of length T, direct segment sums)."""
    return _prefill(_load().oracle_ssd_quadratic, x, dt, A, B, C, D, h0, None, nthreads)


def ssd_magnitudes(x, dt, A, B, C, D, h0=None, nthreads=0):
    """Sum of the absolute values of the terms behind every output of the prefill, (y_mag,
    h_final_mag) in float64: the scale of the rounding error an evaluation of the outputs
    in a given precision carries, used for per-element fp32 tolerances.

    Each output of the recurrence (Eq. 2 with readings R1, R4, R5 of ssd_oracle.c) expands
    into a sum of products:
      y_t[p]  = sum_n C_t[n] (prod_{s<=t} alpha_s h0[p][n]
                              + sum_{s<=t} prod_{s<r<=t} alpha_r dt_s x_s[p] B_s[n]) + D x_t[p]
    and every decay factor alpha = exp(dt*A) and every dt is positive, so the sum of the
    absolute values of those products is the same recurrence run on |x|, |B|, |C|, |D| and
    |h0|.  That is how it is evaluated here."""
    def a(v):
        return None if v is None else np.abs(np.asarray(v, dtype=np.float64))
    return ssd_recurrence(a(x), dt, A, a(B), a(C), a(D), a(h0), nthreads=nthreads)


def decode_step_mag(h_mag, conv_state, xbc, dt, A, D, conv_w, conv_b, act, G, N, nthreads=0):
    """Term magnitudes of one decode step (see oracle_decode_step_mag in ssd_oracle.c).
    ``h_mag`` [layers,b,H,P,N] float64 is updated in place (start it from |h|); conv_state
    is the window BEFORE the step (call this ahead of decode_step).  Returns y_mag
    [layers,b,H,P]."""
    assert h_mag.dtype == np.float64 and h_mag.flags.c_contiguous
    layers, b, H, P, Nn = h_mag.shape
    assert Nn == N
    k = conv_w.shape[2]
    Dc = H * P + 2 * G * N
    cs = _c(conv_state)
    assert cs.shape == (layers, b, Dc, k - 1)
    xbc, dt, A, D, conv_w, conv_b = map(_c, (xbc, dt, A, D, conv_w, conv_b))
    ym = np.zeros((layers, b, H, P), np.float64)
    _load().oracle_decode_step_mag(layers, b, H, P, N, G, k, int(act), _p(h_mag), _p(cs), _p(xbc), _p(dt),
                                   _p(A), _p(D), _p(conv_w), _p(conv_b), _p(ym), int(nthreads))
    return ym


def dt_from_raw(dt_raw, dt_bias=None, dt_min=0.0, dt_max=float("inf")):
    """Step sizes from the raw projection output: clamp(softplus(dt_raw + dt_bias[h]),
    dt_min, dt_max) in float64 (the Mamba-2 block's pre-processing of dt, which the paper's
    compiled graph fuses ahead of the SSD).  dt_raw [..., H]; returns float64 of the same shape."""
    L = _load()
    raw = _c(dt_raw)
    H = raw.shape[-1]
    bias = None if dt_bias is None else _c(dt_bias)
    out = np.empty_like(raw)
    L.oracle_dt_from_raw(raw.size, H, _p(raw), _p(bias), dt_min, dt_max, _p(out))
    return out


def decode_step(h, conv_state, xbc, dt, A, D, conv_w, conv_b, act, G, N, nthreads=0):
    """One decode step over every layer, updating ``h`` and ``conv_state`` IN PLACE.

    h [layers,b,H,P,N] float64 (modified), conv_state [layers,b,Dc,k-1] float64
    (modified), xbc [layers,b,Dc], dt [layers,b,H], A, D [layers,H],
    conv_w [layers,Dc,k], conv_b [layers,Dc].  Returns y [layers,b,H,P].
    """
    assert h.dtype == np.float64 and h.flags.c_contiguous
    assert conv_state.dtype == np.float64 and conv_state.flags.c_contiguous
    layers, b, H, P, Nn = h.shape
    assert Nn == N
    k = conv_w.shape[2]
    Dc = H * P + 2 * G * N
    assert conv_state.shape == (layers, b, Dc, k - 1)
    xbc, dt, A, D, conv_w, conv_b = map(_c, (xbc, dt, A, D, conv_w, conv_b))
    assert xbc.shape == (layers, b, Dc) and dt.shape == (layers, b, H)
    assert A.shape == (layers, H) and D.shape == (layers, H)
    assert conv_w.shape == (layers, Dc, k) and conv_b.shape == (layers, Dc)
    y = np.zeros((layers, b, H, P), np.float64)
    _load().oracle_decode_step(layers, b, H, P, N, G, k, int(act), _p(h), _p(conv_state),
                               _p(xbc), _p(dt), _p(A), _p(D), _p(conv_w), _p(conv_b),
                               _p(y), int(nthreads))
    return y
