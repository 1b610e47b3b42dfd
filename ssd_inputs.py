"""Seeded synthetic inputs for the SSD prefill and decode workloads.

This module is shared by the tests, the benchmark and the smoke check: it is the ONLY code
both the CPU oracle and the CUDA path see, and it holds none of the method's arithmetic.
It draws random numbers, rounds them to the storage dtype and lays them out.

Input recipe (the workloads of "Compiler-First State Space Duality and Portable O(1)
Autoregressive Caching", arXiv 2603.09555; the five configurations below fix shapes and
distributions, the pages' models fix H*P, N, conv width 4 and chunk 256):
  A_h     = -exp(U(ln 1, ln 16))                       fp32, one per head
  dt_bias = softplus^-1(exp(U(ln 1e-3, ln 1e-1)))      one per head
  dt      = softplus(0.5 * N(0,1) + dt_bias_h)         fp32 (already positive)
  x, B, C ~ N(0, 1)                                    rounded to bf16 (RNE) or kept fp32
  D_h     = 1;  h0 = 0, or N(0, 0.1^2) where a configuration asks for a random state
Draw order with numpy default_rng(seed): A, dt_bias, dt noise, x, B, C, h0.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def bf16_round(a: np.ndarray):
    """Round float32 values to bfloat16 (round-to-nearest-even).

    Returns (values as float32 holding exact bf16 numbers, raw uint16 bf16 bits).
    Inputs are finite normal draws, so NaN handling is not needed.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    bits = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16))
    bits = bits.astype(np.uint16)
    vals = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return vals, bits


def _softplus(z):
    return np.logaddexp(0.0, z)


def _inv_softplus(v):
    return np.log(np.expm1(v))


@dataclass
class PrefillCase:
    """One prefill problem.  Arrays are numpy; *_bits are uint16 bf16 payloads (or None)."""
    b: int
    T: int
    H: int
    P: int
    N: int
    G: int
    L: int
    dtype: str            # "bf16" or "f32"
    x: np.ndarray         # float32 values (exact bf16 numbers when dtype == "bf16")
    dt: np.ndarray        # float32 [b,T,H]
    A: np.ndarray         # float32 [H]
    B: np.ndarray         # float32 [b,T,G,N]
    C: np.ndarray         # float32 [b,T,G,N]
    D: np.ndarray         # float32 [H]
    h0: np.ndarray | None  # float32 [b,H,P,N] or None (zero state)
    x_bits: np.ndarray | None = None
    B_bits: np.ndarray | None = None
    C_bits: np.ndarray | None = None


# name -> (b, T, H, P, N, G, L, dtype, h0_std, seed)
PREFILL_CONFIGS = {
    "tiny_f32": (1, 512, 4, 64, 64, 1, 256, "f32", 0.0, 0),
    "mamba2_130m_layer": (1, 4096, 24, 64, 128, 1, 256, "bf16", 0.0, 1),
    "mamba2_2p7b_layer": (8, 4096, 80, 64, 128, 1, 256, "bf16", 0.1, 2),
    "long_context_L64": (1, 65536, 80, 64, 128, 8, 64, "bf16", 0.0, 4),
    "long_context_L128": (1, 65536, 80, 64, 128, 8, 128, "bf16", 0.0, 4),
    "long_context_L256": (1, 65536, 80, 64, 128, 8, 256, "bf16", 0.0, 4),
}


def head_params(rng, H):
    """A (negative, per head) and dt_bias, drawn in that order."""
    A = -np.exp(rng.uniform(np.log(1.0), np.log(16.0), size=H))
    dt_bias = _inv_softplus(np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), size=H)))
    return A.astype(np.float32), dt_bias


def make_prefill(b, T, H, P, N, G, L, dtype="bf16", h0_std=0.0, seed=0,
                 dt_scale=1.0) -> PrefillCase:
    """Draw one prefill problem with the recipe in the module docstring.

    ``dt_scale`` multiplies dt after the draw (1.0 = the recipe); tests use it to
    build strong- or weak-decay edge cases.
    """
    assert H % G == 0
    rng = np.random.default_rng(seed)
    A, dt_bias = head_params(rng, H)
    z = rng.standard_normal((b, T, H), dtype=np.float32)
    dt = (_softplus(0.5 * z.astype(np.float64) + dt_bias[None, None, :]) * dt_scale).astype(np.float32)
    x = rng.standard_normal((b, T, H, P), dtype=np.float32)
    Bm = rng.standard_normal((b, T, G, N), dtype=np.float32)
    Cm = rng.standard_normal((b, T, G, N), dtype=np.float32)
    h0 = None
    if h0_std > 0:
        h0 = (rng.standard_normal((b, H, P, N), dtype=np.float32) * np.float32(h0_std)).astype(np.float32)
    D = np.ones(H, np.float32)
    xb = Bb = Cb = None
    if dtype == "bf16":
        x, xb = bf16_round(x)
        Bm, Bb = bf16_round(Bm)
        Cm, Cb = bf16_round(Cm)
    elif dtype != "f32":
        raise ValueError(dtype)
    return PrefillCase(b, T, H, P, N, G, L, dtype, x, dt, A, Bm, Cm, D, h0, xb, Bb, Cb)


def make_config(name: str, **over) -> PrefillCase:
    b, T, H, P, N, G, L, dtype, h0_std, seed = PREFILL_CONFIGS[name]
    kw = dict(b=b, T=T, H=H, P=P, N=N, G=G, L=L, dtype=dtype, h0_std=h0_std, seed=seed)
    kw.update(over)
    return make_prefill(**kw)


@dataclass
class DecodeCase:
    """Decode workload: per-layer parameters, initial caches and a ring of step inputs."""
    layers: int
    b: int
    H: int
    P: int
    N: int
    G: int
    k: int
    ring: int
    A: np.ndarray        # float32 [layers,H]
    D: np.ndarray        # float32 [layers,H]
    conv_w: np.ndarray   # float32 [layers,Dc,k]
    conv_b: np.ndarray   # float32 [layers,Dc]
    h: np.ndarray        # float32 [layers,b,H,P,N]   initial SSM state
    conv_state: np.ndarray  # float32 [layers,b,Dc,k-1] initial conv window
    xbc: np.ndarray      # float32 [ring,layers,b,Dc] (exact bf16 numbers)
    xbc_bits: np.ndarray  # uint16  [ring,layers,b,Dc]
    dt: np.ndarray       # float32 [ring,layers,b,H]

    @property
    def Dc(self):
        return self.H * self.P + 2 * self.G * self.N


def make_decode(layers, b, H, P, N, G, k=4, ring=8, seed=3, h_std=0.1,
                conv_state_std=1.0) -> DecodeCase:
    """Seeded decode workload.

    Per layer, A and dt_bias follow the prefill recipe; D = 1; conv weights and biases
    ~ U(-0.5, 0.5) (1/sqrt(fan_in) for fan_in = k = 4).  The initial SSM state is
    N(0, h_std^2) and the conv window N(0, conv_state_std^2); the benchmark replaces the
    SSM state with the final state of a prefill.  Step inputs: xbc ~ N(0,1) in bf16 over
    Dc = H*P + 2*G*N channels and dt = softplus(0.5*N(0,1) + dt_bias), ``ring`` steps.
    Draw order: per layer (A, dt_bias); conv_w; conv_b; h; conv_state; xbc; dt noise.
    """
    rng = np.random.default_rng(seed)
    Dc = H * P + 2 * G * N
    A, D, conv_w, conv_b, dt_bias = _decode_params(rng, layers, H, P, N, G, k)
    h = (rng.standard_normal((layers, b, H, P, N), dtype=np.float32) * np.float32(h_std)).astype(np.float32)
    cs = (rng.standard_normal((layers, b, Dc, k - 1), dtype=np.float32) * np.float32(conv_state_std)).astype(np.float32)
    xbc, bits = bf16_round(rng.standard_normal((ring, layers, b, Dc), dtype=np.float32))
    z = rng.standard_normal((ring, layers, b, H), dtype=np.float32).astype(np.float64)
    dt = _softplus(0.5 * z + dt_bias[None, :, None, :]).astype(np.float32)
    return DecodeCase(layers, b, H, P, N, G, k, ring, A, D, conv_w, conv_b, h, cs, xbc, bits, dt)


def _decode_params(rng, layers, H, P, N, G, k):
    Dc = H * P + 2 * G * N
    A = np.empty((layers, H), np.float32)
    dt_bias = np.empty((layers, H), np.float64)
    for l in range(layers):
        A[l], dt_bias[l] = head_params(rng, H)
    conv_w = rng.uniform(-0.5, 0.5, size=(layers, Dc, k)).astype(np.float32)
    conv_b = rng.uniform(-0.5, 0.5, size=(layers, Dc)).astype(np.float32)
    D = np.ones((layers, H), np.float32)
    return A, D, conv_w, conv_b, dt_bias


def make_decode_params(layers, H, P, N, G, k=4, seed=3):
    """Per-layer A, D, conv weights/bias and dt_bias: the first draws of make_decode."""
    return _decode_params(np.random.default_rng(seed), layers, H, P, N, G, k)


def make_decode_ring_device(ring, layers, b, H, P, N, G, dt_bias, seed, device):
    """Large decode step-input rings drawn on the device with a seeded torch generator
    (same distributions as make_decode): xbc ~ N(0,1) in bf16, dt = softplus(0.5 z +
    dt_bias).  Used where host generation of gigabytes would dominate the run."""
    import torch
    gen = torch.Generator(device=device).manual_seed(seed)
    Dc = H * P + 2 * G * N
    xbc = torch.randn((ring, layers, b, Dc), generator=gen, device=device).to(torch.bfloat16)
    z = torch.randn((ring, layers, b, H), generator=gen, device=device)
    bias = torch.as_tensor(dt_bias, dtype=torch.float32, device=device)[None, :, None, :]
    dt = torch.nn.functional.softplus(0.5 * z + bias).contiguous()
    return xbc, dt
