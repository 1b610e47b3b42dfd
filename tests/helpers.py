"""Shared helpers for the GPU parity tests: device copies of seeded cases, oracle runs on
sampled (sequence, head) subsets, and the tolerance metrics.

Tolerances ("Compiler-First State Space Duality ..." validates fp32 against a reference
at float32 rounding scale; the bf16 bar normalises by the largest output):
  fp32 inputs : max_i |d_i| / max(|ref_i|, 1e-2 * max|ref|) <= 1e-4   (element-wise with a
                floor: each output is a sum of products whose terms reach max|ref|, so an
                output that cancels to ~0 still carries an absolute rounding error of a few
                fp32 ulps of max|ref|; the floor allows 1e-6 * max|ref|, about 8 ulps, there)
  bf16 inputs : max |d| / max |ref| <= 2e-2
The same metrics apply to y and to the final / decode state.
"""
import numpy as np
import torch

import oracle

TOL_F32 = 1e-4
F32_FLOOR = 1e-2
TOL_BF16 = 2e-2


def rel_max(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


def rel_floor(got, ref, floor=F32_FLOOR):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.maximum(np.abs(ref), floor * np.abs(ref).max())
    return float((np.abs(got - ref) / np.maximum(den, 1e-300)).max())


def check(got, ref, dtype, what=""):
    """Assert the tolerance for this io dtype; returns the error for reporting."""
    if dtype == "f32":
        e = rel_floor(got, ref)
        assert e <= TOL_F32, "%s: fp32 error %.3e > %.1e (plain max-normalised %.3e)" % (what, e, TOL_F32, rel_max(got, ref))
    else:
        e = rel_max(got, ref)
        assert e <= TOL_BF16, "%s: bf16 error %.3e > %.1e" % (what, e, TOL_BF16)
    return e


def bf16_tensor(bits, dev="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)


def f32_tensor(a, dev="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


def prefill_inputs(case, dev="cuda"):
    """Device tensors for a PrefillCase (bf16 payloads bit-exact with the oracle's view)."""
    if case.dtype == "bf16":
        x, B, C = bf16_tensor(case.x_bits, dev), bf16_tensor(case.B_bits, dev), bf16_tensor(case.C_bits, dev)
    else:
        x, B, C = f32_tensor(case.x, dev), f32_tensor(case.B, dev), f32_tensor(case.C, dev)
    h0 = None if case.h0 is None else f32_tensor(case.h0, dev)
    return dict(x=x, dt=f32_tensor(case.dt, dev), A=f32_tensor(case.A, dev), B=B, C=C,
                D=f32_tensor(case.D, dev), h0=h0)


def oracle_subset(case, seqs, heads, nthreads=0):
    """Oracle recurrence on a (sequence x head) subset.  Heads are independent, so each
    chosen head is run as its own group with its group's B and C."""
    seqs = list(seqs)
    heads = list(heads)
    hpg = case.H // case.G
    groups = [h // hpg for h in heads]
    x = case.x[seqs][:, :, heads]
    dt = case.dt[seqs][:, :, heads]
    B = case.B[seqs][:, :, groups]
    C = case.C[seqs][:, :, groups]
    h0 = None if case.h0 is None else case.h0[seqs][:, heads]
    return oracle.ssd_recurrence(x, dt, case.A[heads], B, C, case.D[heads], h0, nthreads=nthreads)


def run_prefill(ssd, case, chunk=None, **kw):
    t = prefill_inputs(case)
    kw.setdefault("check", True)
    y, hf = ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=chunk or case.L,
                        h0=t["h0"], **kw)
    torch.cuda.synchronize()
    return y, hf, t
