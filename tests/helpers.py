"""Shared helpers for the GPU parity tests: device copies of seeded cases, oracle runs on
sampled (sequence, head) subsets, and the tolerance metrics.

Tolerances ("Compiler-First State Space Duality ..." validates fp32 against a reference
at float32 rounding scale; the bf16 bar normalises by the largest output):
  fp32 inputs : per element, |d_i| <= 1e-4 * |ref_i| + 16 * eps32 * mag_i, where mag_i is
                the sum of the absolute values of the products behind output i (from the
                oracle: oracle.ssd_magnitudes, oracle.decode_step_mag) and eps32 = 2^-23.
                An output is a sum of products; evaluated in fp32 it carries a rounding
                error of a few ulps of that sum of magnitudes, which stays the same when the
                output itself cancels to near zero.  The second term is that allowance (16
                machine epsilons of the term scale); everywhere else the 1e-4 relative bound
                decides.  The reported error is the largest ratio |d_i| / bound_i (<= 1).
  bf16 inputs : max |d| / max |ref| <= 2e-2
The same metrics apply to y and to the final / decode state.
"""
import numpy as np
import torch

import oracle

TOL_F32 = 1e-4
EPS32 = 2.0 ** -23
MAG_EPS = 16
TOL_BF16 = 2e-2


def rel_max(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


def f32_bound_ratio(got, ref, mag, sides=1):
    """Largest |got_i - ref_i| / (sides * (1e-4 |ref_i| + 16 eps32 mag_i)).  sides = 2 when
    both operands are computed results (each carries its own rounding)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    mag = np.broadcast_to(np.asarray(mag, np.float64), ref.shape)
    bound = sides * (TOL_F32 * np.abs(ref) + MAG_EPS * EPS32 * mag)
    return float((np.abs(got - ref) / np.maximum(bound, 1e-300)).max())


def check(got, ref, dtype, what="", mag=None, sides=1):
    """Assert the tolerance for this io dtype; returns the error for reporting.  fp32 needs
    ``mag``, the term magnitudes of ``ref`` (see the module docstring)."""
    if dtype == "f32":
        if mag is None:
            raise ValueError("%s: an fp32 check needs the oracle's term magnitudes" % what)
        e = f32_bound_ratio(got, ref, mag, sides)
        assert e <= 1.0, "%s: fp32 error %.3f of the per-element bound (plain max-normalised %.3e)" % (
            what, e, rel_max(got, ref))
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


def oracle_subset_mag(case, seqs, heads, nthreads=0):
    """Term magnitudes (oracle.ssd_magnitudes) on the same subset as oracle_subset."""
    seqs = list(seqs)
    heads = list(heads)
    hpg = case.H // case.G
    groups = [h // hpg for h in heads]
    x = case.x[seqs][:, :, heads]
    dt = case.dt[seqs][:, :, heads]
    B = case.B[seqs][:, :, groups]
    C = case.C[seqs][:, :, groups]
    h0 = None if case.h0 is None else case.h0[seqs][:, heads]
    return oracle.ssd_magnitudes(x, dt, case.A[heads], B, C, case.D[heads], h0, nthreads=nthreads)


def run_prefill(ssd, case, chunk=None, **kw):
    t = prefill_inputs(case)
    kw.setdefault("check", True)
    y, hf = ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=chunk or case.L,
                        h0=t["h0"], **kw)
    torch.cuda.synchronize()
    return y, hf, t
