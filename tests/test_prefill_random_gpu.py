"""Randomised GPU parity sweep of ssd_prefill against the fp64 oracle.

Each case draws, from its own fixed seed, a batch of 1-3 sequences of 1-900 tokens (ragged
against every block and chunk length), 2-8 heads in 1-H groups, N = 64 or 128, bf16 or
fp32, chunk 64/128/256, a forced segment count (automatic, 1, 2 or 5) and a zero or random
initial state, and compares y and h_final with the oracle within the dtype's bound.  The
draws cover the fused tensor-core path (bf16, N = 128) with and without sequence splits,
and the fp32-FMA path (fp32 or N = 64).
"""
import numpy as np
import pytest
import torch

from ssd_inputs import make_prefill
from tests.helpers import check, oracle_subset, oracle_subset_mag, run_prefill

pytestmark = pytest.mark.gpu

ssd = pytest.importorskip("state_space_model_04_b200")


def _draw(seed):
    rng = np.random.default_rng(1000 + seed)
    H = int(rng.choice([2, 4, 6, 8]))
    G = int(rng.choice([g for g in range(1, H + 1) if H % g == 0]))
    return dict(b=int(rng.integers(1, 4)), T=int(rng.integers(1, 901)), H=H, G=G,
                N=int(rng.choice([64, 128, 128])), dtype=str(rng.choice(["bf16", "bf16", "f32"])),
                chunk=int(rng.choice([64, 128, 256])), nseg=int(rng.choice([0, 1, 2, 5])),
                h0_std=float(rng.choice([0.0, 0.1])))


@pytest.mark.parametrize("seed", range(24))
def test_random_prefill_matches_oracle(seed):
    d = _draw(seed)
    case = make_prefill(d["b"], d["T"], d["H"], 64, d["N"], d["G"], d["chunk"], d["dtype"], h0_std=d["h0_std"],
                        seed=500 + seed)
    ssd.debug_force_prefill_segments(d["nseg"])
    try:
        y, hf, _ = run_prefill(ssd, case)
        torch.cuda.synchronize()
    finally:
        ssd.debug_force_prefill_segments(0)
    y_ref, hf_ref = oracle_subset(case, range(case.b), range(case.H))
    ym, hm = oracle_subset_mag(case, range(case.b), range(case.H)) if case.dtype == "f32" else (None, None)
    check(y.float().cpu().numpy(), y_ref, case.dtype, "y %s" % d, ym)
    check(hf.cpu().numpy(), hf_ref, case.dtype, "h_final %s" % d, hm)
