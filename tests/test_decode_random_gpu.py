"""Randomised GPU parity sweep of the cached decode step against the fp64 oracle.

Each case draws, from its own fixed seed, 1-4 layers, a batch of 1-5 sequences, 2-8 heads
in 1-H groups, N = 64 or 128, bf16 or fp32 step inputs, SiLU or no activation, 1-5 chained
steps, and one of the three entry points (the step with a workspace, the allocation-free
step, or the graph loop). It compares y of every step, the final SSM state and the conv
window with the oracle: y and the state within the dtype's bound, and the window (raw
inputs) exactly.
"""
import numpy as np
import pytest
import torch

from ssd_inputs import make_decode
from tests.helpers import check
from tests.test_decode_gpu import _dev, _oracle_steps

pytestmark = pytest.mark.gpu

ssd = pytest.importorskip("state_space_model_04_b200")


def _draw(seed):
    rng = np.random.default_rng(2000 + seed)
    H = int(rng.choice([2, 4, 6, 8]))
    G = int(rng.choice([g for g in range(1, H + 1) if H % g == 0]))
    return dict(layers=int(rng.integers(1, 5)), b=int(rng.integers(1, 6)), H=H, G=G,
                N=int(rng.choice([64, 128])), io=str(rng.choice(["bf16", "f32"])), act=int(rng.integers(0, 2)),
                steps=int(rng.integers(1, 6)), entry=str(rng.choice(["step", "noalloc", "loop"])))


@pytest.mark.parametrize("seed", range(16))
def test_random_decode_matches_oracle(seed):
    c = _draw(seed)
    d = make_decode(layers=c["layers"], b=c["b"], H=c["H"], P=64, N=c["N"], G=c["G"], ring=c["steps"],
                    seed=700 + seed)
    t = _dev(d, c["io"])
    L, B = d.layers, d.b
    if c["entry"] == "loop":
        y = ssd.decode_loop(t["h"], t["cs"], t["xbc"], t["dt"], t["A"], t["D"], t["w"], t["b"], c["steps"],
                            G=c["G"], act=c["act"])
        y_got = y.float().cpu().numpy().reshape(c["steps"], L * B, d.H, d.P)
    else:
        ys = []
        for s in range(c["steps"]):
            if c["entry"] == "step":
                y = ssd.decode_step(t["h"], t["cs"], t["xbc"][s], t["dt"][s], t["A"], t["D"], t["w"], t["b"],
                                    G=c["G"], act=c["act"])
            else:
                y = torch.empty(L, B, d.H, d.P, dtype=t["xbc"].dtype, device="cuda")
                ssd.decode_step_noalloc(t["h"], t["cs"], t["xbc"][s], t["dt"][s], t["A"], t["D"], t["w"], t["b"],
                                        y, G=c["G"], act=c["act"])
            ys.append(y.float().cpu().numpy())
        y_got = np.stack(ys).reshape(c["steps"], L * B, d.H, d.P)
    torch.cuda.synchronize()
    y_ref, h_ref, cs_ref, y_mag, h_mag = _oracle_steps(d, c["steps"], c["act"], mags=True)
    check(y_got, y_ref, c["io"], "y %s" % c, y_mag)
    check(t["h"].cpu().numpy().reshape(L * B, d.H, d.P, d.N), h_ref, c["io"], "h %s" % c, h_mag)
    np.testing.assert_array_equal(t["cs"].cpu().numpy().reshape(L * B, -1, 3), cs_ref.astype(np.float32))
