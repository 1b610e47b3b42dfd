"""GPU checks of the method's invariants that tie the CUDA paths to each other, beside the
oracle parity tests ("Compiler-First State Space Duality ...": the prefill initialises the
O(1) decode cache; the recurrence is linear in the input and the state; B/C groups are
shared by contiguous blocks of heads).

- A prefill's y and h_final equal T cached decode steps over the same tokens from the same
  h0, with the conv reduced to the identity (taps [0, 0, 0, 1], bias 0) and no activation.
- y(x, h0) = y(x, 0) + y(0, h0).
- G = H with each head's B/C a copy of the single group's equals G = 1, bitwise.
"""
import numpy as np
import pytest
import torch

from ssd_inputs import make_prefill
from tests.helpers import check, oracle_subset, oracle_subset_mag, prefill_inputs, rel_max

pytestmark = pytest.mark.gpu

ssd = pytest.importorskip("state_space_model_04_b200")


def _np(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("dtype,N", [("bf16", 128), ("f32", 64)])
def test_prefill_state_feeds_decode(dtype, N):
    b, T, H, G = 2, 200, 4, 2
    case = make_prefill(b, T, H, 64, N, G, 128, dtype, h0_std=0.1, seed=91 + N)
    t = prefill_inputs(case)
    y_p, h_p = ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=128, h0=t["h0"])
    # decode: one layer, the prefill's batch; the conv passes the current input through
    P, Dc = 64, H * 64 + 2 * G * N
    h = t["h0"].clone().reshape(1, b, H, P, N)
    cs = torch.zeros(1, b, Dc, 3, dtype=torch.float32, device="cuda")
    w = torch.zeros(1, Dc, 4, dtype=torch.float32, device="cuda")
    w[:, :, 3] = 1.0
    bias = torch.zeros(1, Dc, dtype=torch.float32, device="cuda")
    A, D = t["A"].reshape(1, H), t["D"].reshape(1, H)
    ys = []
    for s in range(T):
        xbc = torch.cat([t["x"][:, s].reshape(b, -1), t["B"][:, s].reshape(b, -1), t["C"][:, s].reshape(b, -1)],
                        dim=1).reshape(1, b, Dc).contiguous()
        dt = t["dt"][:, s].reshape(1, b, H).contiguous()
        ys.append(ssd.decode_step(h, cs, xbc, dt, A, D, w, bias, G=G, act=ssd.SSD_ACT_NONE))
    torch.cuda.synchronize()
    y_d = torch.stack(ys, dim=0)[:, 0].permute(1, 0, 2, 3)  # [b, T, H, P]
    y_ref, h_ref = oracle_subset(case, range(b), range(H))
    # with the identity conv and no activation a decode step's products are the recurrence's,
    # so the prefill's term magnitudes bound both paths
    ym, hm = oracle_subset_mag(case, range(b), range(H)) if dtype == "f32" else (None, None)
    # both paths against the oracle, and against each other at the dtype's bound
    check(_np(y_p), y_ref, dtype, "prefill y", ym)
    check(_np(y_d), y_ref, dtype, "decode y", ym)
    check(_np(h_p), h_ref, dtype, "prefill h_final", hm)
    check(_np(h.reshape(b, H, P, N)), h_ref, dtype, "decode h", hm)
    check(_np(y_d), _np(y_p), dtype, "decode y vs prefill y", ym, sides=2)
    check(_np(h.reshape(b, H, P, N)), _np(h_p), dtype, "decode h vs prefill h_final", hm, sides=2)


@pytest.mark.parametrize("dtype,N,tol", [("bf16", 128, 2e-2), ("f32", 64, 1e-5)])
def test_linearity_in_input_and_state(dtype, N, tol):
    case = make_prefill(2, 300, 4, 64, N, 1, 128, dtype, h0_std=0.3, seed=92 + N)
    t = prefill_inputs(case)
    zx = torch.zeros_like(t["x"])
    zh = torch.zeros_like(t["h0"])
    run = lambda x, h0: ssd.prefill(x, t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=128, h0=h0)
    y, hf = run(t["x"], t["h0"])
    y_x, hf_x = run(t["x"], zh)
    y_h, hf_h = run(zx, t["h0"])
    torch.cuda.synchronize()
    assert rel_max(_np(y_x) + _np(y_h), _np(y)) <= tol
    assert rel_max(_np(hf_x) + _np(hf_h), _np(hf)) <= tol


def test_replicated_groups_equal_one_group_bitwise():
    b, T, H, N = 2, 400, 4, 128
    case = make_prefill(b, T, H, 64, N, 1, 256, "bf16", h0_std=0.1, seed=93)
    t = prefill_inputs(case)
    Bh = t["B"].expand(b, T, H, N).contiguous()  # every head its own copy of group 0
    Ch = t["C"].expand(b, T, H, N).contiguous()
    y1, h1 = ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=256, h0=t["h0"])
    yH, hH = ssd.prefill(t["x"], t["dt"], t["A"], Bh, Ch, t["D"], chunk=256, h0=t["h0"])
    torch.cuda.synchronize()
    assert torch.equal(y1, yH) and torch.equal(h1, hH)
