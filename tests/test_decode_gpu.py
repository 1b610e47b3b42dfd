"""GPU parity of the cached decode step and the on-device decode loop against the fp64
oracle (O(1) caching and "Compiled on-device loops" of "Compiler-First State Space
Duality ...").  Steps are chained so the conv window and SSM state carry over; the
graph loop must equal step-by-step calls bitwise; the 2.7B-shaped cache (64 layers x
80 heads x 64 x 128) runs at full size and is checked on sampled (layer, row) pairs.
"""
import numpy as np
import pytest
import torch

import oracle
from ssd_inputs import make_decode
from tests.helpers import bf16_tensor, check, f32_tensor

pytestmark = pytest.mark.gpu

ssd = pytest.importorskip("state_space_model_04_b200")


def _dev(d, io):
    xbc = bf16_tensor(d.xbc_bits) if io == "bf16" else f32_tensor(d.xbc)
    return dict(h=f32_tensor(d.h), cs=f32_tensor(d.conv_state), xbc=xbc, dt=f32_tensor(d.dt),
                A=f32_tensor(d.A), D=f32_tensor(d.D), w=f32_tensor(d.conv_w), b=f32_tensor(d.conv_b))


def _oracle_steps(d, n_steps, act, pairs=None, mags=False):
    """Oracle over n_steps; pairs = list of (layer, row) to run (all if None).  With mags,
    also the term magnitudes of every y and of the final state (fp32 bounds)."""
    if pairs is None:
        pairs = [(l, r) for l in range(d.layers) for r in range(d.b)]
    ls = [p[0] for p in pairs]
    rs = [p[1] for p in pairs]
    # each (layer, row) pair is an independent layer with b = 1
    h = d.h[ls, rs][:, None].astype(np.float64).copy()
    cs = d.conv_state[ls, rs][:, None].astype(np.float64).copy()
    hm = np.abs(h)
    ys, yms = [], []
    for t in range(n_steps):
        s = t % d.ring
        args = (d.xbc[s][ls, rs][:, None], d.dt[s][ls, rs][:, None], d.A[ls], d.D[ls], d.conv_w[ls], d.conv_b[ls])
        if mags:  # before the value step: it reads the window the step starts from
            yms.append(oracle.decode_step_mag(hm, cs, *args, act=act, G=d.G, N=d.N)[:, 0])
        ys.append(oracle.decode_step(h, cs, *args, act=act, G=d.G, N=d.N)[:, 0])
    if mags:
        return np.stack(ys), h[:, 0], cs[:, 0], np.stack(yms), hm[:, 0]
    return np.stack(ys), h[:, 0], cs[:, 0]


@pytest.mark.parametrize("io,act,N,G", [("bf16", 1, 128, 1), ("bf16", 0, 64, 2), ("f32", 1, 64, 1), ("f32", 0, 128, 4)])
def test_decode_steps_vs_oracle(io, act, N, G):
    d = make_decode(layers=3, b=2, H=8, P=64, N=N, G=G, ring=6, seed=31 + N + G)
    t = _dev(d, io)
    ys = []
    for s in range(6):
        y = ssd.decode_step(t["h"], t["cs"], t["xbc"][s], t["dt"][s], t["A"], t["D"], t["w"], t["b"], G=G, act=act)
        ys.append(y.float().cpu().numpy())
    torch.cuda.synchronize()
    y_ref, h_ref, cs_ref, y_mag, h_mag = _oracle_steps(d, 6, act, mags=True)
    L, B = d.layers, d.b
    y_got = np.stack(ys).reshape(6, L * B, d.H, d.P)
    check(y_got, y_ref, io, "y", y_mag)
    check(t["h"].cpu().numpy().reshape(L * B, d.H, d.P, d.N), h_ref, io, "h", h_mag)
    # the conv window holds raw inputs: exact copies
    np.testing.assert_array_equal(t["cs"].cpu().numpy().reshape(L * B, -1, 3), cs_ref.astype(np.float32))


def test_plan_equals_steps_bitwise():
    d = make_decode(layers=2, b=3, H=8, P=64, N=128, G=2, ring=5, seed=41)
    t1, t2 = _dev(d, "bf16"), _dev(d, "bf16")
    n = 13
    ys = []
    for s in range(n):
        ys.append(ssd.decode_step(t1["h"], t1["cs"], t1["xbc"][s % 5], t1["dt"][s % 5], t1["A"], t1["D"],
                                  t1["w"], t1["b"], G=2).clone())
    plan = ssd.DecodePlan(t2["h"], t2["cs"], t2["xbc"], t2["dt"], t2["A"], t2["D"], t2["w"], t2["b"],
                          n_steps=n, G=2)
    yr = plan.launch()
    torch.cuda.synchronize()
    assert torch.equal(t1["h"], t2["h"]) and torch.equal(t1["cs"], t2["cs"])
    for s in range(n - 5, n):  # the ring keeps the last `ring` outputs
        assert torch.equal(yr[s % 5], ys[s])
    # a second launch continues from the carried state, replaying ring slots t % ring
    plan.launch()
    for s in range(n):
        ssd.decode_step(t1["h"], t1["cs"], t1["xbc"][s % 5], t1["dt"][s % 5], t1["A"], t1["D"], t1["w"], t1["b"], G=2)
    torch.cuda.synchronize()
    assert torch.equal(t1["h"], t2["h"])
    plan.close()


def test_plan_vs_oracle_many_steps():
    d = make_decode(layers=2, b=2, H=4, P=64, N=128, G=1, ring=7, seed=43)
    t = _dev(d, "bf16")
    n = 64
    plan = ssd.DecodePlan(t["h"], t["cs"], t["xbc"], t["dt"], t["A"], t["D"], t["w"], t["b"], n_steps=n)
    yr = plan.launch()
    torch.cuda.synchronize()
    y_ref, h_ref, _ = _oracle_steps(d, n, 1)
    check(t["h"].cpu().numpy().reshape(4, 4, 64, 128), h_ref, "bf16", "h")
    for s in range(n - 7, n):
        check(yr[s % 7].float().cpu().numpy().reshape(4, 4, 64), y_ref[s], "bf16", "y step %d" % s)
    plan.close()


@pytest.mark.parametrize("b", [1, 32])
def test_2p7b_cache_full_size_sampled(b):
    """The 2.7B-shaped cache (64 layers, H=80, P=64, N=128, conv over 5376 channels) at
    batch 1 and 32 through the graph loop; (layer, row) pairs sampled against the oracle.
    Non-sampled pairs get seeded device-side random state (pairs are independent)."""
    layers, H, P, N, G, ring, n = 64, 80, 64, 128, 1, 4, 48
    d = make_decode(layers=layers, b=1, H=H, P=P, N=N, G=G, ring=ring, seed=50 + b)
    pairs = [(0, 0), (63, b - 1), (17, b // 2)]
    gen = torch.Generator(device="cuda").manual_seed(1234 + b)
    Dc = H * P + 2 * G * N
    h = torch.randn((layers, b, H, P, N), generator=gen, device="cuda") * 0.1
    cs = torch.randn((layers, b, Dc, 3), generator=gen, device="cuda")
    xbc = torch.randn((ring, layers, b, Dc), generator=gen, device="cuda").to(torch.bfloat16)
    dt = torch.rand((ring, layers, b, H), generator=gen, device="cuda") * 0.1 + 1e-3
    # sampled pairs: host-drawn values the oracle also sees (d has b=1: row 0 of each layer)
    xh = bf16_tensor(d.xbc_bits)
    for (l, r) in pairs:
        h[l, r] = f32_tensor(d.h[l, 0])
        cs[l, r] = f32_tensor(d.conv_state[l, 0])
        xbc[:, l, r] = xh[:, l, 0]
        dt[:, l, r] = f32_tensor(d.dt[:, l, 0])
    plan = ssd.DecodePlan(h, cs, xbc, dt, f32_tensor(d.A), f32_tensor(d.D), f32_tensor(d.conv_w),
                          f32_tensor(d.conv_b), n_steps=n)
    yr = plan.launch()
    torch.cuda.synchronize()
    for (l, r) in pairs:
        # oracle on layer l, row 0 of the host case (same values as device pair (l, r))
        y_ref, h_ref, _ = _oracle_steps(d, n, 1, pairs=[(l, 0)])
        check(h[l, r].cpu().numpy()[None], h_ref, "bf16", "h pair %s" % ((l, r),))
        check(yr[(n - 1) % ring, l, r].float().cpu().numpy()[None], y_ref[n - 1], "bf16", "y pair %s" % ((l, r),))
    assert torch.isfinite(h).all()
    plan.close()
