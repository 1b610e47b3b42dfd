"""The cached decode at the 2.7B shape, run for 4096 on-device steps from the state a
2.7B-layer prefill leaves behind ("Compiler-First State Space Duality and Portable O(1)
Autoregressive Caching": the prefill fills the cache with the final state, and the
compiled decode body updates it one token at a time without the host).

The cache is 64 layers x 80 heads x 64 x 128 fp32 SSM state plus a width-4 conv window over
5120 + 2 * 128 channels, at batch 1 and 32.  Layer l, row r starts from the prefill's final
state of sequence r mod 8 and a conv window holding that sequence's last three tokens of
[x | B | C].  Both sides compute their own prefill: the GPU decode starts from the GPU
prefill, the oracle decode from the fp64 oracle prefill, so the check covers the hand-off as
well as the 4096-step drift of the fp32 state.

Step inputs come from a ring of 64 steps (step t reads slot t mod 64), as in the benchmark.
Sampled (layer, row) pairs carry host-drawn inputs that the oracle sees too; every other
pair gets seeded device-side inputs (pairs are independent, so sampling is exact).  y of the
sampled pairs is compared at EVERY one of the 4096 steps, the state and conv window at the
end.
"""
import numpy as np
import pytest
import torch

import oracle
from ssd_inputs import make_config, make_decode, make_decode_params, make_decode_ring_device
from tests.helpers import bf16_tensor, check, f32_tensor, oracle_subset, prefill_inputs

pytestmark = pytest.mark.gpu

ssd = pytest.importorskip("state_space_model_04_b200")

LAYERS, H, P, N, G, K = 64, 80, 64, 128, 1, 4
DC = H * P + 2 * G * N
RING, STEPS = 64, 4096


def _window(case, seq):
    """Conv window [Dc][3] of sequence `seq`: its last three tokens of [x | B | C], oldest
    first (the channel order of the decode step's packed input)."""
    T = case.T
    x = case.x[seq, T - 3:].reshape(3, H * P)
    Bm = case.B[seq, T - 3:].reshape(3, G * N)
    Cm = case.C[seq, T - 3:].reshape(3, G * N)
    return np.ascontiguousarray(np.concatenate([x, Bm, Cm], axis=1).T, dtype=np.float32)


@pytest.fixture(scope="module")
def prefill_2p7b():
    """The 2.7B-layer prefill (b=8, T=4096, H=80, seeded, h0 ~ N(0, 0.1^2)): the GPU's
    final state, and the oracle's for the sequences the sampled rows map to."""
    case = make_config("mamba2_2p7b_layer")
    t = prefill_inputs(case)
    y, hf = ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=case.L, h0=t["h0"], check=True)
    torch.cuda.synchronize()
    del y, t
    seqs = [0, 7]
    _, hf_ref = oracle_subset(case, seqs, range(H))
    hf_gpu = hf.cpu().numpy()
    for i, s in enumerate(seqs):
        check(hf_gpu[s], hf_ref[i], "bf16", "prefill h_final sequence %d" % s)
    windows = [_window(case, s) for s in range(case.b)]
    return hf, {s: hf_ref[i] for i, s in enumerate(seqs)}, windows


@pytest.mark.parametrize("b", [1, 32])
def test_2p7b_cache_4096_steps_from_prefill(prefill_2p7b, b):
    hf_gpu, hf_ref, windows = prefill_2p7b
    pairs = [(0, 0), (63, b - 1)] + ([(17, b // 2)] if b > 1 else [])
    # per-layer parameters and the sampled pairs' step inputs (row 0 of a b=1 host case)
    d = make_decode(layers=LAYERS, b=1, H=H, P=P, N=N, G=G, k=K, ring=RING, seed=60 + b, h_std=0.0)
    dt_bias = make_decode_params(LAYERS, H, P, N, G, k=K, seed=60 + b)[4]  # the same draws as d's
    dev = "cuda"
    # cache from the prefill: row r <- sequence r mod 8, the same for every layer
    rows = torch.arange(b, device=dev) % hf_gpu.shape[0]
    h = hf_gpu[rows].unsqueeze(0).expand(LAYERS, b, H, P, N).contiguous()
    win = torch.stack([torch.from_numpy(windows[r % len(windows)]) for r in range(b)]).to(dev)
    cs = win.unsqueeze(0).expand(LAYERS, b, DC, K - 1).contiguous()
    xbc, dt = make_decode_ring_device(RING, LAYERS, b, H, P, N, G, dt_bias, seed=4242 + b, device=dev)
    xh = bf16_tensor(d.xbc_bits)
    for (l, r) in pairs:
        xbc[:, l, r] = xh[:, l, 0]
        dt[:, l, r] = f32_tensor(d.dt[:, l, 0])
    plan = ssd.DecodePlan(h, cs, xbc, dt, f32_tensor(d.A), f32_tensor(d.D), f32_tensor(d.conv_w),
                          f32_tensor(d.conv_b), n_steps=RING)
    ys = {p: [] for p in pairs}
    for _ in range(STEPS // RING):
        yr = plan.launch()
        torch.cuda.synchronize()
        for (l, r) in pairs:
            ys[(l, r)].append(yr[:, l, r].float().cpu().numpy())
    plan.close()
    assert torch.isfinite(h).all()

    # oracle: each sampled pair as an independent layer with b = 1, all pairs in one call
    ls = [p[0] for p in pairs]
    h_o = np.stack([hf_ref[r % 8] for (_, r) in pairs])[:, None].astype(np.float64).copy()
    cs_o = np.stack([windows[r % 8] for (_, r) in pairs])[:, None].astype(np.float64).copy()
    xbc_o = d.xbc[:, ls, 0]          # [RING][pairs][Dc]
    dt_o = d.dt[:, ls, 0]            # [RING][pairs][H]
    y_ref = np.empty((STEPS, len(pairs), H, P))
    for t in range(STEPS):
        s = t % RING
        y_ref[t] = oracle.decode_step(h_o, cs_o, xbc_o[s][:, None], dt_o[s][:, None], d.A[ls], d.D[ls],
                                      d.conv_w[ls], d.conv_b[ls], act=1, G=G, N=N)[:, 0]
    worst = 0.0
    for i, (l, r) in enumerate(pairs):
        y_got = np.concatenate(ys[(l, r)])   # [STEPS][H][P], step t at index t
        errs = [check(y_got[t], y_ref[t, i], "bf16", "y pair %s step %d" % ((l, r), t)) for t in range(STEPS)]
        worst = max(worst, max(errs))
        eh = check(h[l, r].cpu().numpy(), h_o[i, 0], "bf16", "h pair %s after %d steps" % ((l, r), STEPS))
        # the conv window holds the last three raw inputs: exact
        np.testing.assert_array_equal(cs[l, r].cpu().numpy(), cs_o[i, 0].astype(np.float32))
        print("pair %s: worst y error over %d steps %.3e, h error %.3e" % ((l, r), STEPS, max(errs), eh))
    assert worst <= 2e-2

