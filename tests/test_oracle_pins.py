"""Pins for the fp64 CPU oracle, checked against things other than the oracle itself.

Source: "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching"
(arXiv 2603.09555).  The pages print no worked example and their display equations were
lost, so the pins are: hand-derived worked examples (tests/golden/), closed forms of the
recurrence, brute-force agreement of three independently written forms (recurrence,
naive chunked dual form, whole-sequence quadratic form), and the invariants the pages
state (static masking / chunking changes nothing, batch invariance, prefill hands its
final state to decode).  Each pin is chosen to catch a specific plausible mistake.
"""
import numpy as np
import pytest

import oracle
from ssd_inputs import make_prefill, make_decode
from tests.conftest import load_golden


def _tiny(b=2, T=12, H=3, P=4, N=5, G=1, seed=11, h0=True, dt_scale=1.0):
    c = make_prefill(b, T, H, P, N, G, L=T, dtype="f32", h0_std=0.3 if h0 else 0.0,
                     seed=seed, dt_scale=dt_scale)
    return c.x, c.dt, c.A, c.B, c.C, c.D, c.h0


def _golden_prefill():
    g = load_golden("recurrence_worked_example.txt")
    T, N = 4, 2
    x = np.array(g["x"]).reshape(1, T, 1, 1)
    dt = np.array(g["dt"]).reshape(1, T, 1)
    A = np.array(g["A"])
    B = np.array(g["B"]).reshape(1, T, 1, N)
    C = np.array(g["C"]).reshape(1, T, 1, N)
    D = np.array(g["D"])
    h0 = np.array(g["h0"]).reshape(1, 1, 1, N)
    return (x, dt, A, B, C, D, h0), np.array(g["y"]), np.array(g["h_final"])


# ---------------------------------------------------------------- worked examples
@pytest.mark.parametrize("form", ["recurrence", "chunked1", "chunked2", "chunked4", "quadratic"])
def test_worked_example_prefill(form):
    """Catches: decay applied after the input, missing dt on the input term, y read
    from the pre-update state, dropped D skip, sign of A, B/C swapped, h0 ignored."""
    args, y_ref, hf_ref = _golden_prefill()
    if form == "recurrence":
        y, hf = oracle.ssd_recurrence(*args[:6], h0=args[6])
    elif form == "quadratic":
        y, hf = oracle.ssd_quadratic(*args[:6], h0=args[6])
    else:
        y, hf = oracle.ssd_chunked(*args[:6], L=int(form[-1]), h0=args[6])
    np.testing.assert_allclose(y.reshape(-1), y_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hf.reshape(-1), hf_ref, rtol=0, atol=1e-12)


def test_worked_example_decode():
    """Catches: conv taps reversed, cache not shifted / shifted the wrong way, bias
    dropped, channel split [x|B|C] out of order, SSM step ordering."""
    g = load_golden("decode_worked_example.txt")
    h = np.array(g["h"]).reshape(1, 1, 1, 1, 1)
    cs = np.array(g["conv_state"]).reshape(1, 1, 3, 3)
    y = oracle.decode_step(h, cs, np.array(g["xbc"]).reshape(1, 1, 3),
                           np.array(g["dt"]).reshape(1, 1, 1), np.array(g["A"]).reshape(1, 1),
                           np.array(g["D"]).reshape(1, 1), np.array(g["conv_w"]).reshape(1, 3, 4),
                           np.array(g["conv_b"]).reshape(1, 3), act=0, G=1, N=1)
    assert abs(y.reshape(-1)[0] - g["y"][0]) < 1e-12
    assert abs(h.reshape(-1)[0] - g["h_new"][0]) < 1e-12
    np.testing.assert_array_equal(cs.reshape(-1), np.array(g["conv_state_new"]))


# ---------------------------------------------------------------- brute force: three forms agree
@pytest.mark.parametrize("shape", [(2, 12, 3, 4, 5, 1), (1, 16, 4, 3, 6, 2), (2, 9, 6, 2, 3, 3)])
def test_three_forms_agree(shape):
    """Recurrence, naive chunked dual form (every L dividing T, L = 1 included) and the
    quadratic form with direct segment sums agree to fp64 rounding."""
    b, T, H, P, N, G = shape
    args = _tiny(b, T, H, P, N, G, seed=sum(shape))
    y0, h0f = oracle.ssd_recurrence(*args[:6], h0=args[6])
    yq, hq = oracle.ssd_quadratic(*args[:6], h0=args[6])
    scale = np.abs(y0).max()
    assert np.abs(yq - y0).max() <= 1e-12 * scale
    assert np.abs(hq - h0f).max() <= 1e-12 * np.abs(h0f).max()
    for L in [d for d in range(1, T + 1) if T % d == 0]:
        yc, hc = oracle.ssd_chunked(*args[:6], L=L, h0=args[6])
        assert np.abs(yc - y0).max() <= 1e-12 * scale, L
        assert np.abs(hc - h0f).max() <= 1e-12 * np.abs(h0f).max(), L


def test_forms_agree_recipe_sizes():
    """Same agreement at the recipe's P=64, N=64 with a realistic decay spread (two
    chunks of 32 plus several heads), catching index mistakes that tiny P/N hide."""
    c = make_prefill(1, 64, 4, 64, 64, 1, L=32, dtype="f32", h0_std=0.1, seed=5)
    y0, hf0 = oracle.ssd_recurrence(c.x, c.dt, c.A, c.B, c.C, c.D, c.h0)
    yc, hc = oracle.ssd_chunked(c.x, c.dt, c.A, c.B, c.C, c.D, 32, c.h0)
    yq, hq = oracle.ssd_quadratic(c.x, c.dt, c.A, c.B, c.C, c.D, c.h0)
    s = np.abs(y0).max()
    assert np.abs(yc - y0).max() < 1e-12 * s and np.abs(yq - y0).max() < 1e-12 * s
    assert np.abs(hc - hf0).max() < 1e-12 * np.abs(hf0).max()
    assert np.abs(hq - hf0).max() < 1e-12 * np.abs(hf0).max()


# ---------------------------------------------------------------- closed forms
def test_dt_zero_keeps_state():
    """dt = 0: no decay and no input, so h_final = h0 and y_t = C_t . h0 + D x_t."""
    x, dt, A, B, C, D, h0 = _tiny()
    dt = np.zeros_like(dt)
    y, hf = oracle.ssd_recurrence(x, dt, A, B, C, D, h0)
    np.testing.assert_allclose(hf, h0, rtol=0, atol=1e-15)
    ref = np.einsum("btgn,bhpn->bthp", C.astype(np.float64), h0.astype(np.float64)) + D[None, None, :, None] * x
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("which", ["B", "C"])
def test_zero_B_or_C_gives_skip_only(which):
    """B = 0 or C = 0 with h0 = 0: y = D x exactly."""
    x, dt, A, B, C, D, _ = _tiny(h0=False)
    if which == "B":
        B = np.zeros_like(B)
    else:
        C = np.zeros_like(C)
    y, _ = oracle.ssd_recurrence(x, dt, A, B, C, D, None)
    np.testing.assert_array_equal(y, D[None, None, :, None].astype(np.float64) * x)


def test_zero_input_decays_state():
    """x = 0: h_t = exp(sum_{k<=t} a_k) h0 and y_t[p] = exp(cs_t) C_t . h0[p]."""
    x, dt, A, B, C, D, h0 = _tiny()
    x = np.zeros_like(x)
    y, hf = oracle.ssd_recurrence(x, dt, A, B, C, D, h0)
    cs = np.cumsum(dt.astype(np.float64) * A[None, None, :].astype(np.float64), axis=1)  # [b,T,H]
    ref = np.exp(cs)[..., None] * np.einsum("btgn,bhpn->bthp", C.astype(np.float64), h0.astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(hf, np.exp(cs[:, -1])[:, :, None, None] * h0, rtol=1e-12)


def test_scalar_impulse_response():
    """P = N = 1, B = C = 1, constant dt and A, impulse x_0 = 1, D = 0:
    y_t = dt * exp(dt*A*t) (the impulse response of a first-order linear filter)."""
    T, d, Av = 40, 0.37, -1.3
    x = np.zeros((1, T, 1, 1)); x[0, 0, 0, 0] = 1.0
    dt = np.full((1, T, 1), d)
    y, _ = oracle.ssd_recurrence(x, dt, np.array([Av]), np.ones((1, T, 1, 1)), np.ones((1, T, 1, 1)),
                                 np.array([0.0]))
    t = np.arange(T)
    np.testing.assert_allclose(y.reshape(-1), d * np.exp(d * Av * t), rtol=1e-13)


@pytest.mark.parametrize("form", ["recurrence", "chunked8", "chunked16", "quadratic"])
def test_step_response_closed_form(form):
    """Constant x, B, C, dt and A with a nonzero h0: the recurrence is a geometric series,
    h_t = q^(t+1) h0 + dt x B^T (1 - q^(t+1)) / (1 - q) with q = exp(dt*A), and
    y_t = h_t C + D x.  T = 48 spans six chunks of 8 and three of 16 (the oracle's chunked
    form takes whole chunks), so a dropped or mis-indexed inter-chunk term, or the initial
    state applied at the wrong token, moves y away from the series."""
    T, P, N, d, Av, Dv = 48, 2, 3, 0.21, -0.8, 0.5
    xv = np.array([0.7, -1.1])
    bv = np.array([0.4, -0.3, 1.2])
    cv = np.array([-0.6, 0.9, 0.25])
    h0v = np.array([[0.3, -0.2, 0.1], [0.05, 0.4, -0.35]])
    x = np.broadcast_to(xv, (1, T, 1, P)).copy()
    dt = np.full((1, T, 1), d)
    Bm = np.broadcast_to(bv, (1, T, 1, N)).copy()
    Cm = np.broadcast_to(cv, (1, T, 1, N)).copy()
    h0 = h0v.reshape(1, 1, P, N)
    args = (x, dt, np.array([Av]), Bm, Cm, np.array([Dv]))
    if form == "recurrence":
        y, hf = oracle.ssd_recurrence(*args, h0)
    elif form == "quadratic":
        y, hf = oracle.ssd_quadratic(*args, h0)
    else:
        y, hf = oracle.ssd_chunked(*args, int(form[len("chunked"):]), h0)
    q = np.exp(d * Av)
    n = np.arange(1, T + 1)[:, None, None]                       # tokens folded in after h0
    h = q ** n * h0v + d * np.outer(xv, bv) * (1 - q ** n) / (1 - q)   # [T, P, N]
    np.testing.assert_allclose(y.reshape(T, P), h @ cv + Dv * xv, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(hf.reshape(P, N), h[-1], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- invariants
def test_split_resume():
    """prefill(T1+T2, h0) == prefill(T2, h_final(prefill(T1, h0))): the cache hand-off."""
    x, dt, A, B, C, D, h0 = _tiny(T=16)
    y, hf = oracle.ssd_recurrence(x, dt, A, B, C, D, h0)
    y1, h1 = oracle.ssd_recurrence(x[:, :7], dt[:, :7], A, B[:, :7], C[:, :7], D, h0)
    y2, h2 = oracle.ssd_chunked(x[:, 7:], dt[:, 7:], A, B[:, 7:], C[:, 7:], D, 3, h1)
    np.testing.assert_allclose(np.concatenate([y1, y2], 1), y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h2, hf, rtol=1e-12, atol=1e-14)


def test_linearity_in_input_and_state():
    """y(x, h0) = y(x, 0) + y(0, h0) (with D applied once)."""
    x, dt, A, B, C, D, h0 = _tiny()
    y, hf = oracle.ssd_recurrence(x, dt, A, B, C, D, h0)
    ya, ha = oracle.ssd_recurrence(x, dt, A, B, C, D, None)
    yb, hb = oracle.ssd_recurrence(np.zeros_like(x), dt, A, B, C, D, h0)
    np.testing.assert_allclose(y, ya + yb, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hf, ha + hb, rtol=1e-12, atol=1e-12)


def test_causality():
    """Perturbing token t leaves y_{<t} unchanged (bitwise in fp64)."""
    x, dt, A, B, C, D, h0 = _tiny(T=16)
    y, _ = oracle.ssd_chunked(x, dt, A, B, C, D, 4, h0)
    x2, B2 = x.copy(), B.copy()
    x2[:, 9] += 1.0
    B2[:, 9] -= 0.5
    y2, _ = oracle.ssd_chunked(x2, dt, A, B2, C, D, 4, h0)
    np.testing.assert_array_equal(y[:, :9], y2[:, :9])
    assert np.abs(y[:, 9:] - y2[:, 9:]).max() > 0


def test_batch_invariance():
    """Sequence r alone gives bitwise the same output as inside the batch."""
    x, dt, A, B, C, D, h0 = _tiny(b=3)
    y, hf = oracle.ssd_recurrence(x, dt, A, B, C, D, h0)
    y1, h1 = oracle.ssd_recurrence(x[1:2], dt[1:2], A, B[1:2], C[1:2], D, h0[1:2])
    np.testing.assert_array_equal(y[1:2], y1)
    np.testing.assert_array_equal(hf[1:2], h1)


def test_groups_match_per_head_slicing():
    """Head h reads group h // (H/G): each head run alone with its group's B, C matches
    the grouped run; G = H with B, C replicated equals G = 1."""
    b, T, H, P, N, G = 1, 10, 6, 3, 4, 3
    x, dt, A, B, C, D, h0 = _tiny(b, T, H, P, N, G, seed=3)
    y, hf = oracle.ssd_recurrence(x, dt, A, B, C, D, h0)
    for h in range(H):
        g = h // (H // G)
        yh, hh = oracle.ssd_recurrence(x[:, :, h:h + 1], dt[:, :, h:h + 1], A[h:h + 1],
                                       B[:, :, g:g + 1], C[:, :, g:g + 1], D[h:h + 1], h0[:, h:h + 1])
        np.testing.assert_array_equal(y[:, :, h:h + 1], yh)
        np.testing.assert_array_equal(hf[:, h:h + 1], hh)
    B1, C1 = B[:, :, :1], C[:, :, :1]
    ya, _ = oracle.ssd_recurrence(x, dt, A, B1, C1, D, h0)
    yb, _ = oracle.ssd_recurrence(x, dt, A, np.repeat(B1, H, 2), np.repeat(C1, H, 2), D, h0)
    np.testing.assert_array_equal(ya, yb)


def test_strong_decay_underflow_is_benign():
    """Very strong decay (exp underflows to 0 inside the chunk) still matches the
    recurrence: the chunked form must not produce inf * 0."""
    x, dt, A, B, C, D, h0 = _tiny(T=16, dt_scale=400.0)
    y0, h0f = oracle.ssd_recurrence(x, dt, A, B, C, D, h0)
    yc, hc = oracle.ssd_chunked(x, dt, A, B, C, D, 8, h0)
    assert np.isfinite(yc).all()
    np.testing.assert_allclose(yc, y0, rtol=1e-12, atol=1e-12 * np.abs(y0).max())


# ---------------------------------------------------------------- decode vs prefill
def test_decode_steps_reproduce_prefill():
    """With an identity conv (taps [0,0,0,1], bias 0) and no activation, T decode steps
    from h0 reproduce the prefill's y and h_final (the prefill initialises the cache)."""
    H, P, N, G, T = 4, 3, 5, 2, 9
    c = make_prefill(1, T, H, P, N, G, L=T, dtype="f32", h0_std=0.2, seed=21)
    Dc = H * P + 2 * G * N
    w = np.zeros((1, Dc, 4)); w[:, :, 3] = 1.0
    bias = np.zeros((1, Dc))
    h = c.h0.astype(np.float64).reshape(1, 1, H, P, N).copy()
    cst = np.zeros((1, 1, Dc, 3))
    ys = []
    for t in range(T):
        xbc = np.concatenate([c.x[0, t].reshape(-1), c.B[0, t].reshape(-1), c.C[0, t].reshape(-1)])
        ys.append(oracle.decode_step(h, cst, xbc.reshape(1, 1, Dc), c.dt[0, t].reshape(1, 1, H),
                                     c.A.reshape(1, H), c.D.reshape(1, H), w, bias, act=0, G=G, N=N))
    y_ref, hf_ref = oracle.ssd_recurrence(c.x, c.dt, c.A, c.B, c.C, c.D, c.h0)
    y_dec = np.stack([v.reshape(H, P) for v in ys])[None]
    np.testing.assert_allclose(y_dec, y_ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h.reshape(1, H, P, N), hf_ref, rtol=1e-13, atol=1e-15)


def test_decode_conv_one_hot_taps_delay_input():
    """Conv taps e_i select window[i]: u_t is the input from (k-1-i) steps ago; with
    B = C channels fed constant 1 the SSM output exposes u_x directly (D = 1, dt = 0)."""
    H, P, N, G, k = 1, 2, 1, 1, 4
    Dc = H * P + 2 * G * N
    for i in range(k):
        w = np.zeros((1, Dc, k)); w[0, :, i] = 1.0
        h = np.zeros((1, 1, H, P, N)); cst = np.zeros((1, 1, Dc, k - 1))
        outs = []
        for t in range(8):
            xbc = np.array([t + 1.0, -(t + 1.0), 1.0, 1.0]).reshape(1, 1, Dc)
            y = oracle.decode_step(h, cst, xbc, np.zeros((1, 1, H)), np.full((1, H), -1.0),
                                   np.ones((1, H)), w, np.zeros((1, Dc)), act=0, G=G, N=N)
            outs.append(y.reshape(-1).copy())
        lag = k - 1 - i
        for t in range(8):
            want = (t + 1.0 - lag) if t >= lag else 0.0
            assert outs[t][0] == want and outs[t][1] == -want


def test_decode_silu_odd_part_identity():
    """SiLU satisfies silu(v) - silu(-v) = v; with D = 1, dt = 0 the decode output is
    u_x itself, so feeding +v and -v through act=SiLU must give outputs differing by v
    (catches a sign error in the sigmoid or applying SiLU to the wrong tensor)."""
    H, P, N, G, k = 1, 8, 1, 1, 4
    Dc = H * P + 2 * G * N
    v = np.linspace(-6, 6, P)
    w = np.zeros((1, Dc, k)); w[0, :, k - 1] = 1.0
    res = []
    for sgn in (1.0, -1.0):
        h = np.zeros((1, 1, H, P, N)); cst = np.zeros((1, 1, Dc, k - 1))
        xbc = np.concatenate([sgn * v, [0.0, 0.0]]).reshape(1, 1, Dc)
        res.append(oracle.decode_step(h, cst, xbc, np.zeros((1, 1, H)), np.full((1, H), -1.0),
                                      np.ones((1, H)), w, np.zeros((1, Dc)), act=1, G=G, N=N).reshape(-1))
    np.testing.assert_allclose(res[0] - res[1], v, rtol=0, atol=1e-14)
    assert res[0][P // 2 - 1] < 0 < res[0][P // 2]  # silu(v) > 0 for v > 0, < 0 for v < 0


def test_decode_layers_and_rows_independent():
    """Each (layer, row) pair of a decode step is independent of the others."""
    d = make_decode(layers=3, b=2, H=2, P=4, N=3, G=1, ring=1, seed=9)
    h = d.h.astype(np.float64).copy(); cs = d.conv_state.astype(np.float64).copy()
    y = oracle.decode_step(h, cs, d.xbc[0], d.dt[0], d.A, d.D, d.conv_w, d.conv_b, act=1, G=1, N=3)
    h1 = d.h[2:3, 1:2].astype(np.float64).copy(); cs1 = d.conv_state[2:3, 1:2].astype(np.float64).copy()
    y1 = oracle.decode_step(h1, cs1, d.xbc[0][2:3, 1:2], d.dt[0][2:3, 1:2], d.A[2:3], d.D[2:3],
                            d.conv_w[2:3], d.conv_b[2:3], act=1, G=1, N=3)
    np.testing.assert_array_equal(y[2:3, 1:2], y1)
    np.testing.assert_array_equal(h[2:3, 1:2], h1)
    np.testing.assert_array_equal(cs[2:3, 1:2], cs1)


# ------------------------------------------------------------------ dt pre-processing
def test_dt_from_raw_closed_forms():
    """softplus(0) = ln 2; softplus(ln(e^k - 1)) = k; softplus(z) - softplus(-z) = z (the
    odd part of softplus is z/2); softplus(z) -> z for large z and -> e^z for very negative z."""
    ks = np.array([0.25, 1.0, 3.0, 10.0])
    got = oracle.dt_from_raw(np.log(np.expm1(ks))[None, :])
    np.testing.assert_allclose(got[0], ks, rtol=1e-14)
    assert abs(oracle.dt_from_raw(np.zeros((1, 1)))[0, 0] - np.log(2.0)) < 1e-15
    z = np.linspace(-30, 30, 121)[None, :]
    np.testing.assert_allclose(oracle.dt_from_raw(z) - oracle.dt_from_raw(-z), z, atol=1e-12)
    np.testing.assert_allclose(oracle.dt_from_raw(np.array([[40.0, 300.0]])), [[40.0, 300.0]], rtol=1e-15)
    np.testing.assert_allclose(oracle.dt_from_raw(np.array([[-40.0, -600.0]])), np.exp([[-40.0, -600.0]]), rtol=1e-12)


def test_dt_from_raw_bias_per_head_and_clamp():
    """The bias is added per head (last axis) before the softplus; the clamp bounds the result."""
    raw = np.zeros((2, 3, 4))
    bias = np.log(np.expm1(np.array([0.001, 0.01, 0.1, 1.0])))
    got = oracle.dt_from_raw(raw, bias)
    np.testing.assert_allclose(got, np.broadcast_to([0.001, 0.01, 0.1, 1.0], raw.shape), rtol=1e-12)
    clamped = oracle.dt_from_raw(raw, bias, dt_min=0.005, dt_max=0.5)
    np.testing.assert_allclose(clamped[0, 0], [0.005, 0.01, 0.1, 0.5], rtol=1e-12)


# ---------------------------------------------------------------- term magnitudes
# The per-element fp32 tolerances scale with the sum of the absolute values of the products
# behind each output.  These pins check that sum against an explicit enumeration of the
# products (written here term by term, independently of the C recurrence) and against the
# two properties that define it.

def _enumerate_prefill_terms(x, dt, A, B, C, D, h0):
    """Every product of the expanded recurrence for one sequence and one head (b = H = 1),
    returned as lists of terms per output: y[t][p] and h_final[p][n]."""
    x, dt, A, B, C, D, h0 = (np.asarray(v, np.float64) for v in (x, dt, A, B, C, D, h0))
    T, P, N = x.shape[1], x.shape[3], B.shape[3]
    a = dt[0, :, 0] * A[0]

    def decay(s, t):  # prod of alpha_r for s < r <= t
        return float(np.exp(a[s + 1:t + 1].sum()))

    y_terms = [[[] for _ in range(P)] for _ in range(T)]
    h_terms = [[[] for _ in range(N)] for _ in range(P)]
    for t in range(T):
        for p in range(P):
            for n in range(N):
                c = C[0, t, 0, n]
                y_terms[t][p].append(c * decay(-1, t) * h0[0, 0, p, n])
                for s in range(t + 1):
                    y_terms[t][p].append(c * decay(s, t) * dt[0, s, 0] * x[0, s, 0, p] * B[0, s, 0, n])
            y_terms[t][p].append(D[0] * x[0, t, 0, p])
    for p in range(P):
        for n in range(N):
            h_terms[p][n].append(decay(-1, T - 1) * h0[0, 0, p, n])
            for s in range(T):
                h_terms[p][n].append(decay(s, T - 1) * dt[0, s, 0] * x[0, s, 0, p] * B[0, s, 0, n])
    return y_terms, h_terms


def test_prefill_magnitudes_enumerated():
    """Catches: a magnitude taken of the wrong operand (C, B, x, h0 or D left signed), the
    decay or dt dropped from a term, h0's term left out."""
    x, dt, A, B, C, D, h0 = _tiny(b=1, T=5, H=1, P=2, N=3, seed=21)
    D = np.array([-0.7])  # a signed skip weight, so |D| matters
    ym, hm = oracle.ssd_magnitudes(x, dt, A, B, C, D, h0)
    y_terms, h_terms = _enumerate_prefill_terms(x, dt, A, B, C, D, h0)
    y_enum = np.array([[sum(abs(v) for v in y_terms[t][p]) for p in range(2)] for t in range(5)])
    h_enum = np.array([[sum(abs(v) for v in h_terms[p][n]) for n in range(3)] for p in range(2)])
    np.testing.assert_allclose(ym[0, :, 0, :], y_enum, rtol=1e-12, atol=0)
    np.testing.assert_allclose(hm[0, 0], h_enum, rtol=1e-12, atol=0)
    # and the enumeration is complete: its signed sums are the outputs themselves
    y, hf = oracle.ssd_recurrence(x, dt, A, B, C, D, h0)
    y_sum = np.array([[sum(y_terms[t][p]) for p in range(2)] for t in range(5)])
    np.testing.assert_allclose(y[0, :, 0, :], y_sum, rtol=1e-12, atol=1e-14)


def test_prefill_magnitudes_bound_and_equality():
    """The magnitude bounds |output| (triangle inequality) and equals it when every input is
    non-negative.  Catches a magnitude that is not a sum of absolute values."""
    x, dt, A, B, C, D, h0 = _tiny(b=2, T=24, H=4, P=3, N=5, G=2, seed=22)
    y, hf = oracle.ssd_recurrence(x, dt, A, B, C, D, h0)
    ym, hm = oracle.ssd_magnitudes(x, dt, A, B, C, D, h0)
    assert (np.abs(y) <= ym * (1 + 1e-12)).all() and (np.abs(hf) <= hm * (1 + 1e-12)).all()
    assert (ym > np.abs(y) * (1 + 1e-6)).any()  # signs cancel somewhere
    ax, aB, aC, ah = np.abs(x), np.abs(B), np.abs(C), np.abs(h0)
    y2, hf2 = oracle.ssd_recurrence(ax, dt, A, aB, aC, D, ah)
    ym2, hm2 = oracle.ssd_magnitudes(ax, dt, A, aB, aC, D, ah)
    np.testing.assert_allclose(ym2, y2, rtol=1e-13, atol=0)
    np.testing.assert_allclose(hm2, hf2, rtol=1e-13, atol=0)


def test_decode_magnitudes_enumerated():
    """One decode step with no activation, P = N = 1 and two conv taps, expanded into every
    product: y = C (alpha h + dt x B) + D x with x, B, C each a sum of two tap products and a
    bias.  Catches: a tap, the bias or the state term left out of the magnitude, |D| or the
    conv weights left signed, the window read after the shift."""
    rng = np.random.default_rng(5)
    layers, b, H, P, N, G, k = 1, 1, 1, 1, 1, 1, 2
    Dc = 3
    h = rng.standard_normal((1, 1, 1, 1, 1))
    cs = rng.standard_normal((1, 1, Dc, 1))
    xbc = rng.standard_normal((1, 1, Dc))
    dt = np.array([[[0.37]]])
    A = np.array([[-1.9]])
    D = np.array([[-0.6]])
    w = rng.standard_normal((1, Dc, k))
    bias = rng.standard_normal((1, Dc))
    alpha = float(np.exp(dt[0, 0, 0] * A[0, 0]))
    # tap products of each channel: [w0 * window0, w1 * current input, bias]
    terms = [[w[0, c, 0] * cs[0, 0, c, 0], w[0, c, 1] * xbc[0, 0, c], bias[0, c]] for c in range(Dc)]
    tx, tB, tC = terms
    prods = [ci * alpha * h.item() for ci in tC]
    prods += [ci * dt[0, 0, 0] * xi * bi for ci in tC for xi in tx for bi in tB]
    prods += [D[0, 0] * xi for xi in tx]
    hm = np.abs(h).copy()
    ym = oracle.decode_step_mag(hm, cs, xbc, dt, A, D, w, bias, act=0, G=G, N=N)
    assert abs(ym.item() - sum(abs(v) for v in prods)) <= 1e-12 * ym.item()
    h_prods = [alpha * h.item()] + [dt[0, 0, 0] * xi * bi for xi in tx for bi in tB]
    assert abs(hm.item() - sum(abs(v) for v in h_prods)) <= 1e-12 * hm.item()
    # the enumeration is complete: its signed sum is the step's output
    h2, cs2 = h.copy(), cs.copy()
    y = oracle.decode_step(h2, cs2, xbc, dt, A, D, w, bias, act=0, G=G, N=N)
    assert abs(y.item() - sum(prods)) <= 1e-12 * max(1.0, abs(y.item()))


@pytest.mark.parametrize("act", [0, 1])
def test_decode_magnitudes_bound_and_equality(act):
    """|y| <= y_mag and |h| <= h_mag over several steps with either activation; with no
    activation and every input, weight and state non-negative the two are equal."""
    d = make_decode(layers=2, b=2, H=4, P=8, N=16, G=2, ring=3, seed=17)
    h = d.h.astype(np.float64).copy()
    cs = d.conv_state.astype(np.float64).copy()
    hm = np.abs(h)
    for s in range(3):
        ym = oracle.decode_step_mag(hm, cs, d.xbc[s], d.dt[s], d.A, d.D, d.conv_w, d.conv_b, act=act, G=2, N=16)
        y = oracle.decode_step(h, cs, d.xbc[s], d.dt[s], d.A, d.D, d.conv_w, d.conv_b, act=act, G=2, N=16)
        assert (np.abs(y) <= ym * (1 + 1e-12)).all() and (np.abs(h) <= hm * (1 + 1e-12)).all()
    if act == 0:
        h = np.abs(d.h).astype(np.float64)
        cs = np.abs(d.conv_state).astype(np.float64)
        hm = h.copy()
        w, bias, xbc = np.abs(d.conv_w), np.abs(d.conv_b), np.abs(d.xbc[0])
        ym = oracle.decode_step_mag(hm, cs, xbc, d.dt[0], d.A, d.D, w, bias, act=0, G=2, N=16)
        y = oracle.decode_step(h, cs, xbc, d.dt[0], d.A, d.D, w, bias, act=0, G=2, N=16)
        np.testing.assert_allclose(ym, y, rtol=1e-13, atol=0)
        np.testing.assert_allclose(hm, h, rtol=1e-13, atol=0)
