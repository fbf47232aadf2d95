"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test fixes the oracle to a closed form, a library routine, a hand-worked
value or an invariant that a plausible mistake (a dropped term, a wrong sign
or index, an off-by-one decay exponent, a transposed operand, a wrong channel
offset) would break.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng


# ---------------------------------------------------------------- elementwise

def test_softplus_closed_forms():
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=0, abs=1e-15)
    for s in (-30.0, -3.0, -0.5, 0.25, 2.0, 30.0):
        # log(1+e^s) - log(1+e^-s) = s for every s
        assert oracle.softplus(s) - oracle.softplus(-s) == pytest.approx(s, abs=1e-12)
    assert oracle.softplus(-50.0) == pytest.approx(math.exp(-50.0), rel=1e-12)
    assert oracle.softplus(float("-inf")) == 0.0
    assert oracle.softplus(800.0) == 800.0  # no overflow


def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), abs=1e-15)
    for s in (-7.0, -1.5, 0.3, 4.0):
        assert oracle.silu(s) - oracle.silu(-s) == pytest.approx(s, abs=1e-12)


# ---------------------------------------------------------------- conv1d + SiLU

def _inv_silu_free_conv(xBC, w, b, state):
    """Pre-activation through numpy's cross-correlation, one channel at a time."""
    L, cd = xBC.shape
    K = w.shape[1]
    left = state[:, 1:].T if state is not None else np.zeros((K - 1, cd))
    padded = np.concatenate([left, xBC], axis=0)
    pre = np.empty((L, cd))
    for c in range(cd):
        pre[:, c] = np.correlate(padded[:, c], w[c], mode="valid") + b[c]
    return pre


@pytest.mark.parametrize("L", [1, 2, 3, 4, 9, 33])
@pytest.mark.parametrize("with_state", [False, True])
def test_conv_matches_numpy_correlate(L, with_state):
    r = rng(L + 10 * with_state)
    cd, K = 7, 4
    xBC = r.standard_normal((L, cd))
    w = r.uniform(-0.5, 0.5, (cd, K))
    b = r.uniform(-0.5, 0.5, cd)
    st = r.standard_normal((cd, K)) if with_state else None
    u, st_out = oracle.conv_silu(xBC, w, b, st)
    pre = _inv_silu_free_conv(xBC, w, b, st)
    np.testing.assert_allclose(u, pre / (1.0 + np.exp(-pre)), rtol=0, atol=1e-13)
    # the state out holds the last K raw inputs, oldest first
    full = np.concatenate([(st.T if st is not None else np.zeros((K, cd))), xBC], axis=0)
    np.testing.assert_array_equal(st_out, full[-K:].T)


def test_conv_tap_order_impulses():
    r = rng(3)
    L, cd, K = 6, 3, 4
    xBC = r.standard_normal((L, cd))
    st = r.standard_normal((cd, K))
    b = np.zeros(cd)
    # tap K-1 multiplies the current token
    w = np.zeros((cd, K)); w[:, K - 1] = 1.0
    u, _ = oracle.conv_silu(xBC, w, b, st)
    np.testing.assert_allclose(u, xBC / (1 + np.exp(-xBC)), atol=1e-15)
    # tap 0 multiplies the input three tokens back (from the state for t < 3)
    w = np.zeros((cd, K)); w[:, 0] = 1.0
    u, _ = oracle.conv_silu(xBC, w, b, st)
    src = np.concatenate([st[:, 1:].T, xBC], axis=0)[:L]
    np.testing.assert_allclose(u, src / (1 + np.exp(-src)), atol=1e-15)


# ---------------------------------------------------------------- the scan

def _rand_scan(seed, L, H=2, P=3, N=4, G=1, h0=True, dt_scale=0.5):
    r = rng(seed)
    x = r.standard_normal((L, H, P))
    B = r.standard_normal((L, G, N))
    C = r.standard_normal((L, G, N))
    dt = dt_scale * r.uniform(0.05, 1.0, (L, H))
    A = -np.exp(r.uniform(0.0, math.log(16.0), H))
    D = r.standard_normal(H)
    hh = r.standard_normal((H, P, N)) if h0 else None
    return x, B, C, dt, A, D, hh


def test_scan_hand_worked_scalar_case():
    g = json.load(open(os.path.join(GOLDEN, "scalar_recurrence.json")))
    L = len(g["x"])
    x = np.array(g["x"]).reshape(L, 1, 1)
    B = np.array(g["B"]).reshape(L, 1, 1)
    C = np.array(g["C"]).reshape(L, 1, 1)
    dt = np.array(g["dt"]).reshape(L, 1)
    for form, q in (("sequential", 0), ("quadratic", 0), ("chunked", 1), ("chunked", 3)):
        y, hL = oracle.scan(x, B, C, dt, [g["A"]], [g["D"]], np.array([[[g["h0"]]]]), form, q)
        np.testing.assert_allclose(y.ravel(), g["y"], rtol=0, atol=1e-12)
        assert hL.item() == pytest.approx(g["hL"], abs=1e-12)


@pytest.mark.parametrize("G", [1, 2])
@pytest.mark.parametrize("with_h0", [False, True])
def test_quadratic_form_equals_sequential(G, with_h0):
    args = _rand_scan(1 + G, L=37, H=4, P=3, N=5, G=G, h0=with_h0)
    y0, h0 = oracle.scan(*args, form="sequential")
    y1, h1 = oracle.scan(*args, form="quadratic")
    np.testing.assert_allclose(y1, y0, rtol=0, atol=1e-11)
    np.testing.assert_allclose(h1, h0, rtol=0, atol=1e-11)


@pytest.mark.parametrize("Q", [1, 2, 3, 5, 16, 64, 50])
def test_chunked_form_equals_sequential(Q):
    # L = 50 is not a multiple of most Q: the last chunk is ragged
    args = _rand_scan(7, L=50, H=4, P=3, N=4, G=2)
    y0, h0 = oracle.scan(*args, form="sequential")
    y1, h1 = oracle.scan(*args, form="chunked", chunk=Q)
    np.testing.assert_allclose(y1, y0, rtol=0, atol=1e-11)
    np.testing.assert_allclose(h1, h0, rtol=0, atol=1e-11)


@pytest.mark.parametrize("form", ["sequential", "chunked"])
def test_A_zero_is_a_cumulative_sum(form):
    x, B, C, dt, A, D, h0 = _rand_scan(11, L=40, H=2, P=3, N=4)
    A = np.zeros_like(A)
    y, hL = oracle.scan(x, B, C, dt, A, D, h0, form=form, chunk=8)
    # h_t = h0 + sum_{s<=t} dt_s x_s B_s^T, computed as a numpy cumsum of outer products
    inc = dt[:, :, None, None] * x[:, :, :, None] * B[:, 0][:, None, None, :]
    hs = h0[None] + np.cumsum(inc, axis=0)
    ref = np.einsum("thpn,tn->thp", hs, C[:, 0]) + D[None, :, None] * x
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-11)
    np.testing.assert_allclose(hL, hs[-1], rtol=0, atol=1e-11)


@pytest.mark.parametrize("form", ["sequential", "quadratic", "chunked"])
def test_dt_zero_gives_D_skip_and_frozen_state(form):
    x, B, C, dt, A, D, h0 = _rand_scan(12, L=20, H=3, P=2, N=3)
    dt = np.zeros_like(dt)
    y, hL = oracle.scan(x, B, C, dt, A, D, h0, form=form, chunk=6)
    ref = np.einsum("hpn,tn->thp", h0, C[:, 0]) + D[None, :, None] * x
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hL, h0, rtol=0, atol=0)


def test_dt_zero_from_softplus_of_minus_inf():
    # dt_raw = -inf gives softplus = 0 exactly, so the mixer's y_pre is D x
    assert oracle.softplus(float("-inf") + 1.0) == 0.0


@pytest.mark.parametrize("form", ["sequential", "chunked"])
def test_very_negative_A_forgets(form):
    x, B, C, dt, A, D, h0 = _rand_scan(13, L=25, H=2, P=3, N=4)
    A = np.full_like(A, -1e4)
    y, hL = oracle.scan(x, B, C, dt, A, D, h0, form=form, chunk=4)
    # exp(dt*A) underflows to 0: h_t = dt_t x_t B_t^T
    ht = dt[:, :, None, None] * x[:, :, :, None] * B[:, 0][:, None, None, :]
    ref = np.einsum("thpn,tn->thp", ht, C[:, 0]) + D[None, :, None] * x
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hL, ht[-1], rtol=0, atol=1e-12)


def test_time_invariant_case_is_a_geometric_convolution():
    # constant dt, B, C: y_t = (C.B) dt sum_j exp(dt A j) x_{t-j} + D x_t, via np.convolve;
    # pins the decay exponent (exp of the sum over r in (s, t], not [s, t])
    L, N = 30, 3
    r = rng(21)
    x = r.standard_normal((L, 1, 1))
    Bv, Cv = r.standard_normal(N), r.standard_normal(N)
    B = np.tile(Bv, (L, 1)).reshape(L, 1, N)
    C = np.tile(Cv, (L, 1)).reshape(L, 1, N)
    dt_c, A_c, D_c = 0.3, -1.7, 0.4
    dt = np.full((L, 1), dt_c)
    kern = (Cv @ Bv) * dt_c * np.exp(dt_c * A_c * np.arange(L))
    ref = np.convolve(x.ravel(), kern)[:L] + D_c * x.ravel()
    for form, q in (("sequential", 0), ("quadratic", 0), ("chunked", 7)):
        y, _ = oracle.scan(x, B, C, dt, [A_c], [D_c], None, form=form, chunk=q)
        np.testing.assert_allclose(y.ravel(), ref, rtol=0, atol=1e-12)


def test_scan_is_causal_and_linear_in_x_and_h0():
    x, B, C, dt, A, D, h0 = _rand_scan(31, L=24, H=2, P=2, N=3)
    x2, _, _, _, _, _, h02 = _rand_scan(32, L=24, H=2, P=2, N=3)
    ya, ha = oracle.scan(x, B, C, dt, A, D, h0)
    yb, hb = oracle.scan(x2, B, C, dt, A, D, h02)
    yc, hc = oracle.scan(2.0 * x - 3.0 * x2, B, C, dt, A, D, 2.0 * h0 - 3.0 * h02)
    np.testing.assert_allclose(yc, 2.0 * ya - 3.0 * yb, atol=1e-11)
    np.testing.assert_allclose(hc, 2.0 * ha - 3.0 * hb, atol=1e-11)
    x3 = x.copy(); x3[15:] += 5.0
    y3, _ = oracle.scan(x3, B, C, dt, A, D, h0)
    np.testing.assert_array_equal(y3[:15], ya[:15])


def test_heads_use_contiguous_groups():
    # H = 4, G = 2: heads 0,1 read group 0's B/C and heads 2,3 read group 1's
    x, B, C, dt, A, D, h0 = _rand_scan(41, L=12, H=4, P=2, N=3, G=2)
    y, _ = oracle.scan(x, B, C, dt, A, D, h0)
    C2 = C.copy(); C2[:, 1] = 0.0
    y2, _ = oracle.scan(x, B, C2, dt, A, D, h0)
    np.testing.assert_array_equal(y2[:, :2], y[:, :2])
    np.testing.assert_allclose(y2[:, 2:], D[None, 2:, None] * x[:, 2:], atol=1e-15)


# ---------------------------------------------------------------- gated RMSNorm

@pytest.mark.parametrize("nbg", [False, True])
@pytest.mark.parametrize("G", [1, 2, 4])
def test_gated_norm_unit_rms_per_group(nbg, G):
    r = rng(50 + G)
    L, di = 5, 24
    y = r.standard_normal((L, di))
    z = r.standard_normal((L, di))
    out = oracle.gated_rmsnorm(y, z, np.ones(di), G, eps=0.0, norm_before_gate=nbg)
    s = 1.0 / (1.0 + np.exp(-z))
    unit = out / (z * s) if nbg else out  # strip the gate when it comes after the norm
    for k in range(G):
        sl = slice(k * di // G, (k + 1) * di // G)
        np.testing.assert_allclose(np.mean(unit[:, sl] ** 2, axis=1), 1.0, rtol=1e-12)
    if not nbg:  # gate first: the sign pattern is that of y * silu(z)
        np.testing.assert_array_equal(np.sign(out), np.sign(y * z * s))


@pytest.mark.parametrize("nbg", [False, True])
def test_gate_is_silu_of_z(nbg):
    # y = 1 and w = 1 (one group, eps = 0): the output is silu(z) up to one positive
    # scale, with silu(0) = 0, silu(+-1) = 0.7310585786300049 / -0.2689414213699951 and
    # silu(2) = 1.7615941559557649 (values of s / (1 + e^-s))
    sil = np.array([0.0, 0.7310585786300049, -0.2689414213699951, 1.7615941559557649])
    z = np.array([[0.0, 1.0, -1.0, 2.0]])
    out = oracle.gated_rmsnorm(np.ones((1, 4)), z, np.ones(4), 1, eps=0.0, norm_before_gate=nbg)
    scale = 1.0 if nbg else 1.0 / math.sqrt(np.mean(sil ** 2))
    np.testing.assert_allclose(out[0], sil * scale, rtol=1e-14, atol=1e-15)


def test_gated_norm_scale_invariance_weight_and_eps():
    r = rng(60)
    L, di = 4, 16
    y, z = r.standard_normal((L, di)), r.standard_normal((L, di))
    w = 1.0 + 0.1 * r.standard_normal(di)
    a = oracle.gated_rmsnorm(y, z, w, 2, eps=0.0)
    b = oracle.gated_rmsnorm(7.5 * y, z, w, 2, eps=0.0)
    np.testing.assert_allclose(a, b, rtol=1e-13)
    one = oracle.gated_rmsnorm(y, z, np.ones(di), 2, eps=0.0)
    np.testing.assert_allclose(a, one * w[None], rtol=1e-13)
    # eps enters inside the root: tiny inputs are damped, not blown up
    tiny = oracle.gated_rmsnorm(1e-6 * y, z, np.ones(di), 1, eps=1e-5)
    assert np.max(np.abs(tiny)) < 1e-2
    # huge z: silu(z) ~ z, a per-channel rescale that the norm does not cancel
    big = oracle.gated_rmsnorm(y, np.full((L, di), 40.0), np.ones(di), 1, eps=0.0)
    plain = oracle.gated_rmsnorm(y, np.full((L, di), 40.0), np.ones(di), 1, eps=0.0,
                                 norm_before_gate=True) / 40.0
    np.testing.assert_allclose(big, plain, rtol=1e-12)


# ---------------------------------------------------------------- whole mixer

def _mixer_case(seed, b=2, L=23, H=4, P=4, N=3, G=2, K=4):
    r = rng(seed)
    cd = H * P + 2 * G * N
    p = {"conv_w": r.uniform(-0.5, 0.5, (cd, K)), "conv_b": r.uniform(-0.5, 0.5, cd),
         "dt_bias": r.uniform(-4.0, -1.0, H), "A": -np.exp(r.uniform(0, math.log(16), H)),
         "D": r.standard_normal(H), "norm_w": 1.0 + 0.1 * r.standard_normal(H * P)}
    inp = {"xBC": r.standard_normal((b, L, cd)), "z": r.standard_normal((b, L, H * P)),
           "dt_raw": r.standard_normal((b, L, H))}
    st = {"conv_state": r.standard_normal((b, cd, K)),
          "ssm_state": 0.1 * r.standard_normal((b, H, P, N))}
    dims = dict(nheads=H, headdim=P, dstate=N, ngroups=G)
    return p, inp, st, dims


def test_mixer_is_the_composition_of_its_steps():
    p, inp, st, dims = _mixer_case(70)
    H, P, N, G = dims["nheads"], dims["headdim"], dims["dstate"], dims["ngroups"]
    out = oracle.mixer_prefill(inp["xBC"], inp["z"], inp["dt_raw"], p, **dims, **st)
    di = H * P
    for bi in range(2):
        u, cs = oracle.conv_silu(inp["xBC"][bi], p["conv_w"], p["conv_b"], st["conv_state"][bi])
        L = u.shape[0]
        x = u[:, :di].reshape(L, H, P)
        B = u[:, di:di + G * N].reshape(L, G, N)
        C = u[:, di + G * N:].reshape(L, G, N)
        dt = np.vectorize(oracle.softplus)(inp["dt_raw"][bi] + p["dt_bias"][None])
        y, hL = oracle.scan(x, B, C, dt, p["A"], p["D"], st["ssm_state"][bi])
        ref = oracle.gated_rmsnorm(y.reshape(L, di), inp["z"][bi], p["norm_w"], G)
        np.testing.assert_allclose(out["y"][bi], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(out["ssm_state"][bi], hL, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(out["conv_state"][bi], cs)


def test_mixer_channel_layout_x_then_B_then_C():
    p, inp, st, dims = _mixer_case(71, G=1)
    H, P, N = dims["nheads"], dims["headdim"], dims["dstate"]
    di = H * P
    # zero the C channels' conv (weight and bias): silu(0) = 0, so y_pre = D x exactly
    pc = dict(p); pc["conv_w"] = p["conv_w"].copy(); pc["conv_b"] = p["conv_b"].copy()
    pc["conv_w"][di + N:] = 0.0; pc["conv_b"][di + N:] = 0.0
    out = oracle.mixer_prefill(inp["xBC"], inp["z"], inp["dt_raw"], pc, **dims, **st)
    for bi in range(2):
        u, _ = oracle.conv_silu(inp["xBC"][bi], pc["conv_w"], pc["conv_b"], st["conv_state"][bi])
        ypre = (u[:, :di].reshape(-1, H, P) * p["D"][None, :, None]).reshape(-1, di)
        ref = oracle.gated_rmsnorm(ypre, inp["z"][bi], p["norm_w"], 1)
        np.testing.assert_allclose(out["y"][bi], ref, atol=1e-12)
    # zero the B channels and the initial state: nothing ever enters the state
    pb = dict(p); pb["conv_w"] = p["conv_w"].copy(); pb["conv_b"] = p["conv_b"].copy()
    pb["conv_w"][di:di + N] = 0.0; pb["conv_b"][di:di + N] = 0.0
    out = oracle.mixer_prefill(inp["xBC"], inp["z"], inp["dt_raw"], pb, **dims,
                               conv_state=st["conv_state"], ssm_state=None)
    assert np.all(out["ssm_state"] == 0.0)


@pytest.mark.parametrize("form,q", [("sequential", 0), ("chunked", 5), ("chunked", 64)])
def test_prefill_splits_into_two_prefills(form, q):
    p, inp, st, dims = _mixer_case(72, L=29)
    full = oracle.mixer_prefill(inp["xBC"], inp["z"], inp["dt_raw"], p, **dims, **st,
                                form=form, chunk=q)
    for L1 in (1, 2, 3, 11, 28):
        a = oracle.mixer_prefill(inp["xBC"][:, :L1], inp["z"][:, :L1], inp["dt_raw"][:, :L1], p,
                                 **dims, **st, form=form, chunk=q)
        b = oracle.mixer_prefill(inp["xBC"][:, L1:], inp["z"][:, L1:], inp["dt_raw"][:, L1:], p,
                                 **dims, conv_state=a["conv_state"], ssm_state=a["ssm_state"],
                                 form=form, chunk=q)
        np.testing.assert_allclose(np.concatenate([a["y"], b["y"]], axis=1), full["y"],
                                   atol=1e-11)
        np.testing.assert_allclose(b["ssm_state"], full["ssm_state"], atol=1e-11)
        np.testing.assert_array_equal(b["conv_state"], full["conv_state"])


def test_prefill_then_decode_steps_equals_prefill():
    p, inp, st, dims = _mixer_case(73, L=20)
    full = oracle.mixer_prefill(inp["xBC"], inp["z"], inp["dt_raw"], p, **dims, **st)
    k = 6
    a = oracle.mixer_prefill(inp["xBC"][:, :-k], inp["z"][:, :-k], inp["dt_raw"][:, :-k], p,
                             **dims, **st)
    cs, hs = a["conv_state"], a["ssm_state"]
    ys = []
    for t in range(20 - k, 20):
        o = oracle.mixer_step(inp["xBC"][:, t], inp["z"][:, t], inp["dt_raw"][:, t], p, cs, hs,
                              **dims)
        cs, hs = o["conv_state"], o["ssm_state"]
        ys.append(o["y"])
    np.testing.assert_allclose(np.stack(ys, axis=1), full["y"][:, -k:], atol=1e-11)
    np.testing.assert_allclose(hs, full["ssm_state"], atol=1e-11)
    np.testing.assert_array_equal(cs, full["conv_state"])


def test_empty_sequence_passes_states_through():
    p, inp, st, dims = _mixer_case(74)
    out = oracle.mixer_prefill(inp["xBC"][:, :0], inp["z"][:, :0], inp["dt_raw"][:, :0], p,
                               **dims, **st)
    assert out["y"].shape[1] == 0
    np.testing.assert_array_equal(out["ssm_state"], st["ssm_state"])
    np.testing.assert_array_equal(out["conv_state"], st["conv_state"])


def test_threads_do_not_change_results():
    p, inp, st, dims = _mixer_case(75, b=3, L=40)
    one = oracle.mixer_prefill(inp["xBC"], inp["z"], inp["dt_raw"], p, **dims, **st, nthreads=1)
    many = oracle.mixer_prefill(inp["xBC"], inp["z"], inp["dt_raw"], p, **dims, **st,
                                nthreads=4)
    for k in one:
        np.testing.assert_array_equal(one[k], many[k])
