"""Pins for the CPU oracle: it is checked here against things other than
itself -- values worked out by hand from the page's definitions
(tests/golden/hand_worked.json), closed forms, identities and invariants --
so that a dropped term, a wrong sign, an off-by-one in the cumulative sum or a
transposed operand in it fails at least one test.

Sources: 2Mamba2Furious (thelatestinai.com summary page), Algorithms 1-6.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from mamba_ssd_sequence_b200 import inputs


def _case_arrays(case, q, k, v):
    B, H, N, d = case["B"], case["H"], case["N"], case["d"]
    q = np.asarray(q, dtype=np.float32).reshape(B, H, N, d)
    k = np.asarray(k, dtype=np.float32).reshape(B, H, N, d)
    v = np.asarray(v, dtype=np.float32).reshape(B, H, N, d)
    dt_p = np.asarray(case["dt_p"], dtype=np.float32).reshape(B, H, N)
    A_log = np.asarray(case["A_log"], dtype=np.float32)
    dt_bias = np.asarray(case["dt_bias"], dtype=np.float32)
    return q, k, v, dt_p, A_log, dt_bias


@pytest.fixture(scope="module")
def golden(golden_dir):
    with open(os.path.join(golden_dir, "hand_worked.json")) as f:
        return {c["name"]: c for c in json.load(f)["cases"]}


# ---------------------------------------------------------------- hand-worked
def test_hand_constant_decay(golden):
    """Algorithms 1/3/4/5 on a 3-token, d=2 case worked out by hand."""
    c = golden["constant-half-decay"]
    q, k, v, dt_p, A_log, dt_bias = _case_arrays(c, c["q"], c["k"], c["v"])
    acs = oracle.log_decay(dt_p, A_log, dt_bias)[0, 0]
    np.testing.assert_allclose(acs, c["acs"], rtol=1e-15)
    Dres = np.asarray(c["D"], dtype=np.float32)
    for e in c["expect"]:
        D = Dres if e["residual"] else None
        for form in (oracle.ssd_quadratic, oracle.ssd_recurrent):
            y, n = form(q, k, v, dt_p, A_log, dt_bias, D, e["order"], e["normalize"],
                        return_norm=True)
            np.testing.assert_allclose(y[0, 0], e["y"], rtol=1e-14, atol=1e-14,
                                       err_msg=f"{form.__name__} {e}")
            if "norm" in e:
                np.testing.assert_allclose(n[0, 0], e["norm"], rtol=1e-14, atol=1e-14)


def test_hand_varying_decay_inclusive_cumsum(golden):
    """The inclusive cumulative sum (decay-then-add, Algorithm 6) on a case
    where an exclusive sum would give different numbers."""
    c = golden["varying-decay-inclusive-cumsum"]
    for var in c["variants"]:
        q, k, v, dt_p, A_log, dt_bias = _case_arrays(c, var["q"], var["k"], var["v"])
        acs = oracle.log_decay(dt_p, A_log, dt_bias)[0, 0]
        # dt_p = ln 3 is stored as float32, so the decay is ln 4 to ~1e-7.
        np.testing.assert_allclose(acs, c["acs"], rtol=1e-7)
        for form in (oracle.ssd_quadratic, oracle.ssd_recurrent):
            y, n = form(q, k, v, dt_p, A_log, dt_bias, None, var["order"], var["normalize"],
                        return_norm=True)
            np.testing.assert_allclose(y[0, 0], var["y"], rtol=2e-7, err_msg=form.__name__)
            if "norm" in var:
                np.testing.assert_allclose(n[0, 0], var["norm"], rtol=2e-7)


# ------------------------------------------------------------ scalar helpers
def test_softplus_closed_forms():
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-16)
    assert oracle.softplus(math.log(3.0)) == pytest.approx(math.log(4.0), rel=1e-15)
    assert oracle.softplus(50.0) == pytest.approx(50.0, rel=1e-16)
    assert oracle.softplus(-50.0) == pytest.approx(math.exp(-50.0), rel=1e-12)
    # softplus(x) - softplus(-x) = x for every x
    for x in (-7.3, -0.1, 0.4, 3.9, 25.0):
        assert oracle.softplus(x) - oracle.softplus(-x) == pytest.approx(x, rel=1e-13, abs=1e-15)


def test_dt_bias_is_softplus_inverse():
    """Algorithm 2: dt_bias = softplus^-1(dt_init), dt_init in [1e-3, 1e-1]."""
    x = inputs.make_inputs(1, 64, 4, 4, "f32", seed=3)
    dt0 = np.array([oracle.softplus(float(b)) for b in x["dt_bias"]])
    assert np.all(dt0 >= inputs.DT_MIN * (1 - 1e-5))
    assert np.all(dt0 <= inputs.DT_MAX * (1 + 1e-5))
    assert np.all((x["A_log"] >= 0) & (x["A_log"] <= math.log(16.0) + 1e-6))


def test_feature_tensor_square_identity():
    """(q . k)^2 = (q (x) q) . (k (x) k)  (Algorithm 5 vs Algorithm 6)."""
    rng = np.random.default_rng(5)
    for d in (1, 3, 16):
        q = rng.standard_normal(d)
        k = rng.standard_normal(d)
        fq, fk = oracle.feature(q, 2), oracle.feature(k, 2)
        assert fq.shape == (d * d,)
        assert np.dot(fq, fk) == pytest.approx(np.dot(q, k) ** 2, rel=1e-12)
        assert np.array_equal(oracle.feature(q, 1), q)
        # entry (a, b) at a*d + b
        assert fq[(d - 1) * d + 0] == pytest.approx(q[d - 1] * q[0])


def test_mask_properties():
    """Algorithm 4: M_ii = 1, 0 < M_ij <= 1 below the diagonal (A < 0, dt > 0),
    zero above it."""
    x = inputs.make_inputs(1, 3, 48, 4, "f32", seed=1)
    acs = oracle.log_decay(x["dt_p"], x["A_log"], x["dt_bias"])
    for h in range(3):
        row = acs[0, h]
        assert np.all(np.diff(row) < 0)  # strictly decreasing: every a_t < 0
        for i in range(48):
            assert oracle.mask(row, i, i) == 1.0
            for j in range(48):
                m = oracle.mask(row, i, j)
                if j > i:
                    assert m == 0.0
                elif j < i:
                    assert 0.0 < m <= 1.0


# --------------------------------------------------------- brute force forms
def _brute(q, k, v, dt_p, A_log, dt_bias, D, order, normalize):
    """Matrix form with explicit N x N A^M and M and explicit tensor-square
    features (Algorithm 4 / 5 as printed), in numpy float64."""
    B, H, N, d = q.shape
    y = np.zeros((B, H, N, d))
    for b in range(B):
        for h in range(H):
            A = -np.exp(np.float64(A_log[h]))
            z = dt_p[b, h].astype(np.float64) + np.float64(dt_bias[h])
            dt = np.log1p(np.exp(z))
            acs = np.cumsum(A * dt)
            AM = np.exp(acs[:, None] - acs[None, :])
            M = np.tril(np.ones((N, N)))
            Q = q[b, h].astype(np.float64)
            K = k[b, h].astype(np.float64)
            if order == 2:
                Q = np.stack([np.kron(r, r) for r in Q])
                K = np.stack([np.kron(r, r) for r in K])
            W = (Q @ K.T) * np.where(M > 0, AM, 0.0)
            yy = W @ v[b, h].astype(np.float64)
            if normalize:
                yy = yy / W.sum(axis=1, keepdims=True)
            if D is not None:
                yy = yy + D[h * d:(h + 1) * d][None, :].astype(np.float64) * v[b, h]
            y[b, h] = yy
    return y


@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("normalize", [False, True])
@pytest.mark.parametrize("residual", [False, True])
def test_quadratic_recurrent_brute_agree(order, normalize, residual):
    """Three independent evaluations: loops over i >= j (Algorithm 5), the
    token recurrence (Algorithm 6) and the explicit matrix form."""
    x = inputs.make_inputs(2, 3, 37, 5, "f32", seed=11, residual=residual)
    q, k = x["q"], x["k"]
    if order == 1 and normalize:
        # Order-1 row sums can pass through zero with SiLU features; positive
        # scores keep the normalised case well conditioned.
        q, k = np.abs(q), np.abs(k)
    args = (q, k, x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], order, normalize)
    yq = oracle.ssd_quadratic(*args)
    yr = oracle.ssd_recurrent(*args)
    yb = _brute(*args)
    scale = np.max(np.abs(yb))
    assert np.max(np.abs(yq - yb)) <= 1e-12 * scale
    assert np.max(np.abs(yr - yb)) <= 1e-12 * scale


def test_sampled_rows_match_full():
    x = inputs.make_inputs(1, 2, 70, 4, "bf16", seed=2)
    args = (x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], 2, True)
    full = oracle.ssd_quadratic(*args)
    rows = [0, 1, 33, 69, 5]
    part = oracle.ssd_quadratic(*args, rows=rows)
    np.testing.assert_array_equal(part, full[:, :, rows, :])


# ------------------------------------------------------------- closed forms
@pytest.mark.parametrize("order", [1, 2])
def test_no_decay_is_prefix_sum_linear_attention(order):
    """A_log -> -inf makes A = 0 and every A^M_ij = 1: plain causal linear
    attention (Algorithm 1 with M only), y_i = phi(q_i)^T sum_{j<=i} phi(k_j) v_j^T."""
    x = inputs.make_inputs(1, 2, 29, 3, "f32", seed=7, residual=False)
    A_log = np.full(2, -1000.0, dtype=np.float32)
    y = oracle.ssd_quadratic(x["q"], x["k"], x["v"], x["dt_p"], A_log, x["dt_bias"], None,
                             order, False)
    for h in range(2):
        Q = x["q"][0, h].astype(np.float64)
        K = x["k"][0, h].astype(np.float64)
        V = x["v"][0, h].astype(np.float64)
        if order == 2:
            Q = np.einsum("ta,tb->tab", Q, Q).reshape(29, -1)
            K = np.einsum("ta,tb->tab", K, K).reshape(29, -1)
        S = np.cumsum(np.einsum("tm,tc->tmc", K, V), axis=0)
        ref = np.einsum("tm,tmc->tc", Q, S)
        np.testing.assert_allclose(y[0, h], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("order", [1, 2])
def test_instant_decay_gives_diagonal(order):
    """A_log huge: every off-diagonal A^M_ij underflows to 0 and only the
    diagonal survives, y_i = (q_i . k_i)^order v_i; normalised, y_i = v_i."""
    x = inputs.make_inputs(1, 2, 17, 4, "f32", seed=8, residual=False)
    A_log = np.full(2, 80.0, dtype=np.float32)
    args = (x["q"], x["k"], x["v"], x["dt_p"], A_log, x["dt_bias"], None, order)
    y = oracle.ssd_quadratic(*args, False)
    s = np.einsum("bhtc,bhtc->bht", x["q"].astype(np.float64), x["k"].astype(np.float64))
    ref = (s ** order)[..., None] * x["v"]
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)
    yn = oracle.ssd_quadratic(*args, True)
    np.testing.assert_allclose(yn, x["v"], rtol=1e-12)


def test_constant_values_normalised_return_the_constant():
    """With the normaliser, the output is a convex-like average of the v_j
    (order 2 weights are >= 0): constant v gives back that constant."""
    x = inputs.make_inputs(2, 2, 40, 6, "f32", seed=9, residual=False)
    v = np.full_like(x["v"], 0.375)
    y = oracle.ssd_quadratic(x["q"], x["k"], v, x["dt_p"], x["A_log"], x["dt_bias"], None, 2, True)
    np.testing.assert_allclose(y, 0.375, rtol=1e-12)


def test_zero_queries_leave_only_the_residual():
    x = inputs.make_inputs(1, 2, 12, 4, "f32", seed=4)
    D = np.arange(8, dtype=np.float32) * 0.25 - 1.0
    q = np.zeros_like(x["q"])
    for order in (1, 2):
        y = oracle.ssd_quadratic(q, x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], D,
                                 order, False)
        ref = x["v"].astype(np.float64) * D.reshape(2, 4).astype(np.float64)[None, :, None, :]
        np.testing.assert_array_equal(y, ref)


def test_single_token():
    x = inputs.make_inputs(1, 1, 1, 5, "f32", seed=6, residual=False)
    s = float(np.dot(x["q"][0, 0, 0].astype(np.float64), x["k"][0, 0, 0].astype(np.float64)))
    for order in (1, 2):
        y = oracle.ssd_recurrent(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"],
                                 None, order, False)
        np.testing.assert_allclose(y[0, 0, 0], s ** order * x["v"][0, 0, 0].astype(np.float64),
                                   rtol=1e-13)


# ---------------------------------------------------------------- invariants
def test_linear_in_v_and_homogeneous_in_q():
    x = inputs.make_inputs(1, 2, 25, 4, "f32", seed=12, residual=False)
    base = (x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], None)
    for order in (1, 2):
        y = oracle.ssd_quadratic(x["q"], *base, order, False)
        ya = oracle.ssd_quadratic(np.float32(2.0) * x["q"], *base, order, False)
        np.testing.assert_allclose(ya, (2.0 ** order) * y, rtol=1e-12, atol=1e-13)
        v2 = x["v"] * np.float32(-2.0)  # exact in float32
        yv = oracle.ssd_quadratic(x["q"], x["k"], v2, x["dt_p"], x["A_log"], x["dt_bias"], None,
                                  order, False)
        np.testing.assert_allclose(yv, -2.0 * y, rtol=1e-12, atol=1e-13)
    yn = oracle.ssd_quadratic(x["q"], *base, 2, True)
    yna = oracle.ssd_quadratic(np.float32(4.0) * x["q"], *base, 2, True)
    np.testing.assert_allclose(yna, yn, rtol=1e-12)


def test_head_and_batch_permutation_equivariance():
    x = inputs.make_inputs(2, 3, 20, 4, "f32", seed=13)
    D = np.arange(12, dtype=np.float32) * 0.1
    args = lambda q, k, v, dt, al, db, DD: (q, k, v, dt, al, db, DD, 2, True)
    y = oracle.ssd_quadratic(*args(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"],
                                   x["dt_bias"], D))
    hp = [2, 0, 1]
    bp = [1, 0]
    Dp = D.reshape(3, 4)[hp].reshape(-1)
    yp = oracle.ssd_quadratic(*args(x["q"][bp][:, hp], x["k"][bp][:, hp], x["v"][bp][:, hp],
                                    x["dt_p"][bp][:, hp], x["A_log"][hp], x["dt_bias"][hp], Dp))
    np.testing.assert_allclose(yp, y[bp][:, hp], rtol=1e-13)


def test_recurrent_final_state_matches_definition():
    """The final H_up from Algorithm 6 equals sum_j exp(A^CS_N-1 - A^CS_j) phi(k_j) v_j^T."""
    x = inputs.make_inputs(1, 1, 15, 3, "f32", seed=14)
    for order in (1, 2):
        _, _, st, zst = oracle.ssd_recurrent(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"],
                                             x["dt_bias"], None, order, False, return_norm=True,
                                             return_state=True)
        acs = oracle.log_decay(x["dt_p"], x["A_log"], x["dt_bias"])[0, 0]
        ref = np.zeros_like(st[0, 0])
        zref = np.zeros_like(zst[0, 0])
        for j in range(15):
            fk = oracle.feature(x["k"][0, 0, j], order)
            w = math.exp(acs[-1] - acs[j])
            ref += w * np.outer(fk, x["v"][0, 0, j])
            zref += w * fk
        np.testing.assert_allclose(st[0, 0], ref, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(zst[0, 0], zref, rtol=1e-12, atol=1e-14)


# ------------------------------------------- Mamba-2S options (Algorithm 4)
def test_hand_mamba2s_log_decay_value_dt(golden):
    """Given per-token log-decays and value discretisation V (.) dt
    (Algorithm 4), on a 3-token case worked out by hand."""
    c = golden["mamba2s-log-decay-value-dt"]
    B, H, N, d = c["B"], c["H"], c["N"], c["d"]
    q = np.asarray(c["q"], np.float32).reshape(B, H, N, d)
    k = np.asarray(c["k"], np.float32).reshape(B, H, N, d)
    v = np.asarray(c["v"], np.float32).reshape(B, H, N, d)
    ld = np.asarray(c["log_decay"], np.float32).reshape(B, H, N)
    dt_p = np.asarray(c["dt_p"], np.float32).reshape(B, H, N)
    dt_bias = np.asarray(c["dt_bias"], np.float32)
    Dres = np.asarray(c["D"], np.float32)
    acs = oracle.log_decay(None, None, None, log_decay_in=ld)[0, 0]
    np.testing.assert_allclose(acs, c["acs"], rtol=1e-7)  # the inputs are float32
    for e in c["expect"]:
        D = Dres if e["residual"] else None
        for form in (oracle.ssd_quadratic, oracle.ssd_recurrent):
            y, n = form(q, k, v, dt_p if e["value_dt"] else None, None,
                        dt_bias if e["value_dt"] else None, D, e["order"], e["normalize"],
                        return_norm=True, log_decay=ld, value_dt=e["value_dt"])
            np.testing.assert_allclose(y[0, 0], e["y"], rtol=3e-7, err_msg=f"{form.__name__} {e}")
            if "norm" in e:
                np.testing.assert_allclose(n[0, 0], e["norm"], rtol=3e-7)


def _small(seed, B=2, H=2, N=19, d=3):
    x = inputs.make_inputs(B, H, N, d, "f32", seed=seed, residual=True)
    return x


@pytest.mark.parametrize("order", [1, 2])
def test_log_decay_input_matches_a_dt(order):
    """Passing a_t = -exp(A_log) softplus(dt_p + dt_bias) as the log-decay
    input reproduces the Algorithm 3 parameterisation."""
    x = _small(3)
    dt = np.log1p(np.exp(-np.abs(x["dt_p"].astype(np.float64) + x["dt_bias"][None, :, None]))) + \
        np.maximum(x["dt_p"].astype(np.float64) + x["dt_bias"][None, :, None], 0.0)
    ld = (-np.exp(x["A_log"].astype(np.float64))[None, :, None] * dt).astype(np.float32)
    for norm in (False, True):
        ref = oracle.ssd_quadratic(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"],
                                   order, norm)
        got = oracle.ssd_quadratic(x["q"], x["k"], x["v"], None, None, None, x["D"], order, norm,
                                   log_decay=ld)
        np.testing.assert_allclose(got, ref, rtol=2e-5, atol=1e-6)


@pytest.mark.parametrize("order", [1, 2])
def test_value_dt_is_prescaled_values(order):
    """value_dt equals the plain operator on V pre-scaled by dt per token
    (the caller-side form of Algorithm 4's V_dt); the normaliser and the
    residual (here off) do not see dt."""
    x = _small(4)
    z = x["dt_p"].astype(np.float64) + x["dt_bias"][None, :, None]
    dt = np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))
    v_dt = (x["v"].astype(np.float64) * dt[..., None]).astype(np.float32)
    for norm in (False, True):
        got, n_got = oracle.ssd_quadratic(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], None,
                                          order, norm, value_dt=True, return_norm=True)
        ref, n_ref = oracle.ssd_quadratic(x["q"], x["k"], v_dt, x["dt_p"], x["A_log"], x["dt_bias"], None,
                                          order, norm, return_norm=True)
        np.testing.assert_allclose(got, ref, rtol=2e-6, atol=1e-7)
        np.testing.assert_allclose(n_got, n_ref, rtol=1e-14)


@pytest.mark.parametrize("order,norm", [(1, False), (2, True), (2, False)])
def test_options_quadratic_equals_recurrent(order, norm):
    """Algorithm 5 and Algorithm 6 agree with both options on."""
    x = _small(5, N=23)
    rng = np.random.default_rng(11)
    ld = (-rng.uniform(0.0, 0.7, size=x["dt_p"].shape)).astype(np.float32)
    kw = dict(log_decay=ld, value_dt=True)
    a = oracle.ssd_quadratic(x["q"], x["k"], x["v"], x["dt_p"], None, x["dt_bias"], x["D"], order, norm, **kw)
    b = oracle.ssd_recurrent(x["q"], x["k"], x["v"], x["dt_p"], None, x["dt_bias"], x["D"], order, norm, **kw)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_zero_log_decay_value_dt_prefix_sums():
    """With a zero log-decay the mask is all ones below the diagonal, so the
    operator is causal linear attention over V (.) dt: prefix sums."""
    x = _small(6, B=1, H=1, N=17, d=4)
    ld = np.zeros_like(x["dt_p"])
    y = oracle.ssd_quadratic(x["q"], x["k"], x["v"], x["dt_p"], None, x["dt_bias"], None, 1, False,
                             log_decay=ld, value_dt=True)[0, 0]
    z = x["dt_p"][0, 0].astype(np.float64) + float(x["dt_bias"][0])
    dt = np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))
    kv = np.einsum("nc,ne->nce", x["k"][0, 0].astype(np.float64), x["v"][0, 0].astype(np.float64) * dt[:, None])
    S = np.cumsum(kv, axis=0)
    ref = np.einsum("nc,nce->ne", x["q"][0, 0].astype(np.float64), S)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------ carried state in and out (Algorithm 6)
def test_hand_decode_step_initial_state(golden):
    """One recurrent step from a given state, worked out by hand."""
    c = golden["decode-step-initial-state"]
    arr = lambda a: np.asarray(a, np.float32).reshape(1, 1, 1, 1)
    q, k, v = arr(c["q"]), arr(c["k"]), arr(c["v"])
    ld = np.asarray(c["log_decay"], np.float32).reshape(1, 1, 1)
    h0 = np.asarray(c["h0"], np.float64).reshape(1, 1, 1, 1)
    z0 = np.asarray(c["z0"], np.float64).reshape(1, 1, 1)
    for e in c["expect"]:
        D = np.asarray(c["D"], np.float32) if e["residual"] else None
        y, _, h, z = oracle.ssd_recurrent(q, k, v, None, None, None, D, e["order"], e["normalize"],
                                          return_norm=True, return_state=True, log_decay=ld, h0=h0, z0=z0)
        np.testing.assert_allclose(y[0, 0], e["y"], rtol=1e-7)
        if "h" in e:
            np.testing.assert_allclose(h[0, 0], e["h"], rtol=1e-7)
            np.testing.assert_allclose(z[0, 0], e["z"], rtol=1e-7)
        yq = oracle.ssd_quadratic(q, k, v, None, None, None, D, e["order"], e["normalize"],
                                  log_decay=ld, h0=h0, z0=z0)
        np.testing.assert_allclose(yq[0, 0], e["y"], rtol=1e-7)


@pytest.mark.parametrize("order,norm", [(1, False), (2, True)])
def test_split_sequence_carries_state(order, norm):
    """Running tokens [0, n) and then [n, N) from the state the first part
    leaves gives the same outputs as running [0, N) at once."""
    x = _small(7, N=21)
    n = 8
    y_all = oracle.ssd_recurrent(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"],
                                 order, norm)
    sl = lambda a, lo, hi: a[:, :, lo:hi]
    y1, h, z = oracle.ssd_recurrent(sl(x["q"], 0, n), sl(x["k"], 0, n), sl(x["v"], 0, n), sl(x["dt_p"], 0, n),
                                    x["A_log"], x["dt_bias"], x["D"], order, norm, return_state=True)
    y2 = oracle.ssd_recurrent(sl(x["q"], n, None), sl(x["k"], n, None), sl(x["v"], n, None),
                              sl(x["dt_p"], n, None), x["A_log"], x["dt_bias"], x["D"], order, norm, h0=h, z0=z)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=2), y_all, rtol=1e-12, atol=1e-12)
    # the quadratic form with the same carried state agrees with the recurrence
    y2q = oracle.ssd_quadratic(sl(x["q"], n, None), sl(x["k"], n, None), sl(x["v"], n, None),
                               sl(x["dt_p"], n, None), x["A_log"], x["dt_bias"], x["D"], order, norm, h0=h, z0=z)
    np.testing.assert_allclose(y2q, y2, rtol=1e-11, atol=1e-12)


def test_zero_decay_initial_state_prefix_sums():
    """Zero log-decay from a given state: y_i = q_i^T (h0 + sum_{j<=i} k_j v_j^T)."""
    x = _small(8, B=1, H=1, N=13, d=3)
    rng = np.random.default_rng(3)
    h0 = rng.standard_normal((1, 1, 3, 3))
    ld = np.zeros_like(x["dt_p"])
    y = oracle.ssd_quadratic(x["q"], x["k"], x["v"], None, None, None, None, 1, False, log_decay=ld, h0=h0)[0, 0]
    S = h0[0, 0] + np.cumsum(np.einsum("nc,ne->nce", x["k"][0, 0].astype(np.float64),
                                       x["v"][0, 0].astype(np.float64)), axis=0)
    ref = np.einsum("nc,nce->ne", x["q"][0, 0].astype(np.float64), S)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------- conv1d + SiLU prologue (Algorithms 3, 6)
def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16
    assert abs(oracle.silu(-1.0) + math.exp(-1.0) / (1.0 + math.exp(-1.0))) < 1e-16
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12          # x sigmoid(x) -> x
    assert abs(oracle.silu(-40.0)) < 1e-15                # -> 0


def test_conv1d_hand_worked():
    """Window 2 on one channel: u_t = 2 x_t - x_{t-1} + 0.5, x_{-1} = 0.
    x = (1, 3, -2): u = (2.5, 5.5, -6.5)."""
    x = np.asarray([1, 3, -2], np.float32).reshape(1, 1, 3, 1)
    w = np.asarray([[2, -1]], np.float32)
    b = np.asarray([0.5], np.float32)
    u = oracle.conv1d(x, w, b, silu=False)[0, 0, :, 0]
    np.testing.assert_array_equal(u, [2.5, 5.5, -6.5])
    y = oracle.conv1d(x, w, b, silu=True)[0, 0, :, 0]
    np.testing.assert_allclose(y, [v / (1 + math.exp(-v)) for v in (2.5, 5.5, -6.5)], rtol=1e-15)


def test_conv1d_identity_and_shift_and_causality():
    """w = (1, 0) is the identity; w = (0, 1) shifts by one token with a zero
    first token; no token depends on a later one; heads never mix."""
    x = _small(9, B=2, H=3, N=11, d=4)["q"]
    H, d = 3, 4
    ident = np.tile(np.asarray([[1, 0]], np.float32), (H * d, 1))
    np.testing.assert_array_equal(oracle.conv1d(x, ident, silu=False), x.astype(np.float64))
    shift = np.tile(np.asarray([[0, 1]], np.float32), (H * d, 1))
    s = oracle.conv1d(x, shift, silu=False)
    np.testing.assert_array_equal(s[:, :, 1:], x[:, :, :-1].astype(np.float64))
    assert np.all(s[:, :, 0] == 0)
    w = np.random.default_rng(1).standard_normal((H * d, 3)).astype(np.float32)
    y = oracle.conv1d(x, w, silu=True)
    x2 = x.copy()
    x2[:, :, 7:] = 100.0                                  # change the future only
    np.testing.assert_array_equal(oracle.conv1d(x2, w, silu=True)[:, :, :7], y[:, :, :7])
    x3 = x.copy()
    x3[:, 1] = 0.0                                        # another head only
    np.testing.assert_array_equal(oracle.conv1d(x3, w, silu=True)[:, 0], y[:, 0])


def test_conv1d_hand_worked_per_head_weights():
    """Two heads of two channels, window 2, with a different weight row for
    every channel h*d + c (the weight row of channel c of head h), and a second
    batch holding the negated tokens.  Worked by hand:
      head 0, w = (1, 10), (2, 20), tokens (1, 2), (3, 4):
        u_0 = (1*1, 2*2) = (1, 4);  u_1 = (1*3 + 10*1, 2*4 + 20*2) = (13, 48)
      head 1, w = (3, 30), (4, 40), tokens (5, 6), (7, 8):
        u_0 = (3*5, 4*6) = (15, 24); u_1 = (3*7 + 30*5, 4*8 + 40*6) = (171, 272)
    The second batch gives the negated values (the weights depend on the head
    only).  Indexing the weights by the channel alone, by b*H + h, or with the
    weight array transposed changes at least one of these values."""
    x = np.asarray([[[[1, 2], [3, 4]], [[5, 6], [7, 8]]]], np.float32)
    x = np.concatenate([x, -x], axis=0)                   # [B=2, H=2, N=2, d=2]
    w = np.asarray([[1, 10], [2, 20], [3, 30], [4, 40]], np.float32)
    u = oracle.conv1d(x, w, None, silu=False)
    want = np.asarray([[[1, 4], [13, 48]], [[15, 24], [171, 272]]], np.float64)
    np.testing.assert_array_equal(u[0], want)
    np.testing.assert_array_equal(u[1], -want)
