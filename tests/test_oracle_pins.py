"""Pins of the fp64 oracle against facts fixed outside the oracle itself:
hand-worked examples (tests/golden), closed forms, invariants of doubly
stochastic matrices, textbook special cases and finite differences.

Each pin is chosen so that a plausible mistake in the oracle fails it:
  * Sinkhorn order (row pass then column pass) and axis: one-iteration
    hand example, exact column sums after a full iteration.
  * Sinkhorn as a diagonal scaling: cross-ratio invariance, the 2x2 limit.
  * Sinkhorn limit is doubly stochastic, non-expansive (spectral norm <= 1),
    closed under products; a dominant permutation is recovered.
  * RMS over all n*C entries, normalisation before the projection, logit
    column order, sigmoid / 2*sigmoid gates: closed forms on constant inputs.
  * Update equation: the n = 1 standard residual x + F, permutations,
    conservation of the stream sum for column-stochastic H_res.
  * Backward: central finite differences of the oracle forward for every
    input (x, phi, b, alpha, f_out), at several Sinkhorn iteration counts.
  * Depth product order and row/column gain: hand-multiplied example.
"""
import json
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed=0):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ Sinkhorn
def test_sinkhorn_one_iteration_hand_worked(oracle_mod):
    g = _golden("sinkhorn_2x2_one_iteration.json")
    H = oracle_mod.sinkhorn(np.log(np.array(g["logits_are_log_of"])), g["iters"])
    exp = np.array(g["expected_num"], float) / np.array(g["expected_den"], float)
    np.testing.assert_allclose(H, exp, rtol=0, atol=1e-15)


def test_sinkhorn_zero_iterations_is_exp(oracle_mod):
    z = _rng(1).normal(0, 2, size=(5, 4, 4))
    np.testing.assert_allclose(oracle_mod.sinkhorn(z, 0), np.exp(z), rtol=1e-15)


@pytest.mark.parametrize("n", [2, 3, 4, 8, 16])
def test_sinkhorn_last_pass_is_columns(oracle_mod, n):
    z = _rng(n).normal(0, 2, size=(20, n, n))
    for iters in (1, 2, 20):
        H = oracle_mod.sinkhorn(z, iters)
        np.testing.assert_allclose(H.sum(axis=1), 1.0, atol=1e-13)  # column sums
    H1 = oracle_mod.sinkhorn(z, 1)
    # after one iteration the row sums are generically not 1 (the row pass came first)
    assert np.max(np.abs(H1.sum(axis=2) - 1.0)) > 1e-3


@pytest.mark.parametrize("n", [2, 4, 8, 16])
def test_sinkhorn_is_a_diagonal_scaling(oracle_mod, n):
    """log H - z = u_i + v_j: every cross ratio of exp(z) survives every step."""
    z = _rng(10 + n).normal(0, 2, size=(8, n, n))
    for iters in (1, 3, 20):
        D = np.log(oracle_mod.sinkhorn(z, iters)) - z
        # double-centering of a rank-(u_i + v_j) matrix vanishes
        Dc = D - D.mean(axis=2, keepdims=True) - D.mean(axis=1, keepdims=True) + D.mean(axis=(1, 2), keepdims=True)
        assert np.max(np.abs(Dc)) < 1e-11


def test_sinkhorn_2x2_limit_closed_form(oracle_mod):
    for case in _golden("sinkhorn_2x2_limit.json")["cases"]:
        H = oracle_mod.sinkhorn(np.log(np.array(case["matrix"])), 2000)
        p = case["p"]
        np.testing.assert_allclose(H, [[p, 1 - p], [1 - p, p]], atol=1e-12)


@pytest.mark.parametrize("n", [4, 8, 16])
def test_sinkhorn_converges_to_doubly_stochastic(oracle_mod, n):
    z = _rng(20 + n).normal(0, 2, size=(16, n, n))
    H = oracle_mod.sinkhorn(z, 20000)
    assert np.all(H >= 0)
    np.testing.assert_allclose(H.sum(axis=2), 1.0, atol=1e-6)
    np.testing.assert_allclose(H.sum(axis=1), 1.0, atol=1e-12)
    # non-expansive: spectral norm <= 1 (a doubly stochastic matrix has norm exactly 1)
    s = np.linalg.svd(H, compute_uv=False)[:, 0]
    assert np.all(s <= 1.0 + 1e-6)
    # at the pages' t_max = 20 the row residual is reported, not asserted
    H20 = oracle_mod.sinkhorn(z, 20)
    print(f"n={n} row-sum residual after 20 iterations: {np.max(np.abs(H20.sum(axis=2) - 1)):.3e}")


@pytest.mark.parametrize("n", [4, 8])
def test_sinkhorn_recovers_dominant_permutation(oracle_mod, n):
    rng = _rng(30 + n)
    perm = rng.permutation(n)
    z = rng.normal(0, 1, size=(n, n))
    z[np.arange(n), perm] += 30.0
    H = oracle_mod.sinkhorn(z[None], 20)[0]
    P = np.zeros((n, n))
    P[np.arange(n), perm] = 1.0
    np.testing.assert_allclose(H, P, atol=1e-9)


def test_products_of_doubly_stochastic_stay_doubly_stochastic(oracle_mod):
    n, L, T = 4, 64, 8
    z = _rng(40).normal(0, 2, size=(T * L, n, n))
    H = oracle_mod.sinkhorn(z, 20000).reshape(T, L, n, n)
    P = np.broadcast_to(np.eye(n), (T, n, n)).copy()
    for l in range(L):
        P = H[:, l] @ P
    np.testing.assert_allclose(P.sum(axis=2), 1.0, atol=1e-9)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-9)
    gf, gb = oracle_mod.depth_amax(H)
    np.testing.assert_allclose(gf, 1.0, atol=1e-9)
    np.testing.assert_allclose(gb, 1.0, atol=1e-9)


def test_sinkhorn_backward_finite_differences(oracle_mod):
    rng = _rng(50)
    for n, iters in ((2, 1), (4, 3), (4, 20), (8, 5)):
        z = rng.normal(0, 1, size=(1, n, n))
        w = rng.normal(0, 1, size=(1, n, n))
        g = oracle_mod.sinkhorn_backward(z, w, iters)
        h = 1e-6
        fd = np.zeros_like(z)
        for idx in np.ndindex(z.shape):
            zp, zm = z.copy(), z.copy()
            zp[idx] += h
            zm[idx] -= h
            fd[idx] = (np.sum(w * oracle_mod.sinkhorn(zp, iters)) -
                       np.sum(w * oracle_mod.sinkhorn(zm, iters))) / (2 * h)
        np.testing.assert_allclose(g, fd, rtol=0, atol=1e-7 * max(1.0, np.max(np.abs(fd))))


# ------------------------------------------------------------- depth gain
def test_depth_amax_hand_multiplied(oracle_mod):
    g = _golden("depth_product_2x2.json")
    H = np.array(g["layers"])[None]
    gf, gb = oracle_mod.depth_amax(H)
    assert gf[0] == g["gain_fwd"] and gb[0] == g["gain_bwd"]


def test_depth_amax_rows_versus_columns(oracle_mod):
    H = np.tile(np.array([[1.0, 1.0], [0.0, 0.0]]), (1, 5, 1, 1))  # idempotent
    gf, gb = oracle_mod.depth_amax(H)
    assert gf[0] == 2.0 and gb[0] == 1.0
    gf0, gb0 = oracle_mod.depth_amax(np.zeros((3, 0, 4, 4)))
    assert np.all(gf0 == 1.0) and np.all(gb0 == 1.0)
    d = np.tile(np.diag([2.0, 1.0]), (1, 10, 1, 1))
    gf, gb = oracle_mod.depth_amax(d)
    assert gf[0] == 2.0 ** 10 and gb[0] == 2.0 ** 10


# ------------------------------------------------------------- the mapping
def _sig(v):
    return 1.0 / (1.0 + math.exp(-v))


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_pre_zero_projection_gives_bias_gates(oracle_mod, n):
    T, C = 3, 8
    M = n * n + 2 * n
    x = _rng(60).normal(size=(T, n, C))
    out = oracle_mod.pre(x, np.zeros((n * C, M)), np.zeros(M), 0.01, iters=20)
    np.testing.assert_allclose(out["H_pre"], 0.5, rtol=0, atol=1e-16)
    np.testing.assert_allclose(out["H_post"], 1.0, rtol=0, atol=1e-16)
    np.testing.assert_allclose(out["H_res"], 1.0 / n, rtol=0, atol=1e-15)
    np.testing.assert_allclose(out["h_in"], 0.5 * x.sum(axis=1), rtol=1e-15, atol=1e-15)
    b = _rng(61).normal(size=M)
    out = oracle_mod.pre(x, np.zeros((n * C, M)), b, 0.01, iters=0)
    np.testing.assert_allclose(out["H_pre"][0], [_sig(v) for v in b[:n]], rtol=1e-15)
    np.testing.assert_allclose(out["H_post"][0], [2 * _sig(v) for v in b[n:2 * n]], rtol=1e-15)
    np.testing.assert_allclose(out["H_res"][0].ravel(), np.exp(b[2 * n:]), rtol=1e-15)


def test_pre_rms_is_over_all_streams(oracle_mod):
    """Stream 0 = 2, other streams 0: mean square over all n*C = 4/n, so r = sqrt(4/n + eps)."""
    n, C, eps, alpha = 4, 8, 1e-6, 0.5
    M = n * n + 2 * n
    x = np.zeros((1, n, C))
    x[0, 0, :] = 2.0
    phi = np.zeros((n * C, M))
    phi[:, 0] = 1.0  # the first pre logit sums the normalised entries
    out = oracle_mod.pre(x, phi, np.zeros(M), alpha, iters=0, eps=eps)
    r = math.sqrt(4.0 / n + eps)
    assert out["r"][0] == pytest.approx(r, rel=1e-15)
    assert out["z"][0, 0] == pytest.approx(alpha * (2.0 * C) / r, rel=1e-14)
    assert out["H_pre"][0, 0] == pytest.approx(_sig(alpha * 16.0 / r), rel=1e-14)


def test_pre_normalises_before_projection(oracle_mod):
    """With eps = 0 the logits do not change when x is scaled."""
    n, C = 4, 16
    M = n * n + 2 * n
    rng = _rng(62)
    x = rng.normal(size=(2, n, C))
    phi = rng.normal(0, 0.3, size=(n * C, M))
    b = rng.normal(size=M)
    z1 = oracle_mod.pre(x, phi, b, 0.7, iters=5, eps=0.0)["z"]
    z2 = oracle_mod.pre(37.0 * x, phi, b, 0.7, iters=5, eps=0.0)["z"]
    np.testing.assert_allclose(z1, z2, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("n", [2, 4])
def test_pre_logit_column_order(oracle_mod, n):
    """One-hot phi column m moves exactly the output that column m names."""
    C = 8
    M = n * n + 2 * n
    x = np.ones((1, n, C))  # r = sqrt(1 + eps); y_m = n*C / r for a column of ones
    eps = 0.0
    for m in range(M):
        phi = np.zeros((n * C, M))
        phi[:, m] = 1.0 / (n * C)  # y_m = 1 exactly
        out = oracle_mod.pre(x, phi, np.zeros(M), 1.0, iters=0, eps=eps)
        pre = np.full(n, 0.5)
        post = np.full(n, 1.0)
        res = np.ones((n, n))
        if m < n:
            pre[m] = _sig(1.0)
        elif m < 2 * n:
            post[m - n] = 2 * _sig(1.0)
        else:
            i, j = divmod(m - 2 * n, n)
            res[i, j] = math.e
        np.testing.assert_allclose(out["H_pre"][0], pre, rtol=1e-15)
        np.testing.assert_allclose(out["H_post"][0], post, rtol=1e-15)
        np.testing.assert_allclose(out["H_res"][0], res, rtol=1e-15)


def test_pre_layer_input_weights_streams(oracle_mod):
    n, C = 4, 8
    M = n * n + 2 * n
    x = np.stack([np.full(C, float(i + 1)) for i in range(n)])[None]
    b = np.zeros(M)
    b[:n] = [-1.0, 0.0, 1.0, 2.0]
    out = oracle_mod.pre(x, np.zeros((n * C, M)), b, 0.0, iters=20)
    expect = sum(_sig(b[i]) * (i + 1) for i in range(n))
    np.testing.assert_allclose(out["h_in"], expect, rtol=1e-15)


# -------------------------------------------------------- the update equation
def test_post_n1_is_standard_residual(oracle_mod):
    x = _rng(70).normal(size=(5, 1, 16))
    f = _rng(71).normal(size=(5, 16))
    out = oracle_mod.post(x, f, np.ones((5, 1)), np.ones((5, 1, 1)))
    np.testing.assert_array_equal(out[:, 0], x[:, 0] + f)


def test_post_permutation_permutes_streams(oracle_mod):
    n, C = 4, 8
    rng = _rng(72)
    perm = rng.permutation(n)
    P = np.zeros((1, n, n))
    P[0, np.arange(n), perm] = 1.0
    x = rng.normal(size=(1, n, C))
    out = oracle_mod.post(x, rng.normal(size=(1, C)), np.zeros((1, n)), P)
    np.testing.assert_array_equal(out[0], x[0, perm])


def test_post_column_stochastic_conserves_stream_sum(oracle_mod):
    n, C, T = 4, 8, 6
    rng = _rng(73)
    H = oracle_mod.sinkhorn(rng.normal(0, 2, size=(T, n, n)), 20)  # exact column sums
    x = rng.normal(size=(T, n, C))
    f = rng.normal(size=(T, C))
    hp = rng.uniform(0, 2, size=(T, n))
    out = oracle_mod.post(x, f, hp, H)
    np.testing.assert_allclose(out.sum(axis=1), x.sum(axis=1) + hp.sum(axis=1)[:, None] * f,
                               atol=1e-12)


# ------------------------------------------------------------- the backward
def _loss(oracle_mod, x, phi, b, alpha, f, G, g, iters, eps):
    o = oracle_mod.pre(x, phi, b, alpha, iters=iters, eps=eps)
    xn = oracle_mod.post(x, f, o["H_post"], o["H_res"])
    return float(np.sum(G * xn) + np.sum(g * o["h_in"]))


@pytest.mark.parametrize("n,iters", [(1, 20), (2, 0), (2, 1), (4, 3), (4, 20), (8, 2), (16, 2)])
def test_backward_matches_finite_differences(oracle_mod, n, iters):
    T, C = 2, (8 if n <= 4 else 2)
    M = n * n + 2 * n
    eps = 1e-6
    rng = _rng(80 + 7 * n + iters)
    x = rng.normal(size=(T, n, C))
    phi = rng.normal(0, 0.3, size=(n * C, M))
    b = rng.normal(0, 1, size=M)
    alpha = 0.8
    f = rng.normal(size=(T, C))
    G = rng.normal(size=(T, n, C))
    g = rng.normal(size=(T, C))
    got = oracle_mod.backward(x, phi, b, alpha, f, G, g, iters=iters, eps=eps)
    h = 1e-6

    def fd(arr, setter):
        out = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            ap, am = arr.copy(), arr.copy()
            ap[idx] += h
            am[idx] -= h
            out[idx] = (setter(ap) - setter(am)) / (2 * h)
        return out

    L = lambda **kw: _loss(oracle_mod, kw.get("x", x), kw.get("phi", phi), kw.get("b", b),
                           kw.get("alpha", alpha), kw.get("f", f), G, g, iters, eps)
    checks = {
        "grad_x": fd(x, lambda a: L(x=a)),
        "grad_phi": fd(phi, lambda a: L(phi=a)),
        "grad_b": fd(b, lambda a: L(b=a)),
        "grad_f_out": fd(f, lambda a: L(f=a)),
    }
    for k, ref in checks.items():
        scale = max(1.0, float(np.max(np.abs(ref))))
        np.testing.assert_allclose(got[k], ref, rtol=0, atol=2e-7 * scale, err_msg=k)
    ga = (L(alpha=alpha + h) - L(alpha=alpha - h)) / (2 * h)
    assert got["grad_alpha"] == pytest.approx(ga, rel=1e-6, abs=1e-7)


def test_backward_parameter_sums_are_token_additive(oracle_mod):
    n, C, T = 4, 8, 7
    M = n * n + 2 * n
    rng = _rng(90)
    args = (rng.normal(size=(T, n, C)), rng.normal(0, 0.3, size=(n * C, M)), rng.normal(size=M),
            0.3, rng.normal(size=(T, C)), rng.normal(size=(T, n, C)), rng.normal(size=(T, C)))
    a = oracle_mod.backward(*args, iters=20)
    bch = oracle_mod.backward(*args, iters=20, chunk=3)
    for k in ("grad_phi", "grad_b"):
        np.testing.assert_allclose(a[k], bch[k], rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(a["grad_x"], bch["grad_x"])


# ------------------------------------- the backward in training order (split)
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_post_backward_finite_differences(oracle_mod, n):
    """The post half against central differences of L = sum G . post(x, f, H_post, H_res):
    grad_f_out = dL/df_out, red = (dL/dH_res row-major, dL/dH_post).  post is linear
    in each argument, so the differences are exact up to rounding."""
    T, C = 3, 5
    rng = _rng(120 + n)
    x = rng.normal(size=(T, n, C))
    f = rng.normal(size=(T, C))
    hp = rng.uniform(0, 2, size=(T, n))
    hr = rng.uniform(0, 1, size=(T, n, n))
    G = rng.normal(size=(T, n, C))
    got = oracle_mod.post_backward(x, f, hp, G)
    h = 1e-6

    def L(f_=f, hp_=hp, hr_=hr):
        return float(np.sum(G * oracle_mod.post(x, f_, hp_, hr_)))

    def fd(arr, which):
        out = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            ap, am = arr.copy(), arr.copy()
            ap[idx] += h
            am[idx] -= h
            out[idx] = (L(**{which: ap}) - L(**{which: am})) / (2 * h)
        return out

    np.testing.assert_allclose(got["grad_f_out"], fd(f, "f_"), rtol=0, atol=1e-8)
    red = got["red"].reshape(T, n * n + n)
    np.testing.assert_allclose(red[:, :n * n].reshape(T, n, n), fd(hr, "hr_"), rtol=0, atol=1e-8)
    np.testing.assert_allclose(red[:, n * n:], fd(hp, "hp_"), rtol=0, atol=1e-8)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_split_backward_equals_whole(oracle_mod, n):
    """post half -> pre half (with grad_h_in given) reproduces the one-call backward,
    whose every gradient is pinned by finite differences above."""
    T, C = 4, 6
    M = n * n + 2 * n
    rng = _rng(130 + n)
    x = rng.normal(size=(T, n, C))
    phi = rng.normal(0, 0.3, size=(n * C, M))
    b = rng.normal(size=M)
    f = rng.normal(size=(T, C))
    G = rng.normal(size=(T, n, C))
    g = rng.normal(size=(T, C))
    whole = oracle_mod.backward(x, phi, b, 0.7, f, G, g, iters=20)
    fwd = oracle_mod.pre(x, phi, b, 0.7, iters=20)
    pb = oracle_mod.post_backward(x, f, fwd["H_post"], G)
    qb = oracle_mod.pre_backward(x, phi, b, 0.7, G, g, pb["red"], iters=20)
    np.testing.assert_allclose(pb["grad_f_out"], whole["grad_f_out"], rtol=1e-13, atol=1e-13)
    for k in ("grad_x", "grad_phi", "grad_b"):
        np.testing.assert_allclose(qb[k], whole[k], rtol=1e-12, atol=1e-12, err_msg=k)
    assert qb["grad_alpha"] == pytest.approx(whole["grad_alpha"], rel=1e-12, abs=1e-12)


# ------------------------------------------------- per-group alpha (pre/post/res)
def test_per_group_alpha_finite_differences(oracle_mod):
    """With alpha = (a_pre, a_post, a_res) each logit group has its own scale:
    grad_alpha[g] against central differences of L in a_g, and grad_x / grad_phi
    against differences too (the groups enter the logits, u and kappa)."""
    n, T, C, iters, eps = 4, 2, 6, 20, 1e-6
    M = n * n + 2 * n
    rng = _rng(140)
    x = rng.normal(size=(T, n, C))
    phi = rng.normal(0, 0.3, size=(n * C, M))
    b = rng.normal(size=M)
    a3 = np.array([0.6, -0.4, 0.9])
    f = rng.normal(size=(T, C))
    G = rng.normal(size=(T, n, C))
    g = rng.normal(size=(T, C))
    got = oracle_mod.backward(x, phi, b, a3, f, G, g, iters=iters, eps=eps)
    assert np.shape(got["grad_alpha"]) == (3,)
    h = 1e-6
    for k in range(3):
        ap, am = a3.copy(), a3.copy()
        ap[k] += h
        am[k] -= h
        fd = (_loss(oracle_mod, x, phi, b, ap, f, G, g, iters, eps) -
              _loss(oracle_mod, x, phi, b, am, f, G, g, iters, eps)) / (2 * h)
        assert got["grad_alpha"][k] == pytest.approx(fd, rel=1e-6, abs=1e-7), k
    for idx in [(0, 1, 2), (1, 3, 5)]:
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd = (_loss(oracle_mod, xp, phi, b, a3, f, G, g, iters, eps) -
              _loss(oracle_mod, xm, phi, b, a3, f, G, g, iters, eps)) / (2 * h)
        assert got["grad_x"][idx] == pytest.approx(fd, rel=1e-6, abs=1e-7)


def test_three_equal_alphas_reproduce_one(oracle_mod):
    """alpha = (a, a, a) is the single-alpha layer; its grad_alpha entries add up to
    the single-alpha gradient."""
    n, T, C = 2, 3, 5
    M = n * n + 2 * n
    rng = _rng(141)
    x, phi, b = rng.normal(size=(T, n, C)), rng.normal(0, 0.3, size=(n * C, M)), rng.normal(size=M)
    f, G, g = rng.normal(size=(T, C)), rng.normal(size=(T, n, C)), rng.normal(size=(T, C))
    one = oracle_mod.backward(x, phi, b, 0.7, f, G, g)
    three = oracle_mod.backward(x, phi, b, np.array([0.7, 0.7, 0.7]), f, G, g)
    np.testing.assert_array_equal(one["grad_x"], three["grad_x"])
    assert one["grad_alpha"] == pytest.approx(float(np.sum(three["grad_alpha"])), rel=1e-14)
    p1, p3 = oracle_mod.pre(x, phi, b, 0.7), oracle_mod.pre(x, phi, b, np.array([0.7, 0.7, 0.7]))
    np.testing.assert_array_equal(p1["H_res"], p3["H_res"])
