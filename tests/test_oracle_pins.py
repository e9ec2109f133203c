"""Pins of the fp64 oracle to facts fixed outside the oracle itself (CPU only).

Each test checks the oracle against a published known-answer vector, a library
routine, a closed form, an invariant or a brute-force special case, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand, an
exclusive instead of inclusive causal sum) fails at least one of them.

Method source: "SLAY: Geometry-Aware Spherical Linearized Attention with Yat-Kernel"
(abstract; nubint.ai review, "Proposed method" steps 1-6).
"""
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ Philox

def _kat_rows():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            w = [int(x, 16) for x in line.split()]
            rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


def test_philox_known_answers():
    rows = _kat_rows()
    assert len(rows) == 3
    for ctr, key, out in rows:
        assert O.philox4x32_10(ctr, key) == out


# --------------------------------------------------------- Gauss-Laguerre

@pytest.mark.parametrize("R", list(range(1, 17)))
def test_gauss_laguerre_moments(R):
    # The R-point rule integrates e^{-t} t^k exactly for k < 2R: int = k!.
    t, w = O.gauss_laguerre(R)
    for k in range(2 * R):
        got = float(np.sum(w * t ** k))
        assert abs(got - math.factorial(k)) <= 1e-11 * math.factorial(k), (R, k, got)
    # ... and not for k = 2R (the degree is exactly 2R-1): the remainder is
    # (R!)^2 > 0, so the rule falls short of (2R)! by exactly (R!)^2.
    got = float(np.sum(w * t ** (2 * R)))
    want = math.factorial(2 * R) - math.factorial(R) ** 2
    assert abs(got - want) <= 1e-9 * math.factorial(2 * R)


def test_gauss_laguerre_two_point_closed_form():
    t, w = O.gauss_laguerre(2)
    r2 = math.sqrt(2.0)
    np.testing.assert_allclose(t, [2 - r2, 2 + r2], rtol=1e-15)
    np.testing.assert_allclose(w, [(2 + r2) / 4, (2 - r2) / 4], rtol=1e-14)


@pytest.mark.parametrize("R", [1, 2, 3, 4, 5, 8, 12, 16, 24, 32])
def test_gauss_laguerre_matches_library_rule(R):
    t, w = O.gauss_laguerre(R)
    tn, wn = np.polynomial.laguerre.laggauss(R)
    np.testing.assert_allclose(t, tn, rtol=1e-12)
    np.testing.assert_allclose(w, wn, rtol=1e-9, atol=1e-300)


# ------------------------------------------------------- Yat kernel, quadrature

def test_yat_kernel_on_sphere_matches_definition():
    # (q.k)^2 / (|q-k|^2 + eps) evaluated from the vectors equals x^2/(2-2x+eps).
    rng = np.random.default_rng(0)
    eps = 1e-6
    for _ in range(50):
        q = rng.standard_normal(7); q /= np.linalg.norm(q)
        k = rng.standard_normal(7); k /= np.linalg.norm(k)
        direct = float(q @ k) ** 2 / (float(np.sum((q - k) ** 2)) + eps)
        assert O.yat_kernel(float(q @ k), eps) == pytest.approx(direct, rel=1e-9)
    assert O.yat_kernel(-1.0, eps) == pytest.approx(1.0 / (4.0 + eps), rel=1e-15)
    assert O.yat_kernel(0.0, eps) == 0.0
    assert O.yat_kernel(1.0, eps) == pytest.approx(1.0 / eps, rel=1e-12)


def test_yat_kernel_positive_definite_and_bounded():
    # The abstract states PD and boundedness on the sphere.
    rng = np.random.default_rng(1)
    X = rng.standard_normal((60, 5))
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    G = X @ X.T
    eps = 1e-2
    K = np.vectorize(lambda x: O.yat_kernel(min(x, 1.0), eps))(G)
    ev = np.linalg.eigvalsh(K)
    assert ev.min() > -1e-9 * ev.max()
    assert K.max() <= 1.0 / eps * (1 + 1e-12)


@pytest.mark.parametrize("x", [-1.0, -0.5, 0.3, 0.5, 0.8])
def test_quadrature_converges_from_below(x):
    # Gauss-Laguerre error for f(t) = e^{ct} is (R!)^2/(2R)! c^{2R} e^{c xi} > 0, so the
    # quadrature kernel stays at or below the closed form and approaches it as R grows.
    eps = 1e-6
    exact = O.yat_kernel(x, eps)
    errs = []
    for R in (2, 4, 8, 16, 32):
        q = O.quad_kernel(x, R, eps)
        errs.append((q - exact) / exact)
        assert q <= exact * (1 + 1e-12)
    assert all(abs(errs[i + 1]) < abs(errs[i]) or abs(errs[i]) < 1e-12 for i in range(4))
    assert abs(errs[-1]) < 1e-8


def test_quadrature_zero_at_x_zero():
    for R in (1, 4, 8):
        assert O.quad_kernel(0.0, R, 1e-6) == 0.0


# ----------------------------------------------------------------- phi

def test_sketch_params_shapes_and_marginals():
    P = O.sketch_params(D=64, R=4, m=256, seed=1234, eps=1e-6)
    assert P.omega.shape == (1024, 64) and P.anchors.shape == (1024, 64)
    # fp32 rounding of the draws
    assert np.array_equal(P.omega, P.omega.astype(np.float32).astype(np.float64))
    assert np.array_equal(P.anchors, P.anchors.astype(np.float32).astype(np.float64))
    # omega ~ N(0,1), anchors ~ N(0, 1/D): moments within a few standard errors
    n = P.omega.size
    assert abs(P.omega.mean()) < 4 / math.sqrt(n)
    assert abs(P.omega.var() - 1.0) < 4 * math.sqrt(2.0 / n)
    assert abs(P.anchors.var() * 64 - 1.0) < 4 * math.sqrt(2.0 / n)
    # fourth moment of a standard normal is 3 (catches a uniform or wrong-scale draw)
    assert abs(np.mean(P.omega ** 4) - 3.0) < 0.1
    # independence of omega and anchors
    assert abs(np.corrcoef(P.omega.ravel(), P.anchors.ravel())[0, 1]) < 4 / math.sqrt(n)
    # quadrature tables
    t, w = O.gauss_laguerre(4)
    np.testing.assert_allclose(P.s, t / (2 + 1e-6), rtol=1e-15)
    np.testing.assert_allclose(P.wt, w / (2 + 1e-6), rtol=1e-15)
    # different seeds give different draws; same seed is reproducible
    P2 = O.sketch_params(D=64, R=4, m=256, seed=1234, eps=1e-6)
    P3 = O.sketch_params(D=64, R=4, m=256, seed=1235, eps=1e-6)
    assert np.array_equal(P.omega, P2.omega)
    assert not np.array_equal(P.omega, P3.omega)


def test_phi_strictly_positive_and_scale_invariant():
    P = O.sketch_params(D=64, R=4, m=64, seed=3, eps=1e-6)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((40, 64))
    phi = O.feature_map(x, P)
    assert phi.shape == (40, 256)
    assert (phi > 0).all()
    np.testing.assert_allclose(O.feature_map(3.7 * x, P), phi, rtol=1e-9)
    np.testing.assert_allclose(O.feature_map(1e-3 * x, P), phi, rtol=1e-9)
    # a zero row is degenerate: x^ = 0, every anchor factor is 0
    z = O.feature_map(np.zeros((1, 64)), P)
    assert (z == 0).all()


@pytest.mark.parametrize("x", [0.35, -0.4])
def test_phi_monte_carlo_mean_per_node(x):
    # For unit q, k with q.k = x, omega ~ N(0,I), a ~ N(0,I/D):
    #   E[exp(sqrt(2s) w.q - s) exp(sqrt(2s) w.k - s)] = exp(2 s x)
    #   E[(a.q)^2 (a.k)^2] = (1 + 2 x^2) / D^2        (Isserlis)
    # so m * mean_j phi_{rj}(q) phi_{rj}(k) -> wt_r exp(2 s_r x) (1 + 2x^2)/D^2.
    D, R, m = 4, 3, 200000
    P = O.sketch_params(D=D, R=R, m=m, seed=11, eps=1e-6)
    q = np.array([1.0, 0.0, 0.0, 0.0])
    k = np.array([x, math.sqrt(1 - x * x), 0.0, 0.0])
    pq = O.feature_map(q[None], P)[0]
    pk = O.feature_map(k[None], P)[0]
    prod = (pq * pk).reshape(R, m) * m
    for r in range(R):
        want = P.wt[r] * math.exp(2 * P.s[r] * x) * (1 + 2 * x * x) / D ** 2
        mean = prod[r].mean()
        sem = prod[r].std() / math.sqrt(m)
        assert abs(mean - want) < 4.5 * sem, (r, mean, want, sem)
        assert sem < 0.2 * want  # informative even for the heavy-tailed top node


# ------------------------------------------------------------ contraction

def _small(seed, B=2, H=2, L=37, D=16, Dv=8):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, L, D))
    k = rng.standard_normal((B, H, L, D))
    v = rng.standard_normal((B, H, L, Dv))
    return q, k, v


@pytest.mark.parametrize("causal", [True, False])
def test_quadratic_equals_recurrent(causal):
    q, k, v = _small(3)
    P = O.sketch_params(D=16, R=3, m=8, seed=5, eps=1e-6)
    o1, d1 = O.attn_quadratic(q, k, v, P, causal)
    o2, d2 = O.attn_recurrent(q, k, v, P, causal)
    np.testing.assert_allclose(o1, o2, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(d1, d2, rtol=1e-11)


def test_rows_variant_equals_full():
    q, k, v = _small(4, L=50)
    P = O.sketch_params(D=16, R=2, m=8, seed=6, eps=1e-6)
    rows = np.array([0, 3, 17, 49])
    for causal in (True, False):
        o, d = O.attn_quadratic(q, k, v, P, causal)
        orow, drow = O.attn_quadratic_rows(q, k, v, P, causal, rows)
        np.testing.assert_allclose(orow, o[:, :, rows], rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(drow, d[:, :, rows], rtol=1e-13)


def test_uniform_keys_closed_form():
    # All keys equal: a_ij = a_i for every j, so the causal output is the running mean
    # of v scaled by (i+1) a_i / ((i+1) a_i + eps).
    L, D, Dv, eps = 20, 16, 5, 1e-3
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 1, L, D))
    k = np.repeat(rng.standard_normal((1, 1, 1, D)), L, axis=2)
    v = rng.standard_normal((1, 1, L, Dv))
    P = O.sketch_params(D=D, R=2, m=4, seed=9, eps=eps)
    out, den = O.attn_quadratic(q, k, v, P, True)
    a = (O.feature_map(q[0, 0], P) @ O.feature_map(k[0, 0, :1], P).T)[:, 0]
    for i in range(L):
        n = i + 1
        want = v[0, 0, :n].mean(axis=0) * (n * a[i]) / (n * a[i] + eps)
        np.testing.assert_allclose(out[0, 0, i], want, rtol=1e-12)
        assert den[0, 0, i] == pytest.approx(n * a[i], rel=1e-12)


def test_single_token_closed_form():
    D, Dv, eps = 8, 3, 0.05
    rng = np.random.default_rng(10)
    q = rng.standard_normal((1, 1, 1, D))
    k = rng.standard_normal((1, 1, 1, D))
    v = rng.standard_normal((1, 1, 1, Dv))
    P = O.sketch_params(D=D, R=2, m=4, seed=1, eps=eps)
    a = float(O.feature_map(q[0, 0], P)[0] @ O.feature_map(k[0, 0], P)[0])
    for causal in (True, False):
        out, den = O.attn_quadratic(q, k, v, P, causal)
        np.testing.assert_allclose(out[0, 0, 0], v[0, 0, 0] * a / (a + eps), rtol=1e-13)


def test_weights_nonnegative_and_sum_to_one():
    # With v = identity (Dv = L) output row i is the weight vector alpha_i.
    L, D = 24, 8
    rng = np.random.default_rng(12)
    q = rng.standard_normal((1, 1, L, D))
    k = rng.standard_normal((1, 1, L, D))
    v = np.eye(L)[None, None]
    P = O.sketch_params(D=D, R=3, m=6, seed=2, eps=1e-6)
    for causal in (True, False):
        out, den = O.attn_quadratic(q, k, v, P, causal)
        W = out[0, 0]
        assert (W >= 0).all()
        if causal:
            assert (np.triu(W, 1) == 0).all()
            assert (np.diag(W) > 0).all()
        np.testing.assert_allclose(W.sum(axis=1), den[0, 0] / (den[0, 0] + 1e-6), rtol=1e-12)
        assert (np.abs(W.sum(axis=1) - 1) < 1e-4).all()


def test_bidir_last_row_and_permutation():
    q, k, v = _small(13, B=1, H=1, L=30)
    P = O.sketch_params(D=16, R=2, m=8, seed=4, eps=1e-6)
    oc, _ = O.attn_quadratic(q, k, v, P, True)
    ob, _ = O.attn_quadratic(q, k, v, P, False)
    np.testing.assert_allclose(ob[0, 0, -1], oc[0, 0, -1], rtol=1e-12)
    perm = np.random.default_rng(0).permutation(30)
    op, _ = O.attn_quadratic(q, k[:, :, perm], v[:, :, perm], P, False)
    np.testing.assert_allclose(op, ob, rtol=1e-11)
    assert not np.allclose(oc[0, 0, :-1], ob[0, 0, :-1])


# ------------------------------------------------------------------ decode

def test_decode_chain_reproduces_causal_and_resumes():
    q, k, v = _small(14, B=2, H=3, L=25)
    P = O.sketch_params(D=16, R=2, m=8, seed=7, eps=1e-6)
    oc, _ = O.attn_quadratic(q, k, v, P, True)
    S = np.zeros((2, 3, P.F, 8))
    z = np.zeros((2, 3, P.F))
    ckpt = None
    for i in range(25):
        out, S, z = O.decode_step(q[:, :, i], k[:, :, i], v[:, :, i], S, z, P)
        np.testing.assert_allclose(out, oc[:, :, i], rtol=1e-11, atol=1e-14)
        if i == 11:
            ckpt = (S.copy(), z.copy())
    S2, z2 = ckpt
    for i in range(12, 25):
        out, S2, z2 = O.decode_step(q[:, :, i], k[:, :, i], v[:, :, i], S2, z2, P)
    np.testing.assert_array_equal(S2, S)
    np.testing.assert_array_equal(z2, z)


# ---------------------------------------------------------------- backward

def test_backward_matches_finite_differences():
    B, H, L, D, Dv = 1, 1, 9, 6, 4
    rng = np.random.default_rng(15)
    q = rng.standard_normal((B, H, L, D))
    k = rng.standard_normal((B, H, L, D))
    v = rng.standard_normal((B, H, L, Dv))
    g = rng.standard_normal((B, H, L, Dv))
    P = O.sketch_params(D=D, R=2, m=3, seed=8, eps=1e-3)

    def loss(q_, k_, v_):
        out, _ = O.attn_quadratic(q_, k_, v_, P, True)
        return float(np.sum(out * g))

    dq, dk, dv = O.attn_causal_bwd(q, k, v, g, P)
    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}; args_p[name] = xp
            args_m = {"q": q, "k": k, "v": v}; args_m[name] = xm
            fd[idx] = (loss(**{a + "_": b for a, b in args_p.items()}) -
                       loss(**{a + "_": b for a, b in args_m.items()})) / (2 * h)
        err = np.linalg.norm(fd - grad) / np.linalg.norm(fd)
        assert err < 1e-7, (name, err)


def test_backward_rows_variant_equals_full():
    q, k, v = _small(16, B=1, H=2, L=21, D=8, Dv=4)
    g = np.random.default_rng(17).standard_normal(v.shape)
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    dq, dk, dv = O.attn_causal_bwd(q, k, v, g, P)
    rows = np.array([0, 5, 20])
    rq, rk, rv = O.attn_causal_bwd_rows(q, k, v, g, P, rows)
    np.testing.assert_allclose(rq, dq[:, :, rows], rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(rk, dk[:, :, rows], rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(rv, dv[:, :, rows], rtol=1e-10, atol=1e-14)


def test_backward_given_output_reduces_to_the_pinned_backward():
    # at the exact forward output the "given" form is the finite-difference-pinned backward
    q, k, v = _small(18, B=1, H=2, L=23, D=8, Dv=4)
    g = np.random.default_rng(19).standard_normal(v.shape)
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    out, den = O.attn_quadratic(q, k, v, P, True)
    want = O.attn_causal_bwd(q, k, v, g, P)
    got = O.attn_causal_bwd_given(q, k, v, out, den, g, P)
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-13)
    rows = np.array([0, 7, 22])
    for a, b in zip(O.attn_causal_bwd_given_rows(q, k, v, out, den, g, P, rows), got):
        np.testing.assert_allclose(a, b[:, :, rows], rtol=1e-10, atol=1e-14)


def test_backward_given_output_depends_on_out_only_through_delta():
    # out enters only through delta_i = -<g_i, out_i>/(den_i + eps): dv does not depend on
    # it, and dq, dk are affine in it (a perturbation's effect doubles when it doubles)
    q, k, v = _small(20, B=1, H=1, L=17, D=8, Dv=4)
    g = np.random.default_rng(21).standard_normal(v.shape)
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    out, den = O.attn_quadratic(q, k, v, P, True)
    u = np.random.default_rng(22).standard_normal(out.shape) * 1e-3
    base = O.attn_causal_bwd_given(q, k, v, out, den, g, P)
    one = O.attn_causal_bwd_given(q, k, v, out + u, den, g, P)
    two = O.attn_causal_bwd_given(q, k, v, out + 2 * u, den, g, P)
    np.testing.assert_allclose(one[2], base[2], rtol=1e-13, atol=1e-15)
    for b, o1, o2 in zip(base[:2], one[:2], two[:2]):
        assert np.linalg.norm(o1 - b) > 0
        np.testing.assert_allclose(o2 - b, 2 * (o1 - b), rtol=1e-6, atol=1e-12)


def _fd_grad(loss, arrays, h=1e-6):
    """Central finite differences of loss(**arrays) with respect to every array."""
    out = {}
    for name, x in arrays.items():
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            fd[idx] = (loss(**{**arrays, name: xp}) - loss(**{**arrays, name: xm})) / (2 * h)
        out[name] = fd
    return out


def test_bidir_backward_matches_finite_differences():
    B, H, L, D, Dv = 1, 1, 7, 6, 4
    rng = np.random.default_rng(25)
    q = rng.standard_normal((B, H, L, D))
    k = rng.standard_normal((B, H, L, D))
    v = rng.standard_normal((B, H, L, Dv))
    g = rng.standard_normal((B, H, L, Dv))
    P = O.sketch_params(D=D, R=2, m=3, seed=8, eps=1e-3)

    def loss(q, k, v):
        out, _ = O.attn_quadratic(q, k, v, P, False)
        return float(np.sum(out * g))

    fd = _fd_grad(loss, {"q": q, "k": k, "v": v})
    dq, dk, dv = O.attn_bidir_bwd(q, k, v, g, P)
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        err = np.linalg.norm(fd[name] - grad) / np.linalg.norm(fd[name])
        assert err < 1e-7, (name, err)


def test_bidir_backward_differs_from_causal_except_where_it_must_agree():
    # the last query sees every key in both forms, and the bidirectional gradient with
    # respect to v is the causal one plus the contributions of earlier queries to later keys
    # (non-zero), so a dropped or kept mask shows
    q, k, v = _small(26, B=1, H=1, L=9, D=8, Dv=4)
    g = np.zeros(v.shape)
    g[..., -1, :] = np.random.default_rng(27).standard_normal(4)   # loss on the last row only
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    cb = O.attn_causal_bwd(q, k, v, g, P)
    bb = O.attn_bidir_bwd(q, k, v, g, P)
    for a, b in zip(cb, bb):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-13)
    g2 = np.random.default_rng(28).standard_normal(v.shape)
    cb = O.attn_causal_bwd(q, k, v, g2, P)
    bb = O.attn_bidir_bwd(q, k, v, g2, P)
    assert np.linalg.norm(cb[2] - bb[2]) > 1e-3 * np.linalg.norm(bb[2])


def test_feature_map_backward_matches_finite_differences():
    rng = np.random.default_rng(29)
    D = 6
    x = rng.standard_normal((5, D))
    x[2] *= 1e-14                      # a row under the norm guard
    x[3] *= 7.0                        # a rescaled row
    P = O.sketch_params(D=D, R=2, m=4, seed=10, eps=1e-3)
    G = rng.standard_normal((5, P.F))

    def loss(x):
        return float(np.sum(O.feature_map(x, P) * G))

    fd = _fd_grad(loss, {"x": x}, h=1e-7)["x"]
    got = O.feature_map_bwd(x, G, P)
    for r in (0, 1, 3, 4):             # finite differences are meaningless at 1e-14 scale
        err = np.linalg.norm(fd[r] - got[r]) / np.linalg.norm(fd[r])
        assert err < 1e-6, (r, err)
    # the guarded row (|x| ~ 1e-14): differences with a step scaled to its size
    fd2 = _fd_grad(lambda x: float(np.sum(O.feature_map(x, P) * G[2:3])), {"x": x[2:3].copy()},
                   h=1e-20)["x"][0]
    err = np.linalg.norm(fd2 - got[2]) / np.linalg.norm(fd2)
    assert err < 1e-6, err


def test_bidir_backward_given_output_reduces_and_is_affine_in_out():
    q, k, v = _small(30, B=1, H=2, L=13, D=8, Dv=4)
    g = np.random.default_rng(31).standard_normal(v.shape)
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    out, den = O.attn_quadratic(q, k, v, P, False)
    want = O.attn_bidir_bwd(q, k, v, g, P)
    base = O.attn_bidir_bwd_given(q, k, v, out, den, g, P)
    for a, b in zip(base, want):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-13)
    u = np.random.default_rng(32).standard_normal(out.shape) * 1e-3
    one = O.attn_bidir_bwd_given(q, k, v, out + u, den, g, P)
    two = O.attn_bidir_bwd_given(q, k, v, out + 2 * u, den, g, P)
    np.testing.assert_allclose(one[2], base[2], rtol=1e-13, atol=1e-15)
    for b, o1, o2 in zip(base[:2], one[:2], two[:2]):
        np.testing.assert_allclose(o2 - b, 2 * (o1 - b), rtol=1e-6, atol=1e-12)


# ----------------------------------------------------------- sketch variants

def test_kind_zero_is_the_default_map():
    P0 = O.sketch_params(D=16, R=3, m=8, seed=5, eps=1e-6)
    Pk = O.sketch_params_kind(16, 3, 8, 5, 1e-6, O.PHI_ANCHOR)
    assert np.array_equal(P0.omega, Pk.omega) and np.array_equal(P0.anchors, Pk.anchors)
    x = np.random.default_rng(40).standard_normal((7, 16))
    assert np.array_equal(O.feature_map(x, P0), O.feature_map_kind(x, Pk))


def test_orthogonal_bank_blocks():
    D, R, m = 8, 2, 20                     # blocks of 8, 8 and 4 rows in each node
    P0 = O.sketch_params(D=D, R=R, m=m, seed=6, eps=1e-6)
    P = O.sketch_params_kind(D, R, m, 6, 1e-6, O.PHI_ORTHOGONAL)
    assert np.array_equal(P.anchors, P0.anchors)
    # every row keeps the length of its Gaussian draw; the first row of a block is unchanged
    np.testing.assert_allclose(np.linalg.norm(P.omega, axis=1), np.linalg.norm(P0.omega, axis=1),
                               rtol=1e-6)
    for r in range(R):
        for b0 in (0, 8, 16):
            f0 = r * m + b0
            nb = min(8, m - b0)
            assert np.array_equal(P.omega[f0], P0.omega[f0])
            blk = P.omega[f0:f0 + nb]
            G = blk @ blk.T
            nrm = np.sqrt(np.diag(G))
            cos = G / np.outer(nrm, nrm)
            assert np.abs(cos - np.eye(nb)).max() < 1e-6
    # rows of different blocks are not made orthogonal
    cross = P.omega[0] @ P.omega[8] / (np.linalg.norm(P.omega[0]) * np.linalg.norm(P.omega[8]))
    assert abs(cross) > 1e-3


def _mc_product(P, x, D, R, m, kind_map):
    q = np.zeros(D); q[0] = 1.0
    k = np.zeros(D); k[0] = x; k[1] = math.sqrt(1 - x * x)
    pq = kind_map(q[None], P)[0]
    pk = kind_map(k[None], P)[0]
    return (pq * pk).reshape(R, m) * m


@pytest.mark.parametrize("x", [0.35, -0.4])
def test_orthogonal_bank_keeps_the_estimator_unbiased(x):
    # every omega row is N(0, I) marginally, so the per-node mean is kind 0's closed form.
    # The top node is left out: its weight exp(sqrt(2 s) w.(q + k) - 2 s) is log-normal with
    # sigma near 4 there, too heavy-tailed for a bound from the sample spread; the lower
    # nodes already fail if the rows lost their Gaussian lengths (unit rows change the mgf).
    D, R, m = 4, 3, 200000
    P = O.sketch_params_kind(D, R, m, 12, 1e-6, O.PHI_ORTHOGONAL)
    prod = _mc_product(P, x, D, R, m, O.feature_map_kind)
    for r in range(R - 1):
        want = P.wt[r] * math.exp(2 * P.s[r] * x) * (1 + 2 * x * x) / D ** 2
        sem = prod[r].std() / math.sqrt(m)
        assert abs(prod[r].mean() - want) < 4.5 * sem, (r, prod[r].mean(), want, sem)


@pytest.mark.parametrize("x", [0.35, -0.4])
def test_signed_anchor_is_unbiased_for_the_square(x):
    # E[(a.q)(b.q)(a.k)(b.k)] = E[(a.q)(a.k)] E[(b.q)(b.k)] = (x / D)^2 for independent a, b
    D, R, m = 4, 3, 200000
    P = O.sketch_params_kind(D, R, m, 13, 1e-6, O.PHI_SIGNED)
    assert not np.array_equal(P.anchors, P.anchors_b)
    prod = _mc_product(P, x, D, R, m, O.feature_map_kind)
    for r in range(R):
        want = P.wt[r] * math.exp(2 * P.s[r] * x) * x * x / D ** 2
        sem = prod[r].std() / math.sqrt(m)
        assert abs(prod[r].mean() - want) < 4.5 * sem, (r, prod[r].mean(), want, sem)
    phi = O.feature_map_kind(np.random.default_rng(41).standard_normal((50, D)), P)
    assert (phi < 0).any() and (phi > 0).any()      # signed: not a positive feature map


def test_per_head_draws():
    P0 = O.sketch_params(D=16, R=2, m=8, seed=7, eps=1e-6)
    h0 = O.sketch_params_kind(16, 2, 8, 7, 1e-6, O.PHI_PER_HEAD, head=0)
    h3 = O.sketch_params_kind(16, 2, 8, 7, 1e-6, O.PHI_PER_HEAD, head=3)
    assert np.array_equal(h0.omega, P0.omega) and np.array_equal(h0.anchors, P0.anchors)
    assert not np.array_equal(h3.omega, h0.omega)
    big = O.sketch_params_kind(64, 4, 256, 7, 1e-6, O.PHI_PER_HEAD, head=5)
    assert abs(big.omega.mean()) < 0.01 and abs(big.omega.var() - 1) < 0.02
    assert abs(big.anchors.var() * 64 - 1) < 0.02


@pytest.mark.parametrize("x", [0.35, -0.4])
def test_performer_features_estimate_exp(x):
    # FAVOR+: E[exp(w.q - 1/2) exp(w.k - 1/2)] = exp(|q + k|^2 / 2 - 1) = exp(q.k) on the
    # sphere, so F * mean_f phi_f(q) phi_f(k) -> exp(x)
    D, R, m = 4, 1, 200000
    P = O.sketch_params_kind(D, R, m, 14, 1e-6, O.PHI_PERFORMER)
    prod = _mc_product(P, x, D, R, m, O.feature_map_kind)[0]
    sem = prod.std() / math.sqrt(m)
    assert abs(prod.mean() - math.exp(x)) < 4.5 * sem, (prod.mean(), math.exp(x), sem)
    assert sem < 0.02 * math.exp(x)
    phi = O.feature_map_kind(np.random.default_rng(42).standard_normal((20, D)), P)
    assert (phi > 0).all()


@pytest.mark.parametrize("causal", [True, False])
def test_contraction_on_given_features_is_the_quadratic_form(causal):
    q, k, v = _small(43, B=1, H=2, L=29, D=16, Dv=8)
    P = O.sketch_params(D=16, R=3, m=8, seed=5, eps=1e-6)
    want, wden = O.attn_quadratic(q, k, v, P, causal)
    got, gden = O.attn_from_phi(O.feature_map(q, P), O.feature_map(k, P), v, P.eps, causal)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(gden, wden, rtol=1e-12)


# ------------------------------------------------------- state continuation

def test_causal_state_from_zero_is_the_causal_form():
    q, k, v = _small(50, B=1, H=2, L=23, D=8, Dv=4)
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    want, wden = O.attn_quadratic(q, k, v, P, True)
    out, den, S1, z1 = O.attn_causal_state(q, k, v, P)
    np.testing.assert_allclose(out, want, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(den, wden, rtol=1e-11)
    # the final state is the total sum phi(k)[v, 1]^T
    pk = O.feature_map(k, P)
    np.testing.assert_allclose(S1, np.einsum("bhlf,bhle->bhfe", pk, v), rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(z1, pk.sum(axis=2), rtol=1e-11)


@pytest.mark.parametrize("cuts", [(9,), (4, 11, 17), (1, 2, 22)])
def test_causal_state_chains_over_a_split_sequence(cuts):
    # sequence parallelism: each part continues from the state the earlier parts end in
    q, k, v = _small(51, B=2, H=1, L=23, D=8, Dv=4)
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    want, wden = O.attn_quadratic(q, k, v, P, True)
    S, z, outs, dens = None, None, [], []
    bounds = (0,) + tuple(cuts) + (23,)
    for a, b in zip(bounds[:-1], bounds[1:]):
        o, d, S, z = O.attn_causal_state(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], P, S, z)
        outs.append(o)
        dens.append(d)
    np.testing.assert_allclose(np.concatenate(outs, axis=2), want, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(np.concatenate(dens, axis=2), wden, rtol=1e-11)


def test_causal_state_is_the_decode_recurrence():
    q, k, v = _small(52, B=1, H=2, L=6, D=8, Dv=4)
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    rng = np.random.default_rng(53)
    S0 = rng.standard_normal((1, 2, P.F, 4)) * 1e-3
    z0 = rng.random((1, 2, P.F)) * 1e-3
    out, den, S1, z1 = O.attn_causal_state(q, k, v, P, S0, z0)
    S, z = S0.copy(), z0.copy()
    for i in range(6):
        o, S, z = O.decode_step(q[:, :, i], k[:, :, i], v[:, :, i], S, z, P)
        np.testing.assert_allclose(out[:, :, i], o, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(S1, S, rtol=1e-12, atol=1e-16)
    np.testing.assert_allclose(z1, z, rtol=1e-12)


# ---------------------------------------------------- backward of a piece of a sequence
def test_piece_backward_without_states_is_the_given_backward():
    # no tokens before or after the piece: the whole-sequence backward at the given output
    q, k, v = _small(54, B=2, H=1, L=17, D=8, Dv=4)
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    out, den = O.attn_quadratic(q, k, v, P, True)
    g = np.random.default_rng(55).standard_normal(v.shape)
    want = O.attn_causal_bwd_given(q, k, v, out, den, g, P)
    got = O.attn_causal_bwd_state(q, k, v, out, den, g, P)
    for a, b in zip(got[:3], want):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("cuts", [(7, 16), (1, 22), (11,)])
def test_piece_backward_chains_to_the_whole_sequence(cuts):
    # sequence parallelism backward: each piece takes the forward state of the pieces before
    # it (S_in, z_in) and the sum of the later pieces' phi(q)[dn, delta] (G_in, zg_in); the
    # pieces' gradients are the whole sequence's (pinned by finite differences)
    q, k, v = _small(56, B=2, H=1, L=23, D=8, Dv=4)
    P = O.sketch_params(D=8, R=2, m=5, seed=9, eps=1e-6)
    g = np.random.default_rng(57).standard_normal(v.shape)
    out, den = O.attn_quadratic(q, k, v, P, True)
    want = O.attn_causal_bwd(q, k, v, g, P)
    bounds = (0,) + tuple(cuts) + (23,)
    pieces = list(zip(bounds[:-1], bounds[1:]))
    S_in, S, z = [], None, None
    for a, b in pieces:                  # forward states entering each piece
        S_in.append((S, z))
        _, _, S, z = O.attn_causal_state(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], P, S, z)
    got = [None] * len(pieces)
    G, zg = None, None
    for p in reversed(range(len(pieces))):   # later pieces first: their G sums the suffix
        a, b = pieces[p]
        sl = (slice(None), slice(None), slice(a, b))
        dq, dk, dv, Go, zgo = O.attn_causal_bwd_state(q[sl], k[sl], v[sl], out[sl], den[sl], g[sl],
                                                      P, *S_in[p], G, zg)
        got[p] = (dq, dk, dv)
        G = Go if G is None else G + Go
        zg = zgo if zg is None else zg + zgo
    for i in range(3):
        np.testing.assert_allclose(np.concatenate([x[i] for x in got], axis=2), want[i],
                                   rtol=1e-9, atol=1e-12)
