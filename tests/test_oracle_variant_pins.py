"""Pins of the oracle's two transition variants (CPU only, no ``gpu`` mark).

Damping regimes ("Understanding Mamba-3 Through Oscillatory Dynamics",
section 2.2 / Table 1, section 4.1, section 4.2 and appendix C.2): rotary pair
i of token t evolves under the generator dt (A I + theta[i] K_s),
K_s = [[0, -1], [s, 0]], s = +1 (underdamped: Mamba-3), 0 (critical), -1
(overdamped), with Mamba-3's exponential-trapezoidal input rule.

Low-rank reflection (the extension's abstract listed on that page; two
reflections compose to a rotation, appendix C.4 of the same paper): the
diagonal part of the transition becomes alpha (I - 2 u u^T / u^T u).

Each pin compares the oracle with a different computation: scipy's matrix
exponential, eigen-decompositions of the one-step transition (probed from the
oracle with unit vectors), dense N x N matrix products written with numpy,
the plain scan where a variant must reduce to it, or a closed form.  Planted
mistakes in copies of the oracle show that the pins catch a wrong sign, a
swapped function, a missing factor or the wrong order of factors.
"""
import math

import numpy as np
import pytest
import scipy.linalg

import oracle

SIGMA = {"under": 1.0, "critical": 0.0, "over": -1.0}


def rand_inputs(seed, b=2, L=30, H=2, G=1, P=3, N=6, R=2, theta_scale=1.0):
    rng = np.random.default_rng(seed)
    A = -np.exp(rng.uniform(-2, 1, size=H))
    return dict(
        x=rng.standard_normal((b, L, H, R, P)),
        B=rng.standard_normal((b, L, G, R, N)),
        C=rng.standard_normal((b, L, G, R, N)),
        dt=np.log1p(np.exp(rng.standard_normal((b, L, H)))),
        A=A,
        lam=1 / (1 + np.exp(-rng.standard_normal((b, L, H)))),
        theta=theta_scale * rng.uniform(-np.pi, np.pi, size=(b, L, G, N // 2)),
    )


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def one_step_transition(run, N, d, A, theta):
    """The N x N matrix M with h_0 = M h_{-1} for one token with no input,
    read off the oracle by feeding the unit vectors as the carry (P = N
    columns at once: column j of init_h is e_j)."""
    P = N
    x = np.zeros((1, 1, 1, 1, P))
    B = np.zeros((1, 1, 1, 1, N))
    C = np.zeros((1, 1, 1, 1, N))
    kw = dict(init_h=np.eye(N).reshape(1, 1, N, P))
    _, hL, _, _ = run(x, B, C, np.full((1, 1, 1), d), np.array([A]), np.full((1, 1, 1), 0.5),
                      np.asarray(theta, dtype=np.float64).reshape(1, 1, 1, N // 2), **kw)
    return hL[0, 0]


# ------------------------------------------------------------ damping regimes
def test_underdamped_regime_is_the_mamba3_scan():
    """s = +1 is Mamba-3's decay-rotation [OSC 4.1: the underdamped variant is
    the model itself]; the oracle's general 2x2 block code must reproduce its
    plain rotation code (a second, separately written step)."""
    I = rand_inputs(1)
    want = oracle.scan(**I)
    got = oracle.scan_damped("under", **I)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("regime", ["under", "critical", "over"])
def test_homogeneous_propagation_is_the_matrix_exponential(regime):
    """[OSC 3, C.1, 4.1]: with no input each pair's update is the exact flow of
    dt (A I + theta K_s) over the interval.  Tokens with varying dt and theta:
    the oracle's state equals the product of scipy.linalg.expm of each
    token's generator applied to the carry-in."""
    s = SIGMA[regime]
    rng = np.random.default_rng(5)
    k, N = 12, 4
    dts = np.log1p(np.exp(rng.standard_normal(k)))
    A = -0.6
    th = rng.uniform(-0.5, 0.5, size=(k, N // 2))
    h0 = rng.standard_normal((N, 2))
    x = np.zeros((1, k, 1, 1, 2))
    B = rng.standard_normal((1, k, 1, 1, N))        # irrelevant: x = 0
    C = rng.standard_normal((1, k, 1, 1, N))
    _, hL, _, _ = oracle.scan_damped(regime, x, B, C, dts.reshape(1, k, 1), np.array([A]),
                                     np.full((1, k, 1), 0.3), th.reshape(1, k, 1, N // 2),
                                     init_h=h0.reshape(1, 1, N, 2))
    want = h0.copy()
    for t in range(k):
        for i in range(N // 2):
            gen = np.array([[A, -th[t, i]], [s * th[t, i], A]])
            want[2 * i:2 * i + 2] = scipy.linalg.expm(dts[t] * gen) @ want[2 * i:2 * i + 2]
    np.testing.assert_allclose(hL[0, 0], want, rtol=1e-11, atol=1e-13)


def test_regimes_share_the_spectral_centre_and_differ_in_eigenstructure():
    """[OSC 2.2 Table 1, 4.1]: underdamped pairs have complex-conjugate
    eigenvalues, critical and overdamped ones real eigenvalues; the damping
    parameter moves them around one shared centre.  Probed from the oracle's
    one-step transition of a single pair: eigenvalues e^{dt(A +- i theta)},
    a double e^{dt A} with a non-trivial Jordan block, and e^{dt(A +- theta)};
    the product of the two eigenvalues is e^{2 dt A} in every regime."""
    d, A, th = 0.7, -0.9, 0.4
    run = lambda r: (lambda *a, **k: oracle.scan_damped(r, *a, **k))
    Mu = one_step_transition(run("under"), 2, d, A, [th])
    Mc = one_step_transition(run("critical"), 2, d, A, [th])
    Mo = one_step_transition(run("over"), 2, d, A, [th])
    ev = np.linalg.eigvals(Mu)
    assert np.all(np.abs(ev.imag) > 1e-3)
    np.testing.assert_allclose(np.sort(np.angle(ev)), [-d * th, d * th], atol=1e-12)
    np.testing.assert_allclose(np.abs(ev), math.exp(d * A), rtol=1e-12)
    ec = np.linalg.eigvals(Mc)
    np.testing.assert_allclose(ec, [math.exp(d * A)] * 2, rtol=1e-7)
    J = Mc - math.exp(d * A) * np.eye(2)
    assert np.linalg.norm(J) > 1e-3                      # not a multiple of I
    np.testing.assert_allclose(J @ J, 0.0, atol=1e-14)  # nilpotent part
    eo = np.sort(np.linalg.eigvals(Mo).real)
    np.testing.assert_allclose(eo, np.exp(d * (A + np.array([-th, th]))), rtol=1e-12)
    for M in (Mu, Mc, Mo):
        np.testing.assert_allclose(np.linalg.det(M), math.exp(2 * d * A), rtol=1e-12)


def test_mode_persistence_across_regimes():
    """[OSC 4.2, C.2]: propagated many steps, the underdamped transition keeps
    two equally decaying modes (both singular values of M^k equal), the
    overdamped one is dominated by its slow eigendirection (the state aligns
    with (1, -1) for theta > 0), and the critical one becomes asymptotically
    rank one (sigma_2 / sigma_1 -> 0), decaying fastest at fixed natural
    frequency."""
    d, A, th, k = 1.0, -0.5, 0.3, 60
    run = lambda r: (lambda *a, **kw: oracle.scan_damped(r, *a, **kw))
    sv = {}
    for r in ("under", "critical", "over"):
        M = one_step_transition(run(r), 2, d, A, [th])
        Mk = np.linalg.matrix_power(M, k)
        sv[r] = np.linalg.svd(Mk, compute_uv=False)
        if r == "over":
            v = Mk @ np.array([0.3, 0.8])
            cosang = abs(v @ np.array([1.0, -1.0])) / (np.linalg.norm(v) * math.sqrt(2))
            assert cosang > 1 - 1e-6
    np.testing.assert_allclose(sv["under"][1] / sv["under"][0], 1.0, rtol=1e-10)
    # critical: sigma_2 / sigma_1 of M^k falls like 1 / k^2
    Mc1 = one_step_transition(run("critical"), 2, d, A, [th])
    ratio = [np.divide(*np.linalg.svd(np.linalg.matrix_power(Mc1, kk), compute_uv=False)[::-1])
             for kk in (k, 4 * k)]
    assert ratio[0] < 1e-2 and ratio[1] < ratio[0] / 10
    # at a fixed natural frequency omega (omega^2 = A^2 + s theta^2 is the
    # underdamped pair's; the critical pair with centre -omega has the same
    # omega) the critical transition decays faster
    omega = math.hypot(A, th)
    Mc = one_step_transition(run("critical"), 2, d, -omega, [th])
    Mu = one_step_transition(run("under"), 2, d, A, [th])
    assert np.linalg.norm(np.linalg.matrix_power(Mc, k), 2) < np.linalg.norm(np.linalg.matrix_power(Mu, k), 2)


def test_zero_phase_makes_every_regime_the_real_diagonal_ssm():
    """With theta = 0 the pair blocks are the identity in every regime, so the
    variants share Mamba-3's input rule exactly [OSC 4.1: same input-update
    rule and state]: all three equal the plain scan at theta = 0."""
    I = rand_inputs(3)
    I["theta"][:] = 0.0
    want = oracle.scan(**I)
    for r in ("critical", "over"):
        for g, w in zip(oracle.scan_damped(r, **I), want):
            np.testing.assert_allclose(g, w, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("regime", ["critical", "over"])
def test_damped_dense_matrix_form(regime):
    """The whole recurrence written with dense N x N block-diagonal matrices
    (numpy), each block scipy.linalg.expm(dt (A I + theta K_s)) / e^{dt A}, and
    the MIMO input / readout as matrix products."""
    s = SIGMA[regime]
    I = rand_inputs(4, b=1, L=14, H=1, G=1, P=3, N=4, R=2, theta_scale=0.2)
    y, hL, _, _ = oracle.scan_damped(regime, **I)
    N, P = 4, 3
    h = np.zeros((N, P))
    prev = np.zeros((N, P))
    for t in range(14):
        d, lam, A = I["dt"][0, t, 0], I["lam"][0, t, 0], I["A"][0]
        T = scipy.linalg.block_diag(*[
            scipy.linalg.expm(d * np.array([[0.0, -w], [s * w, 0.0]])) for w in I["theta"][0, t, 0]])
        cur = I["B"][0, t, 0].T @ I["x"][0, t, 0]
        h = T @ (math.exp(d * A) * h + (1 - lam) * d * math.exp(d * A) * prev) + lam * d * cur
        prev = cur
        np.testing.assert_allclose(y[0, t, 0], I["C"][0, t, 0] @ h, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(hL[0, 0], h, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("regime", ["critical", "over"])
def test_damped_continuation(regime):
    """A split sequence resumed from the carry equals one call (carry semantics
    shared with the plain scan)."""
    I = rand_inputs(6, theta_scale=0.3)
    y, hL, pB, pX = oracle.scan_damped(regime, **I)
    cut = 11
    first = {k: (v[:, :cut] if v.ndim > 1 else v) for k, v in I.items()}
    rest = {k: (v[:, cut:] if v.ndim > 1 else v) for k, v in I.items()}
    y1, h1, b1, x1 = oracle.scan_damped(regime, **first)
    y2, h2, b2, x2 = oracle.scan_damped(regime, **rest, init_h=h1, init_pB=b1, init_pX=x1)
    np.testing.assert_allclose(np.concatenate([y1, y2], 1), y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h2, hL, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ reflection
def test_zero_direction_is_the_plain_scan():
    """u = 0 leaves the diagonal transition unchanged (no reflection)."""
    I = rand_inputs(7)
    u = np.zeros(I["B"].shape[:3] + (I["B"].shape[4],))
    for g, w in zip(oracle.scan_reflect(u, **I), oracle.scan(**I)):
        np.testing.assert_allclose(g, w, rtol=1e-13, atol=1e-13)


def test_reflection_transition_is_orthogonal_times_decay():
    """The one-step transition is alpha R_t H_t with H_t a Householder
    reflection: M^T M = alpha^2 I and det M = -alpha^N (a reflection has
    determinant -1, a rotation +1).  With A = 0 and theta = 0 it is H itself:
    an involution that maps u to -u and fixes the complement of u."""
    rng = np.random.default_rng(8)
    N, d, A = 6, 0.8, -0.7
    u = rng.standard_normal(N)
    th = rng.uniform(-np.pi, np.pi, N // 2)

    def run(*a, **k):
        return oracle.scan_reflect(u.reshape(1, 1, 1, N), *a, **k)

    M = one_step_transition(run, N, d, A, th)
    al = math.exp(d * A)
    np.testing.assert_allclose(M.T @ M, al * al * np.eye(N), atol=1e-13)
    np.testing.assert_allclose(np.linalg.det(M), -al ** N, rtol=1e-12)
    H = one_step_transition(run, N, d, 0.0, np.zeros(N // 2))
    np.testing.assert_allclose(H @ H, np.eye(N), atol=1e-13)
    np.testing.assert_allclose(H @ u, -u, atol=1e-13)
    v = rng.standard_normal(N)
    v -= (v @ u) / (u @ u) * u
    np.testing.assert_allclose(H @ v, v, atol=1e-13)


def test_two_reflections_compose_to_a_rotation():
    """[OSC C.4]: in two dimensions, reflecting along u_1 = (cos a, sin a) and
    then along u_2 = (cos b, sin b) is the rotation by 2 (b - a).  Two tokens,
    A = 0, theta = 0, no input."""
    a, b = 0.4, 1.3
    N, P = 2, 2
    u = np.array([[math.cos(a), math.sin(a)], [math.cos(b), math.sin(b)]]).reshape(1, 2, 1, N)
    x = np.zeros((1, 2, 1, 1, P))
    Z = np.zeros((1, 2, 1, 1, N))
    _, hL, _, _ = oracle.scan_reflect(u, x, Z, Z, np.full((1, 2, 1), 0.5), np.array([0.0]),
                                      np.full((1, 2, 1), 0.5), np.zeros((1, 2, 1, 1)),
                                      init_h=np.eye(2).reshape(1, 1, N, P))
    w = 2 * (b - a)
    np.testing.assert_allclose(hL[0, 0], [[math.cos(w), -math.sin(w)], [math.sin(w), math.cos(w)]],
                               atol=1e-13)


def test_reflection_depends_on_the_order_of_tokens():
    """Noncommutative state tracking (the extension's purpose): two tokens
    with directions neither parallel nor orthogonal give different states in
    the two orders; parallel directions commute."""
    N = 4
    rng = np.random.default_rng(9)
    u1, u2 = rng.standard_normal(N), rng.standard_normal(N)
    h0 = rng.standard_normal((N, 1))

    def two(ua, ub):
        u = np.stack([ua, ub]).reshape(1, 2, 1, N)
        Z = np.zeros((1, 2, 1, 1, N))
        return oracle.scan_reflect(u, np.zeros((1, 2, 1, 1, 1)), Z, Z, np.full((1, 2, 1), 0.5),
                                   np.array([-0.1]), np.full((1, 2, 1), 0.5),
                                   np.zeros((1, 2, 1, N // 2)), init_h=h0.reshape(1, 1, N, 1))[1]
    assert np.linalg.norm(two(u1, u2) - two(u2, u1)) > 1e-3
    np.testing.assert_allclose(two(u1, 2.5 * u1), two(2.5 * u1, u1), atol=1e-13)


def test_reflection_direction_scale_does_not_matter():
    """Only the direction of u enters (u and c u, c != 0, give the same result)."""
    I = rand_inputs(10)
    rng = np.random.default_rng(100)
    u = rng.standard_normal(I["B"].shape[:3] + (I["B"].shape[4],))
    a = oracle.scan_reflect(u, **I)
    b = oracle.scan_reflect(-3.7 * u, **I)
    for g, w in zip(a, b):
        np.testing.assert_allclose(g, w, rtol=1e-12, atol=1e-12)


def test_reflection_dense_matrix_form():
    """The recurrence with dense N x N matrices (numpy): R_t from per-pair
    rotation blocks, H_t = I - 2 u u^T / u^T u, MIMO input and readout as
    matrix products; MIMO rank 2, a shared group of two heads, a carry in."""
    I = rand_inputs(11, b=1, L=16, H=2, G=1, P=3, N=6, R=2)
    rng = np.random.default_rng(110)
    u = rng.standard_normal((1, 16, 1, 6))
    u[0, 5] = 0.0                                     # one token with no reflection
    h0 = rng.standard_normal((1, 2, 6, 3))
    pb0 = rng.standard_normal((1, 2, 2, 6))
    px0 = rng.standard_normal((1, 2, 2, 3))
    y, hL, _, _ = oracle.scan_reflect(u, **I, init_h=h0, init_pB=pb0, init_pX=px0)
    for hh in range(2):
        h = h0[0, hh].copy()
        prev = pb0[0, hh].T @ px0[0, hh]
        for t in range(16):
            d, lam, A = I["dt"][0, t, hh], I["lam"][0, t, hh], I["A"][hh]
            Rt = scipy.linalg.block_diag(*[np.array([[math.cos(d * w), -math.sin(d * w)],
                                                     [math.sin(d * w), math.cos(d * w)]])
                                           for w in I["theta"][0, t, 0]])
            ut = u[0, t, 0]
            Ht = np.eye(6) - (2 * np.outer(ut, ut) / (ut @ ut) if ut @ ut > 0 else 0.0)
            cur = I["B"][0, t, 0].T @ I["x"][0, t, hh]
            h = Rt @ Ht @ (math.exp(d * A) * h + (1 - lam) * d * math.exp(d * A) * prev) + lam * d * cur
            prev = cur
            np.testing.assert_allclose(y[0, t, hh], I["C"][0, t, 0] @ h, rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(hL[0, hh], h, rtol=1e-11, atol=1e-11)


def test_reflection_preserves_the_norm_without_decay():
    """With A = 0 and no input the transition R_t H_t is orthogonal: the
    Frobenius norm of the state never changes over many tokens."""
    rng = np.random.default_rng(12)
    L, N, P = 40, 8, 3
    u = rng.standard_normal((1, L, 1, N))
    Z = np.zeros((1, L, 1, 1, N))
    h0 = rng.standard_normal((1, 1, N, P))
    _, hL, _, _ = oracle.scan_reflect(u, np.zeros((1, L, 1, 1, P)), Z, Z,
                                      np.log1p(np.exp(rng.standard_normal((1, L, 1)))), np.array([0.0]),
                                      np.full((1, L, 1), 0.5), rng.uniform(-np.pi, np.pi, (1, L, 1, N // 2)),
                                      init_h=h0)
    np.testing.assert_allclose(np.linalg.norm(hL), np.linalg.norm(h0), rtol=1e-12)


# ------------------------------------------------------- planted mistakes
def _variant_pin_errors(lib):
    """Largest error of the damped and reflect dense-matrix pins and the
    expm pin, computed with a given oracle build."""
    errs = []
    for regime, s in (("critical", 0.0), ("over", -1.0)):
        I = rand_inputs(4, b=1, L=10, H=1, G=1, P=2, N=4, R=1, theta_scale=0.2)
        y = oracle.scan_damped(regime, **I, lib=lib)[0]
        h = np.zeros((4, 2))
        prev = np.zeros((4, 2))
        for t in range(10):
            d, lam, A = I["dt"][0, t, 0], I["lam"][0, t, 0], I["A"][0]
            T = scipy.linalg.block_diag(*[
                scipy.linalg.expm(d * np.array([[0.0, -w], [s * w, 0.0]])) for w in I["theta"][0, t, 0]])
            cur = I["B"][0, t, 0].T @ I["x"][0, t, 0]
            h = T @ (math.exp(d * A) * h + (1 - lam) * d * math.exp(d * A) * prev) + lam * d * cur
            prev = cur
            errs.append(float(np.max(np.abs(y[0, t, 0] - I["C"][0, t, 0] @ h))))
    I = rand_inputs(11, b=1, L=10, H=1, G=1, P=2, N=4, R=1)
    u = np.random.default_rng(3).standard_normal((1, 10, 1, 4))
    y = oracle.scan_reflect(u, **I, lib=lib)[0]
    h = np.zeros((4, 2))
    prev = np.zeros((4, 2))
    for t in range(10):
        d, lam, A = I["dt"][0, t, 0], I["lam"][0, t, 0], I["A"][0]
        Rt = scipy.linalg.block_diag(*[np.array([[math.cos(d * w), -math.sin(d * w)],
                                                 [math.sin(d * w), math.cos(d * w)]])
                                       for w in I["theta"][0, t, 0]])
        ut = u[0, t, 0]
        Ht = np.eye(4) - 2 * np.outer(ut, ut) / (ut @ ut)
        cur = I["B"][0, t, 0].T @ I["x"][0, t, 0]
        h = Rt @ Ht @ (math.exp(d * A) * h + (1 - lam) * d * math.exp(d * A) * prev) + lam * d * cur
        prev = cur
        errs.append(float(np.max(np.abs(y[0, t, 0] - I["C"][0, t, 0] @ h))))
    return max(errs)


_VARIANT_MUTATIONS = {
    # overdamped block with the rotation's sign pattern (sg = +1)
    "over_sign": [("else { *c = cosh(phi); *sn = sinh(phi); *sg = -1.0; }",
                   "else { *c = cosh(phi); *sn = sinh(phi); *sg = 1.0; }")],
    # cosh and sinh swapped
    "over_swapped": [("else { *c = cosh(phi); *sn = sinh(phi); *sg = -1.0; }",
                      "else { *c = sinh(phi); *sn = cosh(phi); *sg = -1.0; }")],
    # critical shear without dt in the off-diagonal
    "critical_shear": [("else if (regime == 1) { *c = 1.0; *sn = phi; *sg = 0.0; }",
                        "else if (regime == 1) { *c = 1.0; *sn = phi / d_unused; *sg = 0.0; }"),
                       ("static void pair_block(int regime, double phi,",
                        "static const double d_unused = 2.0;\nstatic void pair_block(int regime, double phi,")],
    # reflection without the factor 2 (a projection, not a reflection)
    "reflect_factor": [("const double f = 2.0 * dot / uu;", "const double f = dot / uu;")],
    # reflection applied after the rotation instead of before it
    "reflect_order": [("    /* reflection v <- (I - 2 u u^T / u^T u) v, column by column (u = 0: none) */\n    if (u) {",
                       "    if (0) {"),
                      ("    /* + gamma B_t X_t^T */\n    for (int n = 0; n < N; ++n)\n        for (int p = 0; p < P; ++p) {\n            double cur = 0.0;\n            for (int r = 0; r < R; ++r) cur += xt[r * P + p] * Bt[r * N + n];\n            H[n * P + p] += gamma * cur;",
                       "    if (u) { double uu = 0.0; for (int n = 0; n < N; ++n) uu += u[n] * u[n];"
                       " if (uu > 0.0) for (int p = 0; p < P; ++p) { double dot = 0.0;"
                       " for (int n = 0; n < N; ++n) dot += u[n] * H[n * P + p];"
                       " const double f = 2.0 * dot / uu; for (int n = 0; n < N; ++n) H[n * P + p] -= f * u[n]; } }\n"
                       "    for (int n = 0; n < N; ++n)\n        for (int p = 0; p < P; ++p) {\n            double cur = 0.0;\n            for (int r = 0; r < R; ++r) cur += xt[r * P + p] * Bt[r * N + n];\n            H[n * P + p] += gamma * cur;")],
    # direction not normalised (u u^T instead of u u^T / u^T u)
    "reflect_unnormalised": [("const double f = 2.0 * dot / uu;", "const double f = 2.0 * dot;")],
}


def test_variant_pins_pass_on_the_oracle():
    assert _variant_pin_errors(None) < 1e-10


@pytest.mark.parametrize("name", sorted(_VARIANT_MUTATIONS))
def test_variant_planted_mistakes_are_caught(name):
    """A plausible mistake planted in a copy of the oracle's variant code
    fails the dense-matrix pins."""
    src = oracle.source_text()
    for old, new in _VARIANT_MUTATIONS[name]:
        assert src.count(old) == 1, (name, old)
        src = src.replace(old, new)
    lib = oracle.compile_variant(src, name)
    assert _variant_pin_errors(lib) > 1e-6, f"mutation {name} slipped through"
