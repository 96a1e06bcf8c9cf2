"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Every test here runs on the CPU (no ``gpu`` mark).  None of them re-types the
oracle's own loop: each compares it with a different computation of the same
quantity -- a library routine (scipy lfilter / expm), a closed form, native
complex arithmetic, a dense matrix (SSD) form, an order-of-accuracy
measurement against the exact continuous-time solution, or the counting code
of a worked example.  ``test_planted_mistakes_are_caught`` plants plausible
mistakes in a copy of the oracle and checks that these pins fail on them.

Page references (title, section):
  [M3]  "Mamba-3" summary (b-lab.team): s1 Exponential-Trapezoidal
        Discretization; s2 Complex-Valued SSM, Propositions 2 and 3; s3 MIMO.
  [OSC] "Understanding Mamba-3 Through Oscillatory Dynamics" (paperlayer.ai):
        C.1 matrix exponential of the rotation generator; C.3 accumulation
        under persistent forcing; E.1 phase structure, Figure 5.
  [RD]  "Unlocking Rotational Dynamics via data-RoPE" (aitrending.vip TL;DR;
        the500feed.com s II): exp-trapezoid has O(dt^3) local / O(dt^2)
        global error, exp-Euler O(dt^2) local.
"""
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.signal

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers --
def rand_inputs(seed, b=2, L=40, H=2, G=1, P=3, N=8, R=2):
    rng = np.random.default_rng(seed)
    return dict(
        x=rng.standard_normal((b, L, H, R, P)),
        B=rng.standard_normal((b, L, G, R, N)),
        C=rng.standard_normal((b, L, G, R, N)),
        dt=np.log1p(np.exp(rng.standard_normal((b, L, H)))),
        A=-np.exp(rng.uniform(-2, 1, size=H)),
        lam=1 / (1 + np.exp(-rng.standard_normal((b, L, H)))),
        theta=rng.uniform(-np.pi, np.pi, size=(b, L, G, N // 2)),
    )


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_complex(v):
    """real rows (2i, 2i+1) along the last axis -> complex pair i"""
    return v[..., 0::2] + 1j * v[..., 1::2]


def rot_blockdiag(phis):
    return scipy.linalg.block_diag(*[np.array([[math.cos(f), -math.sin(f)],
                                               [math.sin(f), math.cos(f)]]) for f in phis])


# ------------------------------------------------------------------- pins --
def test_euler_case_is_mamba2_rotation_recurrence():
    """lambda == 1 gives the exp-Euler rule of Proposition 2 [M3 s1, s2]:
    h_t = e^{dt A} R_t h_{t-1} + dt B_t x_t, y_t = C_t^T h_t, written here with
    dense block-diagonal rotation matrices (a different computation)."""
    I = rand_inputs(1)
    I["lam"][:] = 1.0
    y, hL, _, _ = oracle.scan(**I)
    b, L, H, R, P = I["x"].shape
    G, N = I["B"].shape[2], I["B"].shape[4]
    for bb in range(b):
        for h in range(H):
            g = h * G // H
            hs = np.zeros((N, P))
            for t in range(L):
                d = I["dt"][bb, t, h]
                Rt = rot_blockdiag(d * I["theta"][bb, t, g])
                Bt, Ct, xt = I["B"][bb, t, g], I["C"][bb, t, g], I["x"][bb, t, h]
                hs = math.exp(d * I["A"][h]) * (Rt @ hs) + d * (Bt.T @ xt)
                np.testing.assert_allclose(y[bb, t, h], Ct @ hs, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(hL[bb, h], hs, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("lam,order", [(0.5, 2.0), (1.0, 1.0)])
def test_order_of_accuracy_against_exact_solution(lam, order):
    """The exp-trapezoidal rule (lambda = 1/2) is second order globally, the
    exp-Euler rule (lambda = 1) first order [RD; M3 s1 'O(dt^3) local error'].
    Measured on one rotary pair driven by u(s) = cos(w s), against the exact
    solution of dz/ds = (a + i nu) z + b u(s) [M3 s2 complex SSM].  Any error
    in the beta term (index, missing rotation, wrong dt) drops the order."""
    a, nu, w, T = -0.7, 2.3, 1.9, 3.0
    bc = 0.8 - 0.45j                      # complex input column B + i B_hat
    mu = a + 1j * nu

    def exact(T):
        return bc / 2 * ((np.exp(1j * w * T) - np.exp(mu * T)) / (1j * w - mu)
                         + (np.exp(-1j * w * T) - np.exp(mu * T)) / (-1j * w - mu))

    errs = []
    for K in (100, 200, 400):
        dtv = T / K
        s = dtv * np.arange(1, K + 1)      # token t sits at time (t+1) dt
        x = np.cos(w * s).reshape(1, K, 1, 1, 1)
        B = np.tile(np.array([bc.real, bc.imag]), (1, K, 1, 1, 1)).reshape(1, K, 1, 1, 2)
        C = np.tile(np.array([1.0, 0.0]), (1, K, 1, 1, 1)).reshape(1, K, 1, 1, 2)
        dt = np.full((1, K, 1), dtv)
        lamv = np.full((1, K, 1), lam)
        theta = np.full((1, K, 1, 1), nu)
        # the interval (0, dt] starts from z(0) = 0 with input u(0) = 1 pending
        _, hL, _, _ = oracle.scan(x, B, C, dt, np.array([a]), lamv, theta,
                                  init_h=np.zeros((1, 1, 2, 1)),
                                  init_pB=np.array([bc.real, bc.imag]).reshape(1, 1, 1, 2),
                                  init_pX=np.ones((1, 1, 1, 1)))
        z = hL[0, 0, 0, 0] + 1j * hL[0, 0, 1, 0]
        errs.append(abs(z - exact(T)))
    p1 = math.log2(errs[0] / errs[1])
    p2 = math.log2(errs[1] / errs[2])
    assert abs(p1 - order) < 0.15 and abs(p2 - order) < 0.15, (errs, p1, p2)


def test_real_diagonal_case_is_lfilter():
    """theta == 0 and constant dt, lambda: every state entry follows the
    linear filter h_t = alpha h_{t-1} + gamma u_t + beta u_{t-1},
    u_t = B_t x_t^T -- a width-2 FIR on u followed by a one-pole IIR
    [M3 s1 'equivalent to a width-2 data-dependent convolution'], computed by
    scipy.signal.lfilter."""
    I = rand_inputs(2, b=1, L=50, H=1, G=1, P=4, N=6, R=3)
    I["theta"][:] = 0.0
    I["dt"][:] = 0.37
    I["lam"][:] = 0.62
    y, hL, _, _ = oracle.scan(**I)
    d, lam, A = 0.37, 0.62, I["A"][0]
    alpha, beta, gamma = math.exp(d * A), (1 - lam) * d * math.exp(d * A), lam * d
    u = np.einsum("trn,trp->tnp", I["B"][0, :, 0], I["x"][0, :, 0])
    hs = scipy.signal.lfilter([gamma, beta], [1.0, -alpha], u, axis=0)
    ys = np.einsum("trn,tnp->trp", I["C"][0, :, 0], hs)
    np.testing.assert_allclose(y[0, :, 0], ys, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(hL[0, 0], hs[-1], rtol=1e-11, atol=1e-11)


def test_complex_constant_coefficients_is_complex_lfilter():
    """Constant dt, theta, lambda: each complex pair z_i obeys
    z_t = q z_{t-1} + gamma w_t + beta e^{i phi} w_{t-1}, q = e^{dt(A + i theta)},
    w_t = (B + i B_hat) x_t, y = Re((C + i C_hat)^T z) [M3 s2], via lfilter."""
    I = rand_inputs(3, b=1, L=60, H=1, G=1, P=2, N=10, R=2)
    I["dt"][:] = 0.21
    I["lam"][:] = 0.35
    th = np.random.default_rng(33).uniform(-np.pi, np.pi, size=5)
    I["theta"][:] = th
    y, hL, _, _ = oracle.scan(**I)
    d, lam, A = 0.21, 0.35, I["A"][0]
    phi = d * th
    q = np.exp(d * A) * np.exp(1j * phi)
    beta, gamma = (1 - lam) * d * math.exp(d * A), lam * d
    bc = to_complex(I["B"][0, :, 0])                            # [t][r][i]
    w = np.einsum("tri,trp->tip", bc, I["x"][0, :, 0])          # [t][i][p]
    z = np.empty_like(w)
    for i in range(5):
        z[:, i] = scipy.signal.lfilter([gamma, beta * np.exp(1j * phi[i])], [1.0, -q[i]],
                                       w[:, i], axis=0)
    cc = I["C"][0, :, 0, :, 0::2] - 1j * I["C"][0, :, 0, :, 1::2]   # C + i C_hat
    ys = np.real(np.einsum("tri,tip->trp", cc, z))
    np.testing.assert_allclose(y[0, :, 0], ys, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(hL[0, 0, 0::2], z[-1].real, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(hL[0, 0, 1::2], z[-1].imag, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("lam_one", [True, False])
def test_proposition2_complex_state_equals_real_rotation_form(lam_one):
    """Proposition 2 [M3 s2]: the N/2-dim complex SSM (native complex128
    arithmetic) equals the N-dim real SSM with 2x2 rotation blocks.  Mapping:
    pair i <-> rows (2i, 2i+1) = (Re, Im); B_real = (Re b, Im b);
    y = Re(c^T z) so C_real = (Re c, -Im c).  lambda == 1 is the statement as
    printed; general lambda applies e^{dt(A + i theta)} to the beta term too."""
    I = rand_inputs(4, b=2, L=33, H=3, G=3, P=2, N=8, R=2)
    if lam_one:
        I["lam"][:] = 1.0
    rng = np.random.default_rng(44)
    b, L, H, R, P = I["x"].shape
    N = 8
    bcx = rng.standard_normal((b, L, H, R, N // 2)) + 1j * rng.standard_normal((b, L, H, R, N // 2))
    ccx = rng.standard_normal((b, L, H, R, N // 2)) + 1j * rng.standard_normal((b, L, H, R, N // 2))
    Br = np.empty((b, L, H, R, N)); Br[..., 0::2] = bcx.real; Br[..., 1::2] = bcx.imag
    Cr = np.empty((b, L, H, R, N)); Cr[..., 0::2] = ccx.real; Cr[..., 1::2] = -ccx.imag
    I["B"], I["C"] = Br, Cr
    y, hL, _, _ = oracle.scan(**I)
    for bb in range(b):
        for h in range(H):
            z = np.zeros((N // 2, P), dtype=complex)
            wprev = np.zeros((N // 2, P), dtype=complex)
            for t in range(L):
                d, lam = I["dt"][bb, t, h], I["lam"][bb, t, h]
                trans = np.exp(d * (I["A"][h] + 1j * I["theta"][bb, t, h]))     # [i]
                w = bcx[bb, t, h].T @ I["x"][bb, t, h]                           # [i][p]
                z = trans[:, None] * (z + (1 - lam) * d * wprev) + lam * d * w
                ys = np.real(ccx[bb, t, h] @ z)                                  # [r][p]
                np.testing.assert_allclose(y[bb, t, h], ys, rtol=1e-11, atol=1e-11)
                wprev = w
            np.testing.assert_allclose(hL[bb, h, 0::2], z.real, rtol=1e-11, atol=1e-11)
            np.testing.assert_allclose(hL[bb, h, 1::2], z.imag, rtol=1e-11, atol=1e-11)


def test_proposition3_rope_trick():
    """Proposition 3 [M3 s2]: the rotating SSM equals the non-rotating one run
    on B and C rotated by their cumulative phase Phi_t = sum_{s<=t} dt_s theta_s.
    The rotation is done here with complex multiplication by e^{-i Phi}, and
    the final state comes back as h_L = R(Phi_{L-1}) h_tilde.  Also pins the
    oracle's own rope_bc (used for m3_rope_bc parity)."""
    I = rand_inputs(5, b=2, L=37, H=4, G=2, P=3, N=8, R=2)
    y, hL, pB, pX = oracle.scan(**I)
    b, L, H, R, P = I["x"].shape
    G, N = 2, 8
    hpg = H // G
    Bh = np.repeat(I["B"], hpg, axis=2)          # per head
    Ch = np.repeat(I["C"], hpg, axis=2)
    th = np.repeat(I["theta"], hpg, axis=2)
    Phi = np.cumsum(I["dt"][..., None] * th, axis=1)                # [b][t][h][i]
    rot = np.exp(-1j * Phi)[:, :, :, None, :]
    Bt = to_complex(Bh) * rot
    Ct = to_complex(Ch) * rot
    Brot = np.empty_like(Bh); Brot[..., 0::2] = Bt.real; Brot[..., 1::2] = Bt.imag
    Crot = np.empty_like(Ch); Crot[..., 0::2] = Ct.real; Crot[..., 1::2] = Ct.imag
    y2, hT, _, _ = oracle.scan(I["x"], Brot, Crot, I["dt"], I["A"], I["lam"],
                               np.zeros((b, L, H, N // 2)))
    np.testing.assert_allclose(y2, y, rtol=1e-10, atol=1e-10)
    zt = to_complex(np.swapaxes(hT, 2, 3)) * np.exp(1j * Phi[:, -1])[:, :, None, :]
    np.testing.assert_allclose(np.swapaxes(hL, 2, 3)[..., 0::2], zt.real, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(np.swapaxes(hL, 2, 3)[..., 1::2], zt.imag, rtol=1e-10, atol=1e-10)
    # the oracle's rope_bc agrees with the complex rotation and the cumsum
    Bo, Co, ph = oracle.rope_bc(I["B"], I["C"], I["dt"], I["theta"], nheads=H)
    np.testing.assert_allclose(Bo, Brot, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Co, Crot, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ph, Phi, rtol=1e-13, atol=1e-13)


def test_two_band_masked_matrix_brute_force():
    """SSD matrix form [M3 s1: the mask L of Mamba-3 is a decay mask times a
    two-band matrix; RD s II]: Y = (M o (C~ B~^T)) X with
    M = L_decay @ T, L_decay[t,s] = e^{a_t - a_s} (s <= t),
    T[s,s] = gamma_s, T[s,s-1] = beta_s, on rotated C~, B~ (Proposition 3),
    materialised as a dense (L R x L R) matrix.  Also checks the entry-wise
    form M[t,u] = e^{a_t-a_u} (gamma_u + [u<t] (1-lam_{u+1}) dt_{u+1})."""
    I = rand_inputs(6, b=1, L=48, H=1, G=1, P=3, N=6, R=3)
    y, _, _, _ = oracle.scan(**I)
    L, R, P, N = 48, 3, 3, 6
    dt, lam, A = I["dt"][0, :, 0], I["lam"][0, :, 0], I["A"][0]
    a = np.cumsum(dt * A)
    Ld = np.tril(np.exp(a[:, None] - a[None, :]))
    alpha = np.exp(dt * A)
    T = np.diag(lam * dt) + np.diag(((1 - lam) * dt * alpha)[1:], k=-1)
    M = Ld @ T
    Mform = np.zeros((L, L))
    for t in range(L):
        for u in range(t + 1):
            c = lam[u] * dt[u] + ((1 - lam[u + 1]) * dt[u + 1] if u < t else 0.0)
            Mform[t, u] = math.exp(a[t] - a[u]) * c
    np.testing.assert_allclose(M, Mform, rtol=1e-12, atol=1e-14)
    Phi = np.cumsum(dt[:, None] * I["theta"][0, :, 0], axis=0)           # [t][i]
    Bt = to_complex(I["B"][0, :, 0]) * np.exp(-1j * Phi)[:, None, :]
    Ct = to_complex(I["C"][0, :, 0]) * np.exp(-1j * Phi)[:, None, :]
    Bt = np.stack([Bt.real, Bt.imag], -1).reshape(L, R, N)
    Ct = np.stack([Ct.real, Ct.imag], -1).reshape(L, R, N)
    Gm = np.einsum("trn,usn->trus", Ct, Bt).reshape(L * R, L * R)
    Mbig = np.kron(M, np.ones((R, R)))
    Y = (Mbig * Gm) @ I["x"][0, :, 0].reshape(L * R, P)
    np.testing.assert_allclose(y[0, :, 0].reshape(L * R, P), Y, rtol=1e-10, atol=1e-10)


def test_width2_convolution_form():
    """Expanding the trapezoid [M3 s1; RD s II 'size-two convolutional mask']:
    u_t = gamma_t B_t x_t^T + beta_t R_t B_{t-1} x_{t-1}^T is a width-2
    convolution of the rotated inputs and h_t = alpha_t R_t h_{t-1} + u_t.
    The convolution is formed first for all t (vectorised), then the scan."""
    I = rand_inputs(7, b=1, L=30, H=1, G=1, P=2, N=6, R=2)
    y, hL, _, _ = oracle.scan(**I)
    L = 30
    dt, lam, A = I["dt"][0, :, 0], I["lam"][0, :, 0], I["A"][0]
    phi = dt[:, None] * I["theta"][0, :, 0]                              # [t][i]
    bx = to_complex(np.einsum("trn,trp->tpn", I["B"][0, :, 0], I["x"][0, :, 0]))   # [t][p][i]
    beta = (1 - lam) * dt * np.exp(dt * A)
    shifted = np.concatenate([np.zeros_like(bx[:1]), bx[:-1]], axis=0)
    u = (lam * dt)[:, None, None] * bx + (beta[:, None, None] * np.exp(1j * phi)[:, None, :]) * shifted
    z = np.zeros_like(bx[0])
    cc = to_complex(I["C"][0, :, 0, :, :]).conj()                        # C - i*C_odd
    for t in range(L):
        z = np.exp(dt[t] * A) * np.exp(1j * phi[t])[None, :] * z + u[t]
        ys = np.real(np.einsum("ri,pi->rp", cc[t], z))
        np.testing.assert_allclose(y[0, t, 0], ys, rtol=1e-11, atol=1e-11)


def test_closed_form_constant_forcing_and_gap():
    """Constant rho = e^{dt A}, phi = dt theta, lambda and constant input: the
    complex pair follows z_t = K + (z_0 - K) q^t, q = rho e^{i phi},
    K = (gamma + (1-lam) dt q) w / (1 - q), z_0 = gamma w (geometric series).
    Late in the sequence the oracle's state size is |gamma + (1-lam) dt q| |w|
    / |1 - rho e^{i phi}|: the complex gap of [OSC C.3], not the radial gap
    1 - rho, sets how much the forcing accumulates."""
    L = 3000
    d, lam, A = 0.1, 0.4, -0.05
    rho = math.exp(d * A)
    w = 0.6 - 0.3j
    for th in (0.0, 0.5, 2.0, 3.1):
        x = np.ones((1, L, 1, 1, 1))
        B = np.tile([w.real, w.imag], (1, L, 1, 1, 1)).reshape(1, L, 1, 1, 2)
        C = np.tile([1.0, 0.0], (1, L, 1, 1, 1)).reshape(1, L, 1, 1, 2)
        y, hL, _, _ = oracle.scan(x, B, C, np.full((1, L, 1), d), np.array([A]),
                                  np.full((1, L, 1), lam), np.full((1, L, 1, 1), th))
        q = rho * np.exp(1j * d * th)
        K = (lam * d + (1 - lam) * d * q) * w / (1 - q)
        zt = K + (lam * d * w - K) * q ** np.arange(L)
        np.testing.assert_allclose(y[0, :, 0, 0, 0], zt.real, rtol=1e-9, atol=1e-11)
        late = abs(hL[0, 0, 0, 0] + 1j * hL[0, 0, 1, 0])
        gap = abs(1 - rho * np.exp(1j * d * th))
        want = abs(lam * d + (1 - lam) * d * q) * abs(w) / gap
        assert abs(late - want) < 1e-6 * want


def test_c1_homogeneous_decay_rotation_is_matrix_exponential():
    """[OSC C.1]: with no input, one rotary pair evolves by the exponential of
    the generator [[A, -theta], [theta, A]]: after k steps of constant dt it
    equals expm(k dt G) h_0 = e^{k dt A} R(k dt theta) h_0 (scipy.linalg.expm)."""
    k, d, A, th = 25, 0.3, -0.4, 1.1
    h0 = np.array([0.7, -1.3, 0.2, 0.5]).reshape(1, 1, 4, 1)
    x = np.zeros((1, k, 1, 1, 1))
    B = np.zeros((1, k, 1, 1, 4))
    C = np.zeros((1, k, 1, 1, 4))
    theta = np.tile([th, -2 * th], (1, k, 1, 1)).reshape(1, k, 1, 2)
    _, hL, _, _ = oracle.scan(x, B, C, np.full((1, k, 1), d), np.array([A]),
                              np.full((1, k, 1), 0.5), theta, init_h=h0)
    for i, w in enumerate((th, -2 * th)):
        Gen = np.array([[A, -w], [w, A]])
        want = scipy.linalg.expm(k * d * Gen) @ h0[0, 0, 2 * i:2 * i + 2, 0]
        np.testing.assert_allclose(hL[0, 0, 2 * i:2 * i + 2, 0], want, rtol=1e-12, atol=1e-14)


def _read_golden_e1():
    rows = []
    with open(os.path.join(GOLDEN, "e1_phase_increments.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                m, i0, i1, _, _ = line.split()
                rows.append((int(m), float(i0), float(i1)))
    return rows


@pytest.mark.parametrize("row", _read_golden_e1())
def test_e1_phase_counts_ones_modulo_m(row):
    """[OSC E.1, Figure 5]: a pair whose increment is 0 for input 0 and
    360/m degrees for input 1 keeps (count of ones) mod m in its phase.  With
    dt = 1 the oracle's cumulative phase, taken mod 2 pi, must equal the
    prefix count of ones mod m times 2 pi / m."""
    m, inc0, inc1 = row
    bits = np.random.default_rng(100 + m).integers(0, 2, size=300)
    L = bits.size
    theta = np.where(bits == 1, math.radians(inc1), math.radians(inc0)).reshape(1, L, 1, 1)
    B = np.zeros((1, L, 1, 1, 2))
    _, _, ph = oracle.rope_bc(B, B, np.ones((1, L, 1)), theta, nheads=1)
    got = np.mod(ph[0, :, 0, 0], 2 * math.pi)
    want = (np.cumsum(bits) % m) * (2 * math.pi / m)
    diff = np.angle(np.exp(1j * (got - want)))
    assert np.max(np.abs(diff)) < 1e-9


def test_mimo_is_sum_of_siso_runs():
    """MIMO [M3 s3]: the rank-R state update B X^T = sum_r B[:,r] x[r,:]^T is
    a sum of R SISO updates, and y[r'] reads the summed state with C[:,r'].
    By linearity, y_MIMO[r'] = sum_r y_SISO(B[:,r], x[r], C[:,r'])."""
    I = rand_inputs(8, b=1, L=35, H=2, G=2, P=3, N=6, R=3)
    y, hL, _, _ = oracle.scan(**I)
    R = 3
    ysum = np.zeros_like(y)
    hsum = np.zeros_like(hL)
    for r in range(R):
        for r2 in range(R):
            ys, hs, _, _ = oracle.scan(I["x"][:, :, :, r:r + 1], I["B"][:, :, :, r:r + 1],
                                       I["C"][:, :, :, r2:r2 + 1], I["dt"], I["A"], I["lam"],
                                       I["theta"])
            ysum[:, :, :, r2] += ys[:, :, :, 0]
            if r2 == 0:
                hsum += hs
    np.testing.assert_allclose(y, ysum, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(hL, hsum, rtol=1e-11, atol=1e-11)


def test_output_is_linear_in_x_and_the_carry():
    """y and the final state are linear in (x, h_-1, x_-1) jointly, with B, C
    and the coefficients fixed [M3 s1]: nothing in the recurrence adds a term
    that does not carry exactly one factor of the state or of x."""
    I = rand_inputs(15, b=2, L=23, H=2, G=1, P=3, N=6, R=2)
    rng = np.random.default_rng(150)
    x2 = rng.standard_normal(I["x"].shape)
    h1, h2 = rng.standard_normal((2, 2, 2, 6, 3))
    pB = rng.standard_normal((2, 2, 2, 6))
    p1, p2 = rng.standard_normal((2, 2, 2, 2, 3))
    rest = {k: v for k, v in I.items() if k != "x"}
    ya, ha, _, _ = oracle.scan(x=I["x"], **rest, init_h=h1, init_pB=pB, init_pX=p1)
    yb, hb, _, _ = oracle.scan(x=x2, **rest, init_h=h2, init_pB=pB, init_pX=p2)
    yc, hc, _, _ = oracle.scan(x=I["x"] - 2.5 * x2, **rest, init_h=h1 - 2.5 * h2, init_pB=pB,
                               init_pX=p1 - 2.5 * p2)
    np.testing.assert_allclose(yc, ya - 2.5 * yb, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(hc, ha - 2.5 * hb, rtol=1e-11, atol=1e-11)


def test_rank1_equals_siso_shape():
    I = rand_inputs(9, b=1, L=20, H=1, G=1, P=4, N=4, R=1)
    y, hL, _, _ = oracle.scan(**I)
    assert y.shape == (1, 20, 1, 1, 4) and hL.shape == (1, 1, 4, 4)
    assert np.all(np.isfinite(y))


@pytest.mark.parametrize("L1", [1, 17, 39])
def test_continuation_split_sequence(L1):
    """Splitting a sequence across two calls through the carry
    (h, prev_B, prev_x) gives the single-call result: the carry is exactly
    the information the recurrence needs at the cut."""
    I = rand_inputs(10, b=2, L=40, H=2, G=1, P=3, N=6, R=2)
    y, hL, pB, pX = oracle.scan(**I)
    s1 = {k: (v[:, :L1] if k != "A" else v) for k, v in I.items()}
    s2 = {k: (v[:, L1:] if k != "A" else v) for k, v in I.items()}
    ya, ha, pBa, pXa = oracle.scan(**s1)
    yb, hb, pBb, pXb = oracle.scan(**s2, init_h=ha, init_pB=pBa, init_pX=pXa)
    np.testing.assert_allclose(np.concatenate([ya, yb], axis=1), y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hb, hL, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(pBb, pB, rtol=0, atol=0)
    np.testing.assert_allclose(pXb, pX, rtol=0, atol=0)


def test_scan_then_steps_equals_longer_scan():
    """scan(L) followed by k single-token steps equals scan(L + k)."""
    I = rand_inputs(11, b=2, L=30, H=2, G=2, P=3, N=6, R=2)
    L0 = 25
    y, hL, _, _ = oracle.scan(**I)
    s1 = {k: (v[:, :L0] if k != "A" else v) for k, v in I.items()}
    _, h, pB, pX = oracle.scan(**s1)
    for t in range(L0, 30):
        yt, h, pB, pX = oracle.step(h, pB, pX, I["x"][:, t], I["B"][:, t], I["C"][:, t],
                                    I["dt"][:, t], I["A"], I["lam"][:, t], I["theta"][:, t])
        np.testing.assert_allclose(yt, y[:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h, hL, rtol=1e-12, atol=1e-12)


def test_group_sharing_equals_per_head_copies():
    """Heads of one group share B, C and theta; dt, lambda and A stay per head.
    Expanding the groups to per-head copies changes nothing."""
    I = rand_inputs(12, b=1, L=20, H=4, G=2, P=2, N=4, R=2)
    y, hL, _, _ = oracle.scan(**I)
    J = dict(I)
    for k in ("B", "C", "theta"):
        J[k] = np.repeat(I[k], 2, axis=2)
    y2, h2, _, _ = oracle.scan(**J)
    np.testing.assert_array_equal(y, y2)
    np.testing.assert_array_equal(hL, h2)


def test_oracle_rejects_bad_arguments():
    I = rand_inputs(13, b=1, L=4, H=2, G=1, P=2, N=4, R=1)
    with pytest.raises(ValueError):
        oracle.scan(I["x"], I["B"][..., :3], I["C"][..., :3], I["dt"], I["A"], I["lam"],
                    I["theta"][..., :1])          # odd N


def test_thread_count_does_not_change_results():
    """Each (b, h) is one thread's sequential loop, so one thread and all of
    them give bit-identical outputs, forward and backward (the bench times the
    oracle both ways)."""
    I = rand_inputs(14, b=3, L=9, H=4, G=2, P=3, N=4, R=2)
    dy = np.random.default_rng(140).standard_normal(I["x"].shape)
    cores = oracle.num_threads()
    try:
        oracle.set_num_threads(1)
        one = oracle.scan(**I), oracle.scan_bwd(**I, dy=dy)
        oracle.set_num_threads(max(cores, 2))
        many = oracle.scan(**I), oracle.scan_bwd(**I, dy=dy)
    finally:
        oracle.set_num_threads(cores)
    for a, b in zip(one[0], many[0]):
        np.testing.assert_array_equal(a, b)
    assert one[1].keys() == many[1].keys()
    for k in one[1]:
        np.testing.assert_array_equal(one[1][k], many[1][k])


# ------------------------------------------------------- planted mistakes --
def _pin_complex_err(lib):
    """max |oracle - native complex SSM| on time-varying inputs (Prop. 2 reading)."""
    I = rand_inputs(21, b=1, L=24, H=1, G=1, P=2, N=6, R=2)
    rng = np.random.default_rng(210)
    L, R, P, N = 24, 2, 2, 6
    bcx = rng.standard_normal((L, R, N // 2)) + 1j * rng.standard_normal((L, R, N // 2))
    ccx = rng.standard_normal((L, R, N // 2)) + 1j * rng.standard_normal((L, R, N // 2))
    Br = np.empty((1, L, 1, R, N)); Br[0, :, 0, :, 0::2] = bcx.real; Br[0, :, 0, :, 1::2] = bcx.imag
    Cr = np.empty((1, L, 1, R, N)); Cr[0, :, 0, :, 0::2] = ccx.real; Cr[0, :, 0, :, 1::2] = -ccx.imag
    I["B"], I["C"] = Br, Cr
    y = oracle.scan(**I, lib=lib)[0]
    z = np.zeros((N // 2, P), dtype=complex)
    wprev = np.zeros_like(z)
    err = 0.0
    for t in range(L):
        d, lam = I["dt"][0, t, 0], I["lam"][0, t, 0]
        trans = np.exp(d * (I["A"][0] + 1j * I["theta"][0, t, 0]))
        w = bcx[t].T @ I["x"][0, t, 0]
        z = trans[:, None] * (z + (1 - lam) * d * wprev) + lam * d * w
        err = max(err, float(np.max(np.abs(y[0, t, 0] - np.real(ccx[t] @ z)))))
        wprev = w
    return err


def _pin_brute_err(lib):
    """max |oracle - dense SSD two-band form| (rotated via complex multiply)."""
    I = rand_inputs(22, b=1, L=20, H=1, G=1, P=2, N=4, R=2)
    y = oracle.scan(**I, lib=lib)[0]
    L, R, P, N = 20, 2, 2, 4
    dt, lam, A = I["dt"][0, :, 0], I["lam"][0, :, 0], I["A"][0]
    a = np.cumsum(dt * A)
    M = np.tril(np.exp(a[:, None] - a[None, :])) @ (
        np.diag(lam * dt) + np.diag(((1 - lam) * dt * np.exp(dt * A))[1:], k=-1))
    Phi = np.cumsum(dt[:, None] * I["theta"][0, :, 0], axis=0)
    Bt = to_complex(I["B"][0, :, 0]) * np.exp(-1j * Phi)[:, None, :]
    Ct = to_complex(I["C"][0, :, 0]) * np.exp(-1j * Phi)[:, None, :]
    Bt = np.stack([Bt.real, Bt.imag], -1).reshape(L, R, N)
    Ct = np.stack([Ct.real, Ct.imag], -1).reshape(L, R, N)
    Gm = np.einsum("trn,usn->trus", Ct, Bt).reshape(L * R, L * R)
    Y = (np.kron(M, np.ones((R, R))) * Gm) @ I["x"][0, :, 0].reshape(L * R, P)
    return float(np.max(np.abs(y[0, :, 0].reshape(L * R, P) - Y)))


_MUTATIONS = {
    # the beta term added after the rotation instead of before it
    "beta_not_rotated": [
        ("H[n * P + p] = alpha * H[n * P + p] + beta * bx;", "H[n * P + p] = alpha * H[n * P + p];"),
        ("    /* current input: + gamma * B_t X_t^T */",
         "    for (int n = 0; n < N; ++n) for (int p = 0; p < P; ++p) { double bx = 0.0;"
         " for (int r = 0; r < R; ++r) bx += PB[r * N + n] * PX[r * P + p];"
         " H[n * P + p] += beta * bx; }\n    /* current input: + gamma * B_t X_t^T */")],
    # rotation by -phi
    "rotation_sign": [
        ("H[(2 * i) * P + p] = c * u0 - s * u1;", "H[(2 * i) * P + p] = c * u0 + s * u1;"),
        ("H[(2 * i + 1) * P + p] = s * u0 + c * u1;", "H[(2 * i + 1) * P + p] = -s * u0 + c * u1;")],
    # beta weighted by lambda instead of 1 - lambda
    "beta_weight": [("const double beta = (1.0 - lam) * d * exp(d * a);",
                     "const double beta = lam * d * exp(d * a);")],
    # beta term reads B_t x_t instead of B_{t-1} x_{t-1}
    "beta_index": [("bx += PB[r * N + n] * PX[r * P + p];", "bx += Bt[r * N + n] * xt[r * P + p];")],
    # rotation angle without dt
    "angle_without_dt": [("const double phi = d * th[i];", "const double phi = th[i];")],
    # readout always with rank 0 of C
    "readout_rank": [("acc += Ct[r * N + n] * H[n * P + p];", "acc += Ct[n] * H[n * P + p];")],
    # previous x never carried to the next step
    "stale_prev_x": [("memcpy(PX, xt, sizeof(double) * (size_t)R * P);", "/* dropped */")],
}


def test_pins_pass_on_the_oracle():
    assert _pin_complex_err(None) < 1e-10
    assert _pin_brute_err(None) < 1e-10


@pytest.mark.parametrize("name", sorted(_MUTATIONS))
def test_planted_mistakes_are_caught(name):
    """A plausible mistake planted in a copy of the oracle (a dropped or
    misplaced term, a wrong sign or index) fails the complex-SSM pin
    (Proposition 2) or the dense two-band SSD pin."""
    src = oracle.source_text()
    for old, new in _MUTATIONS[name]:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    lib = oracle.compile_variant(src, name)
    errs = (_pin_complex_err(lib), _pin_brute_err(lib))
    assert max(errs) > 1e-6, f"mutation {name} slipped through the pins: {errs}"


# ------------------------------------------------------------- backward --
def _fd_errors(lib, seed=7, b=2, L=6, H=2, G=1, P=3, N=4, R=2, carry=True):
    """Relative error of the oracle's backward against central finite
    differences of its forward, per input (random direction each)."""
    rng = np.random.default_rng(seed)
    rnd = lambda *s: rng.standard_normal(s)
    inp = dict(x=rnd(b, L, H, R, P), B=rnd(b, L, G, R, N), C=rnd(b, L, G, R, N),
               dt=np.log1p(np.exp(rnd(b, L, H))), A=-np.exp(rng.uniform(-2, 1, H)),
               lam=1 / (1 + np.exp(-rnd(b, L, H))), theta=rng.uniform(-np.pi, np.pi, (b, L, G, N // 2)))
    init = dict(init_h=rnd(b, H, N, P), init_pB=rnd(b, H, R, N), init_pX=rnd(b, H, R, P)) if carry else {}
    dy = rnd(b, L, H, R, P)
    fin = dict(dh=rnd(b, H, N, P), dpB=rnd(b, H, R, N), dpX=rnd(b, H, R, P)) if carry else {}

    def J(i, n):
        y, hL, pB, pX = oracle.scan(**i, **n, lib=lib)
        j = float((dy * y).sum())
        if carry:
            j += float((fin["dh"] * hL).sum() + (fin["dpB"] * pB).sum() + (fin["dpX"] * pX).sum())
        return j

    g = oracle.scan_bwd(**inp, dy=dy, **init, **fin, lib=lib)
    errs = {}
    eps = 1e-6
    for k in list(inp) + list(init):
        tgt_inp, tgt_init = dict(inp), dict(init)
        tgt = tgt_inp if k in inp else tgt_init
        base = tgt[k]
        v = rng.standard_normal(base.shape)
        tgt[k] = base + eps * v
        jp = J(tgt_inp, tgt_init)
        tgt[k] = base - eps * v
        jm = J(tgt_inp, tgt_init)
        fd = (jp - jm) / (2 * eps)
        an = float((g[{"init_h": "d_init_h", "init_pB": "d_init_pB", "init_pX": "d_init_pX"}.get(k, "d" + k)]
                    * v).sum())
        errs[k] = abs(fd - an) / max(abs(fd), 1e-12)
    return errs


@pytest.mark.parametrize("case", [
    dict(),                                   # shared group (G=1 of 2 heads), MIMO R=2, carries
    dict(G=2, R=1, seed=8),                   # SISO, one group per head
    dict(carry=False, L=9, seed=9),           # no carry in or out
    dict(R=3, N=6, P=2, seed=10),
])
def test_backward_matches_finite_differences(case):
    """The oracle's backward (its own hand-written adjoint) against central
    finite differences of the forward oracle: a directional derivative per
    input, in float64."""
    errs = _fd_errors(None, **case)
    for k, e in errs.items():
        assert e < 1e-6, (k, e, errs)


_BWD_MUTATIONS = {
    # the beta path of token t+1 left out of dJ/d(B_t x_t^T)
    "bwd_no_beta_path": [("Dt[n * P + p] = ga * gk[n * P + p] + Db[n * P + p];",
                          "Dt[n * P + p] = ga * gk[n * P + p];")],
    # rotation derivative with the wrong sign
    "bwd_dphi_sign": [("dphi += g0 * (-s * v0 - c * v1) + g1 * (c * v0 - s * v1);",
                       "dphi += g0 * (s * v0 + c * v1) + g1 * (-c * v0 + s * v1);")],
    # the phase term of d dt dropped
    "bwd_ddt_no_phase": [("dga * lm + dphi_th;", "dga * lm;")],
    # the adjoint not rotated back (R_t^T) before it is carried
    "bwd_adjoint_unrotated": [("gk[n * P + p] = al * gv[n * P + p];", "gk[n * P + p] = al * gk[n * P + p];")],
    # dA without the beta contribution
    "bwd_dA_no_beta": [("dAh[bh] += dal * dd * al + dbe * (1.0 - lm) * dd * dd * al;",
                        "dAh[bh] += dal * dd * al;")],
    # the gradient arriving at the final prev_B ignored
    "bwd_no_final_pB": [("if (dpB) for (int e = 0; e < R * N; ++e) dBt[e] += dpB[bh * R * N + e];",
                         "/* dropped */")],
}


@pytest.mark.parametrize("name", sorted(_BWD_MUTATIONS))
def test_backward_planted_mistakes_are_caught(name):
    src = oracle.source_text()
    for old, new in _BWD_MUTATIONS[name]:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    lib = oracle.compile_variant(src, name)
    errs = _fd_errors(lib)
    assert max(errs.values()) > 1e-4, f"mutation {name} slipped through: {errs}"


# --------------------------------------------------- phase interventions --
def test_phase_modes_reduce_to_native_where_they_must():
    """With theta == 0 every intervention is the native scan; an identity
    permutation and a 'fixed' frequency equal to the given theta are too."""
    I = rand_inputs(31, b=1, L=30, H=4, G=2, P=3, N=8, R=2)
    I0 = dict(I, theta=np.zeros_like(I["theta"]))
    y0 = oracle.scan(**I0)[0]
    for mode in ("zero", "reverse", "write_only", "read_only"):
        assert rel(oracle.scan_phase(mode, **I0)[0], y0) < 1e-12, mode
    y = oracle.scan(**I)[0]
    assert rel(oracle.scan_phase("shuffle", **I, perm=[0, 1, 2, 3])[0], y) < 1e-12
    Ic = dict(I, theta=np.broadcast_to(np.array([[0.3, -1.1, 2.0, 0.7], [1.5, 0.2, -0.4, 3.0]]),
                                       I["theta"].shape).copy())
    assert rel(oracle.scan_phase("fixed", **Ic, freq=[[0.3, -1.1, 2.0, 0.7], [1.5, 0.2, -0.4, 3.0]])[0],
               oracle.scan(**Ic)[0]) < 1e-12
    # reverse equals the native scan on the mirrored pairs (conjugate rotation)
    Im = dict(I, B=I["B"][..., [1, 0, 3, 2, 5, 4, 7, 6]], C=I["C"][..., [1, 0, 3, 2, 5, 4, 7, 6]])
    yr = oracle.scan_phase("reverse", **I)[0]
    assert rel(yr, oracle.scan(**Im)[0]) < 1e-12


@pytest.mark.parametrize("mode", ["write_only", "read_only"])
def test_one_sided_rotation_is_the_dense_two_band_form(mode):
    """write_only / read_only against the dense two-band SSD matrix built here
    with only one of B, C rotated by the cumulative phase (complex multiply)."""
    I = rand_inputs(32, b=1, L=18, H=1, G=1, P=2, N=4, R=2)
    y = oracle.scan_phase(mode, **I)[0]
    L, R, P, N = 18, 2, 2, 4
    dt, lam, A = I["dt"][0, :, 0], I["lam"][0, :, 0], I["A"][0]
    a = np.cumsum(dt * A)
    M = np.tril(np.exp(a[:, None] - a[None, :])) @ (
        np.diag(lam * dt) + np.diag(((1 - lam) * dt * np.exp(dt * A))[1:], k=-1))
    Phi = np.cumsum(dt[:, None] * I["theta"][0, :, 0], axis=0)
    rot = lambda v: to_complex(v) * np.exp(-1j * Phi)[:, None, :]
    Bc = rot(I["B"][0, :, 0]) if mode == "write_only" else to_complex(I["B"][0, :, 0])
    Cc = to_complex(I["C"][0, :, 0]) if mode == "write_only" else rot(I["C"][0, :, 0])
    Bt = np.stack([Bc.real, Bc.imag], -1).reshape(L, R, N)
    Ct = np.stack([Cc.real, Cc.imag], -1).reshape(L, R, N)
    Gm = np.einsum("trn,usn->trus", Ct, Bt).reshape(L * R, L * R)
    Y = (np.kron(M, np.ones((R, R))) * Gm) @ I["x"][0, :, 0].reshape(L * R, P)
    assert np.max(np.abs(y[0, :, 0].reshape(L * R, P) - Y)) < 1e-10


def test_backward_homogeneity_identities():
    """Exact identities, no finite differences: with a zero carry-in the loss
    J = sum <dy, y> is linear in x, in B and in C separately (homogeneous of
    degree one), so <dJ/dx, x> = <dJ/dB, B> = <dJ/dC, C> = J; and the carry-in
    state enters linearly, so adding h_{-1} adds exactly <dJ/dh_{-1}, h_{-1}>."""
    I = rand_inputs(41, b=2, L=12, H=2, G=1, P=3, N=6, R=2)
    rng = np.random.default_rng(410)
    dy = rng.standard_normal((2, 12, 2, 2, 3))
    y = oracle.scan(**I)[0]
    J = float((dy * y).sum())
    g = oracle.scan_bwd(**I, dy=dy)
    for k in ("x", "B", "C"):
        assert abs(float((g["d" + k] * I[k]).sum()) - J) < 1e-10 * max(1.0, abs(J)), k
    h0 = rng.standard_normal((2, 2, 6, 3))
    J1 = float((dy * oracle.scan(**I, init_h=h0)[0]).sum())
    assert abs((J1 - J) - float((g["d_init_h"] * h0).sum())) < 1e-10 * max(1.0, abs(J1))
