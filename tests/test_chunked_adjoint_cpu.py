"""The chunked (dual) form of the scan's adjoint, checked in float64 against
the oracle's token-by-token reverse mode (CPU only).

Proposition 3 ("Mamba-3" summary, b-lab.team, section 2) turns the scan, in
the frame rotated by the cumulative phase, into a real decaying recurrence
with the two-band trapezoid mask of section 1: with a_t = A sum_{tau<=t} dt_tau,
u_s = B~_s^T x_s and c_s = gamma_s + (1 - lambda_{s+1}) dt_{s+1},

    y_t = C~_t ( sum_{s<=t} w_ts u_s + e^{a_t} S_-1 ),
    w_tt = gamma_t,   w_ts = e^{a_t - a_s} c_s  (s < t).

Its adjoint has the same shape run right to left.  Per chunk [t0, t1], with
rows ordered (t, r) and M the mask broadcast over R x R blocks:

    dC~ = (M o dY X^T) B~   + diag(e^{a_t - a_{t0-1}}) dY S_in^T
    dX  = (M o C~ B~^T)^T dY + diag(e^{a_t1 - a_s} c_s) B~ D
    dB~ = (M o dY X^T)^T C~ + diag(e^{a_t1 - a_s} c_s) X D^T
    D_prev = sum_{t in chunk} e^{a_t - a_{t0-1}} C~_t^T dy_t + e^{a_t1 - a_{t0-1}} D

where S_in is the (augmented) state entering the chunk and D the adjoint of
the state leaving it (R(Phi_{L-1})^T dh after the last chunk).  The scalars
come from dW = blocksum_{R x R}(C~B~^T o dY X^T): row and column sums of
dW o w give dJ/da_t; column sums of dW e^{a_t - a_s} plus <D, u_s> give
dJ/dc_s; the diagonal gives dJ/dgamma.  The rotation gives dPhi_t per pair
from (dB~, B~) and (dC~, C~), and theta and dt take its reverse cumulative sum.

This file writes those equations out in numpy and checks every gradient of
oracle.scan_bwd to rounding on shapes with ragged chunks, carries in and out,
shared groups and R = 1..3.  It states the chunked adjoint a tensor-core
backward computes; nothing in the package imports it.
"""
import numpy as np
import pytest

import oracle


def _rot_t(v, phi):
    """R(phi)^T on interleaved pairs along the last axis."""
    c, s = np.cos(phi), np.sin(phi)
    o = np.empty_like(v)
    o[..., 0::2] = c * v[..., 0::2] + s * v[..., 1::2]
    o[..., 1::2] = -s * v[..., 0::2] + c * v[..., 1::2]
    return o


def _rot(v, phi):
    """R(phi) on interleaved pairs along the last axis."""
    c, s = np.cos(phi), np.sin(phi)
    o = np.empty_like(v)
    o[..., 0::2] = c * v[..., 0::2] - s * v[..., 1::2]
    o[..., 1::2] = s * v[..., 0::2] + c * v[..., 1::2]
    return o


def _pair_dphi(dv, v):
    """sum_r (dv_2i v_2i+1 - dv_2i+1 v_2i): d<dv, R(phi)^T w>/dphi at v = R^T w."""
    return (np.einsum("lrn,lrn->ln", dv[..., 0::2], v[..., 1::2]) -
            np.einsum("lrn,lrn->ln", dv[..., 1::2], v[..., 0::2]))


def chunked_adjoint(x, B, C, dt, A, lam, theta, dy, Q, init_h=None, init_pB=None, init_pX=None,
                    dh=None, dpB=None, dpX=None):
    nb, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    hpg = H // G
    out = {"dx": np.zeros_like(x), "dB": np.zeros_like(B), "dC": np.zeros_like(C),
           "ddt": np.zeros_like(dt), "dA": np.zeros_like(A), "dlam": np.zeros_like(lam),
           "dtheta": np.zeros_like(theta), "d_init_h": np.zeros((nb, H, N, P)),
           "d_init_pB": np.zeros((nb, H, R, N)), "d_init_pX": np.zeros((nb, H, R, P))}
    chunks = [(t0, min(L, t0 + Q) - 1) for t0 in range(0, L, Q)]
    for b in range(nb):
        for h in range(H):
            g = h // hpg
            d, lm, Ah = dt[b, :, h], lam[b, :, h], A[h]
            phi = np.cumsum(d[:, None] * theta[b, :, g], axis=0)
            Bt = _rot_t(B[b, :, g], phi[:, None, :])
            Ct = _rot_t(C[b, :, g], phi[:, None, :])
            X, dY = x[b, :, h], dy[b, :, h]
            cumd = np.cumsum(d)
            a = Ah * cumd
            a_before = np.concatenate([[0.0], a])            # a_{t-1} at index t
            gam = lm * d
            nxt = np.zeros(L)
            nxt[:-1] = (1 - lm[1:]) * d[1:]
            c = gam + nxt
            u = np.einsum("lrn,lrp->lnp", Bt, X)
            h0 = init_h[b, h] if init_h is not None else np.zeros((N, P))
            pB = init_pB[b, h] if init_pB is not None else np.zeros((R, N))
            pX = init_pX[b, h] if init_pX is not None else np.zeros((R, P))
            u_prev = pB.T @ pX
            # forward: state entering each chunk (augmented with the pending beta term)
            S_in = [h0 + ((1 - lm[0]) * d[0] * u_prev if L else 0.0)]
            for t0, t1 in chunks:
                w_exit = np.exp(a[t1] - a[t0:t1 + 1]) * c[t0:t1 + 1]
                S_in.append(np.exp(a[t1] - a_before[t0]) * S_in[-1] + np.einsum("l,lnp->np", w_exit, u[t0:t1 + 1]))
            h_last = S_in[-1]                                # c_{L-1} = gamma_{L-1}: no pending term
            # backward: adjoint of the state leaving each chunk
            D = [None] * (len(chunks) + 1)
            D[-1] = _rot_t(dh[b, h].T, phi[L - 1]).T if (dh is not None and L) else np.zeros((N, P))
            for ci in range(len(chunks) - 1, -1, -1):
                t0, t1 = chunks[ci]
                e_in = np.exp(a[t0:t1 + 1] - a_before[t0])
                D[ci] = (np.exp(a[t1] - a_before[t0]) * D[ci + 1] +
                         np.einsum("l,lrn,lrp->np", e_in, Ct[t0:t1 + 1], dY[t0:t1 + 1]))
            dBt, dCt, dX = np.zeros_like(Bt), np.zeros_like(Ct), np.zeros_like(X)
            da, dgam, eps = np.zeros(L), np.zeros(L), np.zeros(L)
            for ci, (t0, t1) in enumerate(chunks):
                sl = slice(t0, t1 + 1)
                q = t1 - t0 + 1
                tt, ss = np.meshgrid(np.arange(t0, t1 + 1), np.arange(t0, t1 + 1), indexing="ij")
                strict = ss < tt
                E = np.where(strict, np.exp(np.where(strict, a[tt] - a[ss], 0.0)), 0.0)
                W = E * c[ss] + np.where(tt == ss, gam[ss], 0.0)
                Mb = np.kron(W, np.ones((R, R)))
                Cf, Bf = Ct[sl].reshape(q * R, N), Bt[sl].reshape(q * R, N)
                Xf, dYf = X[sl].reshape(q * R, P), dY[sl].reshape(q * R, P)
                CB, YX = Cf @ Bf.T, dYf @ Xf.T
                e_in = np.exp(a[sl] - a_before[t0])
                w_exit = np.exp(a[t1] - a[sl]) * c[sl]
                Dn, Sc = D[ci + 1], S_in[ci]
                dCt[sl] = ((Mb * YX) @ Bf + np.repeat(e_in, R)[:, None] * (dYf @ Sc.T)).reshape(q, R, N)
                dX[sl] = ((Mb * CB).T @ dYf + np.repeat(w_exit, R)[:, None] * (Bf @ Dn)).reshape(q, R, P)
                dBt[sl] = ((Mb * YX).T @ Cf + np.repeat(w_exit, R)[:, None] * (Xf @ Dn.T)).reshape(q, R, N)
                dW = (CB * YX).reshape(q, R, q, R).sum(axis=(1, 3))
                uD = np.einsum("lnp,np->l", u[sl], Dn)
                offd = dW * W * strict
                carry_in = e_in * np.einsum("lrp,lrn,np->l", dY[sl], Ct[sl], Sc)
                da[sl] += offd.sum(axis=1) + carry_in - offd.sum(axis=0) - w_exit * uD
                eps[sl] += (dW * E).sum(axis=0) + np.exp(a[t1] - a[sl]) * uD
                dgam[sl] += np.diag(dW)
            if L:
                da[L - 1] += np.sum(D[-1] * h_last)          # the exported state decays with a_{L-1}
            dgam += eps
            ddt = lm * dgam + Ah * np.cumsum(da[::-1])[::-1]
            dlam = d * dgam
            ddt[1:] += (1 - lm[1:]) * eps[:-1]
            dlam[1:] -= d[1:] * eps[:-1]
            out["dA"][h] += np.sum(cumd * da)
            if L:
                e_prev = np.sum(D[0] * u_prev)
                ddt[0] += (1 - lm[0]) * e_prev
                dlam[0] -= d[0] * e_prev
                du_prev = (1 - lm[0]) * d[0] * D[0]
                out["d_init_pB"][b, h] = pX @ du_prev.T
                out["d_init_pX"][b, h] = pB @ du_prev
            out["d_init_h"][b, h] = D[0]
            dphi = _pair_dphi(dBt, Bt) + _pair_dphi(dCt, Ct)
            if dh is not None and L:
                hf = _rot(h_last.T, phi[L - 1]).T
                dhb = dh[b, h]
                dphi[L - 1] += (dhb[1::2] * hf[0::2] - dhb[0::2] * hf[1::2]).sum(axis=1)
            Psi = np.cumsum(dphi[::-1], axis=0)[::-1]
            out["dtheta"][b, :, g] += d[:, None] * Psi
            ddt += np.sum(theta[b, :, g] * Psi, axis=1)
            out["ddt"][b, :, h] = ddt
            out["dlam"][b, :, h] = dlam
            dBo, dCo = _rot(dBt, phi[:, None, :]), _rot(dCt, phi[:, None, :])
            if L and dpB is not None:
                dBo[L - 1] += dpB[b, h]
            if L and dpX is not None:
                dX[L - 1] += dpX[b, h]
            out["dB"][b, :, g] += dBo
            out["dC"][b, :, g] += dCo
            out["dx"][b, :, h] = dX
    return out


CASES = [  # (batch, L, H, G, P, N, R, Q, carries)
    (1, 7, 1, 1, 2, 4, 1, 3, False),
    (2, 13, 2, 1, 3, 6, 2, 4, False),
    (1, 16, 2, 2, 3, 8, 3, 5, True),
    (2, 21, 4, 2, 2, 4, 2, 8, True),
    (1, 1, 1, 1, 2, 4, 2, 4, True),
    (1, 9, 3, 3, 4, 6, 1, 9, True),
]


@pytest.mark.parametrize("case", CASES, ids=[f"L{c[1]}_R{c[6]}_Q{c[7]}_carry{int(c[8])}" for c in CASES])
def test_chunked_adjoint_equals_token_adjoint(case):
    nb, L, H, G, P, N, R, Q, carry = case
    rng = np.random.default_rng(1000 + L * 7 + Q)
    I = dict(x=rng.standard_normal((nb, L, H, R, P)), B=rng.standard_normal((nb, L, G, R, N)),
             C=rng.standard_normal((nb, L, G, R, N)), dt=np.log1p(np.exp(rng.standard_normal((nb, L, H)))),
             A=-np.exp(rng.uniform(-2, 1, size=H)), lam=1 / (1 + np.exp(-rng.standard_normal((nb, L, H)))),
             theta=rng.uniform(-np.pi, np.pi, size=(nb, L, G, N // 2)))
    dy = rng.standard_normal((nb, L, H, R, P))
    kw = {}
    if carry:
        kw = dict(init_h=rng.standard_normal((nb, H, N, P)), init_pB=rng.standard_normal((nb, H, R, N)),
                  init_pX=rng.standard_normal((nb, H, R, P)), dh=rng.standard_normal((nb, H, N, P)),
                  dpB=rng.standard_normal((nb, H, R, N)), dpX=rng.standard_normal((nb, H, R, P)))
    want = oracle.scan_bwd(**I, dy=dy, **kw)
    got = chunked_adjoint(**I, dy=dy, Q=Q, **kw)
    for k, v in want.items():
        err = np.linalg.norm(got[k] - v) / max(np.linalg.norm(v), 1e-300)
        assert err < 1e-11, f"{k}: relative error {err:.2e}"


def test_chunk_length_does_not_change_the_adjoint():
    """Q = 1 (every token its own chunk) and Q = L (one chunk) agree."""
    rng = np.random.default_rng(7)
    nb, L, H, G, P, N, R = 1, 12, 2, 1, 3, 6, 2
    I = dict(x=rng.standard_normal((nb, L, H, R, P)), B=rng.standard_normal((nb, L, G, R, N)),
             C=rng.standard_normal((nb, L, G, R, N)), dt=np.log1p(np.exp(rng.standard_normal((nb, L, H)))),
             A=-np.exp(rng.uniform(-2, 1, size=H)), lam=1 / (1 + np.exp(-rng.standard_normal((nb, L, H)))),
             theta=rng.uniform(-np.pi, np.pi, size=(nb, L, G, N // 2)))
    dy = rng.standard_normal((nb, L, H, R, P))
    one = chunked_adjoint(**I, dy=dy, Q=1)
    full = chunked_adjoint(**I, dy=dy, Q=L)
    for k in one:
        np.testing.assert_allclose(one[k], full[k], rtol=1e-11, atol=1e-12)
