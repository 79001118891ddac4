"""CPU brute-force check that the chunked re-association the CUDA kernels use is exact.

The kernels never run the token loop. They carry a "primed" state between chunks,
    h'_t = h~_t + (1 - lam_{t+1}) dt_{t+1} v_t,   v_t = sum_r Bbar_t[r] x_t[r]^T,
which folds the trapezoid's pending beta term into the state, so that
    h'_t = alpha_t h'_{t-1} + w_t v_t,   w_t = gamma_t + (1 - lam_{t+1}) dt_{t+1}
(w_{L-1} = gamma_{L-1}), and
    y_t  = Cbar_t^T (alpha_t h'_{t-1} + gamma_t v_t).
Within a chunk this is the SSD form Y = (Cbar Bbar^T o M) X + diag(e^{cum}) Cbar H0 with
M[t,s] = e^{cum_t - cum_s} w_s (s < t), gamma_t (s = t) (the L1 . L2 mask of Sec. 3.1.3
eq. 7, one row per token, expanded by a full R x R block for MIMO), and the chunk-end
state H1 = e^{cum_end} H0 + Bbar^T diag(e^{cum_end - cum_s} w_s) X.

A sequence that starts from a stored state (h~, Phi, prev_B, prev_x) starts from
h'_{-1} = h~_{-1} + (1 - lam_0) dt_0 Bbar_{-1} x_{-1}^T. This file checks the whole scheme
against the sequential oracle for many chunk sizes and ragged lengths.
"""
import math

import numpy as np
import pytest

import oracle
from test_oracle_pins import rand_state, rnd_problem, normed


def rot_T(v, phi):
    half = v.shape[-1] // 2
    c, s = np.cos(phi), np.sin(phi)
    u, w = v[..., :half], v[..., half:]
    return np.concatenate([u * c + w * s, -u * s + w * c], -1)


def chunked(p, Q, state=None):
    x, B, C, th, dt, A, lm = (p[k] for k in ("x", "B", "C", "theta", "dt", "A", "lam"))
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    y = np.zeros_like(x)
    hs = np.zeros((b, H, N, P))
    phis = np.zeros((b, H, N // 2))
    for bb in range(b):
        for hh in range(H):
            g = hh // (H // G)
            Bb = None if p["B_bias"] is None else p["B_bias"][hh]
            Cb = None if p["C_bias"] is None else p["C_bias"][hh]
            if state is None:
                Hc = np.zeros((N, P))
                phi0 = np.zeros(N // 2)
            else:
                phi0 = state.phi[bb, hh]
                Hc = state.h[bb, hh].copy()
                if L > 0:
                    bp = rot_T(normed(state.prev_B[bb, hh], Bb, p["bc_norm"]), phi0)
                    Hc += (1 - lm[bb, 0, hh]) * dt[bb, 0, hh] * bp.T @ state.prev_x[bb, hh]
            phi_run = phi0.copy()
            for c0 in range(0, L, Q):
                c1 = min(L, c0 + Q)
                T = c1 - c0
                d, a, l = dt[bb, c0:c1, hh], A[bb, c0:c1, hh], lm[bb, c0:c1, hh]
                cum = np.cumsum(d * a)
                gam = l * d
                w = gam.copy()
                nxt = (1 - lm[bb, c0 + 1:c1 + 1, hh]) * dt[bb, c0 + 1:c1 + 1, hh]
                w[:len(nxt)] += nxt                      # last token of the sequence: w = gamma
                phi = phi_run + np.cumsum(d[:, None] * th[bb, c0:c1, hh], 0)
                phi_run = phi[-1]
                Bbar = rot_T(normed(B[bb, c0:c1, g], Bb, p["bc_norm"]), phi[:, None, :])
                Cbar = rot_T(normed(C[bb, c0:c1, g], Cb, p["bc_norm"]), phi[:, None, :])
                Bf, Cf = Bbar.reshape(T * R, N), Cbar.reshape(T * R, N)
                X = x[bb, c0:c1, hh].reshape(T * R, P)
                M = np.zeros((T, T))
                for t in range(T):
                    for s in range(t):
                        M[t, s] = math.exp(cum[t] - cum[s]) * w[s]
                    M[t, t] = gam[t]
                Mx = np.kron(M, np.ones((R, R)))
                Yd = ((Cf @ Bf.T) * Mx) @ X
                Yo = np.repeat(np.exp(cum), R)[:, None] * (Cf @ Hc)
                y[bb, c0:c1, hh] = (Yd + Yo).reshape(T, R, P)
                dw = np.repeat(np.exp(cum[-1] - cum) * w, R)
                Hc = math.exp(cum[-1]) * Hc + Bf.T @ (dw[:, None] * X)
            hs[bb, hh] = Hc
            phis[bb, hh] = phi_run
    return y, hs, phis


@pytest.mark.parametrize("Q", [1, 2, 4, 8, 16, 64])
@pytest.mark.parametrize("L", [1, 7, 64, 65])
@pytest.mark.parametrize("R", [1, 2])
@pytest.mark.parametrize("with_state", [False, True])
def test_chunked_equals_sequential(Q, L, R, with_state):
    rng = np.random.default_rng(100 + Q + L + 7 * R + with_state)
    p = rnd_problem(rng, b=1, L=L, H=2, R=R, N=8, P=4)
    st = rand_state(rng, 1, 2, 8, 4, R) if with_state else None
    y, fs = oracle.scan(p["x"], p["B"], p["C"], p["theta"], p["dt"], p["A"], p["lam"],
                        p["B_bias"], p["C_bias"], state=st, bc_norm=True)
    yc, hc, phic = chunked(p, Q, st)
    sc = np.max(np.abs(y))
    np.testing.assert_allclose(yc, y, atol=1e-10 * sc)
    np.testing.assert_allclose(hc, fs.h, atol=1e-10 * np.max(np.abs(fs.h)))
    np.testing.assert_allclose(phic, fs.phi, atol=1e-12)


# ------------------------------------------------------------------------------------------
# The 128-row-chunk kernel's form of the same step: scaled operands. With a reference r per
# chunk (the midpoint of its cumulative log-decay), Bbar rows are scaled by e^{r - cum_s} w_s
# and Cbar rows by e^{cum_t - r}; then (C' B'^T)[t, s] = Cbar_t Bbar_s^T e^{cum_t - cum_s} w_s
# is already the masked score below the diagonal, the diagonal takes gamma_t / w_t, and
#     Y  = P X + C' (e^{r} H0),       H1 = e^{cum_end - r} (e^{r} H0 + B'^T X).
# A chunk that decays by more than MAX_DECAY nats is computed exactly as `chunked` does.
# ------------------------------------------------------------------------------------------
MAX_DECAY = 60.0


def chunked_scaled(p, Q, state=None, max_decay=MAX_DECAY, modes=None):
    x, B, C, th, dt, A, lm = (p[k] for k in ("x", "B", "C", "theta", "dt", "A", "lam"))
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    y = np.zeros_like(x)
    hs = np.zeros((b, H, N, P))
    for bb in range(b):
        for hh in range(H):
            g = hh // (H // G)
            Bb = None if p["B_bias"] is None else p["B_bias"][hh]
            Cb = None if p["C_bias"] is None else p["C_bias"][hh]
            Hc = np.zeros((N, P)) if state is None else state.h[bb, hh].copy()
            phi_run = np.zeros(N // 2) if state is None else state.phi[bb, hh].copy()
            if state is not None and L > 0:
                bp = rot_T(normed(state.prev_B[bb, hh], Bb, p["bc_norm"]), phi_run)
                Hc += (1 - lm[bb, 0, hh]) * dt[bb, 0, hh] * bp.T @ state.prev_x[bb, hh]
            for c0 in range(0, L, Q):
                c1 = min(L, c0 + Q)
                T = c1 - c0
                d, a, l = dt[bb, c0:c1, hh], A[bb, c0:c1, hh], lm[bb, c0:c1, hh]
                cum = np.cumsum(d * a)
                gam = l * d
                w = gam.copy()
                nxt = (1 - lm[bb, c0 + 1:c1 + 1, hh]) * dt[bb, c0 + 1:c1 + 1, hh]
                w[:len(nxt)] += nxt
                phi = phi_run + np.cumsum(d[:, None] * th[bb, c0:c1, hh], 0)
                phi_run = phi[-1]
                Bf = rot_T(normed(B[bb, c0:c1, g], Bb, p["bc_norm"]), phi[:, None, :]).reshape(T * R, N)
                Cf = rot_T(normed(C[bb, c0:c1, g], Cb, p["bc_norm"]), phi[:, None, :]).reshape(T * R, N)
                X = x[bb, c0:c1, hh].reshape(T * R, P)
                rep = lambda v: np.repeat(v, R)
                if -cum[-1] <= max_decay:            # scaled operands
                    r = 0.5 * (cum[0] + cum[-1])
                    fb, fc = np.exp(r - cum) * w, np.exp(cum - r)
                    assert fb.max() <= math.exp(30.0) * max(w.max(), 1.0) and fc.max() <= math.exp(30.0)
                    Bs, Cs = rep(fb)[:, None] * Bf, rep(fc)[:, None] * Cf
                    S = Cs @ Bs.T
                    tok = np.arange(T * R) // R
                    Pm = np.where(tok[:, None] > tok[None, :], S, 0.0)
                    gw = np.where(w > 0, gam / np.where(w > 0, w, 1.0), 0.0)
                    Pm += np.where(tok[:, None] == tok[None, :], S * rep(gw)[:, None], 0.0)
                    y[bb, c0:c1, hh] = (Pm @ X + Cs @ (math.exp(r) * Hc)).reshape(T, R, P)
                    Hc = math.exp(cum[-1] - r) * (math.exp(r) * Hc + Bs.T @ X)
                    if modes is not None:
                        modes.append("scaled")
                else:                                  # exact: unit scales
                    M = np.zeros((T, T))
                    for t in range(T):
                        for s in range(t):
                            M[t, s] = math.exp(cum[t] - cum[s]) * w[s]
                        M[t, t] = gam[t]
                    Yd = ((Cf @ Bf.T) * np.kron(M, np.ones((R, R)))) @ X
                    y[bb, c0:c1, hh] = (Yd + rep(np.exp(cum))[:, None] * (Cf @ Hc)).reshape(T, R, P)
                    Hc = math.exp(cum[-1]) * Hc + Bf.T @ (rep(np.exp(cum[-1] - cum) * w)[:, None] * X)
                    if modes is not None:
                        modes.append("exact")
            hs[bb, hh] = Hc
    return y, hs


@pytest.mark.parametrize("R,Q", [(1, 128), (2, 64), (4, 32), (1, 16)])
@pytest.mark.parametrize("dt_shift", [-2.0, 0.0, 2.0])
@pytest.mark.parametrize("with_state", [False, True])
def test_scaled_operand_chunks_equal_sequential(R, Q, dt_shift, with_state):
    """Both forms of the 128-row-chunk kernel against the sequential oracle: weak decay (all
    chunks scaled), mixed, and strong decay (chunks of more than 60 nats computed exactly)."""
    rng = np.random.default_rng(300 + Q + 7 * R + int(10 * dt_shift) + with_state)
    L = 2 * Q + Q // 2 + 3
    p = rnd_problem(rng, b=1, L=L, H=2, R=R, N=8, P=4, dt_shift=dt_shift)
    st = rand_state(rng, 1, 2, 8, 4, R) if with_state else None
    y, fs = oracle.scan(p["x"], p["B"], p["C"], p["theta"], p["dt"], p["A"], p["lam"],
                        p["B_bias"], p["C_bias"], state=st, bc_norm=True)
    modes = []
    yc, hc = chunked_scaled(p, Q, st, modes=modes)
    np.testing.assert_allclose(yc, y, atol=1e-9 * np.max(np.abs(y)))
    np.testing.assert_allclose(hc, fs.h, atol=1e-9 * np.max(np.abs(fs.h)))
    if dt_shift <= -2.0:
        assert set(modes) == {"scaled"}
    if dt_shift >= 2.0 and Q >= 32:
        assert "exact" in modes


def test_scaled_and_exact_forms_agree_where_both_apply():
    """The same chunks through either form (threshold at infinity: always scaled; at -1: always
    exact) give the same outputs: the scaling is exact arithmetic, not an approximation."""
    rng = np.random.default_rng(333)
    p = rnd_problem(rng, b=1, L=150, H=2, R=2, N=8, P=4, dt_shift=-1.0)
    ys, hs_ = chunked_scaled(p, 64, max_decay=float("inf"))
    ye, he = chunked_scaled(p, 64, max_decay=-1.0)
    np.testing.assert_allclose(ys, ye, atol=1e-10 * np.max(np.abs(ye)))
    np.testing.assert_allclose(hs_, he, atol=1e-10 * np.max(np.abs(he)))
