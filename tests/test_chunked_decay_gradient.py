"""CPU check (fp64) of the chunked backward's direct form of the decay gradient.

The gradient of the loss through the decay term of token t is D_t = <G_t, alpha_t h_{t-1}>,
where G_t = dL/dh_t. The sequential backward gets it as a suffix sum over the sequence of
dy.y - beta db - gamma dg, whose terms nearly cancel; the tensor-core backward instead forms it
per chunk from sums that do not cancel. With the chunk quantities of the forward's chunk mask
("Mamba-3: Improved Sequence Modeling using State Space Principles", Sec. 3.1.3 eq. 7:
cum = chunk-local inclusive sum of dt A, w_s = gamma_s + (1 - lam_{s+1}) dt_{s+1}), H0' the
primed state before the chunk and G_n the state adjoint at the next chunk's first token
(cx_T = cum_end + dt_n A_n; for the last chunk G_n = dL/dh_final, cx_T = cum_end):
    D_t = T1 + T2 + T3 + T4 - beta_t db_t,
    T1 = sum over s' < t <= s of e^{cum_s - cum_s'} w_s' (Cbar_s . Bbar_s') (dy_s . x_s'),
    T2 = sum_{s >= t} e^{cum_s} dy_s . (H0'^T Cbar_s),
    T3 = sum_{s' < t} w_s' e^{cx_T - cum_s'} <G_n, Bbar_s' x_s'^T>,
    T4 = e^{cx_T} <G_n, H0'>.
For MIMO (rank R) the rows are (token, rank) pairs: S' and Z run over rows, the crossing
pairs are rows of different tokens s' < t <= s, and u_t = sum_r Bbar_t[r] x_t[r]^T.
This file checks that form against D_t computed token by token from the plain recurrence and
its adjoint, for several chunk sizes, ranks 1, 2 and 4, ragged ends and both
discretisations, and that the per-token values the kernel hands to the scalar step
(D'_t - D_{t+1} + gamma_t dg_t) give back D_t through that step's suffix sum.
"""
import math

import numpy as np
import pytest

from test_backward_algorithm import rot_T


def problem(rng, L, N, P, zoh, R=1):
    d = np.log1p(np.exp(rng.standard_normal(L) - 1.0))
    a_rate = -np.exp(rng.uniform(-1, 1, L))
    lam = rng.uniform(0.05, 0.95, L)
    al = np.exp(d * a_rate)
    if zoh:
        be = np.zeros(L)
        ga = np.expm1(d * a_rate) / a_rate
        c = np.zeros(L + 1)
    else:
        be = (1 - lam) * d * al
        ga = lam * d
        c = np.zeros(L + 1)
        c[:L] = (1 - lam) * d
    theta = rng.uniform(-math.pi, math.pi, (L, N // 2))
    phi0 = rng.uniform(-math.pi, math.pi, N // 2)
    Phi = phi0 + np.cumsum(d[:, None] * theta, 0)
    Bn = rng.standard_normal((L, R, N))
    Cn = rng.standard_normal((L, R, N))
    Bbar = rot_T(Bn, Phi[:, None])
    Cbar = rot_T(Cn, Phi[:, None])
    Bm1 = rot_T(rng.standard_normal((R, N)), phi0)
    x = rng.standard_normal((L, R, P))
    xm1 = rng.standard_normal((R, P))
    dy = rng.standard_normal((L, R, P))
    h0 = rng.standard_normal((N, P))
    dh1 = rng.standard_normal((N, P))
    return dict(d=d, a=d * a_rate, al=al, be=be, ga=ga, c=c, w=ga + c[1:], Bbar=Bbar,
                Cbar=Cbar, Bm1=Bm1, x=x, xm1=xm1, dy=dy, h0=h0, dh1=dh1)


def sequential(q):
    """h_t, G_t, D_t = alpha_t <G_t, h_{t-1}>, db_t, dg_t and <dh1, h_final>, token by token."""
    L = len(q["d"])
    u = [np.einsum("rn,rp->np", q["Bbar"][t], q["x"][t]) for t in range(L)]
    um1 = np.einsum("rn,rp->np", q["Bm1"], q["xm1"])
    h, prev, uprev = [], q["h0"], um1
    for t in range(L):
        cur = q["al"][t] * prev + q["be"][t] * uprev + q["ga"][t] * u[t]
        h.append(cur)
        prev, uprev = cur, u[t]
    G = [None] * L
    nxt = q["dh1"]
    for t in range(L - 1, -1, -1):
        G[t] = np.einsum("rn,rp->np", q["Cbar"][t], q["dy"][t]) + nxt
        nxt = q["al"][t] * G[t]
    hm = [q["h0"]] + h[:-1]
    um = [um1] + u[:-1]
    D = np.array([q["al"][t] * (G[t] * hm[t]).sum() for t in range(L)])
    db = np.array([(G[t] * um[t]).sum() for t in range(L)])
    dg = np.array([(G[t] * u[t]).sum() for t in range(L)])
    return h, G, D, db, dg, (q["dh1"] * h[-1]).sum()


def chunked_D(q, Q, h, G):
    """D'_t = T1 + T2 + T3 + T4 per chunk, from the chunk-start primed state and G_n only."""
    L = len(q["d"])
    Dp = np.zeros(L)
    for t0 in range(0, L, Q):
        t1 = min(t0 + Q, L)
        T = t1 - t0
        cum = np.cumsum(q["a"][t0:t1])
        if t1 < L:
            cxT, Gn = cum[-1] + q["a"][t1], G[t1]
        else:
            cxT, Gn = cum[-1], q["dh1"]
        hprev = h[t0 - 1] if t0 > 0 else q["h0"]
        uprev = (np.einsum("rn,rp->np", q["Bbar"][t0 - 1], q["x"][t0 - 1]) if t0 > 0
                 else np.einsum("rn,rp->np", q["Bm1"], q["xm1"]))
        H0 = hprev + q["c"][t0] * uprev                       # primed state before the chunk
        R = q["x"].shape[1]
        rows = lambda k: q[k][t0:t1].reshape(T * R, -1)      # row = token * R + rank
        B, C, X, dY = rows("Bbar"), rows("Cbar"), rows("x"), rows("dy")
        w = q["w"][t0:t1]
        tok = np.arange(T * R) // R
        S = B @ C.T                                           # S'[i, j] = Bbar_i . Cbar_j
        Z = X @ dY.T                                          # Z[i, j] = x_i . dy_j
        Acr = np.where(tok[:, None] < tok[None, :],
                       np.exp(cum[tok][None, :] - cum[tok][:, None]) * w[tok][:, None] * S * Z, 0.0)
        v = np.exp(cum[tok]) * np.einsum("jp,np,jn->j", dY, H0, C)
        qv = np.einsum("in,np,ip->i", B, Gn, X)
        T4 = math.exp(cxT) * (Gn * H0).sum()
        for t in range(T):
            before, after = tok < t, tok >= t
            T1 = Acr[np.ix_(before, after)].sum()
            T2 = v[after].sum()
            T3 = (w[tok] * np.exp(cxT - cum[tok]) * qv)[before].sum()
            Dp[t0 + t] = T1 + T2 + T3 + T4
    return Dp


@pytest.mark.parametrize("R", [1, 2, 4])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("Q", [1, 4, 5, 16])
def test_direct_chunk_form_of_the_decay_gradient(Q, zoh, R):
    rng = np.random.default_rng(90 + Q + 7 * zoh + 31 * R)
    L, N, P = 13, 8, 3
    q = problem(rng, L, N, P, zoh, R)
    h, G, D, db, dg, F = sequential(q)
    Dp = chunked_D(q, Q, h, G)
    np.testing.assert_allclose(Dp - q["be"] * db, D, rtol=1e-10, atol=1e-10)
    # the values handed to the scalar step give D back through its suffix sum
    Dn = np.append(D[1:], F)
    slot2 = Dp - Dn + q["ga"] * dg
    back = np.cumsum((slot2 - q["be"] * db - q["ga"] * dg)[::-1])[::-1] + F
    np.testing.assert_allclose(back, D, rtol=1e-10, atol=1e-10)


def test_rectangle_sums_as_prefix_of_row_minus_column_sums():
    """T1_t = sum_{k < t} (row k's sum right of the diagonal - column k's sum above it)."""
    rng = np.random.default_rng(3)
    T = 9
    A = np.triu(rng.standard_normal((T, T)), 1)
    ru, cu = A.sum(1), A.sum(0)
    pref = np.concatenate([[0.0], np.cumsum(ru - cu)[:-1]])
    want = np.array([A[:t, t:].sum() for t in range(T)])
    np.testing.assert_allclose(pref, want, rtol=1e-12, atol=1e-12)
