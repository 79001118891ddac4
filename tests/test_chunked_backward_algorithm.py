"""CPU check of the chunked (parallel-in-time) form of the backward pass.

The backward kernels run two sequential sweeps. The chunked form computes the same gradients
with per-chunk dense products and a recurrence over chunks only. Here M is the forward
scan's chunk mask, the L1 . L2 mask of "Mamba-3: Improved Sequence Modeling using State
Space Principles", Sec. 3.1.3 eq. 7: M[t,s] = e^{cum_t - cum_s} w_s for s < t, gamma_t on
the diagonal, where w_s = gamma_s + (1 - lam_{s+1}) dt_{s+1}. It is one row per (token, rank)
and is expanded by full R x R blocks for MIMO. cum is the chunk-local inclusive sum of dt A.
H0' is the primed state before the chunk.
    dCbar = (M o dY X^T) Bbar + diag(e^{cum}) dY H0'^T                  (h_t dy_t, all t)
    dx    = (M^T o Bbar Cbar^T) dY + diag(w e^{cum_end - cum}) Bbar E      (du_t^T Bbar_t)
    dBbar = (M^T o X dY^T) Cbar + diag(w e^{cum_end - cum}) X E^T          (du_t x_t)
    dg_t, db_t = row sums of (F o Bbar Cbar^T o X dY^T) + their E terms, with F[t,s] =
                 e^{cum_s - cum_t} (s >= t), and Bbar, X of the previous token for db
    E_before = e^{cum_end} E + Cbar^T diag(e^{cum}) dY      (adjoint entering the chunk before)
    H0'_next = e^{cum_end} H0' + Bbar^T diag(e^{cum_end - cum} w) X
Here E is the adjoint entering the chunk's last token from the future, a_{t+1} G_{t+1}; for
the last chunk it is the final state's gradient. The rest is per token and the same as in the
sequential form: the angle adjoint, the decay suffix sum, the chain rule and the norm
backward. These products are the tensor-core work of a chunked backward kernel. This file
checks them against the gradient oracle for several chunk sizes, ragged ends included.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import grad as og
from test_backward_algorithm import cross, norm_backward, rms_scale, rot, rot_T


def chunked_grad(p, st, dy, dfin, bc_norm, flags, Q, eps=1e-6):
    x, B, C, th = p["x"], p["B"], p["C"], p["theta"]
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[-1]
    dt, lam = oracle.step_scalars(p["dt"], p["lam"], p.get("dt_bias"), flags)
    A, Bb, Cb = p["A"], p["B_bias"], p["C_bias"]
    zoh = bool(flags & oracle.DISC_ZOH)
    out = dict(dx=np.zeros_like(x), dtheta=np.zeros_like(th), ddt=np.zeros((b, L, H)),
               dA=np.zeros((b, L, H)), dlam=np.zeros((b, L, H)), dB_bias=np.zeros_like(Bb),
               dC_bias=np.zeros_like(Cb), ddt_bias=np.zeros(H))
    dBn = np.zeros((b, L, H, R, N))
    dCn = np.zeros((b, L, H, R, N))
    dinit = oracle.State.zeros(b, H, N, P, R)
    dprev_n = np.zeros((b, H, R, N))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            d, a_rate, l = dt[bi, :, h], A[bi, :, h], lam[bi, :, h]
            al = np.exp(d * a_rate)
            be = np.zeros(L) if zoh else (1 - l) * d * al
            ga = np.expm1(d * a_rate) / a_rate if zoh else l * d
            c = np.zeros(L + 1)                 # c_t = beta_t / alpha_t, c_L = 0
            c[:L] = 0.0 if zoh else (1 - l) * d
            w = ga + c[1:]
            Phi = st.phi[bi, h] + np.concatenate(
                [np.zeros((1, N // 2)), np.cumsum(d[:, None] * th[bi, :, h], 0)])
            Bbar = rot_T(B[bi, :, g] * rms_scale(B[bi, :, g], bc_norm, eps) + Bb[h], Phi[1:, None])
            Cbar = rot_T(C[bi, :, g] * rms_scale(C[bi, :, g], bc_norm, eps) + Cb[h], Phi[1:, None])
            pB = st.prev_B[bi, h]
            Bm1 = rot_T(pB * rms_scale(pB, bc_norm, eps) + Bb[h], Phi[0])
            xs, dys, xm1 = x[bi, :, h], dy[bi, :, h], st.prev_x[bi, h]
            chunks = [(t0, min(t0 + Q, L)) for t0 in range(0, L, Q)]

            def rows(a, t0, t1):                # [T, R, D] -> [T*R, D], row = t * R + r
                return a[t0:t1].reshape((t1 - t0) * R, -1)

            def prev_rows(a, am1, t0, t1):      # the previous token's rows
                first = am1[None] if t0 == 0 else a[t0 - 1:t0]
                return np.concatenate([first, a[t0:t1 - 1]]).reshape((t1 - t0) * R, -1)

            # forward: primed chunk-start states, then dCbar per chunk
            H0 = st.h[bi, h] + c[0] * np.einsum("rn,rp->np", Bm1, xm1)
            dCbar = np.zeros((L, R, N))
            for t0, t1 in chunks:
                cum = np.cumsum(d[t0:t1] * a_rate[t0:t1])
                T = t1 - t0
                tt = np.arange(T)
                Mt = np.where(tt[:, None] > tt[None, :], np.exp(cum[:, None] - cum[None, :]) * w[t0:t1][None, :], 0.0)
                Mt[tt, tt] = ga[t0:t1]
                Mf = np.kron(Mt, np.ones((R, R)))
                Xf, dYf, Bf = rows(xs, t0, t1), rows(dys, t0, t1), rows(Bbar, t0, t1)
                ecum = np.repeat(np.exp(cum), R)[:, None]
                dCbar[t0:t1] = ((Mf * (dYf @ Xf.T)) @ Bf + ecum * (dYf @ H0.T)).reshape(T, R, N)
                wend = np.repeat(np.exp(cum[-1] - cum) * w[t0:t1], R)[:, None]
                H0 = np.exp(cum[-1]) * H0 + Bf.T @ (wend * Xf)
            # the final state h_{L-1} = H0'_L - c_L u_{L-1} with c_L = 0
            F = (dfin.h[bi, h] * H0).sum()
            # reverse over chunks
            E = dfin.h[bi, h].copy()
            dx = np.zeros((L, R, P))
            dBbar = np.zeros((L, R, N))
            dg = np.zeros(L)
            db = np.zeros(L)
            for t0, t1 in reversed(chunks):
                cum = np.cumsum(d[t0:t1] * a_rate[t0:t1])
                T = t1 - t0
                tt = np.arange(T)
                Mt = np.where(tt[:, None] > tt[None, :], np.exp(cum[:, None] - cum[None, :]) * w[t0:t1][None, :], 0.0)
                Mt[tt, tt] = ga[t0:t1]
                Ft = np.where(tt[None, :] >= tt[:, None], np.exp(cum[None, :] - cum[:, None]), 0.0)
                Mf, Ff = np.kron(Mt, np.ones((R, R))), np.kron(Ft, np.ones((R, R)))
                Xf, dYf = rows(xs, t0, t1), rows(dys, t0, t1)
                Bf, Cf = rows(Bbar, t0, t1), rows(Cbar, t0, t1)
                Bp, Xp = prev_rows(Bbar, Bm1, t0, t1), prev_rows(xs, xm1, t0, t1)
                wend = np.repeat(w[t0:t1] * np.exp(cum[-1] - cum), R)[:, None]
                eend = np.repeat(np.exp(cum[-1] - cum), R)[:, None]
                dx[t0:t1] = ((Mf.T * (Bf @ Cf.T)) @ dYf + wend * (Bf @ E)).reshape(T, R, P)
                dBbar[t0:t1] = ((Mf.T * (Xf @ dYf.T)) @ Cf + wend * (Xf @ E.T)).reshape(T, R, N)
                g_rows = (Ff * (Bf @ Cf.T) * (Xf @ dYf.T)).sum(1) + eend[:, 0] * ((Bf @ E) * Xf).sum(1)
                b_rows = (Ff * (Bp @ Cf.T) * (Xp @ dYf.T)).sum(1) + eend[:, 0] * ((Bp @ E) * Xp).sum(1)
                dg[t0:t1] = g_rows.reshape(T, R).sum(1)
                db[t0:t1] = b_rows.reshape(T, R).sum(1)
                ecum = np.repeat(np.exp(cum), R)[:, None]
                E = np.exp(cum[-1]) * E + Cf.T @ (ecum * dYf)
            # E is now a_0 G_0: the initial state's h gradient; the stored token's du = c_0 E
            out["dx"][bi, :, h] = dx
            out["dx"][bi, L - 1, h] += dfin.prev_x[bi, h]
            dinit.h[bi, h] = E
            du = c[0] * E
            dinit.prev_x[bi, h] = np.einsum("np,rn->rp", du, Bm1)
            dBm1 = np.einsum("np,rp->rn", du, xm1)
            # per token: angle adjoint from the end, rotation back, decay suffix sum
            dPhi = dfin.phi[bi, h].copy()
            thd, dyy = np.zeros(L), np.zeros(L)
            for t in range(L - 1, -1, -1):
                dPhi = dPhi + cross(dBbar[t], Bbar[t]) + cross(dCbar[t], Cbar[t])
                out["dtheta"][bi, t, h] = d[t] * dPhi
                thd[t] = (th[bi, t, h] * dPhi).sum()
                dyy[t] = (Cbar[t] * dCbar[t]).sum()
                dBn[bi, t, h] = rot(dBbar[t], Phi[t + 1])
                dCn[bi, t, h] = rot(dCbar[t], Phi[t + 1])
            dinit.phi[bi, h] = dPhi + cross(dBm1, Bm1)
            dprev_n[bi, h] = rot(dBm1, Phi[0])
            out["dB_bias"][h] += dBn[bi, :, h].sum(0) + dprev_n[bi, h]
            out["dC_bias"][h] += dCn[bi, :, h].sum(0)
            D = np.cumsum((dyy - be * db - ga * dg)[::-1])[::-1] + F
            if zoh:
                ddt = D * a_rate + dg * al + thd
                dA = D * d + dg * (d * al - ga) / a_rate
                dl = np.zeros(L)
            else:
                ddt = D * a_rate + db * (1 - l) * al * (1 + d * a_rate) + dg * l + thd
                dA = D * d + db * (1 - l) * d * d * al
                dl = (dg - db * al) * d
            if flags & oracle.DT_SOFTPLUS:
                ddt = ddt / (1 + np.exp(-(p["dt"][bi, :, h] + p["dt_bias"][h])))
                out["ddt_bias"][h] += ddt.sum()
            if flags & oracle.LAM_SIGMOID:
                dl = dl * l * (1 - l)
            out["ddt"][bi, :, h], out["dA"][bi, :, h], out["dlam"][bi, :, h] = ddt, dA, dl
    heads = [np.arange(H)[np.arange(H) // (H // G) == g] for g in range(G)]
    out["dB"] = np.stack([norm_backward(B[:, :, g], dBn[:, :, hs].sum(2), bc_norm, eps)
                          for g, hs in enumerate(heads)], 2)
    out["dC"] = np.stack([norm_backward(C[:, :, g], dCn[:, :, hs].sum(2), bc_norm, eps)
                          for g, hs in enumerate(heads)], 2)
    for g, hs in enumerate(heads):
        out["dB"][:, L - 1, g] += dfin.prev_B[:, hs].sum(1)
    dinit.prev_B[:] = norm_backward(st.prev_B, dprev_n, bc_norm, eps)
    out["dinit"] = dinit
    return out


@pytest.mark.parametrize("Q", [1, 4, 5, 16])
@pytest.mark.parametrize("flags,bc_norm,R,G,H", [
    (0, True, 1, 1, 2), (0, True, 2, 1, 2), (7, True, 4, 2, 4), (4, False, 1, 2, 2),
])
def test_chunked_backward_equals_gradient(Q, flags, bc_norm, R, G, H):
    rng = np.random.default_rng(60 + Q + flags + R)
    b, L, P, N = 2, 13, 3, 8
    p = dict(x=rng.standard_normal((b, L, H, R, P)), B=rng.standard_normal((b, L, G, R, N)),
             C=rng.standard_normal((b, L, G, R, N)),
             theta=rng.uniform(-math.pi, math.pi, (b, L, H, N // 2)),
             dt=(rng.standard_normal((b, L, H)) - 1.0) if flags & 1
             else np.log1p(np.exp(rng.standard_normal((b, L, H)) - 1.0)),
             A=-np.exp(rng.uniform(-1, 1, (b, L, H))),
             lam=rng.standard_normal((b, L, H)) if flags & 2 else rng.uniform(0.05, 0.95, (b, L, H)),
             B_bias=rng.standard_normal((H, R, N)) * 0.3, C_bias=rng.standard_normal((H, R, N)) * 0.3)
    if flags & 1:
        p["dt_bias"] = rng.standard_normal(H) * 0.5
    st = oracle.State(rng.standard_normal((b, H, N, P)), rng.uniform(-math.pi, math.pi, (b, H, N // 2)),
                      rng.standard_normal((b, H, R, N)), rng.standard_normal((b, H, R, P)))
    dy = rng.standard_normal((b, L, H, R, P))
    dfin = oracle.State(rng.standard_normal((b, H, N, P)), rng.standard_normal((b, H, N // 2)),
                        rng.standard_normal((b, H, R, N)), rng.standard_normal((b, H, R, P)))
    ref = og.scan_grad(p["x"], p["B"], p["C"], p["theta"], p["dt"], p["A"], p["lam"], p["B_bias"],
                       p["C_bias"], st, dy, dfin, bc_norm=bc_norm, dt_bias=p.get("dt_bias"),
                       flags=flags)
    got = chunked_grad(p, st, dy, dfin, bc_norm, flags, Q)
    for k in ("dx", "dB", "dC", "dtheta", "ddt", "dA", "dlam", "dB_bias", "dC_bias", "ddt_bias"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-9, atol=1e-9, err_msg=k)
    for f in ("h", "phi", "prev_B", "prev_x"):
        np.testing.assert_allclose(getattr(got["dinit"], f), getattr(ref["dinit"], f),
                                   rtol=1e-9, atol=1e-9, err_msg="init " + f)
