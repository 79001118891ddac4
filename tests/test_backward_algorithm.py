"""CPU check that the decomposition the backward kernels use is the exact gradient.

The kernels never hold h_t and G_t = dL/dh_t at the same token. Per (batch, head) unit:
  forward sweep:  h_t = a_t h_{t-1} + b_t u_{t-1} + g_t u_t  (u_t = sum_r Bbar_t[r] x_t[r]^T)
                  gives dCbar_t[r] = h_t dy_t[r];
  reverse sweep:  G_t = sum_r Cbar_t[r] dy_t[r]^T + a_{t+1} G_{t+1} (G_{L-1} adds dL/dh_final)
                  gives du_t = g_t G_t + b_{t+1} G_{t+1}, dx_t[r] = du_t^T Bbar_t[r],
                  dBbar_t[r] = du_t x_t[r], db_t = <G_t, u_{t-1}>, dg_t = <G_t, u_t>, and the
                  angle adjoint: Phi_t rotates Bbar_t and Cbar_t, so it collects the pairwise
                  cross products dBbar x Bbar + dCbar x Cbar, summed from the end;
  decay:          the gradient of the log-decay dt_t A_t through the h_{t-1} term is the
                  suffix sum D_t = sum_{s >= t} (dy_s . y_s - b_s db_s - g_s dg_s)
                  + <dL/dh_final, h_final>, with dy_s . y_s = sum_r <Cbar_s[r], dCbar_s[r]>;
  then the chain rule through a = e^{dt A}, b = (1 - lam) dt a, g = lam dt (or the
  zero-order hold's b = 0, g = (a - 1) / A), the raw projections under the flags, the
  inverse rotation and the RMS-norm backward (heads of a group summed, the final state's
  prev_B gradient added after the norm).

Page references are to "Mamba-3: Improved Sequence Modeling using State Space Principles"
(Sec. 3.1.1 Prop. 1, Sec. 3.2.2 Prop. 4, Sec. 3.4). This file restates the decomposition
in numpy float64 and checks it against the gradient oracle (autograd of the plain
recurrence, itself pinned to finite differences of the C oracle).
"""
import math

import numpy as np
import pytest

import oracle
from oracle import grad as og


def rot_T(v, ph):
    h = v.shape[-1] // 2
    c, s = np.cos(ph), np.sin(ph)
    return np.concatenate([v[..., :h] * c + v[..., h:] * s, -v[..., :h] * s + v[..., h:] * c], -1)


def rot(v, ph):
    h = v.shape[-1] // 2
    c, s = np.cos(ph), np.sin(ph)
    return np.concatenate([v[..., :h] * c - v[..., h:] * s, v[..., :h] * s + v[..., h:] * c], -1)


def rms_scale(v, norm, eps):
    return 1.0 / np.sqrt((v * v).mean(-1, keepdims=True) + eps) if norm else np.ones_like(v[..., :1])


def norm_backward(v, dn, norm, eps):
    """Gradient with respect to raw v of v * s(v) + bias, given dn for the normalised value."""
    if not norm:
        return dn
    s = rms_scale(v, True, eps)
    return s * dn - (s ** 3 / v.shape[-1]) * v * (v * dn).sum(-1, keepdims=True)


def cross(dv, v):
    """sum_r (dv_re v_im - dv_im v_re) per pair: the derivative of <dv, R(Phi)^T w> in Phi."""
    h = v.shape[-1] // 2
    return (dv[..., :h] * v[..., h:] - dv[..., h:] * v[..., :h]).sum(0)


def decomposed_grad(p, st, dy, dfin, bc_norm, flags, eps=1e-6):
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
            Phi = st.phi[bi, h] + np.concatenate(
                [np.zeros((1, N // 2)), np.cumsum(d[:, None] * th[bi, :, h], 0)])  # Phi_{-1..L-1}
            Bbar = rot_T(B[bi, :, g] * rms_scale(B[bi, :, g], bc_norm, eps) + Bb[h], Phi[1:, None])
            Cbar = rot_T(C[bi, :, g] * rms_scale(C[bi, :, g], bc_norm, eps) + Cb[h], Phi[1:, None])
            pB = st.prev_B[bi, h]
            Bm1 = rot_T(pB * rms_scale(pB, bc_norm, eps) + Bb[h], Phi[0])
            xs, dys, xm1 = x[bi, :, h], dy[bi, :, h], st.prev_x[bi, h]
            u = lambda t: np.einsum("rn,rp->np", Bbar[t] if t >= 0 else Bm1, xs[t] if t >= 0 else xm1)
            # forward sweep
            hs = st.h[bi, h].copy()
            dCbar = np.zeros((L, R, N))
            for t in range(L):
                hs = al[t] * hs + be[t] * u(t - 1) + ga[t] * u(t)
                dCbar[t] = np.einsum("np,rp->rn", hs, dys[t])
            F = (dfin.h[bi, h] * hs).sum()
            # reverse sweep
            Gn = dfin.h[bi, h].copy()      # a_{t+1} G_{t+1} folded: start with dL/dh_final
            a_n, b_n = 1.0, 0.0
            db, dg, dyy, thd = (np.zeros(L) for _ in range(4))
            dPhi = dfin.phi[bi, h].copy()
            for t in range(L - 1, -1, -1):
                Gt = a_n * Gn + np.einsum("rn,rp->np", Cbar[t], dys[t])
                du = ga[t] * Gt + b_n * Gn
                out["dx"][bi, t, h] = np.einsum("np,rn->rp", du, Bbar[t])
                dBbar = np.einsum("np,rp->rn", du, xs[t])
                dg[t] = (Gt * u(t)).sum()
                db[t] = (Gt * u(t - 1)).sum()
                dPhi = dPhi + cross(dBbar, Bbar[t]) + cross(dCbar[t], Cbar[t])
                out["dtheta"][bi, t, h] = d[t] * dPhi
                thd[t] = (th[bi, t, h] * dPhi).sum()
                dyy[t] = (Cbar[t] * dCbar[t]).sum()
                dBn[bi, t, h] = rot(dBbar, Phi[t + 1])
                dCn[bi, t, h] = rot(dCbar[t], Phi[t + 1])
                Gn, a_n, b_n = Gt, al[t], be[t]
            out["dx"][bi, L - 1, h] += dfin.prev_x[bi, h]
            du = b_n * Gn                  # token -1: the stored previous token
            dinit.h[bi, h] = a_n * Gn
            dinit.prev_x[bi, h] = np.einsum("np,rn->rp", du, Bm1)
            dBm1 = np.einsum("np,rp->rn", du, xm1)
            dinit.phi[bi, h] = dPhi + cross(dBm1, Bm1)
            dprev_n[bi, h] = rot(dBm1, Phi[0])
            out["dB_bias"][h] += dBn[bi, :, h].sum(0) + dprev_n[bi, h]
            out["dC_bias"][h] += dCn[bi, :, h].sum(0)
            # decay suffix sum and the chain rule to the step scalars
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
    # RMS-norm backward of the heads' sum per group
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


@pytest.mark.parametrize("flags,bc_norm,R,G,H", [
    (0, True, 2, 1, 2), (0, False, 1, 2, 2), (3, True, 1, 1, 2), (4, True, 2, 1, 4),
    (7, True, 4, 2, 4),
])
def test_backward_decomposition_equals_gradient(flags, bc_norm, R, G, H):
    rng = np.random.default_rng(40 + flags + R)
    b, L, P, N = 2, 11, 3, 8
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
    got = decomposed_grad(p, st, dy, dfin, bc_norm, flags)
    for k in ("dx", "dB", "dC", "dtheta", "ddt", "dA", "dlam", "dB_bias", "dC_bias", "ddt_bias"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-10, atol=1e-10, err_msg=k)
    for f in ("h", "phi", "prev_B", "prev_x"):
        np.testing.assert_allclose(getattr(got["dinit"], f), getattr(ref["dinit"], f),
                                   rtol=1e-10, atol=1e-10, err_msg="init " + f)
