"""Gradient of the Mamba-3 SSM core scan in float64: reverse-mode differentiation of a plain
token-by-token recurrence.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this module; the library never does, and nothing here comes from
the library.

``scan_torch`` is the forward of "Mamba-3: Improved Sequence Modeling using State Space
Principles" (Sec. 3.1.1 Prop. 1: exponential-trapezoidal update; Sec. 3.2.2 Prop. 4:
rotated B and C; Sec. 3.4: BC norm and bias; Appendix C and Remark 6: rank-R MIMO) written
a second time, in torch float64 ops so that it can be differentiated: vectorised over
(batch, head), one token per loop iteration, no chunking. ``scan_grad`` is torch.autograd of
it for a given output gradient dy and final-state gradient.

Pins (tests/test_oracle_pins.py): the forward equals the C oracle's (``m3_oracle.c``), and
every gradient equals central finite differences of the C oracle, element by element, on
small cases with every option switched on.
"""
from __future__ import annotations

import numpy as np
import torch

from . import DISC_ZOH, DT_SOFTPLUS, LAM_SIGMOID, State


def _t(a, like=None):
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        return a.detach().to("cpu", torch.float64).clone()
    return torch.as_tensor(np.asarray(a, dtype=np.float64)).clone()


def _norm_bias(v, bias, bc_norm, eps):
    """RMS norm over the last axis (no learnable weight), then the bias (Sec. 3.4)."""
    if bc_norm:
        v = v * torch.rsqrt((v * v).mean(-1, keepdim=True) + eps)
    return v if bias is None else v + bias


def _rot_T(v, phi):
    """R(phi)^T v with pair i = (i, i + N/2): (u, w) -> (u cos + w sin, -u sin + w cos)."""
    half = v.shape[-1] // 2
    u, w = v[..., :half], v[..., half:]
    c, s = torch.cos(phi).unsqueeze(-2), torch.sin(phi).unsqueeze(-2)
    return torch.cat([u * c + w * s, -u * s + w * c], dim=-1)


def scan_torch(x, B, C, theta, dt, A, lam, B_bias=None, C_bias=None, h0=None, phi0=None,
               prev_B0=None, prev_x0=None, bc_norm=False, eps=1e-6, dt_bias=None, flags=0):
    """The recurrence over a whole sequence on float64 torch tensors (differentiable).

    Shapes as in ``oracle.scan``; the initial state fields default to zero. Returns
    (y [b,L,H,R,P], h [b,H,N,P], phi [b,H,N/2], prev_B [b,H,R,N], prev_x [b,H,R,P])."""
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[-1]
    heads = torch.arange(H) // (H // G)
    Bh, Ch = B[:, :, heads], C[:, :, heads]                    # per head [b,L,H,R,N]
    if flags & DT_SOFTPLUS:                                    # softplus(d + bias)
        v = dt if dt_bias is None else dt + dt_bias
        dt = torch.logaddexp(v, torch.zeros_like(v))
    if flags & LAM_SIGMOID:
        lam = torch.sigmoid(lam)
    z = torch.zeros
    h = z(b, H, N, P, dtype=x.dtype) if h0 is None else h0
    phi = z(b, H, N // 2, dtype=x.dtype) if phi0 is None else phi0
    Bp = z(b, H, R, N, dtype=x.dtype) if prev_B0 is None else prev_B0
    xp = z(b, H, R, P, dtype=x.dtype) if prev_x0 is None else prev_x0
    ys = []
    for t in range(L):
        d, a_rate, l = dt[:, t], A[:, t], lam[:, t]            # [b,H]
        alpha = torch.exp(d * a_rate)
        if flags & DISC_ZOH:                                   # Mamba-1/2 zero-order hold
            beta = torch.zeros_like(alpha)
            gamma = torch.expm1(d * a_rate) / a_rate
        else:                                                  # Prop. 1
            beta = (1.0 - l) * d * alpha
            gamma = l * d
        phi_prev = phi
        phi = phi + d.unsqueeze(-1) * theta[:, t]
        Bbar = _rot_T(_norm_bias(Bh[:, t], B_bias, bc_norm, eps), phi)
        Cbar = _rot_T(_norm_bias(Ch[:, t], C_bias, bc_norm, eps), phi)
        Bpbar = _rot_T(_norm_bias(Bp, B_bias, bc_norm, eps), phi_prev)
        u_prev = torch.einsum("bhrn,bhrp->bhnp", Bpbar, xp)
        u_cur = torch.einsum("bhrn,bhrp->bhnp", Bbar, x[:, t])
        h = (alpha[..., None, None] * h + beta[..., None, None] * u_prev
             + gamma[..., None, None] * u_cur)
        ys.append(torch.einsum("bhnp,bhrn->bhrp", h, Cbar))
        Bp, xp = Bh[:, t], x[:, t]
    y = torch.stack(ys, 1) if ys else z(b, 0, H, R, P, dtype=x.dtype)
    return y, h, phi, Bp, xp


def scan_grad(x, B, C, theta, dt, A, lam, B_bias=None, C_bias=None, state: State | None = None,
              dy=None, dfinal: State | None = None, bc_norm=False, norm_eps=1e-6,
              dt_bias=None, flags=0):
    """Gradients of  sum(y * dy) + <final state, dfinal>  with respect to every input.

    ``dy`` [b,L,H,R,P] (None = 0); ``dfinal`` a State of the final state's gradients (None or
    any field None = 0). Returns a dict of float64 numpy arrays: dx, dB, dC, dtheta, ddt, dA,
    dlam (with respect to what was passed: the raw projections under the flags), dB_bias,
    dC_bias [H,R,N], ddt_bias [H], and dinit, a State of the initial state's gradients."""
    x, B, C, theta = _t(x), _t(B), _t(C), _t(theta)
    dt, A, lam = _t(dt), _t(A), _t(lam)
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[-1]
    Bb = torch.zeros(H, R, N, dtype=torch.float64) if B_bias is None else _t(B_bias)
    Cb = torch.zeros(H, R, N, dtype=torch.float64) if C_bias is None else _t(C_bias)
    db = torch.zeros(H, dtype=torch.float64) if dt_bias is None else _t(dt_bias)
    st = State.zeros(b, H, N, P, R) if state is None else state
    init = [_t(st.h), _t(st.phi), _t(st.prev_B), _t(st.prev_x)]
    leaves = [x, B, C, theta, dt, A, lam, Bb, Cb, db] + init
    for v in leaves:
        v.requires_grad_(True)
    with torch.enable_grad():
        y, h, phi, Bp, xp = scan_torch(x, B, C, theta, dt, A, lam, Bb, Cb, *init,
                                       bc_norm=bc_norm, eps=norm_eps, dt_bias=db, flags=flags)
        outs = [y, h, phi, Bp, xp]
        dfs = [None, None, None, None] if dfinal is None else [
            dfinal.h, dfinal.phi, dfinal.prev_B, dfinal.prev_x]
        gouts = [torch.zeros_like(y) if dy is None else _t(dy)]
        gouts += [torch.zeros_like(o) if g is None else _t(g) for o, g in zip(outs[1:], dfs)]
        loss = sum((o * g).sum() for o, g in zip(outs, gouts))
        grads = torch.autograd.grad(loss, leaves, allow_unused=True)
    g = [torch.zeros_like(v) if gv is None else gv for v, gv in zip(leaves, grads)]
    n = [t.detach().numpy() for t in g]
    return dict(dx=n[0], dB=n[1], dC=n[2], dtheta=n[3], ddt=n[4], dA=n[5], dlam=n[6],
                dB_bias=n[7], dC_bias=n[8], ddt_bias=n[9],
                dinit=State(n[10], n[11], n[12], n[13]))
