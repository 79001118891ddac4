"""Pins of the gradient oracle (oracle/grad.py) to something other than itself.

1. Its differentiable forward is a second implementation of the recurrence: it must equal
   the C oracle (m3_oracle.c, pinned in test_oracle_pins.py) to rounding.
2. Every gradient it returns must equal the central finite difference of the C oracle's
   output, element by element, for every input and every field of the initial state, with
   the norm, the biases, MIMO rank, shared groups, a nonzero initial state and each flag
   (raw step and trapezoid scalars, zero-order hold) switched on. A dropped term, a wrong
   sign or a transposed operand anywhere in the backward fails here.
3. In the real Euler case (no rotation, lam = 1, no norm or bias) the gradients of x, C and
   A have closed forms as explicit sums over token pairs, checked without autograd or
   finite differences.

Page references are to "Mamba-3: Improved Sequence Modeling using State Space Principles".
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import grad as og


def problem(rng, b, L, H, G, P, N, R, flags=0):
    p = dict(
        x=rng.standard_normal((b, L, H, R, P)),
        B=rng.standard_normal((b, L, G, R, N)),
        C=rng.standard_normal((b, L, G, R, N)),
        theta=rng.uniform(-math.pi, math.pi, (b, L, H, N // 2)),
        dt=(rng.standard_normal((b, L, H)) - 1.0) if flags & oracle.DT_SOFTPLUS
        else np.log1p(np.exp(rng.standard_normal((b, L, H)) - 1.0)),
        A=-np.exp(rng.uniform(-1, 1, (b, L, H))),
        lam=rng.standard_normal((b, L, H)) if flags & oracle.LAM_SIGMOID
        else rng.uniform(0.05, 0.95, (b, L, H)),
        B_bias=rng.standard_normal((H, R, N)) * 0.3,
        C_bias=rng.standard_normal((H, R, N)) * 0.3,
    )
    if flags & oracle.DT_SOFTPLUS:
        p["dt_bias"] = rng.standard_normal(H) * 0.5
    state = oracle.State(rng.standard_normal((b, H, N, P)),
                         rng.uniform(-math.pi, math.pi, (b, H, N // 2)),
                         rng.standard_normal((b, H, R, N)),
                         rng.standard_normal((b, H, R, P)))
    return p, state


def c_forward(p, state, bc_norm, flags):
    return oracle.scan(p["x"], p["B"], p["C"], p["theta"], p["dt"], p["A"], p["lam"],
                       p["B_bias"], p["C_bias"], state, bc_norm=bc_norm, nthreads=1,
                       dt_bias=p.get("dt_bias"), flags=flags)


@pytest.mark.parametrize("flags", [0, 3, 4, 7])
@pytest.mark.parametrize("R,G", [(1, 1), (2, 2)])
@pytest.mark.parametrize("bc_norm", [False, True])
def test_torch_forward_equals_c_oracle(flags, R, G, bc_norm):
    rng = np.random.default_rng(10 + flags + 3 * R)
    p, state = problem(rng, b=2, L=13, H=4, G=G, P=3, N=8, R=R, flags=flags)
    y, st = c_forward(p, state, bc_norm, flags)
    T = {k: torch.as_tensor(v) for k, v in p.items()}
    yt, h, phi, pB, px = og.scan_torch(
        T["x"], T["B"], T["C"], T["theta"], T["dt"], T["A"], T["lam"], T["B_bias"],
        T["C_bias"], torch.as_tensor(state.h), torch.as_tensor(state.phi),
        torch.as_tensor(state.prev_B), torch.as_tensor(state.prev_x), bc_norm=bc_norm,
        dt_bias=T.get("dt_bias"), flags=flags)
    for a, b_ in [(yt, y), (h, st.h), (phi, st.phi), (pB, st.prev_B), (px, st.prev_x)]:
        np.testing.assert_allclose(a.numpy(), b_, rtol=1e-11, atol=1e-11)


def _objective(p, state, dy, dfin, bc_norm, flags):
    y, st = c_forward(p, state, bc_norm, flags)
    return (float((y * dy).sum()) + float((st.h * dfin.h).sum()) + float((st.phi * dfin.phi).sum())
            + float((st.prev_B * dfin.prev_B).sum()) + float((st.prev_x * dfin.prev_x).sum()))


@pytest.mark.parametrize("flags,bc_norm,R,G,H", [
    (0, True, 2, 1, 2),      # MIMO, one group shared by two heads, norm, biases
    (0, False, 1, 2, 2),     # SISO, no norm
    (3, True, 1, 1, 2),      # raw step (softplus + bias) and raw trapezoid weight (sigmoid)
    (4, True, 2, 1, 2),      # zero-order hold
])
def test_gradient_equals_finite_differences_of_c_oracle(flags, bc_norm, R, G, H):
    rng = np.random.default_rng(100 + flags + R)
    b, L, P, N = 1, 4, 2, 4
    p, state = problem(rng, b, L, H, G, P, N, R, flags)
    dy = rng.standard_normal((b, L, H, R, P))
    dfin = oracle.State(rng.standard_normal((b, H, N, P)), rng.standard_normal((b, H, N // 2)),
                        rng.standard_normal((b, H, R, N)), rng.standard_normal((b, H, R, P)))
    g = og.scan_grad(p["x"], p["B"], p["C"], p["theta"], p["dt"], p["A"], p["lam"],
                     p["B_bias"], p["C_bias"], state, dy, dfin, bc_norm=bc_norm,
                     dt_bias=p.get("dt_bias"), flags=flags)
    eps = 1e-6
    targets = [("x", "dx"), ("B", "dB"), ("C", "dC"), ("theta", "dtheta"), ("dt", "ddt"),
               ("A", "dA"), ("lam", "dlam"), ("B_bias", "dB_bias"), ("C_bias", "dC_bias")]
    if "dt_bias" in p:
        targets.append(("dt_bias", "ddt_bias"))
    checked = 0
    for key, gkey in targets:
        arr = p[key]
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + eps
            fp = _objective(p, state, dy, dfin, bc_norm, flags)
            arr[idx] = old - eps
            fm = _objective(p, state, dy, dfin, bc_norm, flags)
            arr[idx] = old
            fd[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(g[gkey], fd, rtol=1e-5, atol=1e-6, err_msg=key)
        checked += arr.size
    for field in ("h", "phi", "prev_B", "prev_x"):
        arr = getattr(state, field)
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + eps
            fp = _objective(p, state, dy, dfin, bc_norm, flags)
            arr[idx] = old - eps
            fm = _objective(p, state, dy, dfin, bc_norm, flags)
            arr[idx] = old
            fd[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(getattr(g["dinit"], field), fd, rtol=1e-5, atol=1e-6,
                                   err_msg="init " + field)
        checked += arr.size
    assert checked > 100
    if flags & oracle.DISC_ZOH:   # lam is not used under the zero-order hold
        assert not np.any(g["dlam"])


def test_gradient_closed_form_real_euler_case():
    """theta = 0, lam = 1 (exponential Euler), no norm, no bias, R = 1, zero initial state:
    y_t = sum_{s<=t} (prod_{k=s+1..t} alpha_k) dt_s (C_t . B_s) x_s (Sec. 3.1.1 with lam = 1 is
    the Mamba-2 recurrence). Then, with K(t,s) = prod_{k=s+1..t} alpha_k dt_s,
        dx_s = sum_{t>=s} K(t,s) (C_t . B_s) dy_t,
        dC_t = sum_{s<=t} K(t,s) (x_s . dy_t) B_s,
        dA_k = sum_{s<k<=t} dt_k K(t,s) (C_t . B_s)(x_s . dy_t),
    written out here as explicit sums (no autograd, no finite differences)."""
    rng = np.random.default_rng(5)
    b, L, H, P, N = 1, 7, 1, 3, 4
    x = rng.standard_normal((b, L, H, 1, P))
    B = rng.standard_normal((b, L, 1, 1, N))
    C = rng.standard_normal((b, L, 1, 1, N))
    dt = np.log1p(np.exp(rng.standard_normal((b, L, H)) - 1.0))
    A = -np.exp(rng.uniform(-1, 1, (b, L, H)))
    dy = rng.standard_normal((b, L, H, 1, P))
    g = og.scan_grad(x, B, C, np.zeros((b, L, H, N // 2)), dt, A, np.ones((b, L, H)),
                     dy=dy)
    al = np.exp(dt[0, :, 0] * A[0, :, 0])
    xs, Bs, Cs, dys, d = x[0, :, 0, 0], B[0, :, 0, 0], C[0, :, 0, 0], dy[0, :, 0, 0], dt[0, :, 0]

    def K(t, s):
        return np.prod(al[s + 1:t + 1]) * d[s]

    dx = np.zeros((L, P))
    dC = np.zeros((L, N))
    dA = np.zeros(L)
    for t in range(L):
        for s in range(t + 1):
            cb, xd = Cs[t] @ Bs[s], xs[s] @ dys[t]
            dx[s] += K(t, s) * cb * dys[t]
            dC[t] += K(t, s) * xd * Bs[s]
            for k in range(s + 1, t + 1):
                dA[k] += d[k] * K(t, s) * cb * xd
    np.testing.assert_allclose(g["dx"][0, :, 0, 0], dx, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dC"][0, :, 0, 0], dC, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dA"][0, :, 0], dA, rtol=1e-12, atol=1e-12)
