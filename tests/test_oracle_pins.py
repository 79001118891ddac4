"""Pins of the fp64 oracle to what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a special case that
reduces to an older, simpler update; an independent complex-valued derivation; the
parallel (masked matrix) form; a closed form; an exact ODE solution's convergence order;
a hand-checkable rotation example; or an invariant. A plausible mistake in the oracle (a
dropped beta term, beta_{t-1} instead of beta_t, a missing alpha in beta, the wrong rotation
direction or pairing, bias before the norm, B and C swapped in MIMO, a state-passing slip)
fails at least one of them.

Page references are to "Mamba-3: Improved Sequence Modeling using State Space Principles".
"""
import math

import numpy as np
import pytest

import oracle


def rnd_problem(rng, b=2, L=24, H=3, G=1, P=5, N=8, R=1, norm=True, bias=True, lam=None,
                theta_scale=math.pi, dt_shift=-1.0):
    x = rng.standard_normal((b, L, H, R, P))
    B = rng.standard_normal((b, L, G, R, N))
    C = rng.standard_normal((b, L, G, R, N))
    th = rng.uniform(-1, 1, (b, L, H, N // 2)) * theta_scale
    dt = np.log1p(np.exp(rng.standard_normal((b, L, H)) + dt_shift))
    A = -np.exp(rng.uniform(-1, 1, (b, L, H)))
    lm = (1 / (1 + np.exp(-rng.standard_normal((b, L, H))))) if lam is None else np.full(
        (b, L, H), float(lam))
    Bb = rng.standard_normal((H, R, N)) * 0.3 if bias else None
    Cb = rng.standard_normal((H, R, N)) * 0.3 if bias else None
    return dict(x=x, B=B, C=C, theta=th, dt=dt, A=A, lam=lm, B_bias=Bb, C_bias=Cb,
                bc_norm=norm)


def rand_state(rng, b, H, N, P, R):
    return oracle.State(rng.standard_normal((b, H, N, P)),
                        rng.uniform(-math.pi, math.pi, (b, H, N // 2)),
                        rng.standard_normal((b, H, R, N)),
                        rng.standard_normal((b, H, R, P)))


def normed(v, bias, norm, eps=1e-6):
    """B or C after the optional RMS norm over N and the bias (Sec. 3.4)."""
    if norm:
        v = v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return v + (0 if bias is None else bias)


# --------------------------------------------------------------------------------------
# Independent complex-valued derivation (Appendix B.3, eq. 25 in complex form; Prop. 2).
# The state is complex of size N/2 in the ORIGINAL (un-rotated) frame: the transition is
# exp(dt (A + i theta)), the previous input gets rotated by the current step's angle, and
# the real readout is Re(c^T h) with c = C_re - i C_im (Prop. 2: C = [C; -C_hat]).
# --------------------------------------------------------------------------------------
def complex_reference(p, state=None):
    x, B, C, th, dt, A, lm = (p[k] for k in ("x", "B", "C", "theta", "dt", "A", "lam"))
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    half = N // 2
    y = np.zeros((b, L, H, R, P))
    out = oracle.State.zeros(b, H, N, P, R)
    for bb in range(b):
        for hh in range(H):
            g = hh // (H // G)
            Bb = None if p["B_bias"] is None else p["B_bias"][hh]
            Cb = None if p["C_bias"] is None else p["C_bias"][hh]
            if state is None:
                phi0 = np.zeros(half)
                hc = np.zeros((half, P), complex)
                bprev = np.zeros((R, half), complex)
                xprev = np.zeros((R, P))
                praw = np.zeros((R, N))
            else:
                phi0 = state.phi[bb, hh].copy()
                ht = state.h[bb, hh]
                hc = np.exp(1j * phi0)[:, None] * (ht[:half] + 1j * ht[half:])
                bn = normed(state.prev_B[bb, hh], Bb, p["bc_norm"])
                bprev = bn[:, :half] + 1j * bn[:, half:]
                xprev = state.prev_x[bb, hh].copy()
                praw = state.prev_B[bb, hh].copy()
            phi = phi0.copy()
            for t in range(L):
                d, a, l = dt[bb, t, hh], A[bb, t, hh], lm[bb, t, hh]
                w = d * th[bb, t, hh]
                bn = normed(B[bb, t, g], Bb, p["bc_norm"])
                cn = normed(C[bb, t, g], Cb, p["bc_norm"])
                bc = bn[:, :half] + 1j * bn[:, half:]
                cc = cn[:, :half] - 1j * cn[:, half:]
                beta = (1 - l) * d * math.exp(d * a)
                gamma = l * d
                hc = (np.exp(d * (a + 1j * th[bb, t, hh]))[:, None] * hc
                      + beta * np.exp(1j * w)[:, None] * np.einsum("rn,rp->np", bprev, xprev)
                      + gamma * np.einsum("rn,rp->np", bc, x[bb, t, hh]))
                y[bb, t, hh] = np.real(np.einsum("rn,np->rp", cc, hc))
                phi = phi + w
                bprev, xprev, praw = bc, x[bb, t, hh].copy(), B[bb, t, g].copy()
            ht = np.exp(-1j * phi)[:, None] * hc
            out.h[bb, hh] = np.concatenate([ht.real, ht.imag], 0)
            out.phi[bb, hh] = phi
            out.prev_B[bb, hh] = praw
            out.prev_x[bb, hh] = xprev
    return y, out


def run(p, state=None, **kw):
    return oracle.scan(p["x"], p["B"], p["C"], p["theta"], p["dt"], p["A"], p["lam"],
                       p["B_bias"], p["C_bias"], state=state, bc_norm=p["bc_norm"], **kw)


def assert_state_close(s1, s2, tol=1e-11):
    for f in ("h", "phi", "prev_B", "prev_x"):
        a, b = getattr(s1, f), getattr(s2, f)
        assert np.max(np.abs(a - b)) <= tol * max(1.0, np.max(np.abs(b))), f


@pytest.mark.parametrize("R,G,H", [(1, 1, 3), (1, 3, 3), (2, 1, 2), (4, 2, 4)])
@pytest.mark.parametrize("with_state", [False, True])
def test_complex_valued_derivation(R, G, H, with_state):
    """Rotated-frame real recurrence == complex recurrence in the original frame (App. B.3).

    Pins the rotation direction (R^T), the (i, i+N/2) pairing, the sign convention of C,
    the beta term's rotation by the current step, and the rotated-frame final state."""
    rng = np.random.default_rng(10 + R + G + H + with_state)
    p = rnd_problem(rng, H=H, G=G, R=R)
    st = rand_state(rng, 2, H, 8, 5, R) if with_state else None
    y, fs = run(p, st)
    yc, fc = complex_reference(p, st)
    np.testing.assert_allclose(y, yc, rtol=0, atol=1e-11 * np.max(np.abs(yc)))
    assert_state_close(fs, fc, 1e-11)


def test_lambda_one_is_exponential_euler():
    """lam == 1 reduces to Mamba-2's exponential-Euler update h = e^{dt A} h + dt B x
    (Sec. 3.1.1 Remark 2, eq. 4), written here in the complex form of Prop. 2."""
    rng = np.random.default_rng(1)
    p = rnd_problem(rng, lam=1.0, R=2)
    y, fs = run(p)
    x, B, C, th, dt, A = (p[k] for k in ("x", "B", "C", "theta", "dt", "A"))
    b, L, H, R, P = x.shape
    half = B.shape[-1] // 2
    for bb in range(b):
        for hh in range(H):
            hc = np.zeros((half, P), complex)
            for t in range(L):
                bn = normed(B[bb, t, 0], p["B_bias"][hh], True)
                cn = normed(C[bb, t, 0], p["C_bias"][hh], True)
                hc = np.exp(dt[bb, t, hh] * (A[bb, t, hh] + 1j * th[bb, t, hh]))[:, None] * hc \
                    + dt[bb, t, hh] * np.einsum("rn,rp->np", bn[:, :half] + 1j * bn[:, half:],
                                                x[bb, t, hh])
                ye = np.real(np.einsum("rn,np->rp", cn[:, :half] - 1j * cn[:, half:], hc))
                np.testing.assert_allclose(y[bb, t, hh], ye, atol=1e-11)


def test_theta_zero_is_real_ssm():
    """theta == 0: no rotation (R_t = I), the angle stays 0 and the state equals the plain
    real exponential-trapezoidal recurrence of Prop. 1 on the normalised, biased B, C."""
    rng = np.random.default_rng(2)
    p = rnd_problem(rng, theta_scale=0.0, R=1, G=1, H=2)
    y, fs = run(p)
    assert np.all(fs.phi == 0)
    x, B, C, dt, A, lm = (p[k] for k in ("x", "B", "C", "dt", "A", "lam"))
    for hh in range(2):
        h = np.zeros((8, 5))
        vprev = np.zeros((8, 5))
        for t in range(x.shape[1]):
            v = np.outer(normed(B[0, t, 0, 0], p["B_bias"][hh, 0], True), x[0, t, hh, 0])
            al = math.exp(dt[0, t, hh] * A[0, t, hh])
            h = al * h + (1 - lm[0, t, hh]) * dt[0, t, hh] * al * vprev + lm[0, t, hh] * dt[0, t, hh] * v
            vprev = v
            np.testing.assert_allclose(
                y[0, t, hh, 0], h.T @ normed(C[0, t, 0, 0], p["C_bias"][hh, 0], True), atol=1e-11)


@pytest.mark.parametrize("R", [1, 3])
def test_parallel_mask_form(R):
    """Y = (L o C B^T) X with L = L1 . L2 (Sec. 3.1.3 eq. 7): L1 the 1-semiseparable decay
    matrix, L2 the 2-band matrix with gamma_t on the diagonal and beta_t below it. For MIMO
    the token mask is expanded by the Kronecker product with a full R x R block of ones.
    Rotations enter through B_bar, C_bar computed as complex products e^{-i Phi} b."""
    rng = np.random.default_rng(3 + R)
    T = 40
    p = rnd_problem(rng, b=1, L=T, H=1, R=R, N=6, P=3)
    y, _ = run(p)
    dt, A, lm = p["dt"][0, :, 0], p["A"][0, :, 0], p["lam"][0, :, 0]
    al = np.exp(dt * A)
    beta = (1 - lm) * dt * al
    gam = lm * dt
    L1 = np.zeros((T, T))
    for t in range(T):
        for s in range(t + 1):
            L1[t, s] = np.prod(al[s + 1:t + 1])
    L2 = np.diag(gam) + np.diag(beta[1:], -1)
    Lm = np.kron(L1 @ L2, np.ones((R, R)))
    phi = np.cumsum(dt[:, None] * p["theta"][0, :, 0], axis=0)  # [T, N/2]
    half = 3

    def bar(v, bias):
        vn = normed(v, bias, True)                    # [T, R, N]
        z = (vn[..., :half] + 1j * vn[..., half:]) * np.exp(-1j * phi)[:, None, :]
        return np.concatenate([z.real, z.imag], -1).reshape(T * R, 2 * half)

    Bb = bar(p["B"][0, :, 0], p["B_bias"][0])
    Cb = bar(p["C"][0, :, 0], p["C_bias"][0])
    X = p["x"][0, :, 0].reshape(T * R, 3)
    Y = (Lm * (Cb @ Bb.T)) @ X
    np.testing.assert_allclose(y[0, :, 0].reshape(T * R, 3), Y, atol=1e-11 * np.max(np.abs(Y)))


def test_mimo_is_sum_of_R2_siso():
    """MIMO output i == sum over j of SISO runs with (B^(j), C^(i), x^(j)) (Sec. 3.3,
    eq. 12-14). Catches B/C or x rank-index mix-ups."""
    rng = np.random.default_rng(4)
    R = 3
    p = rnd_problem(rng, b=1, L=20, H=2, R=R)
    y, _ = run(p)
    acc = np.zeros_like(y)
    for i in range(R):
        for j in range(R):
            q = dict(p)
            q["x"] = p["x"][:, :, :, j:j + 1]
            q["B"] = p["B"][:, :, :, j:j + 1]
            q["C"] = p["C"][:, :, :, i:i + 1]
            q["B_bias"] = p["B_bias"][:, j:j + 1]
            q["C_bias"] = p["C_bias"][:, i:i + 1]
            yij, _ = run(q)
            acc[:, :, :, i] += yij[:, :, :, 0]
    np.testing.assert_allclose(y, acc, atol=1e-11 * np.max(np.abs(acc)))


def test_mimo_rank1_equals_siso_bitwise():
    rng = np.random.default_rng(5)
    p = rnd_problem(rng, R=1)
    y1, s1 = run(p)
    y2, s2 = run(p, nthreads=1)
    assert np.array_equal(y1, y2) and np.array_equal(s1.h, s2.h)


@pytest.mark.parametrize("lam", [0.5, 0.3, 1.0])
def test_constant_alpha_closed_form(lam):
    """Constant dt, A, lam, x, B, C and theta = 0: h_t = v [gamma + w alpha (1-alpha^t)/(1-alpha)]
    with v = B x^T and w = gamma + (1-lam) dt, from unrolling Prop. 1 from h_0 = gamma_0 B_0 x_0."""
    T, N, P = 50, 4, 3
    rng = np.random.default_rng(6)
    Bv, Cv, xv = rng.standard_normal(N), rng.standard_normal(N), rng.standard_normal(P)
    d, a = 0.3, -0.7
    p = dict(x=np.broadcast_to(xv, (1, T, 1, 1, P)).copy(),
             B=np.broadcast_to(Bv, (1, T, 1, 1, N)).copy(),
             C=np.broadcast_to(Cv, (1, T, 1, 1, N)).copy(),
             theta=np.zeros((1, T, 1, N // 2)), dt=np.full((1, T, 1), d),
             A=np.full((1, T, 1), a), lam=np.full((1, T, 1), lam), B_bias=None, C_bias=None,
             bc_norm=False)
    y, fs = run(p)
    al, gam = math.exp(d * a), lam * d
    w = gam + (1 - lam) * d
    for t in range(T):
        coef = gam + w * al * (1 - al ** t) / (1 - al)
        np.testing.assert_allclose(y[0, t, 0, 0], coef * (Cv @ Bv) * xv, rtol=1e-12)
    np.testing.assert_allclose(fs.h[0, 0], (gam + w * al * (1 - al ** (T - 1)) / (1 - al))
                               * np.outer(Bv, xv), rtol=1e-12)


def _ode_error(lam, n_steps, T_end=2.0, a=-0.8):
    """Max error of the scheme against the exact solution of h' = a h + sin(tau), h(0) = 0,
    sampled at tau_t = (t+1) dt, with x(tau) = sin(tau) (so x_{-1} = sin(0) = 0 and the
    all-zero initial state is exact)."""
    d = T_end / n_steps
    tau = d * np.arange(1, n_steps + 1)
    N, P = 2, 1
    p = dict(x=np.sin(tau).reshape(1, -1, 1, 1, 1),
             B=np.broadcast_to(np.array([1.0, 0.0]), (1, n_steps, 1, 1, N)).copy(),
             C=np.broadcast_to(np.array([1.0, 0.0]), (1, n_steps, 1, 1, N)).copy(),
             theta=np.zeros((1, n_steps, 1, 1)), dt=np.full((1, n_steps, 1), d),
             A=np.full((1, n_steps, 1), a), lam=np.full((1, n_steps, 1), lam),
             B_bias=None, C_bias=None, bc_norm=False)
    y, _ = run(p)
    # exact: h(t) = int_0^t e^{a(t-s)} sin s ds = (e^{at} - a sin t - cos t) / (1 + a^2)
    exact = (np.exp(a * tau) - a * np.sin(tau) - np.cos(tau)) / (1 + a * a)
    return np.max(np.abs(y[0, :, 0, 0, 0] - exact))


def test_exact_solution_reference_is_right():
    """The closed form used below solves h' = a h + sin(t), h(0) = 0 (checked by finite
    differences), so the convergence test measures the scheme, not the reference."""
    a = -0.8
    t = np.linspace(0.1, 2, 50)
    f = lambda t: (np.exp(a * t) - a * np.sin(t) - np.cos(t)) / (1 + a * a)
    e = 1e-6
    np.testing.assert_allclose((f(t + e) - f(t - e)) / (2 * e), a * f(t) + np.sin(t), atol=1e-8)
    assert abs(f(0.0)) < 1e-15


def test_convergence_order():
    """lam = 1/2 is the classical trapezoid: global error O(dt^2); lam = 1 (Euler) is O(dt)
    (Sec. 3.1.1 Remark 3, Appendix A.2). A beta without the e^{dt A} factor, or beta_{t-1}
    in place of beta_t, degrades lam = 1/2 to first order and fails here."""
    r_trap = _ode_error(0.5, 200) / _ode_error(0.5, 400)
    r_euler = _ode_error(1.0, 200) / _ode_error(1.0, 400)
    assert 3.6 < r_trap < 4.4, r_trap
    assert 1.8 < r_euler < 2.2, r_euler
    assert _ode_error(0.5, 400) < 1e-4


def test_parity_by_rotation():
    """State tracking by rotation (Sec. 3.2): with alpha = 1, dt = 1, lam = 1, one unit
    impulse at t = 0 and theta_t = pi * bit_t, y_t = cos(pi * sum_{s=1..t} bit_s), i.e. the
    parity of the bits seen after the impulse: +1 even, -1 odd."""
    rng = np.random.default_rng(7)
    T = 33
    bits = rng.integers(0, 2, T)
    x = np.zeros((1, T, 1, 1, 1))
    x[0, 0] = 1.0
    p = dict(x=x, B=np.broadcast_to(np.array([1.0, 0.0]), (1, T, 1, 1, 2)).copy(),
             C=np.broadcast_to(np.array([1.0, 0.0]), (1, T, 1, 1, 2)).copy(),
             theta=(math.pi * bits).reshape(1, T, 1, 1).astype(float),
             dt=np.ones((1, T, 1)), A=np.zeros((1, T, 1)), lam=np.ones((1, T, 1)),
             B_bias=None, C_bias=None, bc_norm=False)
    y, _ = run(p)
    par = np.cumsum(bits) - bits[0]
    expect = np.where(par % 2 == 0, 1.0, -1.0)
    np.testing.assert_allclose(y[0, :, 0, 0, 0], expect, atol=1e-12)


@pytest.mark.parametrize("split", [1, 7, 23])
def test_split_sequence_state_passing(split):
    """scan(L1) -> state -> scan(L2) == scan(L1 + L2) (Appendix G.2 state passing)."""
    rng = np.random.default_rng(8)
    p = rnd_problem(rng, L=24, R=2, G=1, H=2)
    st0 = rand_state(rng, 2, 2, 8, 5, 2)
    y, fs = run(p, st0)
    a = {k: (v[:, :split] if isinstance(v, np.ndarray) and v.ndim >= 3 and k not in ("B_bias", "C_bias") else v) for k, v in p.items()}
    c = {k: (v[:, split:] if isinstance(v, np.ndarray) and v.ndim >= 3 and k not in ("B_bias", "C_bias") else v) for k, v in p.items()}
    y1, s1 = run(a, st0)
    y2, s2 = run(c, s1)
    np.testing.assert_allclose(np.concatenate([y1, y2], 1), y, atol=1e-11)
    assert_state_close(s2, fs)


def test_decode_steps_equal_scan():
    rng = np.random.default_rng(9)
    p = rnd_problem(rng, L=9, R=2, H=2)
    st0 = rand_state(rng, 2, 2, 8, 5, 2)
    y, fs = run(p, st0)
    st = st0
    for t in range(9):
        yt, st = oracle.decode_step(*(p[k][:, t] for k in ("x", "B", "C", "theta", "dt", "A", "lam")),
                                    B_bias=p["B_bias"], C_bias=p["C_bias"], state=st,
                                    bc_norm=True)
        np.testing.assert_allclose(yt, y[:, t], atol=1e-12)
    assert_state_close(st, fs)


def test_bcnorm_scale_invariance_and_bias_after_norm():
    """RMS norm then bias (Sec. 3.4): scaling B_raw and C_raw by any k > 0 per token leaves
    the output unchanged (eps -> 0; 1e-30 keeps the all-zero initial prev_B finite); adding the bias before the norm would break this."""
    rng = np.random.default_rng(11)
    p = rnd_problem(rng, R=2)
    y, _ = oracle.scan(p["x"], p["B"], p["C"], p["theta"], p["dt"], p["A"], p["lam"],
                       p["B_bias"], p["C_bias"], bc_norm=True, norm_eps=1e-30)
    k = rng.uniform(0.1, 10, p["B"].shape[:-1] + (1,))
    y2, _ = oracle.scan(p["x"], p["B"] * k, p["C"] * k[..., ::-1, :], p["theta"], p["dt"],
                        p["A"], p["lam"], p["B_bias"], p["C_bias"], bc_norm=True, norm_eps=1e-30)
    np.testing.assert_allclose(y, y2, atol=1e-11 * np.max(np.abs(y)))
    # RMS norm value itself: a constant vector c*1 normalises to 1 for any c.
    q = dict(p)
    q["B"] = np.full_like(p["B"], 3.7)
    yb, _ = oracle.scan(q["x"], q["B"], p["C"], p["theta"], p["dt"], p["A"], p["lam"],
                        None, p["C_bias"], bc_norm=True, norm_eps=1e-30)
    q["B"] = np.full_like(p["B"], 1.0)
    yc, _ = oracle.scan(q["x"], q["B"], normed(p["C"], None, True, 1e-30), p["theta"], p["dt"],
                        p["A"], p["lam"], None, p["C_bias"], bc_norm=False)
    np.testing.assert_allclose(yb, yc, atol=1e-11 * np.max(np.abs(yc)))


def test_global_angle_offset_invariance():
    """From a zero state, adding a constant to the initial angle leaves y unchanged: scores
    depend only on angle differences (Appendix B.2)."""
    rng = np.random.default_rng(12)
    p = rnd_problem(rng, R=2)
    st = oracle.State.zeros(2, 3, 8, 5, 2)
    st.phi[:] = rng.uniform(-5, 5, st.phi.shape)
    y0, f0 = run(p)
    y1, f1 = run(p, st)
    np.testing.assert_allclose(y0, y1, atol=1e-11 * np.max(np.abs(y0)))
    np.testing.assert_allclose(f1.phi - f0.phi, st.phi, atol=1e-12)


def test_empty_sequence_keeps_state():
    rng = np.random.default_rng(13)
    p = rnd_problem(rng, L=0)
    st = rand_state(rng, 2, 3, 8, 5, 1)
    y, fs = run(p, st)
    assert y.shape[1] == 0
    assert_state_close(fs, st, 0)


# ---------------------------------------------------------------- fused scalar prologue
def test_step_scalars_match_library_softplus_and_sigmoid():
    """softplus and sigmoid of the raw projections (Sec. 2: a positive step; Appendix F:
    lambda_t = sigma(u_t)) against torch's own routines in float64, including the far tails
    where a naive exp overflows."""
    import torch
    rng = np.random.default_rng(21)
    d = np.concatenate([rng.standard_normal((4, 7, 5)).ravel() * 6,
                        [-800.0, -40.0, -20.0, -1e-9, 0.0, 1e-9, 5.0, 20.0, 25.0, 800.0]]).reshape(-1, 5)
    u = np.concatenate([rng.standard_normal((4, 7, 5)).ravel() * 6,
                        [-800.0, -40.0, -20.0, -1e-9, 0.0, 1e-9, 5.0, 20.0, 25.0, 800.0]]).reshape(-1, 5)
    bias = rng.standard_normal(5) - 2.0
    dt, lam = oracle.step_scalars(d, u, bias, oracle.DT_SOFTPLUS | oracle.LAM_SIGMOID)
    v = d + bias
    ref_dt = torch.nn.functional.softplus(torch.from_numpy(v)).numpy()  # linear above 20
    ref_lam = torch.sigmoid(torch.from_numpy(u))
    lin = v > 20   # there the library returns v itself, off by log(1 + e^{-v}) < 2.1e-9
    np.testing.assert_allclose(dt[~lin], ref_dt[~lin], rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(dt[lin], ref_dt[lin], rtol=2.1e-9 / 20, atol=0)
    np.testing.assert_allclose(lam, ref_lam.numpy(), rtol=1e-14, atol=1e-300)
    assert np.all(dt >= 0) and np.all(dt[v > -700] > 0)   # e^{-745} underflows fp64
    assert np.all((lam >= 0) & (lam <= 1))
    # each flag alone transforms only its own input; no flag is the identity
    dt1, lam1 = oracle.step_scalars(d, u, bias, oracle.DT_SOFTPLUS)
    assert np.array_equal(lam1, u) and np.array_equal(dt1, dt)
    dt2, lam2 = oracle.step_scalars(d, u, bias, 0)
    assert np.array_equal(dt2, d) and np.array_equal(lam2, u)


def test_scan_with_raw_scalars_equals_scan_of_library_transformed():
    """Wiring of the prologue inside the scan and decode: per-head bias broadcast over [b, L, H]
    and both flags, against the scan of inputs transformed by torch's softplus / sigmoid."""
    import torch
    rng = np.random.default_rng(22)
    p = rnd_problem(rng, b=2, L=19, H=3, R=2)
    raw_d = rng.standard_normal((2, 19, 3))
    raw_u = rng.standard_normal((2, 19, 3)) * 2
    bias = np.array([-2.0, -0.5, 1.0])
    st = rand_state(rng, 2, 3, 8, 5, 2)
    q = dict(p, dt=raw_d, lam=raw_u)
    y_raw, s_raw = oracle.scan(**{k: v for k, v in q.items() if k != "bc_norm"}, state=st,
                               bc_norm=q["bc_norm"], dt_bias=bias, flags=3)
    ref = dict(p, dt=torch.nn.functional.softplus(torch.from_numpy(raw_d + bias)).numpy(),
               lam=torch.sigmoid(torch.from_numpy(raw_u)).numpy())
    y_ref, s_ref = oracle.scan(**{k: v for k, v in ref.items() if k != "bc_norm"}, state=st,
                               bc_norm=ref["bc_norm"])
    np.testing.assert_allclose(y_raw, y_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s_raw.h, s_ref.h, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s_raw.phi, s_ref.phi, rtol=1e-12, atol=1e-12)
    # one decode step takes the same parameterisation
    tok = {k: (v[:, 0] if k in ("x", "B", "C", "theta") else v) for k, v in q.items()
           if k != "bc_norm"}
    yd, sd = oracle.decode_step(tok["x"], tok["B"], tok["C"], tok["theta"], raw_d[:, 0],
                                p["A"][:, 0], raw_u[:, 0], p["B_bias"], p["C_bias"], st,
                                p["bc_norm"], dt_bias=bias, flags=3)
    y1, s1 = oracle.scan(**{k: (v[:, :1] if k in ("x", "B", "C", "theta", "dt", "A", "lam")
                                else v) for k, v in ref.items() if k != "bc_norm"},
                         state=st, bc_norm=ref["bc_norm"])
    np.testing.assert_allclose(yd, y1[:, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sd.h, s1.h, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- MIMO projections (decode)
def test_decode_step_proj_against_library_gate_and_contraction():
    """O' = sum_r W_O (Y * SiLU(W_Z Z')) with X = W_X X' (Appendix C): against torch's SiLU and
    numpy's einsum applied to the plain decode step of the expanded X; with R = 1 and unit
    weights it is the plain output times SiLU(Z')."""
    import torch
    rng = np.random.default_rng(31)
    for R in (1, 4):
        b, H, P, N = 2, 3, 5, 8
        p = rnd_problem(rng, b=b, L=1, H=H, R=R, P=P, N=N)
        st = rand_state(rng, b, H, N, P, R)
        xp, zp = rng.standard_normal((b, H, P)), rng.standard_normal((b, H, P)) * 3
        WX, WZ, WO = (rng.standard_normal((H, R, P)) for _ in range(3))
        tok = {k: (v[:, 0] if k in ("x", "B", "C", "theta", "dt", "A", "lam") else v)
               for k, v in p.items() if k != "bc_norm"}
        o, so = oracle.decode_step_proj(xp, zp, WX, WZ, WO, tok["B"], tok["C"], tok["theta"],
                                        tok["dt"], tok["A"], tok["lam"], tok["B_bias"],
                                        tok["C_bias"], st, p["bc_norm"])
        X = np.einsum("hrp,bhp->bhrp", WX, xp)
        y, sy = oracle.decode_step(X, tok["B"], tok["C"], tok["theta"], tok["dt"], tok["A"],
                                   tok["lam"], tok["B_bias"], tok["C_bias"], st, p["bc_norm"])
        gate = torch.nn.functional.silu(torch.from_numpy(np.einsum("hrp,bhp->bhrp", WZ, zp)))
        ref = np.einsum("hrp,bhrp->bhp", WO, y * gate.numpy())
        np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(so.h, sy.h, rtol=0, atol=0)
        np.testing.assert_allclose(so.prev_x, X, rtol=0, atol=0)
    # R = 1, unit weights: the plain output gated by SiLU(Z')
    b, H, P, N = 2, 3, 5, 8
    p = rnd_problem(rng, b=b, L=1, H=H, R=1, P=P, N=N)
    st = rand_state(rng, b, H, N, P, 1)
    xp, zp = rng.standard_normal((b, H, P)), rng.standard_normal((b, H, P)) * 3
    one = np.ones((H, 1, P))
    args = [p[k][:, 0] for k in ("B", "C", "theta", "dt", "A", "lam")]
    o1, _ = oracle.decode_step_proj(xp, zp, one, one, one, *args, p["B_bias"], p["C_bias"], st,
                                    p["bc_norm"])
    y1, _ = oracle.decode_step(xp[:, :, None, :], *args, p["B_bias"], p["C_bias"], st,
                               p["bc_norm"])
    ref1 = y1[:, :, 0, :] * torch.nn.functional.silu(torch.from_numpy(zp)).numpy()
    np.testing.assert_allclose(o1, ref1, rtol=1e-12, atol=1e-12)


def test_decode_step_proj_structural_cases_by_hand():
    """Two cases of the projected decode step (Appendix C) fixed without the oracle's own
    contraction code, by plain loops over a tiny problem with no rotation (theta = 0 and a
    zero carried angle), no norm and no bias:
      - W_X = 0: the new token enters nothing, so h' = alpha h + beta sum_r prevB_r prevx_r^T
        (Prop. 1 with x_t = 0), Y[r][p] = sum_n C[r][n] h'[n][p], and O' is the W_O-weighted,
        SiLU(W_Z Z')-gated sum of Y over the ranks; the stored prev_x is 0;
      - W_O one-hot on rank q: O' is rank q's gated output alone, so the outputs of the R
        one-hot choices add up to the output with every weight of W_O at 1 (linear in W_O)."""
    rng = np.random.default_rng(77)
    b, H, R, N, P = 1, 2, 2, 4, 3
    st = oracle.State(rng.standard_normal((b, H, N, P)), np.zeros((b, H, N // 2)),
                      rng.standard_normal((b, H, R, N)), rng.standard_normal((b, H, R, P)))
    B = rng.standard_normal((b, 1, R, N))
    C = rng.standard_normal((b, 1, R, N))
    theta = np.zeros((b, H, N // 2))
    dt = np.array([[0.7, 0.2]])
    A = np.array([[-0.5, -1.3]])
    lam = np.array([[0.3, 0.8]])
    xp, zp = rng.standard_normal((b, H, P)), rng.standard_normal((b, H, P))
    WZ, WO = rng.standard_normal((H, R, P)), rng.standard_normal((H, R, P))
    WX0 = np.zeros((H, R, P))
    o, so = oracle.decode_step_proj(xp, zp, WX0, WZ, WO, B, C, theta, dt, A, lam, state=st)
    for h in range(H):
        al = math.exp(dt[0, h] * A[0, h])
        be = (1.0 - lam[0, h]) * dt[0, h] * al
        hn = [[al * st.h[0, h, n, p] + be * sum(st.prev_B[0, h, r, n] * st.prev_x[0, h, r, p]
                                              for r in range(R))
               for p in range(P)] for n in range(N)]
        for n in range(N):
            for p in range(P):
                assert abs(so.h[0, h, n, p] - hn[n][p]) < 1e-12
        for p in range(P):
            want = 0.0
            for r in range(R):
                y = sum(C[0, 0, r, n] * hn[n][p] for n in range(N))
                z = WZ[h, r, p] * zp[0, h, p]
                want += WO[h, r, p] * y * (z / (1.0 + math.exp(-z)))
            assert abs(o[0, h, p] - want) < 1e-12 * max(1.0, abs(want))
    assert np.all(so.prev_x == 0.0)
    # one-hot W_O: rank q alone, and the ranks add up to W_O = 1
    WX = rng.standard_normal((H, R, P))
    ones = np.ones((H, R, P))
    o_all, _ = oracle.decode_step_proj(xp, zp, WX, WZ, ones, B, C, theta, dt, A, lam, state=st)
    y_all, _ = oracle.decode_step(WX[None] * xp[:, :, None, :], B, C, theta, dt, A, lam,
                                  state=st)
    total = np.zeros_like(o_all)
    for q in range(R):
        e = np.zeros((H, R, P))
        e[:, q, :] = 1.0
        oq, _ = oracle.decode_step_proj(xp, zp, WX, WZ, e, B, C, theta, dt, A, lam, state=st)
        for h in range(H):
            for p in range(P):
                z = WZ[h, q, p] * zp[0, h, p]
                assert abs(oq[0, h, p] - y_all[0, h, q, p] * z / (1.0 + math.exp(-z))) < 1e-12
        total += oq
    np.testing.assert_allclose(total, o_all, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- zero-order hold
def test_zoh_is_exact_for_piecewise_constant_input():
    """The zero-order-hold weights ("Mamba-3：推理优先的状态空间模型", Sec. 1.2) are the exact
    solution of h' = A h + B x when A, B and x are held constant over each step: the oracle
    with DISC_ZOH against scipy's ODE integrator over the same steps (theta = 0, no norm)."""
    from scipy.integrate import solve_ivp
    rng = np.random.default_rng(41)
    L, N, P = 12, 2, 3
    x = rng.standard_normal((1, L, 1, 1, P))
    B = np.zeros((1, L, 1, 1, N)); B[..., 0] = 1.0 + rng.random((1, L, 1, 1))
    C = np.zeros((1, L, 1, 1, N)); C[..., 0] = 1.0
    dt = rng.uniform(0.1, 0.6, (1, L, 1))
    A = -rng.uniform(0.2, 2.5, (1, L, 1))
    lam = rng.random((1, L, 1))            # unused under zero-order hold
    y, st = oracle.scan(x, B, C, np.zeros((1, L, 1, N // 2)), dt, A, lam, flags=oracle.DISC_ZOH)
    h = np.zeros(P)
    for t in range(L):
        a, b, xt = A[0, t, 0], B[0, t, 0, 0, 0], x[0, t, 0, 0]
        sol = solve_ivp(lambda _, v: a * v + b * xt, (0.0, dt[0, t, 0]), h, rtol=1e-12, atol=1e-14)
        h = sol.y[:, -1]
        np.testing.assert_allclose(y[0, t, 0, 0], h, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(st.h[0, 0, 0], h, rtol=1e-9, atol=1e-12)
    # lam does not enter, and the previous token does not either
    y2, _ = oracle.scan(x, B, C, np.zeros((1, L, 1, N // 2)), dt, A, 1 - lam, flags=oracle.DISC_ZOH)
    np.testing.assert_array_equal(y, y2)
