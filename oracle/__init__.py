"""Plain sequential fp64 CPU oracle for the Mamba-3 SSM core.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package. The library under
``state_space_sequence_mamba_b200`` never imports it, and this package imports nothing
from there.

The arithmetic lives in ``m3_oracle.c``: a token-by-token loop over the
exponential-trapezoidal, rotated-frame recurrence of "Mamba-3: Improved Sequence Modeling
using State Space Principles" (Sec. 3.1.1 Prop. 1, Sec. 3.2.2 Prop. 4, Appendix C and
Remark 6). This module only marshals arrays: it upcasts every input to float64, calls the C
loop and returns float64 arrays.

Parity pins for every function here are in ``tests/test_oracle_pins.py``. None is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m3_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_m3_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compiles ``m3_oracle.c`` into ``_m3_oracle.so`` with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math", "-std=c11",
             _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
        ("ngroups", ctypes.c_int64), ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64),
        ("rank", ctypes.c_int64), ("bc_norm", ctypes.c_int32), ("norm_eps", ctypes.c_double),
        ("zoh", ctypes.c_int32),
    ]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.m3o_scan.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 14 + [ctypes.c_int]
        lib.m3o_scan.restype = ctypes.c_int
        lib.m3o_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    """Threads an OpenMP region of the oracle would use on this host."""
    return int(_load().m3o_max_threads())


def _f64(a) -> np.ndarray:
    """Any array-like (numpy, torch CPU tensor of any float dtype) -> contiguous float64."""
    if hasattr(a, "detach"):  # torch tensor; bf16 has no numpy dtype, go through float64
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


@dataclass
class State:
    """Recurrent state of every (batch, head) unit, float64.

    h [b,H,N,P] is the state in the rotated (RoPE) frame; phi [b,H,N/2] the cumulative
    angle; prev_B [b,H,R,N] and prev_x [b,H,R,P] the previous token's raw B and x."""

    h: np.ndarray
    phi: np.ndarray
    prev_B: np.ndarray
    prev_x: np.ndarray

    @staticmethod
    def zeros(batch, nheads, dstate, headdim, rank) -> "State":
        return State(
            np.zeros((batch, nheads, dstate, headdim)),
            np.zeros((batch, nheads, dstate // 2)),
            np.zeros((batch, nheads, rank, dstate)),
            np.zeros((batch, nheads, rank, headdim)),
        )

    def copy(self) -> "State":
        return State(self.h.copy(), self.phi.copy(), self.prev_B.copy(), self.prev_x.copy())


DT_SOFTPLUS, LAM_SIGMOID, DISC_ZOH = 1, 2, 4


def step_scalars(dt, lam, dt_bias=None, flags: int = 0):
    """The step scalars from the layer's raw projections, in float64 (dt, lam [..., H];
    dt_bias [H] or None).

    DT_SOFTPLUS: the step is softplus(dt + dt_bias) = log(1 + e^{dt + dt_bias}). The paper
    says only that the step is a positive projection of the token (Sec. 2, the Mamba-2
    parameterisation); softplus is the reading taken. LAM_SIGMOID: the trapezoid weight is
    sigmoid(u) = 1 / (1 + e^{-u}) (Appendix F, default parameterisation lambda_t = sigma(u_t))."""
    dt, lam = _f64(dt), _f64(lam)
    if flags & DT_SOFTPLUS:
        v = dt + (0.0 if dt_bias is None else _f64(dt_bias))
        dt = np.logaddexp(0.0, v)
    if flags & LAM_SIGMOID:
        e = np.exp(-np.abs(lam))
        lam = np.where(lam >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return dt, lam


def scan(x, B, C, theta, dt, A, lam, B_bias=None, C_bias=None, state: State | None = None,
         bc_norm: bool = False, norm_eps: float = 1e-6, nthreads: int = 0, dt_bias=None,
         flags: int = 0):
    """Runs the sequential recurrence over a whole sequence.

    Shapes: x [b,L,H,R,P]; B, C [b,L,G,R,N]; theta [b,L,H,N/2]; dt, A, lam [b,L,H];
    B_bias, C_bias [H,R,N] or None. ``state`` (float64, not modified) is the state before
    the first token, or None for a fresh sequence (all zeros). ``flags`` and ``dt_bias``:
    dt and lam are raw projections, see ``step_scalars``; DISC_ZOH: zero-order-hold weights
    beta = 0, gamma = (e^{dt A} - 1) / A ("Mamba-3：推理优先的状态空间模型", Sec. 1.2).

    Returns (y [b,L,H,R,P] float64, final State)."""
    x, B, C, theta = _f64(x), _f64(B), _f64(C), _f64(theta)
    dt, lam = step_scalars(dt, lam, dt_bias, flags)
    A = _f64(A)
    B_bias = None if B_bias is None else _f64(B_bias)
    C_bias = None if C_bias is None else _f64(C_bias)
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    assert B.shape == (b, L, G, R, N) and C.shape == B.shape
    assert theta.shape == (b, L, H, N // 2)
    assert dt.shape == (b, L, H) and A.shape == dt.shape and lam.shape == dt.shape
    st = State.zeros(b, H, N, P, R) if state is None else State(
        _f64(state.h).copy(), _f64(state.phi).copy(), _f64(state.prev_B).copy(),
        _f64(state.prev_x).copy())
    assert st.h.shape == (b, H, N, P) and st.phi.shape == (b, H, N // 2)
    assert st.prev_B.shape == (b, H, R, N) and st.prev_x.shape == (b, H, R, P)
    y = np.zeros((b, L, H, R, P))
    d = _Dims(b, L, H, G, P, N, R, 1 if bc_norm else 0, float(norm_eps),
              1 if flags & DISC_ZOH else 0)
    rc = _load().m3o_scan(ctypes.byref(d), _ptr(x), _ptr(B), _ptr(C), _ptr(theta), _ptr(dt),
                          _ptr(A), _ptr(lam), _ptr(B_bias), _ptr(C_bias), _ptr(st.h),
                          _ptr(st.phi), _ptr(st.prev_B), _ptr(st.prev_x), _ptr(y),
                          int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the dimensions")
    return y, st


def decode_step(x, B, C, theta, dt, A, lam, B_bias=None, C_bias=None,
                state: State | None = None, bc_norm: bool = False, norm_eps: float = 1e-6,
                nthreads: int = 0, dt_bias=None, flags: int = 0):
    """One token: x [b,H,R,P]; B, C [b,G,R,N]; theta [b,H,N/2]; dt, A, lam [b,H].

    Exactly one iteration of ``scan``. Returns (y [b,H,R,P], new State)."""
    def tok(a):
        a = _f64(a)
        return a[:, None]
    y, st = scan(tok(x), tok(B), tok(C), tok(theta), tok(dt), tok(A), tok(lam), B_bias,
                 C_bias, state, bc_norm, norm_eps, nthreads, dt_bias, flags)
    return y[:, 0], st


def decode_step_proj(xp, zp, W_X, W_Z, W_O, B, C, theta, dt, A, lam, B_bias=None,
                     C_bias=None, state: State | None = None, bc_norm: bool = False,
                     norm_eps: float = 1e-6, nthreads: int = 0, dt_bias=None, flags: int = 0):
    """One token with the MIMO projections around the SSM (Appendix C):
        X[r][p] = W_X[h][r][p] X'[p],   Z[r][p] = W_Z[h][r][p] Z'[p],
        Y = the SSM output of X (decode_step),   Y' = Y * SiLU(Z),
        O'[p] = sum_r W_O[h][r][p] Y'[r][p],   SiLU(z) = z / (1 + e^{-z}).
    xp, zp [b,H,P]; W_X, W_Z, W_O [H,R,P] (per head: the reading of the paper's per-layer
    P x R weights with H heads). The new state's prev_x is X. Returns (O' [b,H,P], State)."""
    xp, zp = _f64(xp), _f64(zp)
    W_X, W_Z, W_O = _f64(W_X), _f64(W_Z), _f64(W_O)
    X = W_X[None] * xp[:, :, None, :]                      # [b,H,R,P]
    y, st = decode_step(X, B, C, theta, dt, A, lam, B_bias, C_bias, state, bc_norm, norm_eps,
                        nthreads, dt_bias, flags)
    Z = W_Z[None] * zp[:, :, None, :]
    silu = Z / (1.0 + np.exp(-Z))
    return (W_O[None] * y * silu).sum(axis=2), st
