"""ctypes binding of the C ABI in include/m3.h. Argument marshalling only.

torch supplies device memory and streams; every step of the computation runs in the CUDA
kernels of ``libm3.so``. If the library is missing this module raises: there is no fallback
implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libm3.so")

M3_OK, M3_ERR_INVALID_ARG, M3_ERR_UNSUPPORTED, M3_ERR_CUDA, M3_ERR_TIMEOUT = range(5)
M3_F32, M3_BF16 = 0, 1
# m3_dims.flags: the step scalars arrive raw and the kernels apply softplus / sigmoid; the
# zero-order-hold discretisation; the backward in fp32 on the CUDA cores
M3_DT_SOFTPLUS, M3_LAM_SIGMOID, M3_DISC_ZOH, M3_BWD_FP32 = 1, 2, 4, 8
BWD_FP32 = M3_BWD_FP32


class M3Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"m3 status {status}: {msg}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64),
                ("rank", ctypes.c_int64), ("chunk", ctypes.c_int64),
                ("in_dtype", ctypes.c_int32), ("bc_norm", ctypes.c_int32),
                ("norm_eps", ctypes.c_float), ("flags", ctypes.c_uint32)]


class Inputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("x", "B", "C", "theta", "dt", "A", "lam", "B_bias", "C_bias", "dt_bias")]


class StateC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("h", "phi", "prev_B", "prev_x")]


class SegState(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("h", "phi", "lam_sum")]


class Proj(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("x_in", "z_in", "W_X", "W_Z", "W_O")]


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dx", "dB", "dC", "dtheta", "ddt", "dA", "dlam",
                                               "dB_bias", "dC_bias", "ddt_bias")]


# Symbols include/m3.h declares (checked by the CPU test suite).
EXPORTS = ("m3_scan_workspace_bytes", "m3_scan_fwd", "m3_decode_step", "m3_scan_check",
           "m3_status_str", "m3_last_error", "m3_scan_fwd_noalloc", "m3_decode_step_proj",
           "m3_scan_state", "m3_state_combine", "m3_scan_bwd_workspace_bytes", "m3_scan_bwd")

_lib = None


def load_library(path: str = LIB_PATH):
    """Loads libm3.so and declares the signatures. Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m state_space_sequence_mamba_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    lib.m3_scan_workspace_bytes.argtypes = [P(Dims)]
    lib.m3_scan_workspace_bytes.restype = ctypes.c_size_t
    lib.m3_scan_fwd.argtypes = [P(Dims), P(Inputs), P(StateC), P(StateC), ctypes.c_void_p,
                                ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    lib.m3_scan_fwd.restype = ctypes.c_int
    lib.m3_decode_step.argtypes = [P(Dims), P(Inputs), P(StateC), P(StateC), ctypes.c_void_p,
                                   ctypes.c_void_p]
    lib.m3_decode_step.restype = ctypes.c_int
    lib.m3_decode_step_proj.argtypes = [P(Dims), P(Inputs), P(Proj), P(StateC), P(StateC),
                                        ctypes.c_void_p, ctypes.c_void_p]
    lib.m3_decode_step_proj.restype = ctypes.c_int
    lib.m3_scan_state.argtypes = [P(Dims), P(Inputs), P(StateC), P(SegState), ctypes.c_void_p,
                                  ctypes.c_size_t, ctypes.c_void_p]
    lib.m3_scan_state.restype = ctypes.c_int
    lib.m3_state_combine.argtypes = [P(Dims), ctypes.c_int, P(SegState), ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p]
    lib.m3_state_combine.restype = ctypes.c_int
    lib.m3_scan_bwd_workspace_bytes.argtypes = [P(Dims)]
    lib.m3_scan_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.m3_scan_bwd.argtypes = [P(Dims), P(Inputs), P(StateC), ctypes.c_void_p, P(StateC),
                                P(Grads), P(StateC), ctypes.c_void_p, ctypes.c_size_t,
                                ctypes.c_void_p]
    lib.m3_scan_bwd.restype = ctypes.c_int
    lib.m3_scan_check.argtypes = [ctypes.c_void_p]
    lib.m3_scan_check.restype = ctypes.c_int
    lib.m3_status_str.argtypes = [ctypes.c_int]
    lib.m3_status_str.restype = ctypes.c_char_p
    lib.m3_last_error.argtypes = []
    lib.m3_last_error.restype = ctypes.c_char_p
    lib.m3_scan_fwd_noalloc.argtypes = [P(Dims), P(Inputs), P(StateC), P(StateC),
                                        ctypes.c_void_p, ctypes.c_void_p]
    lib.m3_scan_fwd_noalloc.restype = ctypes.c_int
    _lib = lib
    return lib


def _check(rc: int):
    if rc != M3_OK:
        lib = load_library()
        raise M3Error(rc, lib.m3_last_error().decode() or lib.m3_status_str(rc).decode())


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return M3_BF16
    if dt == torch.float32:
        return M3_F32
    raise ValueError(f"unsupported input dtype {dt}")


class State:
    """Device state of every (batch, head) unit: h [b,H,N,P] fp32, phi [b,H,N/2] fp32,
    prev_B [b,H,R,N] and prev_x [b,H,R,P] in the input dtype."""

    def __init__(self, h, phi, prev_B, prev_x):
        self.h, self.phi, self.prev_B, self.prev_x = h, phi, prev_B, prev_x

    @staticmethod
    def empty(batch, nheads, dstate, headdim, rank, dtype, device):
        return State(torch.empty(batch, nheads, dstate, headdim, device=device),
                     torch.empty(batch, nheads, dstate // 2, device=device),
                     torch.empty(batch, nheads, rank, dstate, dtype=dtype, device=device),
                     torch.empty(batch, nheads, rank, headdim, dtype=dtype, device=device))

    @staticmethod
    def from_dict(d):
        return State(d["h"], d["phi"], d["prev_B"], d["prev_x"])

    def as_dict(self):
        return dict(h=self.h, phi=self.phi, prev_B=self.prev_B, prev_x=self.prev_x)

    def c(self):
        return StateC(*(_ptr(t) for t in (self.h, self.phi, self.prev_B, self.prev_x)))


def make_dims(x, B, chunk, bc_norm, norm_eps, flags=0):
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    return Dims(b, L, H, G, P, N, R, int(chunk), _dtype_code(x.dtype), 1 if bc_norm else 0,
                float(norm_eps), int(flags))


def scan_workspace_bytes(dims: Dims) -> int:
    return int(load_library().m3_scan_workspace_bytes(ctypes.byref(dims)))


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def scan_fwd(x, B, C, theta, dt, A, lam, B_bias=None, C_bias=None, init: State | None = None,
             final: State | None | bool = True, y=None, workspace=None, chunk=64,
             bc_norm=False, norm_eps=1e-6, stream=None, dt_bias=None, flags=0):
    """m3_scan_fwd on torch CUDA tensors (shapes as in include/m3.h). ``flags``
    (M3_DT_SOFTPLUS | M3_LAM_SIGMOID) passes dt and lam raw, with ``dt_bias`` [H].

    ``final=True`` allocates a new State for the result, ``False``/None skips it, or pass a
    State (it may be ``init`` itself). Returns (y, final State or None)."""
    lib = load_library()
    dims = make_dims(x, B, chunk, bc_norm, norm_eps, flags)
    dev = x.device
    if y is None:
        y = torch.empty_like(x)
    if final is True:
        final = State.empty(dims.batch, dims.nheads, dims.dstate, dims.headdim, dims.rank,
                            x.dtype, dev)
    elif final is False:
        final = None
    need = scan_workspace_bytes(dims)
    if need == 0:
        # invalid or unsupported dims: let the call report why
        need = 256
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    ins = Inputs(*(_ptr(t) for t in (x, B, C, theta, dt, A, lam, B_bias, C_bias, dt_bias)))
    ic = init.c() if init is not None else None
    fc = final.c() if final is not None else None
    rc = lib.m3_scan_fwd(ctypes.byref(dims), ctypes.byref(ins),
                         ctypes.byref(ic) if ic is not None else None,
                         ctypes.byref(fc) if fc is not None else None,
                         _ptr(y), _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(rc)
    return y, final


def scan_check(workspace):
    _check(load_library().m3_scan_check(_ptr(workspace)))


def decode_step(x, B, C, theta, dt, A, lam, B_bias=None, C_bias=None, state_in: State = None,
                state_out: State | None = None, y=None, bc_norm=False, norm_eps=1e-6,
                stream=None, dt_bias=None, flags=0):
    """m3_decode_step: x [b,1,H,R,P], B, C [b,1,G,R,N], theta [b,1,H,N/2], dt/A/lam [b,1,H].

    ``state_out`` defaults to ``state_in`` (in-place). Returns (y [b,H,R,P], state_out)."""
    lib = load_library()
    dims = make_dims(x, B, 1, bc_norm, norm_eps, flags)
    if state_out is None:
        state_out = state_in
    if y is None:
        y = torch.empty(dims.batch, dims.nheads, dims.rank, dims.headdim, dtype=x.dtype,
                        device=x.device)
    ins = Inputs(*(_ptr(t) for t in (x, B, C, theta, dt, A, lam, B_bias, C_bias, dt_bias)))
    si, so = state_in.c(), state_out.c()
    rc = lib.m3_decode_step(ctypes.byref(dims), ctypes.byref(ins), ctypes.byref(si),
                            ctypes.byref(so), _ptr(y), _stream_handle(stream))
    _check(rc)
    return y, state_out


def decode_step_proj(xp, zp, W_X, W_Z, W_O, B, C, theta, dt, A, lam, B_bias=None, C_bias=None,
                     state_in: State = None, state_out: State | None = None, o=None,
                     bc_norm=False, norm_eps=1e-6, stream=None, dt_bias=None, flags=0):
    """m3_decode_step_proj: one token with the MIMO projections. xp, zp [b,1,H,P] (X', Z');
    W_X, W_Z, W_O [H,R,P] fp32; B, C [b,1,G,R,N]; theta [b,1,H,N/2]; dt/A/lam [b,1,H].
    ``state_out`` defaults to ``state_in``. Returns (O' [b,H,P], state_out)."""
    lib = load_library()
    b, _, H, P = xp.shape
    R = W_X.shape[1]
    dims = make_dims(xp.reshape(b, 1, H, 1, P).expand(b, 1, H, R, P), B, 1, bc_norm, norm_eps,
                     flags)
    if state_out is None:
        state_out = state_in
    if o is None:
        o = torch.empty(b, H, P, dtype=xp.dtype, device=xp.device)
    ins = Inputs(*(_ptr(t) for t in (None, B, C, theta, dt, A, lam, B_bias, C_bias, dt_bias)))
    pr = Proj(*(_ptr(t) for t in (xp, zp, W_X, W_Z, W_O)))
    si, so = state_in.c(), state_out.c()
    rc = lib.m3_decode_step_proj(ctypes.byref(dims), ctypes.byref(ins), ctypes.byref(pr),
                                 ctypes.byref(si), ctypes.byref(so), _ptr(o),
                                 _stream_handle(stream))
    _check(rc)
    return o, state_out


def scan_state(x, B, C, theta, dt, A, lam, B_bias=None, C_bias=None, init: State | None = None,
               chunk=64, bc_norm=False, norm_eps=1e-6, stream=None, dt_bias=None, flags=0,
               workspace=None):
    """m3_scan_state: the state after the last token (h [b,H,N,P], phi [b,H,N/2]) and the summed
    log-decay [b,H], without y. Returns (h, phi, lam_sum)."""
    lib = load_library()
    dims = make_dims(x, B, chunk, bc_norm, norm_eps, flags)
    b, L, H, R, P = x.shape
    N = B.shape[4]
    dev = x.device
    h = torch.empty(b, H, N, P, device=dev)
    phi = torch.empty(b, H, N // 2, device=dev)
    lam_sum = torch.empty(b, H, device=dev)
    if workspace is None:
        workspace = torch.zeros(max(256, scan_workspace_bytes(dims)), dtype=torch.uint8,
                                device=dev)
    ins = Inputs(*(_ptr(t) for t in (x, B, C, theta, dt, A, lam, B_bias, C_bias, dt_bias)))
    ic = init.c() if init is not None else None
    out = SegState(_ptr(h), _ptr(phi), _ptr(lam_sum))
    rc = lib.m3_scan_state(ctypes.byref(dims), ctypes.byref(ins),
                           ctypes.byref(ic) if ic is not None else None, ctypes.byref(out),
                           _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(rc)
    return h, phi, lam_sum


def state_combine(h, phi, lam_sum, stream=None):
    """m3_state_combine on stacked segment states h [S,b,H,N,P], phi [S,b,H,N/2], lam_sum
    [S,b,H]: the state after segment S-1. Returns (h [b,H,N,P], phi [b,H,N/2])."""
    lib = load_library()
    S, b, H, N, P = h.shape
    dims = Dims(b, 1, H, 1, P, N, 1, 1, M3_F32, 0, 1e-6, 0)
    h_out = torch.empty(b, H, N, P, device=h.device)
    phi_out = torch.empty(b, H, N // 2, device=h.device)
    seg = SegState(_ptr(h), _ptr(phi), _ptr(lam_sum))
    rc = lib.m3_state_combine(ctypes.byref(dims), int(S), ctypes.byref(seg), _ptr(h_out),
                              _ptr(phi_out), _stream_handle(stream))
    _check(rc)
    return h_out, phi_out


def scan_bwd_workspace_bytes(dims: Dims) -> int:
    return int(load_library().m3_scan_bwd_workspace_bytes(ctypes.byref(dims)))


def scan_bwd(x, B, C, theta, dt, A, lam, dy, B_bias=None, C_bias=None, init: State | None = None,
             dfinal: dict | None = None, bc_norm=False, norm_eps=1e-6, stream=None, dt_bias=None,
             flags=0, want_init=True, workspace=None):
    """m3_scan_bwd: gradients of sum(y * dy) + <final state, dfinal> for the forward that
    scan_fwd runs on the same arguments. ``dfinal``: dict of fp32 h, phi, prev_B, prev_x (any
    may be missing = 0). Returns a dict of fp32 tensors dx, dB, dC, dtheta, ddt, dA, dlam,
    dB_bias, dC_bias, ddt_bias and (with want_init) dinit, a dict of the initial state's."""
    lib = load_library()
    dims = make_dims(x, B, 1, bc_norm, norm_eps, flags)
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    dev = x.device
    f32 = dict(device=dev, dtype=torch.float32)
    g = dict(dx=torch.empty(b, L, H, R, P, **f32), dB=torch.empty(b, L, G, R, N, **f32),
             dC=torch.empty(b, L, G, R, N, **f32), dtheta=torch.empty(b, L, H, N // 2, **f32),
             ddt=torch.empty(b, L, H, **f32), dA=torch.empty(b, L, H, **f32),
             dlam=torch.empty(b, L, H, **f32), dB_bias=torch.empty(H, R, N, **f32),
             dC_bias=torch.empty(H, R, N, **f32), ddt_bias=torch.empty(H, **f32))
    gc = Grads(*(_ptr(g[k]) for k in ("dx", "dB", "dC", "dtheta", "ddt", "dA", "dlam",
                                       "dB_bias", "dC_bias", "ddt_bias")))
    dinit = None
    if want_init:
        dinit = dict(h=torch.empty(b, H, N, P, **f32), phi=torch.empty(b, H, N // 2, **f32),
                     prev_B=torch.empty(b, H, R, N, **f32), prev_x=torch.empty(b, H, R, P, **f32))
    if workspace is None:
        workspace = torch.empty(max(256, scan_bwd_workspace_bytes(dims)), dtype=torch.uint8,
                                device=dev)
    ins = Inputs(*(_ptr(t) for t in (x, B, C, theta, dt, A, lam, B_bias, C_bias, dt_bias)))
    ic = init.c() if init is not None else None
    df = None
    if dfinal is not None:
        df = StateC(*(_ptr(dfinal.get(k)) for k in ("h", "phi", "prev_B", "prev_x")))
    di = StateC(*(_ptr(dinit[k]) for k in ("h", "phi", "prev_B", "prev_x"))) if dinit else None
    rc = lib.m3_scan_bwd(ctypes.byref(dims), ctypes.byref(ins),
                         ctypes.byref(ic) if ic is not None else None, _ptr(dy),
                         ctypes.byref(df) if df is not None else None, ctypes.byref(gc),
                         ctypes.byref(di) if di is not None else None, _ptr(workspace),
                         workspace.numel(), _stream_handle(stream))
    _check(rc)
    g["dinit"] = dinit
    return g
