"""Shared helpers for the GPU parity tests: run the CUDA library and the oracle on the same
stored inputs and compare them with the tolerances of the workloads.

Tolerance rule: err = max|gpu - oracle| / max|oracle| per output tensor (y, and each field of
the final state), at most 1e-4 for fp32 inputs and 2e-2 for bf16 inputs with fp32 state.
"""
import os

import numpy as np
import torch

import oracle
from state_space_sequence_mamba_b200 import binding as m3

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}

# errors measured by every comparison of the run, by test id; written out at the end of the
# session when M3_PARITY_REPORT names a file (see conftest.py)
ERRORS: dict = {}


def record(errs: dict) -> None:
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    ERRORS.setdefault(test, []).append({k: float(v) for k, v in errs.items()})


def rel(g, o) -> float:
    g = g.detach().double().cpu().numpy() if torch.is_tensor(g) else np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    if o.size == 0:
        return 0.0
    return float(np.max(np.abs(g - o)) / max(float(np.max(np.abs(o))), 1e-30))


def oracle_state(st: dict | None):
    if st is None:
        return None
    return oracle.State(*(st[k].double().cpu().numpy() for k in ("h", "phi", "prev_B", "prev_x")))


def gpu_scan(pr, dev, use_state=True, chunk=None, final=True):
    g = pr.to(dev)
    init = m3.State.from_dict(g.state) if (use_state and g.state is not None) else None
    y, fin = m3.scan_fwd(**g.tensors(), **g.scalar_args(), init=init, final=final,
                         chunk=chunk or pr.dims.chunk, bc_norm=pr.dims.bc_norm)
    torch.cuda.synchronize()
    return y, fin


def oracle_scan(pr, use_state=True, heads=None, batches=None):
    """The oracle on problem pr, optionally on some heads and / or batch rows only."""
    t = pr.tensors()
    t.update(pr.scalar_args())
    st = pr.state if use_state else None
    if batches is not None:
        bs = torch.as_tensor(batches)
        for k in ("x", "B", "C", "theta", "dt", "A", "lam"):
            t[k] = t[k][bs]
        if st is not None:
            st = {k: v[bs] for k, v in st.items()}
    if heads is not None:
        hs = torch.as_tensor(heads)
        for k in ("x", "theta", "dt", "A", "lam"):
            t[k] = t[k][:, :, hs]
        for k in ("B_bias", "C_bias", "dt_bias"):
            if t[k] is not None:
                t[k] = t[k][hs]
        if st is not None:
            st = {k: v[:, hs] for k, v in st.items()}
        assert pr.dims.ngroups == 1
    return oracle.scan(**t, state=oracle_state(st), bc_norm=pr.dims.bc_norm,
                       norm_eps=pr.dims.norm_eps)


def compare(pr, y, fin, yo, so, heads=None, tol=None, batches=None):
    tol = tol or TOL[pr.dims.dtype]
    hs = slice(None) if heads is None else torch.as_tensor(heads)
    if batches is not None:
        bs = torch.as_tensor(batches, device=y.device)
        y = y[bs]
        if fin is not None:
            fin = type(fin)(*(getattr(fin, k)[bs] for k in ("h", "phi", "prev_B", "prev_x")))
    errs = {"y": rel(y[:, :, hs], yo)}
    if fin is not None:
        errs["h"] = rel(fin.h[:, hs], so.h)
        errs["phi"] = rel(fin.phi[:, hs], so.phi)
        # the previous-token fields are byte copies of inputs: exact
        errs["prev_B"] = rel(fin.prev_B[:, hs], so.prev_B)
        errs["prev_x"] = rel(fin.prev_x[:, hs], so.prev_x)
        assert errs["prev_B"] == 0.0 and errs["prev_x"] == 0.0, errs
    record(errs)
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"errors above {tol}: {errs}"
    return errs
