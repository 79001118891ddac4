"""m3_scan_fwd_noalloc, the prefill scan for callers that cannot allocate device memory when
they run it (a serving runtime whose device memory is all planned before it starts, or a
step whose memory is fixed in advance). It takes its scratch from a fixed array inside the
library instead of a caller-provided workspace, so its results must be those of m3_scan_fwd.

The file is named to be collected last: a run that stops at the first failure has then
already run every other test. It also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

from gpu_common import TOL, rel
from state_space_sequence_mamba_b200 import binding as m3
from state_space_sequence_mamba_b200.inputs import make_problem

pytestmark = pytest.mark.gpu


def noalloc_scan(g, chunk, bc_norm):
    """Calls m3_scan_fwd_noalloc through the C ABI on the device tensors of problem g."""
    lib = m3.load_library()
    dims = m3.make_dims(g.x, g.B, chunk, bc_norm, 1e-6)
    y = torch.empty_like(g.x)
    fin = m3.State.empty(dims.batch, dims.nheads, dims.dstate, dims.headdim, dims.rank,
                         g.x.dtype, g.x.device)
    ins = m3.Inputs(*(m3._ptr(t) for t in (g.x, g.B, g.C, g.theta, g.dt, g.A, g.lam,
                                           g.B_bias, g.C_bias)))
    init = m3.State.from_dict(g.state).c()
    fc = fin.c()
    rc = lib.m3_scan_fwd_noalloc(ctypes.byref(dims), ctypes.byref(ins), ctypes.byref(init),
                                 ctypes.byref(fc), m3._ptr(y),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    m3._check(rc)
    return y, fin


def reference_scan(g, chunk, bc_norm):
    return m3.scan_fwd(**g.tensors(), init=m3.State.from_dict(g.state), chunk=chunk,
                       bc_norm=bc_norm)


def test_noalloc_matches_scan_fwd_on_two_calls_in_a_row(cuda_dev):
    # SISO with BC normalisation (tensor-core path, per-token scales in the scratch), then a
    # longer MIMO problem that needs more scratch than the first left behind.
    cases = [
        (make_problem(2, 200, 4, 1, 64, 128, rank=1, chunk=64, bc_norm=True, bias_std=0.1,
                      seed=71, with_state=True), 64),
        (make_problem(3, 333, 8, 1, 64, 128, rank=4, chunk=16, bc_norm=True, bias_std=0.1,
                      seed=72, with_state=True), 16),
    ]
    for pr, chunk in cases:
        g = pr.to(cuda_dev)
        y_na, f_na = noalloc_scan(g, chunk, True)
        y_ref, f_ref = reference_scan(g, chunk, True)
        torch.cuda.synchronize()
        tol = TOL[torch.bfloat16]
        assert rel(y_na, y_ref.double().cpu().numpy()) <= tol
        assert rel(f_na.h, f_ref.h.double().cpu().numpy()) <= tol
        assert rel(f_na.phi, f_ref.phi.double().cpu().numpy()) <= tol
        assert torch.equal(f_na.prev_B, f_ref.prev_B) and torch.equal(f_na.prev_x, f_ref.prev_x)


def test_noalloc_rejects_dims_beyond_its_scratch(cuda_dev):
    lib = m3.load_library()
    dims = m3.Dims(64, 4096, 64, 1, 64, 128, 1, 64, m3.M3_BF16, 1, 1e-6)  # 262144 rows
    fake = ctypes.c_void_p(0x10000)
    ins = m3.Inputs(*([fake] * 9))
    rc = lib.m3_scan_fwd_noalloc(ctypes.byref(dims), ctypes.byref(ins), None, None, fake, None)
    assert rc == m3.M3_ERR_UNSUPPORTED
    assert b"1 MiB" in lib.m3_last_error()


def test_noalloc_runs_long_sequences_in_fewer_segments(cuda_dev):
    # b1 H4 L2543 is cut into 5 segments by m3_scan_fwd; its 5 state slots per sequence
    # (~0.6 MiB) plus the RMS scales fit the fixed scratch. For b1 H32 L2543 one slot per
    # sequence alone (~1 MiB) does not: it runs as one segment. Both must match m3_scan_fwd.
    for H, seed in ((4, 81), (32, 82)):
        pr = make_problem(1, 2543, H, 1, 64, 128, rank=1, chunk=64, bc_norm=True, bias_std=0.1,
                          seed=seed, with_state=True)
        g = pr.to(cuda_dev)
        y_na, f_na = noalloc_scan(g, 64, True)
        y_ref, f_ref = reference_scan(g, 64, True)
        torch.cuda.synchronize()
        tol = TOL[torch.bfloat16]
        assert rel(y_na, y_ref.double().cpu().numpy()) <= tol
        assert rel(f_na.h, f_ref.h.double().cpu().numpy()) <= tol
