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

from gpu_common import TOL, compare, oracle_scan, rel
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


def one_segment_scan(g, chunk, bc_norm, copies=80):
    """m3_scan_fwd on `copies` copies of the problem stacked along the batch: with that many
    (batch, head) units every SM is busy without cutting sequences, so each copy runs as one
    segment. Returns the first copy's y and final state."""
    t = g.tensors()
    rep = lambda v: v.repeat(copies, *([1] * (v.dim() - 1)))
    ts = {k: (rep(v) if (v is not None and k not in ("B_bias", "C_bias")) else v)
          for k, v in t.items()}
    st = m3.State.from_dict({k: rep(v) for k, v in g.state.items()})
    assert g.x.shape[0] * copies * g.x.shape[2] >= 2 * 148 + 1
    y, fin = m3.scan_fwd(**ts, init=st, chunk=chunk, bc_norm=bc_norm)
    b = g.x.shape[0]
    return y[:b], m3.State(fin.h[:b], fin.phi[:b], fin.prev_B[:b], fin.prev_x[:b])


def assert_identical(y_a, f_a, y_b, f_b):
    assert torch.equal(y_a, y_b)
    for k in ("h", "phi", "prev_B", "prev_x"):
        assert torch.equal(getattr(f_a, k), getattr(f_b, k)), k


def check_oracle(pr, y, fin):
    yo, so = oracle_scan(pr)
    compare(pr, y, fin, yo, so)


NOALLOC = [
    # problem, chunk, how m3_scan_fwd and the no-alloc call split the sequences
    (dict(b=2, L=200, H=4, R=1, seed=71), 64, "same"),    # one segment each
    (dict(b=3, L=333, H=8, R=4, seed=72), 16, "one"),     # two segments vs one (scratch)
    (dict(b=2, L=300, H=4, R=1, seed=73), 128, "same"),   # 128-row chunks: never cut
    (dict(b=2, L=150, H=4, R=4, seed=74), 32, "same"),
]


def test_noalloc_matches_scan_fwd_on_calls_in_a_row(cuda_dev):
    """Four calls in a row (SISO, then a longer MIMO problem that needs more scratch than the
    first left behind, then the 128-row-chunk kernel): bit-identical to m3_scan_fwd where
    both run the same segments, to m3_scan_fwd run as one segment per sequence where the
    no-alloc call's scratch holds fewer segment states, and within tolerance of the oracle."""
    for kw, chunk, split in NOALLOC:
        pr = make_problem(kw["b"], kw["L"], kw["H"], 1, 64, 128, rank=kw["R"], chunk=chunk,
                          bc_norm=True, bias_std=0.1, seed=kw["seed"], with_state=True)
        g = pr.to(cuda_dev)
        y_na, f_na = noalloc_scan(g, chunk, True)
        if split == "same":
            y_ref, f_ref = reference_scan(g, chunk, True)
        else:
            y_ref, f_ref = one_segment_scan(g, chunk, True)
        torch.cuda.synchronize()
        assert_identical(y_na, f_na, y_ref, f_ref)
        check_oracle(pr, y_na, f_na)


def test_noalloc_rejects_dims_beyond_its_scratch(cuda_dev):
    lib = m3.load_library()
    dims = m3.Dims(64, 4096, 64, 1, 64, 128, 1, 64, m3.M3_BF16, 1, 1e-6)  # 262144 rows
    fake = ctypes.c_void_p(0x10000)
    ins = m3.Inputs(*([fake] * 9))
    rc = lib.m3_scan_fwd_noalloc(ctypes.byref(dims), ctypes.byref(ins), None, None, fake, None)
    assert rc == m3.M3_ERR_UNSUPPORTED
    assert b"1 MiB" in lib.m3_last_error()


def test_noalloc_runs_long_sequences_in_fewer_segments(cuda_dev):
    """b1 H4 L2543 is cut into 5 segments by m3_scan_fwd; its 5 state slots per sequence
    (~0.6 MiB) plus the RMS scales fit the fixed scratch, so the no-alloc call runs the same
    5 segments: bit-identical. For b1 H32 L2543 one slot per sequence alone (~1 MiB) does
    not fit: it runs as one segment, bit-identical to m3_scan_fwd forced to one segment per
    sequence. Both within tolerance of the oracle."""
    for H, seed in ((4, 81), (32, 82)):
        pr = make_problem(1, 2543, H, 1, 64, 128, rank=1, chunk=64, bc_norm=True, bias_std=0.1,
                          seed=seed, with_state=True)
        g = pr.to(cuda_dev)
        y_na, f_na = noalloc_scan(g, 64, True)
        if H == 4:
            y_ref, f_ref = reference_scan(g, 64, True)
        else:
            y_ref, f_ref = one_segment_scan(g, 64, True, copies=10)
            y_seg, _ = reference_scan(g, 64, True)   # the segmented form differs by rounding
            torch.cuda.synchronize()
            assert not torch.equal(y_seg, y_na)
            assert rel(y_na, y_seg.double().cpu().numpy()) <= TOL[torch.bfloat16]
        torch.cuda.synchronize()
        assert_identical(y_na, f_na, y_ref, f_ref)
        check_oracle(pr, y_na, f_na)
