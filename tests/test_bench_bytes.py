"""The algorithmic byte counts behind the benchmark's roofline fractions.

bench.py divides `scan_bytes` (forward) and `bwd_bytes` (backward) by the measured time.
These tests recount both from the sizes of the tensors themselves. Every input is read
once, and every output and gradient (fp32) is written once. The tests also pin the figures
that the measurement notes quote for the workloads.
"""
import importlib.util
import os
from types import SimpleNamespace

import torch

from state_space_sequence_mamba_b200.inputs import Dims, make_problem

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def test_scan_bytes_recount():
    bench = _bench()
    pr = make_problem(2, 10, 4, 2, 16, 32, rank=2, dtype=torch.bfloat16, bias_std=0.1, seed=1)
    inputs = sum(nbytes(v) for v in pr.tensors().values())
    y = nbytes(pr.x)
    b, H, N, P, R = 2, 4, 32, 16, 2
    final = b * H * (N * P * 4 + N // 2 * 4 + R * N * 2 + R * P * 2)
    assert bench.scan_bytes(pr) == inputs + y + final


def test_bwd_bytes_recount():
    bench = _bench()
    pr = make_problem(2, 10, 4, 2, 16, 32, rank=2, dtype=torch.bfloat16, bias_std=0.1, seed=1,
                      with_state=True)
    t = pr.tensors()
    dy = torch.empty_like(pr.x)
    reads = sum(nbytes(v) for v in t.values()) + nbytes(dy) + sum(nbytes(v) for v in pr.state.values())
    f32 = lambda v: v.numel() * 4
    writes = (f32(pr.x) + f32(pr.B) + f32(pr.C) + f32(pr.theta) + f32(pr.dt) * 3
              + f32(t["B_bias"]) * 2 + sum(f32(v) for v in pr.state.values()))
    assert bench.bwd_bytes(pr) == reads + writes


def test_quoted_workload_bytes():
    bench = _bench()
    # SISO prefill b4 H64 P64 N128 L2048 bf16 with biases; MIMO R4 the same shapes
    for R, bwd_b in ((1, 512262144), (4, 1356595200)):
        d = Dims(4, 2048, 64, 1, 64, 128, R, 64 // R, torch.bfloat16, True, 1e-6)
        fake = SimpleNamespace(dims=d, state={"h": None})
        assert bench.bwd_bytes(fake) == bwd_b
    pr = make_problem(4, 2048, 64, 1, 64, 128, rank=1, dtype=torch.bfloat16, bc_norm=True,
                      bias_std=0.1, seed=1)
    assert bench.scan_bytes(pr) == 220430336


def test_backward_form_follows_the_library():
    """The form the backward bench line reports is the one the library picks: the chunked
    tensor-core form for the bf16 prefill workloads (SISO and MIMO R4), the fp32 sweeps with
    M3_BWD_FP32, for fp32 inputs and for a head size the chunked form does not take."""
    from state_space_sequence_mamba_b200 import binding as m3
    from state_space_sequence_mamba_b200.inputs import make_config
    b = _bench()
    for cfg in (1, 2):
        pr = make_config(cfg, with_state=True, batch=1, nheads=4, seqlen=64)
        dims = m3.make_dims(pr.x, pr.B, 1, True, 1e-6, 0)
        assert b.bwd_chunked(m3, dims), cfg
        dims.flags = m3.BWD_FP32
        assert not b.bwd_chunked(m3, dims), cfg
    for kw in (dict(dtype=torch.float32), dict(P=32)):
        P = kw.get("P", 64)
        pr = make_problem(1, 64, 4, 1, P, 128, rank=1, chunk=64,
                          dtype=kw.get("dtype", torch.bfloat16), bc_norm=True, seed=3)
        dims = m3.make_dims(pr.x, pr.B, 1, True, 1e-6, 0)
        assert not b.bwd_chunked(m3, dims), kw
