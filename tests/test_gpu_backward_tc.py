"""GPU parity of the chunked tensor-core backward (m3_scan_bwd without M3_BWD_FP32 on SISO
bf16 inputs with N = 128, P = 64 and H a multiple of 4) with the gradient oracle.

The chunk products run with bf16 operands and fp32 accumulators, as the forward scan's do, so
the bound is the bf16 one of the forward: max|gpu - oracle| / max|oracle| <= 2e-2 per gradient
tensor. The sums have a fixed order, so two runs give identical bits. The measured errors are
recorded (M3_PARITY_REPORT).
"""
import pytest
import torch

from test_gpu_backward import PER_HEAD, compare_grads, draw_grads, gpu_grads, oracle_grads
from state_space_sequence_mamba_b200 import binding as m3
from state_space_sequence_mamba_b200.inputs import make_config, make_problem

pytestmark = pytest.mark.gpu

TC_TOL = 2e-2
TC_KEYS = ("dx", "dB", "dC", "dtheta", "ddt", "dA", "dlam", "dB_bias", "dC_bias", "ddt_bias")

CASES = [
    # b, L, H, G, bc_norm, bias, state, raw, extra flags
    (1, 64, 4, 1, True, 0.1, True, False, 0),     # one full chunk
    (2, 150, 4, 2, True, 0.1, True, False, 0),    # ragged third chunk, two groups
    (1, 200, 8, 1, True, 0.1, True, True, 0),     # raw scalars
    (1, 100, 4, 1, True, 0.1, True, True, 4),     # raw scalars, zero-order hold
    (2, 65, 4, 1, False, 0.0, False, False, 0),   # no norm, no bias, fresh state
    (1, 1, 4, 1, True, 0.1, True, False, 0),      # one token
    (1, 129, 4, 4, True, 0.3, True, False, 0),    # G = H, a token past two chunks
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"b{c[0]}L{c[1]}H{c[2]}G{c[3]}"
                         f"n{int(c[4])}s{int(c[6])}raw{int(c[7])}z{c[8]}")
def test_tc_backward_matches_gradient_oracle(cuda_dev, case):
    b, L, H, G, norm, bias, state, raw, flags = case
    pr = make_problem(b, L, H, G, 64, 128, rank=1, chunk=64, dtype=torch.bfloat16,
                      bc_norm=norm, bias_std=bias, seed=1000 + L + H, with_state=state,
                      raw_scalars=raw)
    pr.flags |= flags
    dy, dfin = draw_grads(pr, seed=L + 3)
    got = gpu_grads(pr, dy, dfin, cuda_dev, exact=False)
    ref = oracle_grads(pr, dy, dfin)
    compare_grads(got, ref, keys=TC_KEYS, tol=TC_TOL)


def test_tc_backward_without_final_gradient(cuda_dev):
    pr = make_problem(1, 130, 4, 1, 64, 128, rank=1, chunk=64, dtype=torch.bfloat16,
                      bc_norm=True, bias_std=0.1, seed=41, with_state=True)
    dy, _ = draw_grads(pr, seed=5, with_final=False)
    got = gpu_grads(pr, dy, None, cuda_dev, exact=False)
    compare_grads(got, oracle_grads(pr, dy, None), keys=TC_KEYS, tol=TC_TOL)


def test_tc_backward_is_reproducible(cuda_dev):
    """Fixed summation order: two runs give the same bits in every gradient."""
    pr = make_problem(2, 300, 8, 1, 64, 128, rank=1, chunk=64, dtype=torch.bfloat16,
                      bc_norm=True, bias_std=0.1, seed=42, with_state=True)
    dy, dfin = draw_grads(pr, seed=6)
    a = gpu_grads(pr, dy, dfin, cuda_dev, exact=False)
    b = gpu_grads(pr, dy, dfin, cuda_dev, exact=False)
    for k in TC_KEYS:
        assert torch.equal(a[k], b[k]), k
    for f in ("h", "phi", "prev_B", "prev_x"):
        assert torch.equal(a["dinit"][f], b["dinit"][f]), f


def test_tc_backward_full_length_every_gradient(cuda_dev):
    """Every gradient element by element at the SISO workload's full length on a reduced head
    count (b1 H8 L2048), with a carried state."""
    pr = make_config(1, with_state=True, batch=1, nheads=8)
    dy, dfin = draw_grads(pr, seed=14)
    got = gpu_grads(pr, dy, dfin, cuda_dev, exact=False)
    compare_grads(got, oracle_grads(pr, dy, dfin), keys=TC_KEYS, tol=TC_TOL)


def test_tc_backward_full_size_sampled_heads(cuda_dev):
    """The SISO prefill workload (b4 H64 L2048) with a carried state: the per-head gradients
    and the initial-state gradients of sampled units against the oracle, and the gradients
    that sum over heads against the fp32 sequential path on the same inputs."""
    pr = make_config(1, with_state=True)
    dy, dfin = draw_grads(pr, seed=11)
    got = gpu_grads(pr, dy, dfin, cuda_dev, exact=False)
    heads, batches = [0, 37], [1, 3]
    ref = oracle_grads(pr, dy, dfin, heads=heads, batches=batches)
    compare_grads(got, ref, keys=PER_HEAD, heads=heads, batches=batches, tol=TC_TOL)
    exact = gpu_grads(pr, dy, dfin, cuda_dev, exact=True)
    for k in ("dB", "dC", "dB_bias", "dC_bias", "ddt_bias"):
        den = float(exact[k].abs().max())
        e = float((got[k] - exact[k]).abs().max())
        assert (e <= TC_TOL * den) if den > 0 else e == 0.0, (k, e, den)
