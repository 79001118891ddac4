"""GPU parity of the chunked tensor-core backward (m3_scan_bwd without M3_BWD_FP32 on bf16
inputs with N = 128, P = 64, R in {1, 2, 4, 8} and H a multiple of 4) with the gradient
oracle.

The chunk products run with bf16 operands and fp32 accumulators, as the forward scan's do, so
the bound is the bf16 one of the forward: max|gpu - oracle| / max|oracle| <= 2e-2 per gradient
tensor. The sums have a fixed order, so two runs give identical bits. The measured errors are
recorded (M3_PARITY_REPORT).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import record, rel
from test_gpu_backward import PER_HEAD, compare_grads, draw_grads, gpu_grads, oracle_grads
from state_space_sequence_mamba_b200 import binding as m3
from state_space_sequence_mamba_b200.inputs import make_config, make_problem

pytestmark = pytest.mark.gpu

TC_TOL = 2e-2
TC_KEYS = ("dx", "dB", "dC", "dtheta", "ddt", "dA", "dlam", "dB_bias", "dC_bias", "ddt_bias")


def compare_tc(got, ref, pr):
    """Every gradient within TC_TOL of max|oracle| per tensor, except the initial angle's:
    dPhi_{-1} is the last value of the angle adjoint's suffix sum over the sequence, whose
    per-token values dPhi_t = dtheta_t / dt_t are the other members of the same sum (checked
    through dtheta). Its terms nearly cancel (|dPhi_{-1}| can be 1/40 of sum_t |dl_t|), so its
    error is measured against the largest |dPhi_t| of that sum rather than against its own
    maximum."""
    errs = compare_grads(got, ref, keys=TC_KEYS, init=False, tol=TC_TOL)
    init = {}
    for f in ("h", "prev_B", "prev_x"):
        init["init_" + f] = rel(got["dinit"][f], getattr(ref["dinit"], f))
    dt, _ = oracle.step_scalars(pr.dt.double().numpy(), pr.lam.double().numpy(),
                                None if pr.dt_bias is None else pr.dt_bias.double().numpy(),
                                pr.flags)
    dphi_t = np.asarray(ref["dtheta"]) / dt[..., None]
    phi_ref = np.asarray(ref["dinit"].phi)
    den = max(float(np.abs(phi_ref).max()), float(np.abs(dphi_t).max()))
    init["init_phi"] = float((got["dinit"]["phi"].double().cpu().numpy() - phi_ref).__abs__().max()) / den
    record(init)
    bad = {k: v for k, v in init.items() if not v <= TC_TOL}
    assert not bad, f"initial-state gradient errors above {TC_TOL}: {init}"
    errs.update(init)
    return errs

CASES = [
    # b, L, H, G, bc_norm, bias, state, raw, extra flags, rank
    (1, 64, 4, 1, True, 0.1, True, False, 0),     # one full chunk
    (2, 150, 4, 2, True, 0.1, True, False, 0),    # ragged third chunk, two groups
    (1, 200, 8, 1, True, 0.1, True, True, 0),     # raw scalars
    (1, 100, 4, 1, True, 0.1, True, True, 4),     # raw scalars, zero-order hold
    (2, 65, 4, 1, False, 0.0, False, False, 0),   # no norm, no bias, fresh state
    (1, 1, 4, 1, True, 0.1, True, False, 0),      # one token
    (1, 129, 4, 4, True, 0.3, True, False, 0),    # G = H, a token past two chunks
    (2, 77, 4, 1, True, 0.1, True, False, 0, 2),  # MIMO R2: chunks of 32 tokens, ragged
    (1, 50, 4, 2, True, 0.1, True, False, 0, 4),  # MIMO R4: chunks of 16 tokens, two groups
    (1, 40, 4, 1, True, 0.1, True, True, 0, 4),   # MIMO R4, raw scalars
    (1, 30, 4, 1, True, 0.1, True, True, 4, 4),   # MIMO R4, raw scalars, zero-order hold
    (1, 21, 4, 1, True, 0.1, False, False, 0, 8), # MIMO R8: chunks of 8 tokens, fresh state
    (1, 1, 4, 1, True, 0.1, True, False, 0, 4),   # MIMO R4, one token
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"b{c[0]}L{c[1]}H{c[2]}G{c[3]}"
                         f"n{int(c[4])}s{int(c[6])}raw{int(c[7])}z{c[8]}R{c[9] if len(c) > 9 else 1}")
def test_tc_backward_matches_gradient_oracle(cuda_dev, case):
    b, L, H, G, norm, bias, state, raw, flags = case[:9]
    R = case[9] if len(case) > 9 else 1
    pr = make_problem(b, L, H, G, 64, 128, rank=R, chunk=64 // R, dtype=torch.bfloat16,
                      bc_norm=norm, bias_std=bias, seed=1000 + L + H, with_state=state,
                      raw_scalars=raw)
    pr.flags |= flags
    dy, dfin = draw_grads(pr, seed=L + 3)
    got = gpu_grads(pr, dy, dfin, cuda_dev, exact=False)
    compare_tc(got, oracle_grads(pr, dy, dfin), pr)


def test_tc_backward_without_final_gradient(cuda_dev):
    pr = make_problem(1, 130, 4, 1, 64, 128, rank=1, chunk=64, dtype=torch.bfloat16,
                      bc_norm=True, bias_std=0.1, seed=41, with_state=True)
    dy, _ = draw_grads(pr, seed=5, with_final=False)
    got = gpu_grads(pr, dy, None, cuda_dev, exact=False)
    compare_tc(got, oracle_grads(pr, dy, None), pr)


@pytest.mark.parametrize("R", [1, 4])
def test_tc_backward_is_reproducible(cuda_dev, R):
    """Fixed summation order: two runs give the same bits in every gradient, the bias and
    dt_bias sums over units included (raw scalars, so dt_bias has a gradient)."""
    pr = make_problem(2, 300, 8, 1, 64, 128, rank=R, chunk=64 // R, dtype=torch.bfloat16,
                      bc_norm=True, bias_std=0.1, seed=42, with_state=True, raw_scalars=True)
    dy, dfin = draw_grads(pr, seed=6)
    a = gpu_grads(pr, dy, dfin, cuda_dev, exact=False)
    b = gpu_grads(pr, dy, dfin, cuda_dev, exact=False)
    for k in TC_KEYS:
        assert torch.equal(a[k], b[k]), k
    for f in ("h", "phi", "prev_B", "prev_x"):
        assert torch.equal(a["dinit"][f], b["dinit"][f]), f


@pytest.mark.parametrize("cfg,kw", [(1, dict(batch=1, nheads=8)),
                                    (2, dict(batch=1, nheads=4, seqlen=1024))])
def test_tc_backward_full_length_every_gradient(cuda_dev, cfg, kw):
    """Every gradient element by element at the workloads' full length on a reduced head
    count (SISO b1 H8 L2048; MIMO R4 b1 H4 L1024), with a carried state."""
    pr = make_config(cfg, with_state=True, **kw)
    dy, dfin = draw_grads(pr, seed=14 + cfg)
    got = gpu_grads(pr, dy, dfin, cuda_dev, exact=False)
    compare_tc(got, oracle_grads(pr, dy, dfin), pr)


@pytest.mark.parametrize("cfg,kw", [(1, {}), (2, dict(seqlen=512))])
def test_tc_backward_full_size_sampled_heads(cuda_dev, cfg, kw):
    """The prefill workloads (SISO b4 H64 L2048; MIMO R4 b4 H64 at L512) with a carried
    state: the per-head gradients and the initial-state gradients of sampled units against
    the oracle, and the gradients that sum over heads against the fp32 sequential path on
    the same inputs."""
    pr = make_config(cfg, with_state=True, **kw)
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
