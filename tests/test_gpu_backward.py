"""GPU parity of the backward pass (m3_scan_bwd) with the gradient oracle (oracle/grad.py).

Both sides take the same stored inputs (bf16 inputs are compared after the same rounding),
so the only difference is the kernels' fp32 arithmetic. Tolerance: for every gradient tensor
max|gpu - oracle| / max|oracle| <= 1e-4, the bound of the fp32 forward. fp32 sums over L
tokens and over N * P, and the decay gradient's suffix sum over the sequence, stay near
1e-6 relative even at L = 2048; the measured errors are recorded (M3_PARITY_REPORT).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import grad as og
from gpu_common import oracle_state, record, rel
from state_space_sequence_mamba_b200 import binding as m3
from state_space_sequence_mamba_b200.inputs import make_config, make_problem

pytestmark = pytest.mark.gpu

GTOL = 1e-4
KEYS = ("dx", "dB", "dC", "dtheta", "ddt", "dA", "dlam", "dB_bias", "dC_bias", "ddt_bias")
PER_HEAD = ("dx", "dtheta", "ddt", "dA", "dlam")


def draw_grads(pr, seed, with_final=True):
    d = pr.dims
    g = torch.Generator().manual_seed(seed)
    b, L, H, R, P, N = d.batch, d.seqlen, d.nheads, d.rank, d.headdim, d.dstate
    dy = torch.randn(b, L, H, R, P, generator=g).to(d.dtype)
    if not with_final:
        return dy, None
    dfin = dict(h=torch.randn(b, H, N, P, generator=g), phi=torch.randn(b, H, N // 2, generator=g),
                prev_B=torch.randn(b, H, R, N, generator=g), prev_x=torch.randn(b, H, R, P, generator=g))
    return dy, dfin


def gpu_grads(pr, dy, dfin, dev, exact=True):
    """exact: the fp32 sequential sweeps (M3_BWD_FP32); else the path m3_scan_bwd picks, the
    chunked tensor-core form where it applies."""
    g = pr.to(dev)
    init = m3.State.from_dict(g.state) if g.state is not None else None
    sa = g.scalar_args()
    if exact:
        sa["flags"] = sa["flags"] | m3.BWD_FP32
    out = m3.scan_bwd(**g.tensors(), dy=dy.to(dev), **sa, init=init,
                      dfinal=None if dfin is None else {k: v.to(dev) for k, v in dfin.items()},
                      bc_norm=pr.dims.bc_norm, norm_eps=pr.dims.norm_eps)
    torch.cuda.synchronize()
    return out


def oracle_grads(pr, dy, dfin, heads=None, batches=None):
    t = pr.tensors()
    t.update(pr.scalar_args())
    st = pr.state
    bs = slice(None) if batches is None else torch.as_tensor(batches)
    if heads is not None:
        hs = torch.as_tensor(heads)
        assert pr.dims.ngroups == 1
        for k in ("x", "theta", "dt", "A", "lam"):
            t[k] = t[k][:, :, hs]
        for k in ("B_bias", "C_bias", "dt_bias"):
            if t[k] is not None:
                t[k] = t[k][hs]
        st = None if st is None else {k: v[:, hs] for k, v in st.items()}
        dy = dy[:, :, hs]
        dfin = None if dfin is None else {k: v[:, hs] for k, v in dfin.items()}
    if batches is not None:
        for k in ("x", "B", "C", "theta", "dt", "A", "lam"):
            t[k] = t[k][bs]
        st = None if st is None else {k: v[bs] for k, v in st.items()}
        dy = dy[bs]
        dfin = None if dfin is None else {k: v[bs] for k, v in dfin.items()}
    dfs = None if dfin is None else oracle.State(
        *(dfin[k].double().numpy() for k in ("h", "phi", "prev_B", "prev_x")))
    return og.scan_grad(**t, state=oracle_state(st), dy=dy, dfinal=dfs,
                        bc_norm=pr.dims.bc_norm, norm_eps=pr.dims.norm_eps)


def compare_grads(got, ref, keys=KEYS, init=True, heads=None, batches=None, tol=GTOL):
    hs = slice(None) if heads is None else torch.as_tensor(heads)
    bs = slice(None) if batches is None else torch.as_tensor(batches)
    errs = {}
    for k in keys:
        g = got[k]
        if heads is not None or batches is not None:
            g = g[bs][:, :, hs] if k in PER_HEAD else g
        errs[k] = rel(g, ref[k])
    if init:
        for f in ("h", "phi", "prev_B", "prev_x"):
            g = got["dinit"][f][bs][:, hs]
            errs["init_" + f] = rel(g, getattr(ref["dinit"], f))
    record(errs)
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"gradient errors above {tol}: {errs}"
    return errs


CASES = [
    # b, L, H, G, P, N, R, dtype, bc_norm, bias, state, raw, extra flags
    (2, 100, 4, 2, 16, 32, 1, torch.float32, True, 0.1, True, False, 0),   # ragged chunks
    (1, 37, 2, 1, 64, 128, 1, torch.bfloat16, True, 0.1, True, False, 0),
    (2, 50, 2, 1, 64, 128, 2, torch.bfloat16, True, 0.1, True, False, 0),
    (1, 33, 2, 2, 64, 128, 4, torch.bfloat16, True, 0.1, True, False, 0),
    (1, 9, 2, 1, 32, 64, 8, torch.float32, True, 0.1, True, False, 0),
    (2, 40, 2, 1, 128, 64, 1, torch.bfloat16, False, 0.0, False, False, 0),  # fresh state
    (1, 48, 2, 1, 32, 256, 1, torch.float32, True, 0.1, True, False, 0),   # 512 threads
    (1, 21, 3, 1, 16, 16, 2, torch.float32, True, 0.1, True, False, 0),    # one warp
    (2, 64, 2, 1, 64, 128, 1, torch.bfloat16, True, 0.1, True, True, 0),   # raw scalars
    (1, 45, 2, 1, 64, 128, 2, torch.float32, True, 0.1, True, False, 4),   # zero-order hold
    (1, 30, 2, 1, 64, 128, 4, torch.bfloat16, True, 0.1, True, True, 4),   # raw + ZOH
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"L{c[1]}H{c[2]}G{c[3]}P{c[4]}N{c[5]}R{c[6]}"
                         f"{'bf' if c[7] == torch.bfloat16 else 'f32'}raw{int(c[11])}z{c[12]}")
def test_backward_matches_gradient_oracle(cuda_dev, case):
    b, L, H, G, P, N, R, dt, norm, bias, state, raw, flags = case
    pr = make_problem(b, L, H, G, P, N, rank=R, chunk=16, dtype=dt, bc_norm=norm,
                      bias_std=bias, seed=L + 7 * R + P, with_state=state, raw_scalars=raw)
    pr.flags |= flags
    dy, dfin = draw_grads(pr, seed=L + R)
    got = gpu_grads(pr, dy, dfin, cuda_dev)
    ref = oracle_grads(pr, dy, dfin)
    compare_grads(got, ref)


@pytest.mark.parametrize("L", [1, 16, 17])
def test_backward_short_sequences(cuda_dev, L):
    """One token, exactly one staged chunk, one chunk and a token; no final-state gradient."""
    pr = make_problem(1, L, 2, 1, 64, 128, rank=1, dtype=torch.float32, bc_norm=True,
                      bias_std=0.1, seed=300 + L, with_state=True)
    dy, _ = draw_grads(pr, seed=L, with_final=False)
    got = gpu_grads(pr, dy, None, cuda_dev)
    compare_grads(got, oracle_grads(pr, dy, None))


def test_backward_partial_final_gradient(cuda_dev):
    """Only the final h has a gradient (NULL phi, prev_B, prev_x count as zero)."""
    pr = make_problem(2, 40, 2, 1, 64, 128, rank=1, dtype=torch.bfloat16, bc_norm=True,
                      bias_std=0.1, seed=77, with_state=True, raw_scalars=True)
    dy, dfin = draw_grads(pr, seed=3)
    part = {"h": dfin["h"]}
    got = gpu_grads(pr, dy, part, cuda_dev)
    zero = {k: torch.zeros_like(v) for k, v in dfin.items()}
    zero["h"] = dfin["h"]
    compare_grads(got, oracle_grads(pr, dy, zero))


def test_backward_empty_sequence_passes_final_gradient_through(cuda_dev):
    pr = make_problem(2, 0, 2, 1, 16, 16, dtype=torch.float32, with_state=True, seed=9)
    dy, dfin = draw_grads(pr, seed=1)
    got = gpu_grads(pr, dy, dfin, cuda_dev)
    for f in ("h", "phi", "prev_B", "prev_x"):
        assert torch.equal(got["dinit"][f].cpu(), dfin[f])
    assert not got["dB_bias"].any() and not got["ddt_bias"].any()


def test_backward_full_size_prefill_sampled_heads(cuda_dev):
    """The SISO prefill workload (b4 H64 P64 N128 L2048, bf16, norm + bias) with a carried state:
    the per-head gradients and the initial-state gradients of sampled (batch, head) units
    against the oracle run on those units alone. dB, dC and the bias gradients sum over all
    heads; they are compared element by element in the smaller cases above and only checked
    for finiteness here."""
    pr = make_config(1, with_state=True)
    dy, dfin = draw_grads(pr, seed=11)
    got = gpu_grads(pr, dy, dfin, cuda_dev)
    heads, batches = [0, 37], [1, 3]
    ref = oracle_grads(pr, dy, dfin, heads=heads, batches=batches)
    compare_grads(got, ref, keys=PER_HEAD, heads=heads, batches=batches)
    for k in ("dB", "dC", "dB_bias", "dC_bias"):
        assert torch.isfinite(got[k]).all(), k


@pytest.mark.slow
@pytest.mark.parametrize("cfg,kw", [(1, dict(batch=1, nheads=8)),
                                    (2, dict(batch=1, nheads=4, seqlen=1024))])
def test_backward_full_length_every_gradient(cuda_dev, cfg, kw):
    """Every gradient, dB, dC and the bias gradients (sums over all heads and tokens) too,
    element by element at the workloads' full sequence length on a reduced head count: SISO
    b1 H8 L2048 and MIMO R4 b1 H4 L1024, with a carried state."""
    pr = make_config(cfg, with_state=True, **kw)
    dy, dfin = draw_grads(pr, seed=13 + cfg)
    got = gpu_grads(pr, dy, dfin, cuda_dev)
    ref = oracle_grads(pr, dy, dfin)
    compare_grads(got, ref)


def test_backward_full_size_mimo_sampled_heads(cuda_dev):
    pr = make_config(2, seqlen=512, with_state=True)
    dy, dfin = draw_grads(pr, seed=12)
    got = gpu_grads(pr, dy, dfin, cuda_dev)
    heads, batches = [5, 63], [0]
    ref = oracle_grads(pr, dy, dfin, heads=heads, batches=batches)
    compare_grads(got, ref, keys=PER_HEAD, heads=heads, batches=batches)
