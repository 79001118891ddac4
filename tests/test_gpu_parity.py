"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle on the same
seeded inputs. Small cases span several chunks plus a ragged tail; the full-size workloads
are checked on sampled heads / units that the oracle computes one by one."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_common import TOL, compare, gpu_scan, oracle_scan, oracle_state, record, rel
from state_space_sequence_mamba_b200 import binding as m3
from state_space_sequence_mamba_b200.inputs import make_config, make_decode, make_problem

pytestmark = pytest.mark.gpu


def test_config0_fp32_exact_path(cuda_dev):
    pr = make_config(0)
    y, fin = gpu_scan(pr, cuda_dev)
    yo, so = oracle_scan(pr)
    errs = compare(pr, y, fin, yo, so, tol=1e-4)
    assert errs["y"] < 1e-4


SMALL = [
    # b, L, H, G, P, N, R, chunk, dtype, norm, bias, state
    (2, 200, 4, 1, 64, 128, 1, 64, torch.bfloat16, True, 0.1, True),
    (2, 200, 4, 1, 64, 128, 1, 64, torch.bfloat16, True, 0.1, False),
    (1, 65, 4, 2, 64, 128, 1, 64, torch.bfloat16, False, 0.0, True),
    (1, 63, 4, 4, 64, 128, 1, 64, torch.bfloat16, True, 0.1, True),
    (2, 64, 3, 1, 64, 128, 1, 64, torch.bfloat16, True, 0.1, True),
    (1, 1, 4, 1, 64, 128, 1, 64, torch.bfloat16, True, 0.1, True),
    (2, 100, 4, 1, 64, 128, 4, 16, torch.bfloat16, True, 0.1, True),
    (1, 17, 2, 1, 64, 128, 4, 16, torch.bfloat16, True, 0.1, False),
    (1, 70, 2, 1, 32, 64, 2, 32, torch.bfloat16, True, 0.1, True),
    (1, 40, 2, 2, 16, 16, 8, 8, torch.bfloat16, False, 0.0, True),
    (1, 130, 2, 1, 64, 128, 1, 64, torch.float32, True, 0.1, True),
    (1, 90, 2, 1, 128, 32, 1, 32, torch.float32, False, 0.0, True),
    (1, 77, 2, 1, 16, 16, 4, 16, torch.float32, True, 0.3, True),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "b{}L{}H{}G{}P{}N{}R{}Q{}{}{}{}".format(
    *c[:8], "f32" if c[8] == torch.float32 else "bf16", "n" if c[9] else "", "s" if c[11] else ""))
def test_scan_small(cuda_dev, case):
    b, L, H, G, P, N, R, Q, dt, norm, bias, st = case
    pr = make_problem(b, L, H, G, P, N, rank=R, chunk=Q, dtype=dt, bc_norm=norm,
                      bias_std=bias, seed=L + 13 * R + P, with_state=True)
    y, fin = gpu_scan(pr, cuda_dev, use_state=st)
    yo, so = oracle_scan(pr, use_state=st)
    compare(pr, y, fin, yo, so)


# Few units and long sequences take the sequence-parallel form: each sequence is cut into
# segments (a state-only pass, then all segments at once from their assembled start states).
# With 4-8 units on a B200 these lengths give 2-5 segments, the last one ragged.
SEGMENTED = [
    # b, L, H, G, R, chunk, state
    (1, 2543, 4, 1, 1, 64, True),     # 40 chunks -> 5 segments of 8
    (1, 2543, 4, 1, 1, 64, False),
    (1, 700, 4, 1, 4, 16, True),      # 44 chunks -> 5 segments of 9
    (1, 900, 4, 1, 2, 32, True),      # 29 chunks -> 3 segments of 10
    (1, 333, 4, 1, 8, 8, True),       # 42 chunks -> 5 segments of 9
    (1, 1100, 4, 2, 1, 64, True),     # 18 chunks, two B/C groups -> 2 segments of 9
    (2, 1500, 4, 1, 1, 64, True),     # 24 chunks, 8 units -> 3 segments of 8
]


@pytest.mark.parametrize("case", SEGMENTED, ids=lambda c: "b{}L{}H{}G{}R{}Q{}{}".format(
    *c[:6], "s" if c[6] else ""))
def test_scan_segmented(cuda_dev, case):
    b, L, H, G, R, Q, st = case
    pr = make_problem(b, L, H, G, 64, 128, rank=R, chunk=Q, dtype=torch.bfloat16, bc_norm=True,
                      bias_std=0.1, seed=7 * L + R, with_state=True)
    y, fin = gpu_scan(pr, cuda_dev, use_state=st)
    yo, so = oracle_scan(pr, use_state=st)
    compare(pr, y, fin, yo, so)


def test_segmented_final_state_may_alias_init(cuda_dev):
    """In place with the sequence-parallel form (b1 H4 L2543: 5 segments): the last segment
    writes the final state while segment 0 runs, so the full pass must not read the caller's
    initial state; the result must match the oracle from the original state."""
    pr = make_problem(1, 2543, 4, 1, 64, 128, rank=1, chunk=64, bc_norm=True, bias_std=0.1,
                      seed=23, with_state=True)
    g = pr.to(cuda_dev)
    st = m3.State.from_dict({k: v.clone() for k, v in g.state.items()})
    y, fin = m3.scan_fwd(**g.tensors(), init=st, final=st, chunk=64, bc_norm=True)
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr, use_state=True)
    compare(pr, y, fin, yo, so)


def test_final_state_may_alias_init(cuda_dev):
    pr = make_problem(2, 150, 4, 1, 64, 128, rank=1, chunk=64, bc_norm=True, bias_std=0.1,
                      seed=5, with_state=True)
    g = pr.to(cuda_dev)
    st = m3.State.from_dict({k: v.clone() for k, v in g.state.items()})
    y, fin = m3.scan_fwd(**g.tensors(), init=st, final=st, chunk=64, bc_norm=True)
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr)
    compare(pr, y, fin, yo, so)


def test_empty_sequence(cuda_dev):
    pr = make_problem(2, 0, 4, 1, 64, 128, seed=6, with_state=True)
    g = pr.to(cuda_dev)
    y, fin = m3.scan_fwd(**g.tensors(), init=m3.State.from_dict(g.state), chunk=64)
    torch.cuda.synchronize()
    for k in ("h", "phi", "prev_B", "prev_x"):
        assert torch.equal(getattr(fin, k), g.state[k])
    y, fin = m3.scan_fwd(**g.tensors(), init=None, chunk=64)
    torch.cuda.synchronize()
    assert float(fin.h.abs().max()) == 0.0 and float(fin.phi.abs().max()) == 0.0


def test_split_sequence_on_gpu(cuda_dev):
    """scan(L1) -> state -> scan(L2) matches the oracle's single scan(L1 + L2)."""
    pr = make_problem(2, 300, 4, 1, 64, 128, rank=1, chunk=64, bc_norm=True, bias_std=0.1,
                      seed=21, with_state=True)
    g = pr.to(cuda_dev)
    t = g.tensors()
    cut = 137
    first = {k: (v[:, :cut].contiguous() if k not in ("B_bias", "C_bias") else v) for k, v in t.items()}
    second = {k: (v[:, cut:].contiguous() if k not in ("B_bias", "C_bias") else v) for k, v in t.items()}
    y1, s1 = m3.scan_fwd(**first, init=m3.State.from_dict(g.state), chunk=64, bc_norm=True)
    y2, s2 = m3.scan_fwd(**second, init=s1, chunk=64, bc_norm=True)
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr)
    compare(pr, torch.cat([y1, y2], 1), s2, yo, so)


def test_deterministic(cuda_dev):
    pr = make_problem(2, 200, 4, 1, 64, 128, rank=4, chunk=16, bc_norm=True, bias_std=0.1,
                      seed=9, with_state=True)
    y1, f1 = gpu_scan(pr, cuda_dev)
    y2, f2 = gpu_scan(pr, cuda_dev)
    assert torch.equal(y1, y2) and torch.equal(f1.h, f2.h)


def test_nan_stays_in_its_unit(cuda_dev):
    pr = make_problem(2, 100, 4, 1, 64, 128, rank=1, chunk=64, bc_norm=True, bias_std=0.1,
                      seed=10, with_state=True)
    pr.x[1, 50, 2, 0, 3] = float("nan")
    y, fin = gpu_scan(pr, cuda_dev)
    bad = torch.isnan(y).any(dim=(1, 3, 4))  # [b, H]
    assert bad[1, 2]
    bad[1, 2] = False
    assert not bad.any()
    assert torch.isfinite(fin.h[0]).all() and torch.isfinite(fin.h[1, :2]).all()
    assert torch.isfinite(fin.h[1, 3]).all()


def test_unsupported_shape_reports_cleanly(cuda_dev):
    pr = make_problem(1, 8, 2, 1, 128, 256, rank=1, chunk=64, seed=11)
    with pytest.raises(m3.M3Error) as ei:
        gpu_scan(pr, cuda_dev, use_state=False)
    assert ei.value.status == m3.M3_ERR_UNSUPPORTED


# ---------------------------------------------------------------- decode
@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_decode_steps_small(cuda_dev, R):
    steps = 5
    pr = make_problem(2, steps, 4, 1, 64, 128, rank=R, chunk=1, bc_norm=True, bias_std=0.1,
                      seed=30 + R, with_state=True)
    g = pr.to(cuda_dev)
    st = m3.State.from_dict({k: v.clone() for k, v in g.state.items()})
    ys = []
    for t in range(steps):
        tok = {k: (v[:, t:t + 1].contiguous() if k not in ("B_bias", "C_bias") else v)
               for k, v in g.tensors().items()}
        y, st = m3.decode_step(**tok, state_in=st, bc_norm=True)
        ys.append(y.clone())
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr)
    compare(pr, torch.stack(ys, 1), st, yo, so)


def test_decode_out_of_place_and_fp32(cuda_dev):
    pr = make_problem(2, 1, 4, 2, 32, 64, rank=2, chunk=1, dtype=torch.float32, bc_norm=True,
                      bias_std=0.2, seed=40, with_state=True)
    g = pr.to(cuda_dev)
    sin = m3.State.from_dict(g.state)
    sout = m3.State.empty(2, 4, 64, 32, 2, torch.float32, cuda_dev)
    y, sout = m3.decode_step(**g.tensors(), state_in=sin, state_out=sout, bc_norm=True)
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr)
    compare(pr, y[:, None], sout, yo, so, tol=1e-4)
    for k in ("h", "phi"):
        assert torch.equal(getattr(sin, k), g.state[k])  # input state untouched


# ---------------------------------------------------------------- 128-row chunks
# The warp-specialised scan takes chunks of 128 (token, rank) rows: chunk 128 / R. Cases span
# several chunks with a ragged tail; dt_shift > 0 makes chunks decay by more than 60 nats,
# which that kernel computes in its exact (unscaled) form, dt_shift 0 mixes both forms.
PIPE = [
    # b, L, H, G, R, norm, bias, state, dt_shift, raw scalars, zoh
    (1, 300, 4, 1, 1, True, 0.1, True, -2.0, False, False),
    (2, 130, 4, 1, 2, False, 0.0, False, -2.0, False, False),
    (2, 77, 4, 1, 4, True, 0.1, True, -2.0, False, False),
    (1, 1, 4, 1, 1, True, 0.1, True, -2.0, False, False),
    (2, 128, 4, 2, 1, True, 0.1, False, -2.0, False, False),
    (1, 257, 8, 4, 2, True, 0.1, True, -2.0, False, False),
    (1, 400, 4, 1, 1, True, 0.1, True, 1.5, False, False),
    (1, 300, 4, 1, 2, True, 0.1, True, 1.5, False, False),
    (1, 300, 4, 1, 4, False, 0.0, True, 1.0, False, False),
    (2, 700, 4, 1, 1, True, 0.1, True, 0.0, False, False),
    (2, 333, 4, 1, 1, True, 0.1, True, -2.0, True, False),
    (2, 150, 4, 1, 4, True, 0.1, True, -2.0, True, True),
    (1, 260, 4, 1, 2, True, 0.1, True, -2.0, False, True),
]


@pytest.mark.parametrize("case", PIPE, ids=lambda c: "b{}L{}H{}G{}R{}{}{}d{}{}{}".format(
    *c[:5], "n" if c[5] else "", "s" if c[7] else "", c[8], "raw" if c[9] else "",
    "zoh" if c[10] else ""))
def test_scan_128_row_chunks(cuda_dev, case):
    b, L, H, G, R, norm, bias, st, dts, raw, zoh = case
    pr = make_problem(b, L, H, G, 64, 128, rank=R, chunk=128 // R, bc_norm=norm,
                      bias_std=bias, seed=11 * L + R, with_state=True, dt_shift=dts,
                      raw_scalars=raw)
    if zoh:
        pr.flags |= m3.M3_DISC_ZOH
    y, fin = gpu_scan(pr, cuda_dev, use_state=st)
    yo, so = oracle_scan(pr, use_state=st)
    compare(pr, y, fin, yo, so)


@pytest.mark.parametrize("R", [1, 4])
def test_128_row_chunks_final_state_may_alias_init(cuda_dev, R):
    pr = make_problem(2, 290, 4, 1, 64, 128, rank=R, chunk=128 // R, bc_norm=True,
                      bias_std=0.1, seed=17 + R, with_state=True)
    g = pr.to(cuda_dev)
    st = m3.State.from_dict({k: v.clone() for k, v in g.state.items()})
    y, fin = m3.scan_fwd(**g.tensors(), init=st, final=st, chunk=128 // R, bc_norm=True)
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr)
    compare(pr, y, fin, yo, so)


def test_128_row_chunks_deterministic_and_split(cuda_dev):
    """Two runs are bit-identical; scan(L1) -> state -> scan(L2) matches the oracle's
    single scan over L1 + L2 with the cut inside a chunk."""
    pr = make_problem(2, 300, 4, 1, 64, 128, rank=1, chunk=128, bc_norm=True, bias_std=0.1,
                      seed=29, with_state=True)
    y1, f1 = gpu_scan(pr, cuda_dev)
    y2, f2 = gpu_scan(pr, cuda_dev)
    assert torch.equal(y1, y2) and torch.equal(f1.h, f2.h) and torch.equal(f1.phi, f2.phi)
    g = pr.to(cuda_dev)
    t = g.tensors()
    cut = 170
    part = lambda sl: {k: (v[:, sl].contiguous() if k not in ("B_bias", "C_bias") else v)
                       for k, v in t.items()}
    ya, sa = m3.scan_fwd(**part(slice(0, cut)), init=m3.State.from_dict(g.state), chunk=128,
                         bc_norm=True)
    yb, sb = m3.scan_fwd(**part(slice(cut, None)), init=sa, chunk=128, bc_norm=True)
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr)
    compare(pr, torch.cat([ya, yb], 1), sb, yo, so)


# ---------------------------------------------------------------- full-size workloads
@pytest.mark.slow
def test_config1_full_size_all_heads_of_one_sequence(cuda_dev):
    """The SISO prefill workload as the benchmark launches it (chunk 64): all 64 heads of
    sequence 2 against the oracle."""
    pr = make_config(1)
    y, fin = gpu_scan(pr, cuda_dev, use_state=False)
    yo, so = oracle_scan(pr, use_state=False, batches=[2])
    compare(pr, y, fin, yo, so, batches=[2])


@pytest.mark.slow
def test_config2_mimo_full_size_sampled_heads(cuda_dev):
    """MIMO R4 as the benchmark launches it (chunk 16): 8 heads of sequences 0 and 3."""
    pr = make_config(2)
    y, fin = gpu_scan(pr, cuda_dev, use_state=False)
    heads = [1, 9, 18, 27, 36, 45, 54, 63]
    yo, so = oracle_scan(pr, use_state=False, heads=heads, batches=[0, 3])
    compare(pr, y, fin, yo, so, heads=heads, batches=[0, 3])


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [1, 2])
def test_full_size_128_row_chunks(cuda_dev, cfg):
    """The two b4 L2048 prefill workloads with 128-row chunks (chunk 128 and 32): 16 heads of
    sequence 1 (SISO), 8 heads of sequence 2 (MIMO R4)."""
    pr = make_config(cfg)
    y, fin = gpu_scan(pr, cuda_dev, use_state=False, chunk=128 // pr.dims.rank)
    heads = list(range(3, 64, 4)) if cfg == 1 else [0, 8, 16, 24, 32, 40, 48, 56]
    bsel = [1] if cfg == 1 else [2]
    yo, so = oracle_scan(pr, use_state=False, heads=heads, batches=bsel)
    compare(pr, y, fin, yo, so, heads=heads, batches=bsel)


@pytest.mark.slow
def test_config4_long_context_with_carry_in(cuda_dev):
    """L = 65536 from the final state of the SISO prefill workload's sequence 0 (computed by
    the oracle, stored as fp32 / bf16 like any state), checked on sampled heads."""
    p1 = make_config(1)
    for k in ("x", "B", "C", "theta", "dt", "A", "lam"):
        setattr(p1, k, getattr(p1, k)[:1])
    _, s1 = oracle_scan(p1, use_state=False)
    pr = make_config(4)
    pr.B_bias, pr.C_bias = p1.B_bias, p1.C_bias   # same layer parameters as the carried state
    pr.state = dict(h=torch.from_numpy(s1.h).float(), phi=torch.from_numpy(s1.phi).float(),
                    prev_B=torch.from_numpy(s1.prev_B).to(torch.bfloat16),
                    prev_x=torch.from_numpy(s1.prev_x).to(torch.bfloat16))
    y, fin = gpu_scan(pr, cuda_dev, use_state=True)
    heads = [3, 60]
    yo, so = oracle_scan(pr, use_state=True, heads=heads)
    compare(pr, y, fin, yo, so, heads=heads)


@pytest.mark.slow
@pytest.mark.parametrize("R", [1, 4])
def test_config3_decode_1000_steps_sampled_units(cuda_dev, R):
    steps = 1000
    pr = make_decode(R, steps, device=cuda_dev)
    st = m3.State.from_dict({k: v.clone() for k, v in pr.state.items()})
    bsel = [0, 77]
    hsel = list(range(0, 64, 8)) if R == 4 else list(range(0, 64, 2))
    ys = []
    for t in range(steps):
        y, st = m3.decode_step(pr.x[t], pr.B[t], pr.C[t], pr.theta[t], pr.dt[t], pr.A[t],
                               pr.lam[t], state_in=st)
        ys.append(y[bsel][:, hsel].float())
    torch.cuda.synchronize()
    ys = torch.stack(ys, 1)  # [nb, steps, nh, R, P]
    b_i, h_i = torch.as_tensor(bsel), torch.as_tensor(hsel)
    cpu = lambda t: t.cpu()
    xo = cpu(pr.x[:, b_i][:, :, 0][:, :, h_i]).transpose(0, 1)
    Bo = cpu(pr.B[:, b_i][:, :, 0]).transpose(0, 1)
    Co = cpu(pr.C[:, b_i][:, :, 0]).transpose(0, 1)
    tho = cpu(pr.theta[:, b_i][:, :, 0][:, :, h_i]).transpose(0, 1)
    sc = lambda t: cpu(t[:, b_i][:, :, 0][:, :, h_i]).transpose(0, 1)
    s0 = {k: cpu(v[b_i][:, h_i]) for k, v in pr.state.items()}
    yo, so = oracle.scan(xo, Bo, Co, tho, sc(pr.dt), sc(pr.A), sc(pr.lam),
                         state=oracle_state(s0))
    e_y = rel(ys, yo)
    e_h = rel(st.h[b_i][:, h_i], so.h)
    e_phi = rel(st.phi[b_i][:, h_i], so.phi)
    record({"y": e_y, "h": e_h, "phi": e_phi})
    assert e_y <= TOL[torch.bfloat16] and e_h <= TOL[torch.bfloat16] and e_phi <= 2e-2, \
        (e_y, e_h, e_phi)


# ---------------------------------------------------------------- fused scalar prologue
# dt and lam passed raw (M3_DT_SOFTPLUS | M3_LAM_SIGMOID, per-head dt_bias): every kernel
# applies softplus / sigmoid to real tokens only.
RAW = [
    # b, L, H, P, N, R, chunk, dtype
    (2, 200, 4, 64, 128, 1, 64, torch.bfloat16),    # tensor-core scan, SISO, ragged tail
    (2, 100, 4, 64, 128, 4, 16, torch.bfloat16),    # tensor-core scan, MIMO
    (1, 2543, 4, 64, 128, 1, 64, torch.bfloat16),   # sequence-parallel form, 5 segments
    (1, 130, 2, 64, 128, 1, 64, torch.float32),     # exact fp32 path
]


@pytest.mark.parametrize("case", RAW, ids=lambda c: "b{}L{}H{}P{}N{}R{}Q{}{}".format(
    *c[:7], "f32" if c[7] == torch.float32 else "bf16"))
def test_scan_raw_scalars(cuda_dev, case):
    b, L, H, P, N, R, Q, dt = case
    pr = make_problem(b, L, H, 1, P, N, rank=R, chunk=Q, dtype=dt, bc_norm=True,
                      bias_std=0.1, seed=3 * L + R, with_state=True, raw_scalars=True)
    assert pr.flags == m3.M3_DT_SOFTPLUS | m3.M3_LAM_SIGMOID
    y, fin = gpu_scan(pr, cuda_dev)
    yo, so = oracle_scan(pr)
    compare(pr, y, fin, yo, so, tol=1e-4 if dt == torch.float32 else None)


@pytest.mark.parametrize("R,dt", [(1, torch.bfloat16), (2, torch.bfloat16), (4, torch.bfloat16),
                                  (2, torch.float32)])
def test_decode_raw_scalars(cuda_dev, R, dt):
    steps = 4
    pr = make_problem(2, steps, 4, 1, 64, 128, rank=R, chunk=1, dtype=dt, bc_norm=True,
                      bias_std=0.1, seed=50 + R, with_state=True, raw_scalars=True)
    g = pr.to(cuda_dev)
    st = m3.State.from_dict({k: v.clone() for k, v in g.state.items()})
    ys = []
    for t in range(steps):
        tok = {k: (v[:, t:t + 1].contiguous() if k not in ("B_bias", "C_bias") else v)
               for k, v in g.tensors().items()}
        y, st = m3.decode_step(**tok, **g.scalar_args(), state_in=st, bc_norm=True)
        ys.append(y.clone())
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr)
    compare(pr, torch.stack(ys, 1), st, yo, so, tol=1e-4 if dt == torch.float32 else None)


# ---------------------------------------------------------------- decode with MIMO projections
@pytest.mark.parametrize("R,dt", [(1, torch.bfloat16), (2, torch.bfloat16), (4, torch.bfloat16),
                                  (8, torch.bfloat16), (4, torch.float32)])
def test_decode_proj(cuda_dev, R, dt):
    """m3_decode_step_proj over a few steps (X = W_X X' in, O' = sum_r W_O Y SiLU(W_Z Z') out,
    Appendix C) against the oracle; the stored previous token is the expanded X, rounded to
    the storage type, so it is compared within the tolerance rather than bit for bit."""
    from state_space_sequence_mamba_b200.inputs import make_proj
    steps, b, H, P, N = 3, 2, 4, 64, 128
    pr = make_problem(b, steps, H, 1, P, N, rank=R, chunk=1, dtype=dt, bc_norm=True,
                      bias_std=0.1, seed=60 + R, with_state=True)
    xp, zp, WX, WZ, WO = make_proj(steps, b, H, P, R, dtype=dt, seed=70 + R)
    g = pr.to(cuda_dev)
    st = m3.State.from_dict({k: v.clone() for k, v in g.state.items()})
    so = oracle_state(pr.state)
    tol = TOL[dt]
    Wd = [w.to(cuda_dev) for w in (WX, WZ, WO)]
    for t in range(steps):
        tok = {k: (v[:, t:t + 1].contiguous() if k not in ("B_bias", "C_bias") else v)
               for k, v in g.tensors().items() if k != "x"}
        o, st = m3.decode_step_proj(xp[t].to(cuda_dev), zp[t].to(cuda_dev), *Wd, **tok,
                                    state_in=st, bc_norm=True)
        oo, so = oracle.decode_step_proj(xp[t][:, 0], zp[t][:, 0], WX, WZ, WO,
                                         pr.B[:, t], pr.C[:, t], pr.theta[:, t], pr.dt[:, t],
                                         pr.A[:, t], pr.lam[:, t], pr.B_bias, pr.C_bias, so,
                                         bc_norm=True)
        torch.cuda.synchronize()
        errs = {"o": rel(o, oo)}
        record(errs)
        assert errs["o"] <= tol, errs
    errs = {"h": rel(st.h, so.h), "phi": rel(st.phi, so.phi), "prev_x": rel(st.prev_x, so.prev_x),
            "prev_B": rel(st.prev_B, so.prev_B)}
    record(errs)
    assert errs["prev_B"] == 0.0 and all(v <= tol for v in errs.values()), errs


# ---------------------------------------------------------------- context parallelism
@pytest.mark.parametrize("b,L,R", [(2, 300, 1), (1, 2543, 1), (1, 700, 4)])
def test_scan_state_matches_final_state(cuda_dev, b, L, R):
    """m3_scan_state (no y): its h and phi against the oracle's final state and its summed
    log-decay against sum_t dt_t A_t, in one segment (8 units: then also equal to
    m3_scan_fwd's final state to rounding) and in the sequence-parallel form (4 units, 5
    segments combined on the device, each segment's operands rounded in its own frame)."""
    pr = make_problem(b, L, 4, 1, 64, 128, rank=R, chunk=64 // R, bc_norm=True, bias_std=0.1,
                      seed=91 + L, with_state=True)
    g = pr.to(cuda_dev)
    init = m3.State.from_dict(g.state)
    h, phi, lsum = m3.scan_state(**g.tensors(), init=init, chunk=64 // R, bc_norm=True)
    _, fin = m3.scan_fwd(**g.tensors(), init=init, chunk=64 // R, bc_norm=True)
    torch.cuda.synchronize()
    _, so = oracle_scan(pr)
    errs = {"h": rel(h, so.h), "phi": rel(phi, so.phi),
            "lam_sum": rel(lsum, (pr.dt.double() * pr.A.double()).sum(1).numpy())}
    record(errs)
    assert errs["h"] <= TOL[torch.bfloat16] and errs["phi"] < 1e-5 and errs["lam_sum"] < 1e-5, errs
    if b * 4 >= 8:   # one segment: the same arithmetic as the scan's own state chain
        assert rel(h, fin.h.double().cpu().numpy()) < 1e-5


@pytest.mark.parametrize("world,R,raw", [(2, 1, False), (4, 1, True), (3, 4, False)])
def test_context_parallel_phases_on_gpu(cuda_dev, world, R, raw):
    """The context-parallel phases with the library's kernels, the ranks run one after another
    on one device (no collective: the gathered lists are built locally): the concatenated
    outputs and the last rank's final state against the oracle's single scan."""
    from state_space_sequence_mamba_b200 import context_parallel as cp
    Q = 64 // R
    pr = make_problem(2, 900 + 7 * world, 4, 1, 64, 128, rank=R, chunk=Q, bc_norm=True,
                      bias_std=0.1, seed=93 + world, with_state=True, raw_scalars=raw)
    g = pr.to(cuda_dev)
    L = pr.dims.seqlen
    cut = [L * k // world for k in range(world + 1)]
    ts = [{k: (v[:, cut[r]:cut[r + 1]].contiguous() if k not in ("B_bias", "C_bias") else v)
           for k, v in g.tensors().items()} for r in range(world)]
    init = m3.State.from_dict(g.state)
    scalar = g.scalar_args()
    ops = cp.DeviceOps()
    lasts = [cp.last_token(t) for t in ts]
    prevs = [None] + lasts[:-1]
    segs = [cp.segment_state(r, ts[r], init, prevs[r], Q, True, scalar, ops) for r in range(world)]
    seg_h, seg_phi, seg_lam = (torch.stack([s[i] for s in segs]) for i in range(3))
    outs = [cp.finish(r, world, ts[r], init, prevs[r], seg_h, seg_phi, seg_lam, Q, True,
                      scalar, ops) for r in range(world)]
    torch.cuda.synchronize()
    y = torch.cat([o[0] for o in outs], 1)
    assert all(o[1] is None for o in outs[:-1])
    yo, so = oracle_scan(pr)
    compare(pr, y, outs[-1][1], yo, so)


# ---------------------------------------------------------------- degenerate regimes
def _degenerate(pr, kind):
    """Rewrites one problem's step scalars / angles into a limiting regime of the method."""
    if kind == "euler":            # lam = 1: exponential Euler, no previous-token term
        pr.lam.fill_(1.0)
    elif kind == "prev_only":      # lam = 0: only the previous token enters
        pr.lam.fill_(0.0)
    elif kind == "no_rotation":    # theta = 0: the real-valued SSM
        pr.theta.zero_()
    elif kind == "strong_decay":   # dt A down to about -11 per token: decays underflow within a chunk
        pr.dt.copy_(pr.dt * 0 + 4.0)
        pr.A.copy_(pr.A.clamp(max=-2.0))
    elif kind == "tiny_step":      # dt = 1e-6: alpha = 1, gamma ~ 0
        pr.dt.fill_(1e-6)
    elif kind == "fast_angle":     # dt theta up to 3 pi per token: the carried angle wraps often
        pr.dt.fill_(3.0)
    return pr


@pytest.mark.parametrize("kind", ["euler", "prev_only", "no_rotation", "strong_decay",
                                  "tiny_step", "fast_angle"])
@pytest.mark.parametrize("R,L,b,rows", [(1, 333, 2, 64), (4, 150, 2, 64), (1, 2543, 1, 64),
                                        (1, 333, 2, 128), (4, 150, 2, 128)])
def test_scan_degenerate_regimes(cuda_dev, kind, R, L, b, rows):
    """Limits of the recurrence through the tensor-core scans (SISO, MIMO, the
    sequence-parallel form at b1 L2543, and 128-row chunks) against the oracle."""
    pr = make_problem(b, L, 4, 1, 64, 128, rank=R, chunk=rows // R, bc_norm=True, bias_std=0.1,
                      seed=101 + L + R, with_state=True)
    pr = _degenerate(pr, kind)
    y, fin = gpu_scan(pr, cuda_dev)
    assert torch.isfinite(y.float()).all() and torch.isfinite(fin.h).all()
    yo, so = oracle_scan(pr)
    compare(pr, y, fin, yo, so)


@pytest.mark.parametrize("kind", ["euler", "strong_decay", "fast_angle"])
@pytest.mark.parametrize("R", [1, 4])
def test_decode_degenerate_regimes(cuda_dev, kind, R):
    steps = 3
    pr = make_problem(2, steps, 4, 1, 64, 128, rank=R, chunk=1, bc_norm=True, bias_std=0.1,
                      seed=121 + R, with_state=True)
    pr = _degenerate(pr, kind)
    g = pr.to(cuda_dev)
    st = m3.State.from_dict({k: v.clone() for k, v in g.state.items()})
    ys = []
    for t in range(steps):
        tok = {k: (v[:, t:t + 1].contiguous() if k not in ("B_bias", "C_bias") else v)
               for k, v in g.tensors().items()}
        y, st = m3.decode_step(**tok, state_in=st, bc_norm=True)
        ys.append(y.clone())
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr)
    compare(pr, torch.stack(ys, 1), st, yo, so)


# ---------------------------------------------------------------- zero-order hold
ZOH = [
    # b, L, H, P, N, R, chunk, dtype, raw scalars too
    (2, 333, 4, 64, 128, 1, 64, torch.bfloat16, False),   # tensor-core scan, SISO
    (2, 150, 4, 64, 128, 4, 16, torch.bfloat16, True),    # tensor-core scan, MIMO, flags 7
    (1, 2543, 4, 64, 128, 1, 64, torch.bfloat16, False),  # sequence-parallel form
    (1, 130, 2, 64, 128, 1, 64, torch.float32, False),    # exact fp32 path
]


@pytest.mark.parametrize("case", ZOH, ids=lambda c: "b{}L{}R{}{}{}".format(
    c[0], c[1], c[5], "f32" if c[7] == torch.float32 else "bf16", "raw" if c[8] else ""))
def test_scan_zoh(cuda_dev, case):
    """M3_DISC_ZOH (beta = 0, gamma = (alpha - 1) / A) through every scan path."""
    b, L, H, P, N, R, Q, dt, raw = case
    pr = make_problem(b, L, H, 1, P, N, rank=R, chunk=Q, dtype=dt, bc_norm=True,
                      bias_std=0.1, seed=5 * L + R, with_state=True, raw_scalars=raw)
    pr.flags |= m3.M3_DISC_ZOH
    y, fin = gpu_scan(pr, cuda_dev)
    yo, so = oracle_scan(pr)
    compare(pr, y, fin, yo, so, tol=1e-4 if dt == torch.float32 else None)


@pytest.mark.parametrize("R,dt", [(1, torch.bfloat16), (4, torch.bfloat16), (2, torch.float32)])
def test_decode_zoh(cuda_dev, R, dt):
    steps = 4
    pr = make_problem(2, steps, 4, 1, 64, 128, rank=R, chunk=1, dtype=dt, bc_norm=True,
                      bias_std=0.1, seed=140 + R, with_state=True)
    pr.flags |= m3.M3_DISC_ZOH
    g = pr.to(cuda_dev)
    st = m3.State.from_dict({k: v.clone() for k, v in g.state.items()})
    ys = []
    for t in range(steps):
        tok = {k: (v[:, t:t + 1].contiguous() if k not in ("B_bias", "C_bias") else v)
               for k, v in g.tensors().items()}
        y, st = m3.decode_step(**tok, **g.scalar_args(), state_in=st, bc_norm=True)
        ys.append(y.clone())
    torch.cuda.synchronize()
    yo, so = oracle_scan(pr)
    compare(pr, torch.stack(ys, 1), st, yo, so, tol=1e-4 if dt == torch.float32 else None)
