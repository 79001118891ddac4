"""Seeded synthetic inputs for the Mamba-3 SSM core.

This module draws random tensors and nothing else: it holds none of the recurrence's
arithmetic. The tests feed the same stored tensors (bf16 or fp32, exactly as drawn here) to
the CUDA library and to the CPU oracle.

Value distributions follow the 1.5B-scale layer workloads (H=64 heads, head dim P=64,
state N=128, B/C shared by all heads):

* x, B_raw, C_raw ~ N(0, 1), or N(0, 1/R) for rank-R MIMO;
* B/C bias ~ N(0, 0.1) per (head, rank, channel) when BC normalisation is on, else 0;
* dt = softplus(N(0,1) + dt_shift) with dt_shift = -2 (-4 for the long-memory regime);
* A = -exp(U(-1, 1)); lam = sigmoid(N(0, 1)); theta ~ U(-pi, pi) on the N/2 pairs.

Draw order for one seed is fixed: x, B, C, bias_B, bias_C, dt_raw, A_raw, lam_raw, theta,
then the initial state (h ~ N(0,1), phi ~ U(-pi,pi), prev_B ~ N(0,1), prev_x ~ N(0,1)).
fp32 draws are cast to the stored dtype once; every consumer reads those stored bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass
class Dims:
    batch: int
    seqlen: int
    nheads: int
    ngroups: int
    headdim: int
    dstate: int
    rank: int = 1
    chunk: int = 64
    dtype: torch.dtype = torch.bfloat16
    bc_norm: bool = False
    norm_eps: float = 1e-6


@dataclass
class Problem:
    """One scan problem: dims, inputs in their stored dtypes, optional initial state."""

    dims: Dims
    x: torch.Tensor          # [b, L, H, R, P]   dtype
    B: torch.Tensor          # [b, L, G, R, N]   dtype (raw, before normalisation)
    C: torch.Tensor          # [b, L, G, R, N]   dtype
    theta: torch.Tensor      # [b, L, H, N/2]    dtype
    dt: torch.Tensor         # [b, L, H]         fp32, > 0
    A: torch.Tensor          # [b, L, H]         fp32, < 0
    lam: torch.Tensor        # [b, L, H]         fp32, in (0, 1)
    B_bias: torch.Tensor | None = None   # [H, R, N] fp32
    C_bias: torch.Tensor | None = None   # [H, R, N] fp32
    state: dict | None = field(default=None)  # h, phi (fp32), prev_B, prev_x (dtype)
    # raw step scalars: flags = 3 (dt and lam are the raw projections), dt_bias [H] fp32
    dt_bias: torch.Tensor | None = None
    flags: int = 0

    def tensors(self):
        return dict(x=self.x, B=self.B, C=self.C, theta=self.theta, dt=self.dt, A=self.A,
                    lam=self.lam, B_bias=self.B_bias, C_bias=self.C_bias)

    def scalar_args(self):
        """How dt and lam are to be read: flags 0 (ready to use) or 3 (raw, with dt_bias)."""
        return dict(dt_bias=self.dt_bias, flags=self.flags)

    def to(self, device) -> "Problem":
        mv = lambda t: None if t is None else t.to(device)
        st = None if self.state is None else {k: mv(v) for k, v in self.state.items()}
        return Problem(self.dims, mv(self.x), mv(self.B), mv(self.C), mv(self.theta),
                       mv(self.dt), mv(self.A), mv(self.lam), mv(self.B_bias),
                       mv(self.C_bias), st, mv(self.dt_bias), self.flags)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def random_state(batch, nheads, dstate, headdim, rank, dtype, g, device="cpu") -> dict:
    """h ~ N(0,1) fp32, phi ~ U(-pi,pi) fp32, prev_B, prev_x ~ N(0,1) in ``dtype``."""
    h = torch.randn(batch, nheads, dstate, headdim, generator=g, device=device)
    phi = (torch.rand(batch, nheads, dstate // 2, generator=g, device=device) * 2 - 1) * math.pi
    prev_B = torch.randn(batch, nheads, rank, dstate, generator=g, device=device).to(dtype)
    prev_x = torch.randn(batch, nheads, rank, headdim, generator=g, device=device).to(dtype)
    return dict(h=h, phi=phi, prev_B=prev_B, prev_x=prev_x)


def make_problem(batch, seqlen, nheads, ngroups, headdim, dstate, rank=1, chunk=64,
                 dtype=torch.bfloat16, bc_norm=False, bias_std=0.0, dt_shift=-2.0,
                 seed=0, with_state=False, device="cpu", lead=(), input_std=None,
                 raw_scalars=False) -> Problem:
    """Draws one problem. ``lead`` prepends extra leading dims (used for stacks of decode
    steps: lead=(steps,) gives x [steps, b, 1, H, R, P] and so on).

    ``raw_scalars``: dt and lam are stored as their raw N(0,1) draws (the layer's projections
    before softplus and sigmoid) and a per-head dt_bias ~ N(dt_shift, 0.5^2) is drawn after
    everything else; the problem's flags ask the consumer to apply the parameterisation."""
    g = _gen(seed, device)
    d = Dims(batch, seqlen, nheads, ngroups, headdim, dstate, rank, chunk, dtype,
             bool(bc_norm), 1e-6)
    b, L, H, G, P, N, R = batch, seqlen, nheads, ngroups, headdim, dstate, rank
    sd = 1.0 / math.sqrt(R) if input_std is None else float(input_std)
    shp = tuple(lead)
    x = (torch.randn(*shp, b, L, H, R, P, generator=g, device=device) * sd).to(dtype)
    B = (torch.randn(*shp, b, L, G, R, N, generator=g, device=device) * sd).to(dtype)
    C = (torch.randn(*shp, b, L, G, R, N, generator=g, device=device) * sd).to(dtype)
    if bias_std > 0:
        B_bias = torch.randn(H, R, N, generator=g, device=device) * bias_std
        C_bias = torch.randn(H, R, N, generator=g, device=device) * bias_std
    else:
        B_bias = C_bias = None
    dt_raw = torch.randn(*shp, b, L, H, generator=g, device=device)
    A = -torch.exp(torch.rand(*shp, b, L, H, generator=g, device=device) * 2 - 1)
    lam_raw = torch.randn(*shp, b, L, H, generator=g, device=device)
    theta = ((torch.rand(*shp, b, L, H, N // 2, generator=g, device=device) * 2 - 1)
             * math.pi).to(dtype)
    st = random_state(b, H, N, P, R, dtype, g, device) if with_state else None
    if raw_scalars:
        dt_bias = torch.randn(H, generator=g, device=device) * 0.5 + dt_shift
        return Problem(d, x, B, C, theta, dt_raw.float(), A.float(), lam_raw.float(), B_bias,
                       C_bias, st, dt_bias.float(), 3)
    dt = torch.nn.functional.softplus(dt_raw + dt_shift)
    lam = torch.sigmoid(lam_raw)
    return Problem(d, x, B, C, theta, dt.float(), A.float(), lam.float(), B_bias, C_bias, st)


# The five workloads. Each entry: (description, keyword arguments of make_problem).
CONFIGS = {
    0: ("SISO scan fp32: b1 H1 P16 N16 L64",
        dict(batch=1, seqlen=64, nheads=1, ngroups=1, headdim=16, dstate=16, rank=1,
             chunk=64, dtype=torch.float32, bc_norm=False, bias_std=0.0, seed=0)),
    1: ("SISO prefill bf16: b4 H64 P64 N128 L2048 chunk 64, BCNorm + bias",
        dict(batch=4, seqlen=2048, nheads=64, ngroups=1, headdim=64, dstate=128, rank=1,
             chunk=64, dtype=torch.bfloat16, bc_norm=True, bias_std=0.1, seed=1)),
    2: ("MIMO R4 prefill bf16: b4 H64 P64 N128 L2048 chunk 16, BCNorm + bias",
        dict(batch=4, seqlen=2048, nheads=64, ngroups=1, headdim=64, dstate=128, rank=4,
             chunk=16, dtype=torch.bfloat16, bc_norm=True, bias_std=0.1, seed=2)),
    4: ("long SISO prefill bf16: b1 H64 P64 N128 L65536 chunk 64, dt=softplus(N-4)",
        dict(batch=1, seqlen=65536, nheads=64, ngroups=1, headdim=64, dstate=128, rank=1,
             chunk=64, dtype=torch.bfloat16, bc_norm=True, bias_std=0.1, dt_shift=-4.0,
             seed=4)),
}


def make_config(idx: int, device="cpu", **overrides) -> Problem:
    """Problem for workload ``idx`` (0, 1, 2 or 4); keyword overrides replace fields."""
    kw = dict(CONFIGS[idx][1])
    kw.update(overrides)
    return make_problem(device=device, **kw)


def make_decode(rank: int, steps: int, batch=128, nheads=64, headdim=64, dstate=128,
                seed=3, device="cpu", raw_scalars=False):
    """Decode workload: per-step inputs drawn as for the fp32 scan workload (N(0,1) x, B, C;
    no normalisation, zero bias), stored bf16, stacked over ``steps``; initial state drawn
    after them (h ~ N(0,1) fp32, phi ~ U(-pi,pi), prev_B, prev_x ~ N(0,1) bf16).

    Returns (Problem with leading step dim: x [steps, b, 1, H, R, P] ...)."""
    return make_problem(batch, 1, nheads, 1, headdim, dstate, rank=rank, chunk=1,
                        dtype=torch.bfloat16, bc_norm=False, bias_std=0.0, dt_shift=-2.0,
                        seed=seed, with_state=True, device=device, lead=(steps,),
                        input_std=1.0, raw_scalars=raw_scalars)


def make_proj(steps: int, batch: int, nheads: int, headdim: int, rank: int,
              dtype=torch.bfloat16, seed=0, device="cpu"):
    """Inputs of the MIMO projections around decode steps: X', Z' ~ N(0, 1) per step
    [steps, b, 1, H, P] in ``dtype``, and per-head weights W_X, W_Z, W_O ~ N(0, 1) [H, R, P]
    fp32 (drawn in that order)."""
    g = _gen(seed, device)
    xp = torch.randn(steps, batch, 1, nheads, headdim, generator=g, device=device).to(dtype)
    zp = torch.randn(steps, batch, 1, nheads, headdim, generator=g, device=device).to(dtype)
    W = [torch.randn(nheads, rank, headdim, generator=g, device=device) for _ in range(3)]
    return xp, zp, W[0], W[1], W[2]
