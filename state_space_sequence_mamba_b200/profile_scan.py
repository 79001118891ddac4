"""Runs the prefill scan on one of the seeded workloads a few times and checks its status,
for a profiler to capture one launch of it:

    python -m state_space_sequence_mamba_b200.profile_scan CONFIG CHUNK REPS
    python -m state_space_sequence_mamba_b200.profile_scan bwd CONFIG REPS [fp32]

CONFIG is a workload of ``inputs.CONFIGS`` (1: SISO b4 L2048, 2: MIMO R4 b4 L2048, 4: b1
L65536), CHUNK the chunk length (64 / R for the 64-row tensor-core scan, 128 / R for the
128-row one), REPS the number of calls; BC normalisation is on. With ``bwd`` it runs the
backward (m3_scan_bwd) of the workload with its carried initial state and a seeded dy, in
the form the call picks, or the fp32 sweeps with ``fp32``. Prints ``ok``."""
from __future__ import annotations

import sys


def main(argv=None) -> None:
    import torch
    from . import binding as m3
    from .inputs import make_config
    args = list(sys.argv[1:] if argv is None else argv)
    if args and args[0] == "bwd":
        backward(int(args[1]) if len(args) > 1 else 1, int(args[2]) if len(args) > 2 else 3,
                 len(args) > 3 and args[3] == "fp32")
        return
    cfg = int(args[0]) if args else 1
    chunk = int(args[1]) if len(args) > 1 else 64
    reps = int(args[2]) if len(args) > 2 else 3
    dev = torch.device("cuda:0")
    t = make_config(cfg).to(dev).tensors()
    dims = m3.make_dims(t["x"], t["B"], chunk, True, 1e-6, 0)
    ws = torch.zeros(m3.scan_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    y = torch.empty_like(t["x"])
    for _ in range(reps):
        m3.scan_fwd(**t, chunk=chunk, bc_norm=True, y=y, workspace=ws)
    torch.cuda.synchronize()
    m3.scan_check(ws)
    print("ok")


def backward(cfg: int, reps: int, fp32: bool) -> None:
    import torch
    from . import binding as m3
    from .inputs import make_config
    dev = torch.device("cuda:0")
    pr = make_config(cfg, with_state=True).to(dev)
    g = torch.Generator(device=dev).manual_seed(cfg + 1)
    dy = torch.randn(pr.x.shape, generator=g, device=dev).to(pr.x.dtype)
    sa = pr.scalar_args()
    if fp32:
        sa["flags"] = sa["flags"] | m3.BWD_FP32
    dims = m3.make_dims(pr.x, pr.B, 1, pr.dims.bc_norm, pr.dims.norm_eps, sa["flags"])
    ws = torch.empty(m3.scan_bwd_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    init = m3.State.from_dict(pr.state)
    for _ in range(reps):
        m3.scan_bwd(**pr.tensors(), dy=dy, init=init, bc_norm=pr.dims.bc_norm,
                    norm_eps=pr.dims.norm_eps, workspace=ws, **sa)
    torch.cuda.synchronize()
    m3.scan_check(ws)
    print("ok")


if __name__ == "__main__":
    main()
