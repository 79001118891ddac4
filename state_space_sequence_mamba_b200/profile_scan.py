"""Runs the prefill scan on one of the seeded workloads a few times and checks its status,
for a profiler to capture one launch of it:

    python -m state_space_sequence_mamba_b200.profile_scan CONFIG CHUNK REPS

CONFIG is a workload of ``inputs.CONFIGS`` (1: SISO b4 L2048, 2: MIMO R4 b4 L2048, 4: b1
L65536), CHUNK the chunk length (64 / R for the 64-row tensor-core scan, 128 / R for the
128-row one), REPS the number of calls; BC normalisation is on. Prints ``ok``."""
from __future__ import annotations

import sys


def main(argv=None) -> None:
    import torch
    from . import binding as m3
    from .inputs import make_config
    args = list(sys.argv[1:] if argv is None else argv)
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


if __name__ == "__main__":
    main()
