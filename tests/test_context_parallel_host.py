"""The context-parallel prefill's orchestration (state_space_sequence_mamba_b200.
context_parallel) run as gloo ranks on the CPU, with stand-ins for the three kernels backed by
the fp64 oracle and a direct fp64 combine: the ranks' outputs, concatenated, must equal the
oracle's single scan of the whole sequence, and the last rank's final state its final state.
This checks the exchange (which previous token and which end states each rank uses, in which
frame) independently of the kernels, which the GPU tests check."""
import json
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = textwrap.dedent("""
    import json, os, sys
    sys.path.insert(0, os.environ["REPO_ROOT"])
    sys.path.insert(0, os.path.join(os.environ["REPO_ROOT"], "tests"))
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle
    from state_space_sequence_mamba_b200 import binding as m3
    from state_space_sequence_mamba_b200 import context_parallel as cp
    from state_space_sequence_mamba_b200.inputs import make_problem

    def to_oracle(st):
        if st is None:
            return None
        return oracle.State(*(getattr(st, k).double().numpy() for k in ("h", "phi", "prev_B", "prev_x")))

    class OracleOps:
        def scan_state(self, t, init, chunk, bc_norm, scalar):
            _, s = oracle.scan(**t, state=to_oracle(init), bc_norm=bc_norm, **scalar)
            dt, _ = oracle.step_scalars(t["dt"], t["lam"], scalar["dt_bias"], scalar["flags"])
            lsum = (dt * t["A"].double().numpy()).sum(axis=1)       # [b, H]
            return torch.from_numpy(s.h), torch.from_numpy(s.phi), torch.from_numpy(lsum)

        def state_combine(self, h, phi, lam):
            h, phi, lam = h.numpy(), phi.numpy(), lam.numpy()
            S, b, H, N, P = h.shape
            half = N // 2
            acc, ang = h[0].copy(), phi[0].copy()
            for j in range(1, S):
                c, s = np.cos(ang)[..., None], np.sin(ang)[..., None]
                top, bot = h[j][:, :, :half], h[j][:, :, half:]
                rot = np.concatenate([top * c + bot * s, bot * c - top * s], axis=2)
                acc = np.exp(lam[j])[..., None, None] * acc + rot
                ang = ang + phi[j]
            return torch.from_numpy(acc), torch.from_numpy(ang)

        def scan_fwd(self, t, init, final, chunk, bc_norm, scalar):
            y, s = oracle.scan(**t, state=to_oracle(init), bc_norm=bc_norm, **scalar)
            fin = m3.State(*(torch.from_numpy(getattr(s, k)) for k in ("h", "phi", "prev_B", "prev_x")))
            return torch.from_numpy(y), (fin if final else None)

    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", rank=rank, world_size=world)
    R, raw = int(os.environ["RANKS_R"]), os.environ["RAW"] == "1"
    pr = make_problem(2, 3 * 37, 4, 2, 16, 16, rank=R, chunk=8, dtype=torch.bfloat16,
                      bc_norm=True, bias_std=0.2, seed=11, with_state=True, raw_scalars=raw)
    L = pr.dims.seqlen
    cut = [L * k // world for k in range(world + 1)]
    sl = lambda v: v[:, cut[rank]:cut[rank + 1]].contiguous()
    t = {k: (sl(v) if k not in ("B_bias", "C_bias") else v) for k, v in pr.tensors().items()}
    init = m3.State(*(pr.state[k].double() if k in ("h", "phi") else pr.state[k]
                      for k in ("h", "phi", "prev_B", "prev_x"))) if rank == 0 else None
    y, fin = cp.scan_context_parallel(**t, init=init, chunk=8, bc_norm=True,
                                      **pr.scalar_args(), ops=OracleOps())
    out = {"rank": rank}
    yo, so = oracle.scan(**pr.tensors(), state=to_oracle(m3.State(*(pr.state[k] for k in ("h", "phi", "prev_B", "prev_x")))),
                         bc_norm=True, **pr.scalar_args())
    ref = yo[:, cut[rank]:cut[rank + 1]]
    out["y_err"] = float(np.max(np.abs(y.numpy() - ref)) / np.max(np.abs(yo)))
    if rank == world - 1:
        out["h_err"] = float(np.max(np.abs(fin.h.numpy() - so.h)) / np.max(np.abs(so.h)))
        out["phi_err"] = float(np.max(np.abs(fin.phi.numpy() - so.phi)) / np.max(np.abs(so.phi)))
        out["prev_ok"] = bool(np.array_equal(fin.prev_B.numpy(), so.prev_B)
                              and np.array_equal(fin.prev_x.numpy(), so.prev_x))
    else:
        out["fin_none"] = fin is None
    dist.barrier()
    dist.destroy_process_group()
    with open(os.environ["OUT_FILE"], "w") as f:
        json.dump(out, f)
""")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,R,raw", [(2, 1, False), (3, 2, True)])
def test_context_parallel_orchestration(tmp_path, world, R, raw):
    script = tmp_path / "rank.py"
    script.write_text(RANK_SCRIPT)
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), REPO_ROOT=ROOT,
                   OUT_FILE=str(tmp_path / f"out{rank}.json"), CUDA_VISIBLE_DEVICES="",
                   RANKS_R=str(R), RAW="1" if raw else "0")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT))
    for p in procs:
        try:
            out, _ = p.communicate(timeout=240)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("gloo ranks did not finish")
        assert p.returncode == 0, out.decode(errors="replace")[-3000:]
    res = [json.loads((tmp_path / f"out{r}.json").read_text()) for r in range(world)]
    for r in res:
        assert r["y_err"] < 1e-12, res
    last = res[-1]
    assert last["h_err"] < 1e-12 and last["phi_err"] < 1e-12 and last["prev_ok"], last
    assert all(r["fin_none"] for r in res[:-1])
