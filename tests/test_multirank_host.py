"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on the CPU.

Each rank of `bench.py --gpus N` processes its own independent sequences (weak scaling) and the
reported time is the slowest rank's. These tests start two processes with the gloo backend
and check that every rank gets the maximum of the ranks' times, that the whole-job rate counts
every rank's units, and that the ranks draw different inputs.
"""
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
    import torch
    import torch.distributed as dist
    import bench
    from state_space_sequence_mamba_b200.inputs import make_config

    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = 10.0 + 7.5 * rank          # the ranks see different times
    ms = bench.max_over_ranks(local_ms, world, dist, "cpu")
    rate = bench.weak_throughput(8192, world, 5, ms)
    pr = make_config(0, seed=bench.rank_seed(rank, 0))
    out = {"rank": rank, "ms": ms, "rate": rate, "x0": float(pr.x.flatten()[0])}
    dist.barrier()
    dist.destroy_process_group()
    with open(os.environ["OUT_FILE"], "w") as f:
        json.dump(out, f)
""")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks(tmp_path):
    world = 2
    script = tmp_path / "rank.py"
    script.write_text(RANK_SCRIPT)
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), REPO_ROOT=ROOT,
                   OUT_FILE=str(tmp_path / f"out{rank}.json"), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT))
    for p in procs:
        try:
            out, _ = p.communicate(timeout=240)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("gloo ranks did not finish")
        assert p.returncode == 0, out.decode(errors="replace")[-2000:]
    res = [json.loads((tmp_path / f"out{r}.json").read_text()) for r in range(world)]
    slowest = 10.0 + 7.5 * (world - 1)
    for r in res:
        assert r["ms"] == pytest.approx(slowest)            # max over ranks, on every rank
        assert r["rate"] == pytest.approx(8192 * world * 5 / (slowest / 1e3))
    assert res[0]["x0"] != res[1]["x0"]                     # independent inputs per rank


def test_weak_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.weak_throughput(8192, 1, 10, 2.0)
    eight = bench.weak_throughput(8192, 8, 10, 2.0)
    assert eight == pytest.approx(8 * one)
    assert bench.rank_seed(0, 0) != bench.rank_seed(1, 0) != bench.rank_seed(0, 1)


def test_bench_spawns_its_ranks_and_reports_the_slowest():
    """`bench.py --gpus 2` without a launcher starts two ranks under torch.distributed.run
    (rendezvous on 127.0.0.1). With --host-plumbing the ranks are gloo CPU processes whose
    step is a fixed wait (rank 1's is the longer, 15 ms): rank 0 alone prints one line whose
    n_gpus is 2, whose step time is the slowest rank's and whose rate counts both ranks."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    env.pop("WORLD_SIZE", None)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                          "--steps", "4", "--warmup", "1", "--host-plumbing"],
                         capture_output=True, text=True, timeout=240, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, out.stdout
    r = lines[0]
    assert r["n_gpus"] == 2 and r["steps"] == 4 and r["scaling"] == "weak"
    assert r["ms_per_step"] >= 15.0                     # rank 1's wait, not rank 0's 10 ms
    want = r["units_per_rank_step"] * 2 * 4 / (r["ms_per_step"] * 4 / 1e3)
    assert abs(r["value"] - want) <= 1e-9 * want


def test_bench_rejects_a_rank_count_that_disagrees_with_the_launcher():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                          "--host-plumbing"], capture_output=True, text=True, timeout=120,
                         env=env, cwd=ROOT)
    assert out.returncode != 0 and "WORLD_SIZE=3" in out.stderr
