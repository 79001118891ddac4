"""Benchmark of the Mamba-3 SSM core on B200.

Headline: prefill throughput (tokens/s) of the SISO chunked scan at 1.5B-layer shapes
(batch 4, 64 heads, head dim 64, state 128, L 2048, chunk 64, bf16 inputs, fp32 state,
BC norm + bias), one m3_scan_fwd per step, inputs resident in HBM. Also reported: the
decode step (batch 128, 64 heads, SISO and MIMO R=4) as us/step over 1000 consecutive steps
captured in one CUDA graph, the end-to-end prefill through the public API with host buffers,
the roofline of the dominant kernel, SM clocks during the timed region, and the CPU oracle.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-decode]
For N > 1 it runs under torch.distributed.run (started by itself when no launcher set
WORLD_SIZE); every rank runs its own copy of the workload (independent sequences: weak
scaling, no collective on the data path) and the reported time is the slowest rank's.
--context-parallel adds the long-sequence prefill split along the sequence over the ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSM prefill tokens/s + decode µs/step at 1.5B shapes; % of HBM/TC roofline"
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the dominant
# scan kernel on this workload, from one ncu capture, keyed by the SHA-256 of the kernel's
# source file when it was captured: reported while that file is unchanged, else null.
SCAN_TRAFFIC = {"kernel": "scan_tc_kernel",
                "source": "state_space_sequence_mamba_b200/csrc/m3_scan_tc.cu",
                "sha256": "0987a86f8a47ce05cb03c949cc42428ab50417a13d9b95527b7e1b7b1338848d",
                "bytes": 186.534144e6}
# kernels one scan launches: the per-token RMS-scale pre-pass of B and C, then the scan
KERNELS_PER_SCAN = 2
WORKLOAD = "SISO prefill b4 H64 P64 N128 L2048 chunk64 bf16/fp32-state BCNorm+bias"


def scan_traffic():
    """The captured DRAM bytes per launch, or None when the kernel source has changed since
    (or no capture is recorded)."""
    import hashlib
    if SCAN_TRAFFIC["sha256"] is None:
        return None
    with open(os.path.join(ROOT, SCAN_TRAFFIC["source"]), "rb") as f:
        same = hashlib.sha256(f.read()).hexdigest() == SCAN_TRAFFIC["sha256"]
    return SCAN_TRAFFIC["bytes"] if same else None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the backward pass (SISO and MIMO R4) and print its numbers")
    ap.add_argument("--bwd-seqlen", type=int, default=None,
                    help="sequence length of the --backward-only workloads (default: theirs)")
    ap.add_argument("--context-parallel", action="store_true",
                    help="also time the long-sequence prefill (b1 H64 L65536) split along the "
                         "sequence over the ranks (N > 1)")
    ap.add_argument("--host-plumbing", action="store_true",
                    help="check the multi-rank launch, max-over-ranks timing and report on "
                         "CPU ranks (gloo), with a fixed per-rank wait as the step: no GPU")
    return ap.parse_args()


def spawn_ranks(args) -> int:
    """`--gpus N` (N > 1) started without a launcher: run this script again under
    torch.distributed.run with N processes on this node, one per GPU, rendezvous on
    127.0.0.1. Rank 0 prints the line; returns the launcher's exit code."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def run_host_plumbing(args):
    """The multi-rank path of the report without a GPU: gloo ranks whose step is a fixed
    wait (10 + 5 * rank ms), timed on each rank, maximised over the ranks, turned into the
    whole-job rate of `units` per rank and step, and printed by rank 0."""
    import datetime
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    wait = 0.010 + 0.005 * rank
    units = 8192
    for _ in range(args.warmup):
        time.sleep(wait)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time.sleep(wait)
    local_ms = (time.perf_counter() - t0) * 1e3
    total_ms = max_over_ranks(local_ms, world, dist, "cpu")
    if rank == 0:
        print(json.dumps({"check": "host-plumbing", "n_gpus": world, "steps": args.steps,
                          "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
                          "value": weak_throughput(units, world, args.steps, total_ms),
                          "units_per_rank_step": units, "scaling": "weak"}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(ms, world, dist, device):
    """The slowest rank's time (every rank calls this at the same point of the run)."""
    if world == 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_throughput(units_per_rank, world, steps, total_ms):
    """Whole-job rate when every rank processes its own units_per_rank per step."""
    return units_per_rank * world * steps / (total_ms / 1e3)


def rank_seed(rank, i):
    """Seed of input set i on a rank: every rank draws its own independent sequences."""
    return 1 + 100 * rank + i


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.index, f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r)
                          if v.lower() == "active"})
        sm = sorted(r[0] for r in rows)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def scan_bytes(pr) -> int:
    """Algorithmic HBM bytes of one scan: every input read once, y written once, final
    state written once (no initial state)."""
    t = pr.tensors()
    n = sum(v.numel() * v.element_size() for v in t.values() if v is not None)
    n += t["x"].numel() * t["x"].element_size()  # y
    d = pr.dims
    es = t["x"].element_size()
    units = d.batch * d.nheads
    n += units * (d.dstate * d.headdim * 4 + d.dstate // 2 * 4 + d.rank * (d.dstate + d.headdim) * es)
    return int(n)


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from state_space_sequence_mamba_b200 import binding as m3
    from state_space_sequence_mamba_b200.inputs import make_config, make_decode
    m3.load_library()
    hbm, tc, peak_kind = peaks()
    if args.backward_only:
        out = {"backward": {
            name: bench_backward(m3, dev, cfg, hbm, world, dist, rank_seed(rank, 11 + cfg),
                                 reps=args.steps, seqlen=args.bwd_seqlen, exact=exact)
            for name, cfg, exact in (("siso_b4", 1, False), ("siso_b4_fp32", 1, True),
                                     ("mimo_r4_b4", 2, False))}, "peak_hbm_gbs": hbm,
            "seqlen": args.bwd_seqlen or 2048}
        if rank == 0:
            print(json.dumps(out), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    # two input sets (each > L2) alternate between steps so no step reads the previous
    # step's inputs from L2
    sets = [make_config(1, device=dev, seed=rank_seed(rank, i)) for i in range(2)]
    d = sets[0].dims
    y = torch.empty_like(sets[0].x)
    fin = m3.State.empty(d.batch, d.nheads, d.dstate, d.headdim, d.rank, d.dtype, dev)
    ws = torch.zeros(max(256, m3.scan_workspace_bytes(m3.make_dims(sets[0].x, sets[0].B,
                                                                   d.chunk, True, 1e-6))),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        m3.scan_fwd(**sets[i % 2].tensors(), init=None, final=fin, y=y, workspace=ws,
                    chunk=d.chunk, bc_norm=True, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    props = torch.cuda.get_device_properties(dev)
    gpu_id = ("GPU-" + str(props.uuid)) if getattr(props, "uuid", None) else str(local)
    with ClockSampler(gpu_id) as clk:
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            step(i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    m3.scan_check(ws)
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), world, dist, dev)
    per_launch = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    tokens = d.batch * d.seqlen
    value = weak_throughput(tokens, world, args.steps, total_ms)
    byts = scan_bytes(sets[0])
    launch_ms = sum(per_launch) / len(per_launch)
    achieved = byts / (launch_ms / 1e3) / 1e9

    # ---- end to end through the public API: pinned host inputs in, y and the final state
    # out, every step ----
    # Steps are pipelined over three streams with two buffer sets, as a serving loop would
    # run them: step i+1's inputs go host -> device while step i's results go device -> host
    # (the two directions use separate copy engines). Each step still copies all of its
    # inputs in and its whole y and final state (h, phi, prev_B, prev_x) out inside the timed
    # region.
    host = {k: (v.cpu().pin_memory() if v is not None else None)
            for k, v in sets[0].tensors().items()}
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    dev_in = [{k: (torch.empty_like(v, device=dev) if v is not None else None)
               for k, v in host.items()} for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]
    fin_dev = [m3.State.empty(d.batch, d.nheads, d.dstate, d.headdim, d.rank, d.dtype, dev)
               for _ in range(2)]
    fin_fields = ("h", "phi", "prev_B", "prev_x")
    fin_host = [{k: torch.empty(getattr(fin_dev[0], k).shape,
                                dtype=getattr(fin_dev[0], k).dtype).pin_memory()
                 for k in fin_fields} for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = y_host[0].numel() * y_host[0].element_size() + sum(
        v.numel() * v.element_size() for v in fin_host[0].values())
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    for j in range(2):          # every buffer starts free
        comp_done[j].record(stream)
        out_done[j].record(stream)

    def e2e_step(i):
        j = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(comp_done[j])         # the scan of step i-2 has read these inputs
            for k, v in host.items():
                if v is not None:
                    dev_in[j][k].copy_(v, non_blocking=True)
            in_done[j].record(s_in)
        stream.wait_event(in_done[j])
        stream.wait_event(out_done[j])            # y of step i-2 has left the device
        m3.scan_fwd(**dev_in[j], init=None, final=fin_dev[j], y=y_dev[j], workspace=ws,
                    chunk=d.chunk, bc_norm=True, stream=stream)
        comp_done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[j])
            y_host[j].copy_(y_dev[j], non_blocking=True)
            for k in fin_fields:
                fin_host[j][k].copy_(getattr(fin_dev[j], k), non_blocking=True)
            out_done[j].record(s_out)

    e2e_steps = max(3, min(args.steps, 10))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev)
    e2e_val = weak_throughput(tokens, world, e2e_steps, e2e_ms)
    del host, dev_in, y_host, y_dev, fin_dev, fin_host

    # ---- decode: 1000 consecutive steps in one CUDA graph, SISO and MIMO R=4 ----
    decode = {}
    if not args.no_decode:
        for R in (1, 4):
            decode[f"R{R}"] = bench_decode(m3, dev, R, args.decode_steps, hbm, world, dist)

    # ---- the other prefill workloads (parity configurations, reported beside the headline):
    # MIMO R4 (b4 L2048) and the long sequence (b1 L65536, sequence-parallel form) ----
    others = {}
    if not args.no_decode:
        for name, cfg in (("mimo_r4_b4_L2048", 2), ("long_b1_L65536", 4)):
            po = make_config(cfg, device=dev, seed=rank_seed(rank, cfg))
            do = po.dims
            yo = torch.empty_like(po.x)
            fo = m3.State.empty(do.batch, do.nheads, do.dstate, do.headdim, do.rank, do.dtype, dev)
            wso = torch.zeros(max(256, m3.scan_workspace_bytes(m3.make_dims(
                po.x, po.B, do.chunk, True, 1e-6))), dtype=torch.uint8, device=dev)

            def step_o():
                m3.scan_fwd(**po.tensors(), init=None, final=fo, y=yo, workspace=wso,
                            chunk=do.chunk, bc_norm=True, stream=stream)

            for _ in range(3):
                step_o()
            torch.cuda.synchronize()
            reps = 3 if cfg == 4 else 10
            e0.record(stream)
            for _ in range(reps):
                step_o()
            e1.record(stream)
            torch.cuda.synchronize()
            oms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev) / reps
            others[name] = {"ms_per_scan": oms,
                            "tokens_per_s": do.batch * do.seqlen * world / (oms / 1e3),
                            "frac_hbm": scan_bytes(po) / (oms / 1e3) / 1e9 / hbm}
            del po, yo, fo, wso

    # ---- the fused scalar prologue: dt and lam passed raw, softplus / sigmoid applied in the
    # kernels (same workloads, one input set each) ----
    prologue = {}
    if not args.no_decode:
        praw = make_config(1, device=dev, seed=rank_seed(rank, 0), raw_scalars=True)

        def step_raw():
            m3.scan_fwd(**praw.tensors(), **praw.scalar_args(), init=None, final=fin, y=y,
                        workspace=ws, chunk=d.chunk, bc_norm=True, stream=stream)

        for _ in range(3):
            step_raw()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(10):
            step_raw()
        e1.record(stream)
        torch.cuda.synchronize()
        pms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev) / 10
        prologue["prefill_ms"] = pms
        prologue["prefill_frac_hbm"] = scan_bytes(praw) / (pms / 1e3) / 1e9 / hbm
        del praw
        prologue["decode_R4"] = bench_decode(m3, dev, 4, args.decode_steps, hbm, world, dist,
                                             raw=True)
        decode["R4_proj"] = bench_decode(m3, dev, 4, args.decode_steps, hbm, world, dist,
                                         proj=True)

    # ---- the backward pass of the scan (training side), SISO and MIMO R4 workloads ----
    backward = {}
    if not args.no_decode:
        backward["siso_b4_L2048"] = bench_backward(m3, dev, 1, hbm, world, dist,
                                                   rank_seed(rank, 11),
                                                   cpu=(rank == 0 and world == 1))
        backward["siso_b4_L2048_fp32"] = bench_backward(m3, dev, 1, hbm, world, dist,
                                                        rank_seed(rank, 11), exact=True)
        backward["mimo_r4_b4_L2048"] = bench_backward(m3, dev, 2, hbm, world, dist,
                                                      rank_seed(rank, 12))

    cp_leg = None
    if args.context_parallel:
        cp_leg = (bench_context_parallel(m3, dev, hbm, world, dist, stream) if world > 1 else
                  {"skipped": "needs more than one rank"})
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch_per_gpu": d.batch, "seq_len": d.seqlen,
                   "nheads": d.nheads, "headdim": d.headdim, "dstate": d.dstate,
                   "chunk": d.chunk, "parallelism": f"independent sequences x{world}",
                   "l2": "two alternating input sets of 144 MB each (> 126 MB L2), no flush"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": scan_traffic(),
                     "bytes_per_launch": byts, "launch_ms": launch_ms,
                     "peak_source": peak_kind},
        "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * KERNELS_PER_SCAN,
        "clocks": clk.summary(),
        "decode": decode,
        "fused_scalar_prologue": prologue,
        "other_prefill": others,
        "backward": backward,
    }
    if cp_leg is not None:
        line["context_parallel"] = cp_leg
    if rank == 0:
        line["cpu_baseline"] = cpu_baseline(sets[0]) if world == 1 else None
        if world == 1 and not args.no_decode:
            line["cpu_baselines"] = cpu_baselines()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def bench_context_parallel(m3, dev, hbm, world, dist, stream, reps=3):
    """The long-sequence prefill (b1 H64 L65536) split along the sequence over the ranks:
    rank k scans tokens [k L / N, (k + 1) L / N) of the same sequence after one exchange of
    the last tokens and the segments' end states (two NCCL all-gathers, no peer loads), and
    the time is the slowest rank's. Strong scaling: the sequence is fixed."""
    import torch
    from state_space_sequence_mamba_b200 import context_parallel as cp
    from state_space_sequence_mamba_b200.inputs import make_config
    rank = dist.get_rank()
    pr = make_config(4, device=dev, seed=rank_seed(0, 40))   # the same sequence on every rank
    d = pr.dims
    L = d.seqlen
    lo, hi = L * rank // world, L * (rank + 1) // world
    t = {k: (v[:, lo:hi].contiguous() if k not in ("B_bias", "C_bias") else v)
         for k, v in pr.tensors().items()}
    del pr

    def run():
        return cp.scan_context_parallel(**t, chunk=d.chunk, bc_norm=True)

    for _ in range(2):
        run()
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev) / reps
    return {"workload": "long SISO prefill b1 H64 L65536 split over the ranks", "world": world,
            "ms_per_scan": ms, "tokens_per_s": d.batch * L / (ms / 1e3), "scaling": "strong",
            "exchange": "two all-gathers of last tokens and end states (NCCL)"}


def bwd_bytes(pr) -> int:
    """Algorithmic HBM bytes of one backward pass: every forward input, dy and the initial
    state read once; every gradient (fp32) written once."""
    import torch
    d = pr.dims
    es = 2 if d.dtype == torch.bfloat16 else 4
    b, L, H, G, P, N, R = d.batch, d.seqlen, d.nheads, d.ngroups, d.headdim, d.dstate, d.rank
    units = b * H
    reads = (es * (2 * b * L * H * R * P + 2 * b * L * G * R * N + b * L * H * N // 2)
             + 12 * b * L * H + 8 * H * R * N)
    writes = 4 * (b * L * H * R * P + 2 * b * L * G * R * N + b * L * H * N // 2 + 3 * b * L * H
                  + 2 * H * R * N)
    if pr.state is not None:
        reads += units * (4 * N * P + 4 * N // 2 + es * R * (N + P))
        writes += units * 4 * (N * P + N // 2 + R * (N + P))
    return reads + writes


def bwd_chunked(m3, dims) -> bool:
    """Whether m3_scan_bwd runs the chunked tensor-core form for these dims, as the library
    decides it: only that form needs workspace beyond the fp32 sweeps' (its chunk states)."""
    import copy
    fp32 = copy.copy(dims)
    fp32.flags = dims.flags | m3.BWD_FP32
    return m3.scan_bwd_workspace_bytes(dims) > m3.scan_bwd_workspace_bytes(fp32)


def bench_backward(m3, dev, cfg, hbm, world, dist, seed, reps=5, seqlen=None, cpu=False,
                   exact=False):
    """m3_scan_bwd on a prefill workload with a carried initial state and dy ~ N(0,1); with
    exact, the fp32 sequential sweeps (M3_BWD_FP32) instead of the path the call picks."""
    import torch
    from state_space_sequence_mamba_b200.inputs import make_config
    kw = {} if seqlen is None else {"seqlen": seqlen}
    pr = make_config(cfg, device=dev, seed=seed, with_state=True, **kw)
    d = pr.dims
    g = torch.Generator(device=dev).manual_seed(seed + 1)
    dy = torch.randn(pr.x.shape, generator=g, device=dev).to(d.dtype)
    init = m3.State.from_dict(pr.state)
    sa = pr.scalar_args()
    if exact:
        sa["flags"] = sa["flags"] | m3.BWD_FP32
    dims = m3.make_dims(pr.x, pr.B, 1, d.bc_norm, d.norm_eps, sa["flags"])
    ws = torch.empty(m3.scan_bwd_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    tc = bwd_chunked(m3, dims)
    stream = torch.cuda.current_stream()

    def step():   # the config's own BC norm, eps and scalar form, as the CPU baseline reads them
        return m3.scan_bwd(**pr.tensors(), dy=dy, init=init, bc_norm=d.bc_norm,
                           norm_eps=d.norm_eps, workspace=ws, stream=stream, **sa)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev) / reps
    byts = bwd_bytes(pr)
    out = {"ms_per_backward": ms, "tokens_per_s": d.batch * d.seqlen * world / (ms / 1e3),
           "bytes": byts, "frac_hbm": byts / (ms / 1e3) / 1e9 / hbm,
           # chunked: [RMS scales], state pass, chunk kernel, bias sums, scalar, norm;
           # sequential: [RMS scales], two sweeps, scalar, norm
           "form": "tensor-core chunked" if tc else "fp32 sequential sweeps",
           "kernels_per_call": (5 if tc else 4) + (1 if d.bc_norm else 0),
           "workspace_bytes": ws.numel()}
    if cpu:   # an auxiliary field: a failure here is reported, not fatal to the bench line
        try:
            out["cpu_baseline"] = cpu_baseline_backward(pr, dy)
        except Exception as e:  # noqa: BLE001
            out["cpu_baseline"] = {"error": f"{type(e).__name__}: {e}"[:200]}
    del pr, dy, init, ws
    torch.cuda.empty_cache()
    return out


def bench_decode(m3, dev, R, steps, hbm, world, dist, raw=False, proj=False):
    import torch
    from state_space_sequence_mamba_b200.inputs import make_decode, make_proj
    pr = make_decode(R, steps, device=dev, raw_scalars=raw)
    if proj:   # MIMO projections fused: x' and z' [P] in, O' [P] out
        xp, zp, WX, WZ, WO = make_proj(steps, pr.dims.batch, pr.dims.nheads, pr.dims.headdim,
                                       R, dtype=torch.bfloat16, seed=5, device=dev)
        ob = torch.empty(pr.dims.batch, pr.dims.nheads, pr.dims.headdim, dtype=torch.bfloat16,
                         device=dev)
    st = m3.State.from_dict({k: v.clone() for k, v in pr.state.items()})
    yb = torch.empty(pr.dims.batch, pr.dims.nheads, R, pr.dims.headdim, dtype=torch.bfloat16,
                     device=dev)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())

    def run(n):
        for t in range(n):
            if proj:
                m3.decode_step_proj(xp[t], zp[t], WX, WZ, WO, pr.B[t], pr.C[t], pr.theta[t],
                                    pr.dt[t], pr.A[t], pr.lam[t], dt_bias=pr.dt_bias,
                                    flags=pr.flags, state_in=st, o=ob, stream=s)
            else:
                m3.decode_step(pr.x[t], pr.B[t], pr.C[t], pr.theta[t], pr.dt[t], pr.A[t],
                               pr.lam[t], dt_bias=pr.dt_bias, flags=pr.flags,
                               state_in=st, y=yb, stream=s)

    with torch.cuda.stream(s):
        run(3)  # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run(steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):  # replay() launches on the current stream
        g.replay()  # warm-up replay
        torch.cuda.synchronize()
        e0.record(s)
        g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev)
    us = ms * 1e3 / steps
    units = pr.dims.batch * pr.dims.nheads
    es = 2
    N, P = pr.dims.dstate, pr.dims.headdim
    # state h and phi read + written, prev_B and prev_x read + written, x and y (or x', z'
    # and O'), theta, dt/A/lam; B and C once per batch row; the projection weights once
    io = 3 * P * es if proj else 2 * R * P * es
    per_unit = (2 * N * P * 4 + 2 * (N // 2) * 4 + 2 * R * N * es + 2 * R * P * es
                + io + (N // 2) * es + 3 * 4)
    byts = units * per_unit + pr.dims.batch * 2 * R * N * es
    if proj:
        byts += 3 * pr.dims.nheads * R * P * 4
    ach = byts / (us / 1e6) / 1e9
    del g
    return {"us_per_step": us, "steps": steps, "graph": True, "bytes_per_step": byts,
            "achieved_gbs": ach, "frac_hbm": ach / hbm, "gpu_launches": steps}


def cpu_baseline(pr, min_s=10.0, max_reps=30):
    """The fp64 oracle as it stands, on all host cores, on the whole workload (every sequence,
    head and token), repeated until about min_s seconds of CPU work have been timed."""
    import oracle
    t = {k: (v.cpu() if v is not None else None) for k, v in pr.tensors().items()}
    cores = oracle.max_threads()
    reps, el = 0, 0.0
    while reps < max_reps and (reps == 0 or el < min_s):
        t0 = time.perf_counter()
        oracle.scan(**t, bc_norm=True, nthreads=cores)
        el += time.perf_counter() - t0
        reps += 1
    tokens = t["x"].shape[0] * t["x"].shape[1] * reps
    return {"value": tokens / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"the whole workload ({pr.dims.batch} sequences x {pr.dims.nheads} heads x "
                      f"L={pr.dims.seqlen}) x {reps} passes, {el:.1f} s"}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _timed_oracle(make, start, limit, target_s, nthreads):
    """The oracle scan on samples of growing size (`make(k)` builds one of k units) until one
    takes at least target_s or k reaches limit. Returns (k, seconds)."""
    import oracle
    k = start
    while True:
        t = make(k)
        t0 = time.perf_counter()
        oracle.scan(**t, nthreads=nthreads)
        el = time.perf_counter() - t0
        if el >= target_s or k >= limit:
            return k, el
        k = min(limit, max(2 * k, int(k * target_s / max(el, 1e-3) * 1.2)))


def cpu_baselines(target_s=1.5):
    """The fp64 oracle as it stands on every workload of the measurement: one thread and all
    host cores, each on a bounded sample (reduced head count, or reduced batch for the
    decode steps, at full length), scaled to the workload's unit. Prefill: tokens/s of the
    whole workload (a sample of k of H heads runs k/H of its work). Decode: us per step of
    the whole batch over 1000 consecutive steps, from a sample of heads of one sequence (the
    oracle's scan over those steps is the same recurrence)."""
    import oracle
    from state_space_sequence_mamba_b200.inputs import make_config, make_decode
    cores = oracle.max_threads()
    out = {"cpu_model": cpu_model(), "nproc": os.cpu_count(), "kind": "oracle"}

    def prefill(cfg):
        H = 64

        def make(k):
            pr = make_config(cfg, batch=1, nheads=k)
            t = {kk: v for kk, v in pr.tensors().items()}
            t.update(bc_norm=True)
            return t
        L = make_config(cfg, batch=1, nheads=1).dims.seqlen
        res = {}
        for name, nt, start in (("one_thread", 1, 1), ("all_cores", cores, min(H, cores))):
            k, el = _timed_oracle(make, start, H, target_s, nt)
            res[name] = {"value": L * k / H / el, "unit": "tokens/s", "threads": nt,
                         "sample": f"1 sequence, {k} of {H} heads, L={L}, {el:.2f} s"}
        return res

    def decode(R, steps=1000, batch=128, H=64):
        def make(k):
            pr = make_decode(R, steps, batch=1, nheads=k)
            sq = lambda v: v[:, :, 0].transpose(0, 1).contiguous()
            st = oracle.State(*(pr.state[f].double().numpy()
                                for f in ("h", "phi", "prev_B", "prev_x")))
            return dict(x=sq(pr.x), B=sq(pr.B), C=sq(pr.C), theta=sq(pr.theta), dt=sq(pr.dt),
                        A=sq(pr.A), lam=sq(pr.lam), state=st)
        res = {}
        for name, nt, start in (("one_thread", 1, 1), ("all_cores", cores, min(H, cores))):
            k, el = _timed_oracle(make, start, H, target_s, nt)
            res[name] = {"value": el / steps * batch * H / k * 1e6, "unit": "us/step",
                         "threads": nt, "sample": f"1 of {batch} sequences, {k} of {H} heads, "
                                                  f"{steps} steps, {el:.2f} s"}
        return res

    for key, fn in (("siso_prefill_b4_L2048", lambda: prefill(1)),
                    ("mimo_r4_prefill_b4_L2048", lambda: prefill(2)),
                    ("decode_siso_b128_1000_steps", lambda: decode(1)),
                    ("decode_mimo_r4_b128_1000_steps", lambda: decode(4)),
                    ("long_prefill_b1_L65536", lambda: prefill(4))):
        try:
            out[key] = fn()
        except Exception as e:  # noqa: BLE001  (an auxiliary field: reported, not fatal)
            out[key] = {"error": f"{type(e).__name__}: {e}"[:200]}
    return out


def cpu_baseline_backward(pr, dy, heads=8):
    """The gradient oracle (float64 autograd of the plain recurrence) as it stands, on the host
    cores, on a bounded sample of a backward workload: sequence 0 and its first `heads` heads,
    every token. The rate counts the sample as that fraction of the workload's tokens."""
    import torch
    import oracle
    from oracle import grad as og
    hs = torch.arange(heads)
    t = {}
    for k, v in pr.tensors().items():
        if v is None:
            t[k] = None
        elif k in ("x", "theta", "dt", "A", "lam"):
            t[k] = v[:1, :, hs].cpu()
        elif k in ("B_bias", "C_bias"):
            t[k] = v[hs].cpu()
        else:
            t[k] = v[:1].cpu()
    st = None if pr.state is None else oracle.State(
        *(pr.state[k][:1, hs].double().cpu().numpy() for k in ("h", "phi", "prev_B", "prev_x")))
    t0 = time.perf_counter()
    og.scan_grad(**t, state=st, dy=dy[:1, :, hs].cpu(), bc_norm=pr.dims.bc_norm,
                 norm_eps=pr.dims.norm_eps)
    el = time.perf_counter() - t0
    tokens = pr.dims.seqlen * heads / pr.dims.nheads
    return {"value": tokens / el, "unit": "tokens/s", "cores": torch.get_num_threads(),
            "kind": "oracle",
            "sample": f"sequence 0, heads 0-{heads - 1} of {pr.dims.nheads}, L={pr.dims.seqlen} "
                      f"(= {tokens:.0f} workload tokens), {el:.1f} s"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from state_space_sequence_mamba_b200.inputs import make_config
    pr = make_config(1)
    t = {k: (v[:1] if (v is not None and k not in ("B_bias", "C_bias")) else v)
         for k, v in pr.tensors().items()}
    cores = oracle.max_threads()
    for _ in range(args.warmup):
        oracle.scan(**t, bc_norm=True, nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.scan(**t, bc_norm=True, nthreads=cores)
    el = time.perf_counter() - t0
    tokens = t["x"].shape[1]
    v = tokens * args.steps / el
    sample = (f"1 of {pr.dims.batch} sequences per step (all {pr.dims.nheads} heads, "
              f"L={pr.dims.seqlen})")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(a))
    if int(os.environ.get("WORLD_SIZE", 1)) != a.gpus:
        sys.exit(f"--gpus {a.gpus} but WORLD_SIZE={os.environ.get('WORLD_SIZE')}")
    if a.host_plumbing:
        run_host_plumbing(a)
    elif a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
