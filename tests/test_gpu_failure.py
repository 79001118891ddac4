"""Failure detection and out-of-bounds writes on the GPU, without faulting it.

- The timeout path: the tensor-core scan's test hook (environment variable
  M3_TEST_SKIP_THETA_LOAD=k) makes CTA 0 skip the theta load of chunk k, so that its bounded
  mbarrier wait (about 2e9 SM clocks, about a second) runs out. The CTA then records the
  status word, waits for the copies and tensor-core work it did start, releases its tensor
  memory and exits; every other CTA finishes normally. m3_scan_check must report
  M3_ERR_TIMEOUT and zero the header, and the next call on the same workspace must be exact.
- Guard bands: y and every field of the final state are views into larger buffers whose
  surrounding bytes hold a fixed pattern; ragged-length scans (SISO, MIMO, 64- and 128-row
  chunks, one and several segments) must leave the pattern untouched and match the oracle.
"""
import os

import pytest
import torch

from gpu_common import compare, oracle_scan
from state_space_sequence_mamba_b200 import binding as m3
from state_space_sequence_mamba_b200.inputs import make_problem

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("R,chunk", [(1, 64), (1, 128), (4, 32)])
def test_timeout_is_reported_and_the_workspace_reusable(cuda_dev, R, chunk):
    """Through the 64-row (chunk 64) and the 128-row (chunk 128 / R) tensor-core scans."""
    pr = make_problem(2, 300, 4, 1, 64, 128, rank=R, chunk=chunk, bc_norm=True, bias_std=0.1,
                      seed=151 + R, with_state=True)
    g = pr.to(cuda_dev)
    t = g.tensors()
    dims = m3.make_dims(t["x"], t["B"], chunk, True, 1e-6)
    ws = torch.zeros(m3.scan_workspace_bytes(dims), dtype=torch.uint8, device=cuda_dev)
    init = m3.State.from_dict(g.state)
    os.environ["M3_TEST_SKIP_THETA_LOAD"] = "1"
    try:
        m3.scan_fwd(**t, init=init, chunk=chunk, bc_norm=True, workspace=ws)
        torch.cuda.synchronize()
    finally:
        del os.environ["M3_TEST_SKIP_THETA_LOAD"]
    with pytest.raises(m3.M3Error) as ei:
        m3.scan_check(ws)
    assert ei.value.status == m3.M3_ERR_TIMEOUT
    assert int(ws[:256].count_nonzero()) == 0          # the header is zero again
    # the same workspace, the same stream, right after: a normal call, checked exactly
    y, fin = m3.scan_fwd(**t, init=init, chunk=chunk, bc_norm=True, workspace=ws)
    torch.cuda.synchronize()
    m3.scan_check(ws)
    yo, so = oracle_scan(pr)
    compare(pr, y, fin, yo, so)


@pytest.mark.parametrize("R", [1, 4])
def test_backward_timeout_is_reported_and_the_workspace_reusable(cuda_dev, R):
    """The chunked tensor-core backward: CTA 0 skips one load group (theta, dY, raw C) of its
    second step, so its bounded wait gives up; m3_scan_check reports the timeout on the
    backward's workspace and the next call on the same workspace matches the oracle (the
    drain of the CTA's copies and MMAs and the TMEM release worked)."""
    from test_gpu_backward import draw_grads, oracle_grads
    from test_gpu_backward_tc import compare_tc
    pr = make_problem(1, 200, 4, 1, 64, 128, rank=R, chunk=64 // R, dtype=torch.bfloat16,
                      bc_norm=True, bias_std=0.1, seed=171 + R, with_state=True)
    dy, dfin = draw_grads(pr, seed=5)
    g = pr.to(cuda_dev)
    t = g.tensors()
    dims = m3.make_dims(t["x"], t["B"], 1, True, 1e-6)
    ws = torch.zeros(m3.scan_bwd_workspace_bytes(dims), dtype=torch.uint8, device=cuda_dev)
    init = m3.State.from_dict(g.state)
    df = {k: v.to(cuda_dev) for k, v in dfin.items()}

    def call():
        return m3.scan_bwd(**t, dy=dy.to(cuda_dev), init=init, dfinal=df, bc_norm=True,
                           workspace=ws)

    os.environ["M3_TEST_SKIP_THETA_LOAD"] = "1"
    try:
        call()
        torch.cuda.synchronize()
    finally:
        del os.environ["M3_TEST_SKIP_THETA_LOAD"]
    with pytest.raises(m3.M3Error) as ei:
        m3.scan_check(ws)
    assert ei.value.status == m3.M3_ERR_TIMEOUT
    assert int(ws[:256].count_nonzero()) == 0          # the header is zero again
    got = call()
    torch.cuda.synchronize()
    m3.scan_check(ws)
    compare_tc(got, oracle_grads(pr, dy, dfin), pr)


PAT = 0x5A   # the guard bytes
BAND = 4096  # bytes before and after each output


def guarded(shape, dtype, dev):
    """A tensor of `shape` inside a byte buffer with BAND pattern bytes on each side."""
    n = int(torch.Size(shape).numel()) * torch.empty(0, dtype=dtype).element_size()
    buf = torch.full((BAND + n + BAND,), PAT, dtype=torch.uint8, device=dev)
    return buf, buf[BAND:BAND + n].view(dtype).view(shape)


def bands_intact(buf):
    n = buf.numel()
    return bool((buf[:BAND] == PAT).all()) and bool((buf[n - BAND:] == PAT).all())


GUARD = [
    # b, L, H, G, R, chunk: ragged tails; the b1 L2543 cases run in 5 segments
    (2, 77, 4, 1, 1, 64),
    (1, 2543, 4, 1, 1, 64),
    (2, 51, 4, 2, 4, 16),
    (1, 700, 4, 1, 4, 16),
    (2, 201, 4, 1, 1, 128),
    (2, 59, 4, 1, 4, 32),
    (1, 33, 2, 1, 8, 8),
]


@pytest.mark.parametrize("case", GUARD, ids=lambda c: "b{}L{}H{}G{}R{}Q{}".format(*c))
def test_outputs_stay_inside_their_buffers(cuda_dev, case):
    b, L, H, G, R, Q = case
    P, N = 64, 128
    pr = make_problem(b, L, H, G, P, N, rank=R, chunk=Q, bc_norm=True, bias_std=0.1,
                      seed=160 + L + R, with_state=True)
    g = pr.to(cuda_dev)
    dt = g.x.dtype
    bufs = {}
    bufs["y"], y = guarded(g.x.shape, dt, cuda_dev)
    bufs["h"], h = guarded((b, H, N, P), torch.float32, cuda_dev)
    bufs["phi"], phi = guarded((b, H, N // 2), torch.float32, cuda_dev)
    bufs["prev_B"], pB = guarded((b, H, R, N), dt, cuda_dev)
    bufs["prev_x"], px = guarded((b, H, R, P), dt, cuda_dev)
    fin = m3.State(h, phi, pB, px)
    y, fin = m3.scan_fwd(**g.tensors(), init=m3.State.from_dict(g.state), final=fin, y=y,
                         chunk=Q, bc_norm=True)
    torch.cuda.synchronize()
    for k, buf in bufs.items():
        assert bands_intact(buf), k
    yo, so = oracle_scan(pr)
    compare(pr, y, fin, yo, so)


@pytest.mark.parametrize("R", [1, 4])
def test_decode_outputs_stay_inside_their_buffers(cuda_dev, R):
    b, H, P, N = 3, 4, 64, 128
    pr = make_problem(b, 1, H, 1, P, N, rank=R, chunk=1, bc_norm=True, bias_std=0.1,
                      seed=170 + R, with_state=True)
    g = pr.to(cuda_dev)
    dt = g.x.dtype
    bufs = {}
    bufs["y"], y = guarded((b, H, R, P), dt, cuda_dev)
    bufs["h"], h = guarded((b, H, N, P), torch.float32, cuda_dev)
    bufs["phi"], phi = guarded((b, H, N // 2), torch.float32, cuda_dev)
    bufs["prev_B"], pB = guarded((b, H, R, N), dt, cuda_dev)
    bufs["prev_x"], px = guarded((b, H, R, P), dt, cuda_dev)
    out = m3.State(h, phi, pB, px)
    y, out = m3.decode_step(**g.tensors(), state_in=m3.State.from_dict(g.state),
                            state_out=out, y=y, bc_norm=True)
    torch.cuda.synchronize()
    for k, buf in bufs.items():
        assert bands_intact(buf), k
    yo, so = oracle_scan(pr)
    compare(pr, y[:, None], out, yo, so)
