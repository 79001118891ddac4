"""Host-side checks of the C ABI that need no GPU: the library loads, exports every entry
point include/m3.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import __graft_entry__
from state_space_sequence_mamba_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    __graft_entry__.build()
    return bd.load_library()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(m3_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(lib):
    decl = declared_functions()
    assert {"m3_scan_fwd", "m3_decode_step", "m3_scan_workspace_bytes", "m3_scan_check"} <= decl
    for name in decl:
        assert hasattr(lib, name), name
    assert set(bd.EXPORTS) == decl


def test_status_strings(lib):
    for s in range(5):
        assert lib.m3_status_str(s).decode()
    assert lib.m3_status_str(99).decode() == "unknown status"


def dims(**kw):
    d = dict(batch=2, seqlen=10, nheads=4, ngroups=1, headdim=64, dstate=128, rank=1, chunk=64,
             in_dtype=bd.M3_BF16, bc_norm=1, norm_eps=1e-6, flags=0)
    d.update(kw)
    return bd.Dims(*(d[f] for f, _ in bd.Dims._fields_))


def test_struct_layout_matches_header(lib):
    assert ctypes.sizeof(bd.Dims) == 8 * 8 + 4 + 4 + 4 + 4  # ..., norm_eps, flags
    assert ctypes.sizeof(bd.Inputs) == 10 * 8 and ctypes.sizeof(bd.StateC) == 4 * 8


@pytest.mark.parametrize("kw,ok", [
    ({}, True), (dict(nheads=3, ngroups=2), False), (dict(dstate=15), False),
    (dict(headdim=48), False), (dict(rank=3), False), (dict(chunk=0), False),
    (dict(chunk=64, rank=4), False), (dict(chunk=16, rank=4), True), (dict(in_dtype=7), False),
    (dict(dstate=272), False), (dict(norm_eps=-1.0), False), (dict(batch=-1), False),
    (dict(flags=7), True), (dict(flags=8), True), (dict(flags=16), False),
])
def test_workspace_query_validates(lib, kw, ok):
    n = lib.m3_scan_workspace_bytes(ctypes.byref(dims(**kw)))
    assert (n >= 256) == ok


def test_workspace_holds_segment_states_for_long_sequences(lib):
    """Few long sequences run in segments: the workspace grows by one state slot (fp32 h [N][P],
    angle [N/2], log-decay, padding) per unit and segment (the segments' end states but the
    last's, and the primed initial state); many short sequences do not. Without a GPU the SM
    count is taken as 148 (two CTAs each: 296 slots)."""
    stride = (128 * 64 + 64 + 4) * 4
    def ws(**kw):
        return lib.m3_scan_workspace_bytes(ctypes.byref(dims(bc_norm=0, **kw)))
    base = ws(batch=1, nheads=64, seqlen=64)              # one chunk: never segmented
    assert ws(batch=4, nheads=64, seqlen=2048) == base     # 256 units fill the SMs already
    # b1 H64 L65536: 296 // 64 = 4 segments of 256 chunks -> 4 slots per unit
    r256 = lambda n: (n + 255) // 256 * 256                # the body is 256-byte aligned
    assert ws(batch=1, nheads=64, seqlen=65536) == base + r256(64 * 4 * stride)
    # b1 H4 L2543: 40 chunks, at least 8 per segment -> 5 segments
    assert ws(batch=1, nheads=4, seqlen=2543) == base + r256(4 * 5 * stride)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails before any launch


def fake_inputs(**kw):
    f = {n: FAKE for n, _ in bd.Inputs._fields_}
    f.update(kw)
    return bd.Inputs(*(f[n] for n, _ in bd.Inputs._fields_))


def test_scan_rejects_bad_arguments_without_launching(lib):
    d = dims()
    ins = fake_inputs()
    ws = ctypes.c_void_p(0x100000)
    call = lambda dd=d, ii=ins, y=FAKE, w=ws, nb=4096, init=None, fin=None: lib.m3_scan_fwd(
        ctypes.byref(dd), ctypes.byref(ii), init, fin, y, w, nb, None)
    assert call(ii=fake_inputs(x=None)) == bd.M3_ERR_INVALID_ARG
    assert b"x" in lib.m3_last_error()
    assert call(ii=fake_inputs(theta=FAKE + 2)) == bd.M3_ERR_INVALID_ARG
    assert call(y=None) == bd.M3_ERR_INVALID_ARG
    assert call(w=None) == bd.M3_ERR_INVALID_ARG
    assert call(nb=16) == bd.M3_ERR_INVALID_ARG
    assert call(w=ctypes.c_void_p(0x100010)) == bd.M3_ERR_INVALID_ARG  # not 256-aligned
    bad = bd.StateC(FAKE, None, FAKE, FAKE)
    assert call(init=ctypes.byref(bad)) == bd.M3_ERR_INVALID_ARG
    assert b"phi" in lib.m3_last_error()
    assert call(dd=dims(headdim=48)) == bd.M3_ERR_UNSUPPORTED
    assert call(dd=dims(nheads=3, ngroups=2)) == bd.M3_ERR_INVALID_ARG
    assert lib.m3_scan_fwd(None, ctypes.byref(ins), None, None, FAKE, ws, 4096, None) == \
        bd.M3_ERR_INVALID_ARG


def test_backward_workspace_and_argument_checks(lib):
    """m3_scan_bwd_workspace_bytes follows its documented size; m3_scan_bwd rejects bad
    arguments before anything is launched."""
    d = dims(batch=2, seqlen=100, nheads=4, dstate=128, rank=1)
    T = 16
    r64 = lambda v: (v + 63) // 64 * 64
    units, nch = 2 * 4, (100 + T - 1) // T
    simt = 4 * (2 * r64(2 * 100 * 4 * 128) + r64(units * nch * 64) + r64(units)
                + r64(units * 100 * 4) + r64(units * 128) + r64(2 * 2 * 100 * 4) + r64(units))
    r256 = lambda v: (v + 255) // 256 * 256
    base = 256 + r256(simt)   # status header, the sequential sweeps' buffers
    # bf16, R = 1, N = 128, P = 64, H % 4 == 0: the chunked tensor-core form's chunk states
    # (16 KB and the chunk's angle per unit and 64-token chunk), final state, bias sums, scales
    n64 = (100 + 63) // 64
    tc = (r256(units * n64 * 16384) + r256(units * n64 * 64 * 4) + r256(units * 128 * 64 * 4)
          + r256(units * 65 * 4) + r256(units * 2 * 128 * 4) + r256(2 * n64 * 64 * 1 * 8))
    assert lib.m3_scan_bwd_workspace_bytes(ctypes.byref(d)) == base + tc
    assert lib.m3_scan_bwd_workspace_bytes(ctypes.byref(dims(batch=2, seqlen=100, nheads=4,
                                                             flags=bd.M3_BWD_FP32))) == base
    assert lib.m3_scan_bwd_workspace_bytes(ctypes.byref(dims(batch=2, seqlen=100, nheads=4,
                                                             in_dtype=bd.M3_F32))) == base
    # MIMO R4: chunks of 16 tokens (64 rows), the bias sums and scales per rank
    d4 = dims(batch=2, seqlen=100, nheads=4, dstate=128, rank=4, chunk=16)
    nch4 = (100 + 3) // 4   # the sweeps stage 16 / R = 4 tokens at a time
    simt4 = 4 * (2 * r64(2 * 100 * 4 * 4 * 128) + r64(units * nch4 * 64) + r64(units)
                 + r64(units * 100 * 4) + r64(units * 4 * 128) + r64(2 * 2 * 100 * 4 * 4)
                 + r64(units * 4))
    n16 = (100 + 15) // 16
    tc4 = (r256(units * n16 * 16384) + r256(units * n16 * 64 * 4) + r256(units * 128 * 64 * 4)
           + r256(units * 65 * 4) + r256(units * 2 * 4 * 128 * 4) + r256(2 * n16 * 16 * 1 * 4 * 8))
    assert lib.m3_scan_bwd_workspace_bytes(ctypes.byref(d4)) == 256 + r256(simt4) + tc4
    d4f = dims(batch=2, seqlen=100, nheads=4, dstate=128, rank=4, chunk=16, flags=bd.M3_BWD_FP32)
    assert lib.m3_scan_bwd_workspace_bytes(ctypes.byref(d4f)) == 256 + r256(simt4)
    assert lib.m3_scan_bwd_workspace_bytes(ctypes.byref(dims(rank=3))) == 0
    assert ctypes.sizeof(bd.Grads) == 10 * 8
    ins = fake_inputs()
    g = bd.Grads(*([FAKE] * 10))
    ws = ctypes.c_void_p(0x100000)
    call = lambda dd=d, ii=ins, dy=FAKE, gg=g, w=ws, nb=1 << 40: lib.m3_scan_bwd(
        ctypes.byref(dd), ctypes.byref(ii), None, dy, None,
        ctypes.byref(gg) if gg is not None else None, None, w, nb, None)
    assert call(gg=None) == bd.M3_ERR_INVALID_ARG
    assert call(dy=None) == bd.M3_ERR_INVALID_ARG
    assert b"dy" in lib.m3_last_error()
    assert call(gg=bd.Grads(FAKE, FAKE, None, *([FAKE] * 7))) == bd.M3_ERR_INVALID_ARG
    assert b"dC" in lib.m3_last_error()
    assert call(gg=bd.Grads(*([FAKE] * 7), FAKE + 4, FAKE, FAKE)) == bd.M3_ERR_INVALID_ARG
    assert call(w=None) == bd.M3_ERR_INVALID_ARG
    assert call(nb=16) == bd.M3_ERR_INVALID_ARG
    assert call(dd=dims(headdim=48)) == bd.M3_ERR_UNSUPPORTED


def test_decode_rejects_bad_arguments_without_launching(lib):
    d = dims(seqlen=1)
    ins = fake_inputs()
    st = bd.StateC(FAKE, FAKE, FAKE, FAKE)
    assert lib.m3_decode_step(ctypes.byref(dims(seqlen=2)), ctypes.byref(ins), ctypes.byref(st),
                              ctypes.byref(st), FAKE, None) == bd.M3_ERR_INVALID_ARG
    assert lib.m3_decode_step(ctypes.byref(d), ctypes.byref(ins), None, ctypes.byref(st), FAKE,
                              None) == bd.M3_ERR_INVALID_ARG
    assert lib.m3_decode_step(ctypes.byref(d), ctypes.byref(fake_inputs(lam=None)),
                              ctypes.byref(st), ctypes.byref(st), FAKE, None) == bd.M3_ERR_INVALID_ARG
    assert lib.m3_decode_step(ctypes.byref(d), ctypes.byref(ins), ctypes.byref(st),
                              ctypes.byref(st), None, None) == bd.M3_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        bd._lib_backup = bd._lib
        try:
            bd._lib = None
            bd.load_library(str(tmp_path / "nope.so"))
        finally:
            bd._lib = bd._lib_backup


@pytest.mark.parametrize("kw,fits", [
    # rows = batch * ceil(seqlen / chunk) * chunk * ngroups * rank; chunks hold 64 or 128 rows,
    # so the largest count that fits is 130944 or 131008 (131040 is not a multiple of 64)
    (dict(batch=1, seqlen=131008, chunk=64), True),     # 2047 chunks: 131008 rows
    (dict(batch=1, seqlen=131009, chunk=64), False),    # 2048 chunks: 131072 rows
    (dict(batch=2, seqlen=65472, chunk=64), True),      # 2 * 1023 chunks: 130944 rows
    (dict(batch=2, seqlen=65473, chunk=64), False),     # 130946 tokens, padded to 131072 rows
    (dict(batch=2, seqlen=65500, chunk=64), False),     # 131000 tokens, padded to 131072 rows
    (dict(batch=1, seqlen=130944, chunk=128), True),    # 1023 chunks of 128
    (dict(batch=1, seqlen=130945, chunk=128), False),   # 1024 chunks: 131072 rows
    (dict(batch=1, seqlen=32736, chunk=32, rank=4), True),    # 1023 chunks of 32 tokens x 4
    (dict(batch=1, seqlen=32737, chunk=32, rank=4), False),
    (dict(batch=2, seqlen=65521, chunk=64, bc_norm=0), True),  # no scales: no limit
])
def test_noalloc_limit_on_both_sides(lib, kw, fits):
    """m3_scan_fwd_noalloc runs when batch * ceil(seqlen / chunk) * chunk * ngroups * rank
    <= 131040 with BC norm on, and returns M3_ERR_UNSUPPORTED above it. x is null, so a call
    within the bound stops at argument validation (or at the missing device) and never
    launches."""
    d = dims(nheads=4, **kw)
    ins = fake_inputs(x=None)
    st = lib.m3_scan_fwd_noalloc(ctypes.byref(d), ctypes.byref(ins), None, None, FAKE, None)
    if fits:
        assert st in (bd.M3_ERR_INVALID_ARG, bd.M3_ERR_CUDA), st
    else:
        assert st == bd.M3_ERR_UNSUPPORTED
        assert b"131040" in lib.m3_last_error()
