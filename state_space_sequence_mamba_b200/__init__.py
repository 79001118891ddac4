"""Mamba-3 selective-SSM core for NVIDIA B200 (sm_100a): chunked prefill scan and one-token
decode step, exposed through the C ABI in ``include/m3.h``.

``inputs`` draws seeded synthetic workloads. ``scan_fwd`` / ``decode_step`` (from
``binding``) marshal torch CUDA tensors into the C ABI; every step of the computation runs
in the library's CUDA kernels. Importing the package does not load the library; the first
call does, and raises if the compiled library is missing.
"""
from .inputs import Dims, Problem, make_problem, make_config, make_decode, CONFIGS  # noqa: F401


def __getattr__(name):
    if name in ("scan_fwd", "decode_step", "scan_workspace_bytes", "M3Error", "load_library",
                "State"):
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
