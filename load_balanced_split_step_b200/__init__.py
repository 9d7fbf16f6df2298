"""Load-balanced split-KV decode attention for B200 (sm_100a).

The compute path is the C-ABI library ``libhpcdecode.so``, built from ``csrc/``. Its
entry points are declared in ``include/hpc_decode.h``. ``binding`` marshals torch
tensors into those calls and does nothing else. Importing ``binding`` (or any name
below) loads the library and raises if it is missing: there is no CPU fallback.

``workloads`` holds the seeded synthetic inputs and needs no library.
"""
_API = ("plan", "plan_static", "plan_host", "attention", "merge", "prologue", "decode_step", "decode_step_fused",
        "decode_step_noalloc",
        "Plan", "HpcError", "library_path", "status_string", "DEV_STATUS")


def __getattr__(name):
    if name in _API:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
