"""B200-native selective scan (S6) forward pass and recurrent state update.

The compute lives in ``libmamba_scan.so`` (CUDA kernels for sm_100a behind a
C ABI declared in ``include/mamba_scan.h``).  :mod:`.binding` marshals torch
tensors into that ABI; nothing here computes on the host.  The library is
loaded on first use, and a missing or unloadable library raises an error:
there is no fallback path.
"""
from __future__ import annotations

__all__ = ["mamba_scan_fwd", "mamba_state_update", "mamba_scan_plan", "load_library"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
