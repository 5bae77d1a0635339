"""Gated DeltaNet-2 token-mixer forward on NVIDIA B200 (sm_100a).

``chunk_fwd`` (chunked prefill) and ``decode_step`` (recurrent decode) call the
C ABI of ``libgdn2.so`` (declared in ``include/gdn2.h``).  The binding module is
loaded on first use so that ``inputs`` (the seeded workload generator) can be
imported on machines without the built library.
"""
from __future__ import annotations

import importlib

__all__ = ["chunk_fwd", "decode_step", "check_status", "GDN2Error", "gdn2", "inputs", "build"]


def __getattr__(name):
    if name in ("chunk_fwd", "decode_step", "check_status", "GDN2Error"):
        mod = importlib.import_module(".gdn2", __name__)
        return getattr(mod, name)
    if name in ("gdn2", "inputs", "build"):
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
