"""Float64 CPU oracle for the Gated DeltaNet-2 token mixer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA product path never calls it and shares no code with it.

* ``gdn2_fwd`` -- the plain sequential recurrence in float64 (C, OpenMP over
  independent (sequence, head) units), following the step order of the pages:
  decay, erase read of the decayed state, erase with b, write with w, read with
  q after the update (see ``gdn2_oracle.c`` for the citations).
* ``gdn2_decode_step`` -- the same recurrence for one token per sequence.
* ``gdn2_bwd`` -- reverse-mode gradients of that recurrence in float64 (C),
  pinned by central finite differences of ``gdn2_fwd``.
* ``prologue`` -- the activations (q, k L2-normalised; sigmoid gates) that
  turn pre-activations into the recurrence inputs, and their gradient.
* ``chunked.gdn2_chunked_fwd`` -- the float64 chunkwise (WY) form, used only to
  prove the chunk algebra equal to the recurrence on tiny inputs.

Parity pins live in ``tests/test_oracle_pins.py``.  The erase/write decoupling
with b != w has no printed example on the pages ("parity unpinned" for that
combination by a worked example); it is pinned by the hand-derived closed forms
in those tests (transposed-operand and write-only/erase-only cases).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

SCALAR_DECAY = 1
SCALAR_GATES = 2
TIED_GATES = 4
GATE_FORM_P3 = 8

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (plain -O2, no fast-math) into ``oracle/liboracle.so``."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, dp = ctypes.c_int64, ctypes.POINTER(ctypes.c_double)
        lib.oracle_gdn2_fwd.restype = ctypes.c_int
        lib.oracle_gdn2_fwd.argtypes = [i64, i64, i64, i64, i64, ctypes.POINTER(ctypes.c_int64),
                                        dp, dp, dp, dp, dp, dp, dp, dp, dp, i64]
        lib.oracle_gdn2_bwd.restype = ctypes.c_int
        lib.oracle_gdn2_bwd.argtypes = [i64, i64, i64, i64, i64, ctypes.POINTER(ctypes.c_int64),
                                        dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                        dp, dp, dp, dp, dp, dp, dp, i64]
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _f64(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def gdn2_fwd(q, k, v, log_a, b, w=None, S0=None, cu_seqlens=None, flags: int = 0,
             n_threads: int = 0):
    """Sequential float64 forward.

    q, k: [T_tot, H, d_k]; v: [T_tot, H, d_v]; log_a, b, w: [T_tot, H, d_k]
    (or [T_tot, H] with the scalar flags; w is [T_tot, H, d_v] in the
    GATE_FORM_P3 form; w may be None with TIED_GATES).  S0: [N, H, d_k, d_v]
    or None (zeros).  cu_seqlens: [N+1] offsets, default one sequence.
    Returns (o [T_tot, H, d_v], S_T [N, H, d_k, d_v]) as float64 arrays.
    """
    q, k, v, log_a, b = (_f64(t) for t in (q, k, v, log_a, b))
    w = _f64(w)
    S0 = _f64(S0)
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, T_tot], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != T_tot:
        raise ValueError("cu_seqlens must start at 0 and end at T_tot")
    if w is None and not (flags & TIED_GATES):
        raise ValueError("w is required unless TIED_GATES")
    if S0 is not None and S0.shape != (N, H, dk, dv):
        raise ValueError(f"S0 shape {S0.shape} != {(N, H, dk, dv)}")
    o = np.zeros((T_tot, H, dv), dtype=np.float64)
    S_T = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().oracle_gdn2_fwd(N, H, dk, dv, int(flags),
                                 cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(b), _ptr(w),
                                 _ptr(S0), _ptr(o), _ptr(S_T), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_gdn2_fwd rejected its arguments")
    return o, S_T


def gdn2_decode_step(q, k, v, log_a, b, w, S, flags: int = 0, n_threads: int = 0):
    """One recurrent step for N sequences: q, k [N, H, d_k], v [N, H, d_v],
    gates [N, H, d_k] (or [N, H]), S [N, H, d_k, d_v].  Returns (o, S_new)."""
    q = _f64(q)
    N = q.shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    return gdn2_fwd(q, k, v, log_a, b, w, S0=S, cu_seqlens=cu, flags=flags, n_threads=n_threads)


def gdn2_bwd(q, k, v, log_a, b, w, dO, S0=None, dS_T=None, cu_seqlens=None, flags: int = 0,
             n_threads: int = 0):
    """Float64 gradients of  sum <dO, o> + <dS_T, S_T>  for ``gdn2_fwd`` with the same
    arguments.  Returns a dict with dq, dk, dv, dlog_a, db, dw (None with TIED_GATES,
    whose w gradient is added into db) and dS0, each shaped like its input."""
    q, k, v, log_a, b = (_f64(t) for t in (q, k, v, log_a, b))
    w, dO, S0, dS_T = _f64(w), _f64(dO), _f64(S0), _f64(dS_T)
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    cu = np.array([0, T_tot], dtype=np.int64) if cu_seqlens is None else \
        np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != T_tot:
        raise ValueError("cu_seqlens must start at 0 and end at T_tot")
    tied = bool(flags & TIED_GATES)
    if w is None and not tied:
        raise ValueError("w is required unless TIED_GATES")
    if dO.shape != (T_tot, H, dv):
        raise ValueError(f"dO shape {dO.shape} != {(T_tot, H, dv)}")
    for name, t in (("S0", S0), ("dS_T", dS_T)):
        if t is not None and t.shape != (N, H, dk, dv):
            raise ValueError(f"{name} shape {t.shape} != {(N, H, dk, dv)}")
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), dlog_a=np.zeros_like(log_a),
               db=np.zeros_like(b), dw=None if tied else np.zeros_like(w),
               dS0=np.zeros((N, H, dk, dv), dtype=np.float64))
    rc = _load().oracle_gdn2_bwd(N, H, dk, dv, int(flags), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(b), _ptr(None if tied else w),
                                 _ptr(S0), _ptr(dO), _ptr(dS_T),
                                 _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dlog_a"]),
                                 _ptr(out["db"]), _ptr(out["dw"]), _ptr(out["dS0"]), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_gdn2_bwd rejected its arguments")
    return out
