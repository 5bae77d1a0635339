"""ctypes binding of ``libgdn2.so`` (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; PyTorch is
used only to allocate device memory and to name the current stream.  Importing
this module loads the shared library and raises ``ImportError`` if it is
missing: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn2.so")

# enum gdn2_status / gdn2_dtype / gdn2_flags (include/gdn2.h)
OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_TIMEOUT = -4
ERR_WORKSPACE = -5
ERR_RANGE = -6
BF16 = 0
F32 = 1
SCALAR_DECAY = 1
SCALAR_GATES = 2
TIED_GATES = 4
GATE_FORM_P3 = 8
FUSED_PROLOGUE = 16

EXPORTED = ("gdn2_chunk_fwd", "gdn2_chunk_fwd_workspace_size", "gdn2_check_status",
            "gdn2_decode_step", "gdn2_decode_step_indexed", "gdn2_decode_status", "gdn2_bwd",
            "gdn2_bwd_workspace_size", "gdn2_chunk_bwd", "gdn2_chunk_bwd_workspace_size", "gdn2_chunk_fwd_split", "gdn2_chunk_fwd_split_workspace_size",
            "gdn2_segment_maps", "gdn2_segment_maps_workspace_size", "gdn2_affine_prefix",
            "gdn2_segment_correct", "gdn2_segment_correct_workspace_size",
            "gdn2_chunk_fwd_split_varlen", "gdn2_chunk_fwd_split_varlen_workspace_size",
            "gdn2_chunk_fwd_noalloc", "gdn2_chunk_fwd_noalloc_status", "gdn2_debug_timeout_once",
            "gdn2_last_error", "gdn2_version")
DEBUG_CHUNK = 1
DEBUG_DECODE = 2
DEBUG_BWD = 3


class Dims(ctypes.Structure):
    _fields_ = [("n_seqs", ctypes.c_int32), ("seq_len", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("dtype_in", ctypes.c_int32), ("dtype_out", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("reserved", ctypes.c_int32)]


class GDN2Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"gdn2 status {status}: {message}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m gated_delta_rule_159_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.gdn2_chunk_fwd.restype = ctypes.c_int
    lib.gdn2_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(Dims), vp, sz, vp]
    lib.gdn2_chunk_fwd_workspace_size.restype = sz
    lib.gdn2_chunk_fwd_workspace_size.argtypes = [ctypes.POINTER(Dims)]
    lib.gdn2_check_status.restype = ctypes.c_int
    lib.gdn2_check_status.argtypes = [vp, vp]
    lib.gdn2_decode_step.restype = ctypes.c_int
    lib.gdn2_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(Dims), vp]
    lib.gdn2_decode_step_indexed.restype = ctypes.c_int
    lib.gdn2_decode_step_indexed.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_int32, vp, vp,
                                             ctypes.POINTER(Dims), vp]
    lib.gdn2_chunk_fwd_split.restype = ctypes.c_int
    lib.gdn2_chunk_fwd_split.argtypes = [vp] * 9 + [ctypes.POINTER(Dims), ctypes.c_int32, vp, sz, vp]
    lib.gdn2_chunk_fwd_split_workspace_size.restype = sz
    lib.gdn2_chunk_fwd_split_workspace_size.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32]
    lib.gdn2_segment_maps.restype = ctypes.c_int
    lib.gdn2_segment_maps.argtypes = [vp] * 10 + [ctypes.POINTER(Dims), vp, sz, vp]
    lib.gdn2_segment_maps_workspace_size.restype = sz
    lib.gdn2_segment_maps_workspace_size.argtypes = [ctypes.POINTER(Dims)]
    lib.gdn2_affine_prefix.restype = ctypes.c_int
    lib.gdn2_affine_prefix.argtypes = [vp, vp, vp, vp] + [ctypes.c_int32] * 4 + [vp]
    lib.gdn2_segment_correct.restype = ctypes.c_int
    lib.gdn2_segment_correct.argtypes = [vp] * 7 + [ctypes.POINTER(Dims), vp, sz, vp]
    lib.gdn2_segment_correct_workspace_size.restype = sz
    lib.gdn2_segment_correct_workspace_size.argtypes = [ctypes.POINTER(Dims)]
    lib.gdn2_decode_status.restype = ctypes.c_int
    lib.gdn2_decode_status.argtypes = [vp]
    lib.gdn2_chunk_fwd_split_varlen.restype = ctypes.c_int
    lib.gdn2_chunk_fwd_split_varlen.argtypes = [vp] * 11 + [ctypes.POINTER(Dims), vp, sz, vp]
    lib.gdn2_chunk_fwd_split_varlen_workspace_size.restype = sz
    lib.gdn2_chunk_fwd_split_varlen_workspace_size.argtypes = [ctypes.POINTER(Dims), vp]
    lib.gdn2_debug_timeout_once.restype = ctypes.c_int
    lib.gdn2_debug_timeout_once.argtypes = [ctypes.c_int32, ctypes.c_uint64]
    lib.gdn2_bwd.restype = ctypes.c_int
    lib.gdn2_bwd.argtypes = [vp] * 17 + [ctypes.POINTER(Dims), vp, sz, vp]
    lib.gdn2_bwd_workspace_size.restype = sz
    lib.gdn2_bwd_workspace_size.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32]
    lib.gdn2_chunk_bwd.restype = ctypes.c_int
    lib.gdn2_chunk_bwd.argtypes = [vp] * 17 + [ctypes.POINTER(Dims), vp, sz, vp]
    lib.gdn2_chunk_bwd_workspace_size.restype = sz
    lib.gdn2_chunk_bwd_workspace_size.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32]
    lib.gdn2_last_error.restype = ctypes.c_char_p
    lib.gdn2_last_error.argtypes = []
    lib.gdn2_version.restype = ctypes.c_int
    lib.gdn2_version.argtypes = []
    return lib


lib = _load()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return BF16
    if t == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t}")


def _torch_dtype(code: int) -> torch.dtype:
    return torch.bfloat16 if code == BF16 else torch.float32


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("gdn2 tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("gdn2 tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(rc: int):
    if rc != OK:
        raise GDN2Error(rc, lib.gdn2_last_error().decode())


def make_dims(n_seqs, seq_len, n_heads, d_k, d_v, chunk, dtype_in, dtype_out, flags) -> Dims:
    return Dims(int(n_seqs), int(seq_len), int(n_heads), int(d_k), int(d_v), int(chunk), int(dtype_in),
                int(dtype_out), int(flags), 0)


def flags_of(scalar_decay=False, scalar_gates=False, tied_gates=False, gate_form_p3=False,
             fused_prologue=False) -> int:
    return (SCALAR_DECAY if scalar_decay else 0) | (SCALAR_GATES if scalar_gates else 0) | \
           (TIED_GATES if tied_gates else 0) | (GATE_FORM_P3 if gate_form_p3 else 0) | \
           (FUSED_PROLOGUE if fused_prologue else 0)


def workspace_size(dims: Dims) -> int:
    return int(lib.gdn2_chunk_fwd_workspace_size(ctypes.byref(dims)))


def split_workspace_size(dims: Dims, n_split: int) -> int:
    """Workspace bytes of ``gdn2_chunk_fwd_split`` (0 for invalid arguments)."""
    return int(lib.gdn2_chunk_fwd_split_workspace_size(ctypes.byref(dims), int(n_split)))


def bwd_workspace_size(dims: Dims, packed: bool = False) -> int:
    """Workspace bytes of ``gdn2_bwd``; ``packed``: the call passes cu_seqlens (seq_len = T_tot)."""
    return int(lib.gdn2_bwd_workspace_size(ctypes.byref(dims), 1 if packed else 0))


def chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_a: torch.Tensor, b: torch.Tensor,
              w: Optional[torch.Tensor] = None, S0: Optional[torch.Tensor] = None,
              cu_seqlens: Optional[torch.Tensor] = None, *, chunk: int = 64, scalar_decay: bool = False,
              scalar_gates: bool = False, tied_gates: bool = False, gate_form_p3: bool = False,
              fused_prologue: bool = False, out_dtype: Optional[torch.dtype] = None,
              output_final_state: bool = True, cu_seqlens_host: Optional[Sequence[int]] = None,
              o: Optional[torch.Tensor] = None, S_T: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None):
    """Chunked GDN-2 forward through ``gdn2_chunk_fwd``.

    q, k: [B, T, H, d_k] (equal lengths) or [T_tot, H, d_k] with ``cu_seqlens``
    (int32 [N+1] on the device); v: same with d_v.  log_a, b, w: like k, or
    [.., H] with the scalar flags; with ``gate_form_p3`` (the gist.science gate
    placement) w has d_v channels.  S0: fp32 [N, H, d_k, d_v] or None.
    Returns (o [.., H, d_v], S_T fp32 [N, H, d_k, d_v] or None).
    """
    if q.dim() == 4:
        if cu_seqlens is not None:
            raise ValueError("4-D inputs take no cu_seqlens")
        N, T, H, dk = q.shape
        seq_len = T
    elif q.dim() == 3:
        if cu_seqlens is None:
            N, (T, H, dk) = 1, q.shape
            seq_len = T
        else:
            N = cu_seqlens.numel() - 1
            T_tot, H, dk = q.shape
            seq_len = T_tot
            if cu_seqlens.dtype != torch.int32:
                raise TypeError("cu_seqlens must be int32")
    else:
        raise ValueError("q must be [B, T, H, d_k] or [T_tot, H, d_k]")
    dv = v.shape[-1]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    flags = flags_of(scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue)
    dims = make_dims(N, seq_len, H, dk, dv, chunk, _dtype_code(q.dtype), _dtype_code(out_dtype), flags)
    dev = q.device
    if o is None:
        o = torch.empty(*v.shape[:-1], dv, dtype=out_dtype, device=dev)
    if S_T is None and output_final_state:
        S_T = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(workspace_size(dims), dtype=torch.uint8, device=dev)
    host_cu = None
    if cu_seqlens_host is not None:
        host_cu = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
    rc = lib.gdn2_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(b), _ptr(w), _ptr(S0),
                            _ptr(cu_seqlens), host_cu, _ptr(o), _ptr(S_T), ctypes.byref(dims),
                            _ptr(workspace), workspace.numel(), _stream(dev))
    _check(rc)
    return o, S_T


def debug_timeout_once(site: int, wait_ns: int) -> None:
    """Test hook: the next launch of the kernel at ``site`` (DEBUG_CHUNK / DEBUG_DECODE) runs
    its bounded waits with a ``wait_ns`` limit and lets one of them run out (see
    ``gdn2_debug_timeout_once`` in include/gdn2.h).  Not for production use."""
    _check(lib.gdn2_debug_timeout_once(int(site), int(wait_ns)))


def decode_status(device=None) -> int:
    """Synchronise and read (and clear) the decode kernels' status: OK or ERR_TIMEOUT."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    return int(lib.gdn2_decode_status(_stream(dev)))


def chunk_fwd_split(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_a: torch.Tensor, b: torch.Tensor,
                    w: Optional[torch.Tensor] = None, S0: Optional[torch.Tensor] = None, *,
                    n_split: Optional[int] = None,
                    scalar_decay: bool = False, scalar_gates: bool = False, tied_gates: bool = False,
                    gate_form_p3: bool = False, fused_prologue: bool = False,
                    out_dtype: Optional[torch.dtype] = None, workspace: Optional[torch.Tensor] = None):
    """Sequence-parallel chunked forward through ``gdn2_chunk_fwd_split``: inputs
    [B, T, H, d] (equal lengths), every sequence cut into up to ``n_split`` segments
    (default: as many as keep the B x H x n_split segment units within the SM count).
    Returns (o [B, T, H, d_v], S_T fp32 [B, H, d_k, d_v])."""
    N, T, H, dk = q.shape
    if n_split is None:
        n_split = max(1, torch.cuda.get_device_properties(q.device).multi_processor_count // (N * H))
    dv = v.shape[-1]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    flags = flags_of(scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue)
    dims = make_dims(N, T, H, dk, dv, 64, _dtype_code(q.dtype), _dtype_code(out_dtype), flags)
    dev = q.device
    o = torch.empty(N, T, H, dv, dtype=out_dtype, device=dev)
    S_T = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(split_workspace_size(dims, n_split), 256), dtype=torch.uint8, device=dev)
    rc = lib.gdn2_chunk_fwd_split(_ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
                                  _ptr(S_T), ctypes.byref(dims), int(n_split), _ptr(workspace), workspace.numel(),
                                  _stream(dev))
    _check(rc)
    return o, S_T


def split_varlen_workspace_size(dims: Dims, cu_seqlens_host: Sequence[int]) -> int:
    """Workspace bytes of ``gdn2_chunk_fwd_split_varlen`` for these lengths (0 if invalid)."""
    host_cu = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
    return int(lib.gdn2_chunk_fwd_split_varlen_workspace_size(ctypes.byref(dims), host_cu))


def chunk_fwd_split_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_a: torch.Tensor,
                           b: torch.Tensor, w: Optional[torch.Tensor], S0: Optional[torch.Tensor],
                           cu_seqlens: torch.Tensor, cu_seqlens_host: Sequence[int], *,
                           scalar_decay: bool = False, scalar_gates: bool = False, tied_gates: bool = False,
                           gate_form_p3: bool = False, fused_prologue: bool = False,
                           out_dtype: Optional[torch.dtype] = None, o: Optional[torch.Tensor] = None,
                           S_T: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """Packed varlen forward through ``gdn2_chunk_fwd_split_varlen``: sequences far longer
    than the balanced per-SM share are cut into segments that run side by side.
    q, k: [T_tot, H, d_k]; v: [T_tot, H, d_v]; cu_seqlens int32 [N + 1] on the device and its
    host copy.  Returns (o [T_tot, H, d_v], S_T fp32 [N, H, d_k, d_v])."""
    T_tot, H, dk = q.shape
    N = cu_seqlens.numel() - 1
    dv = v.shape[-1]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    flags = flags_of(scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue)
    dims = make_dims(N, T_tot, H, dk, dv, 64, _dtype_code(q.dtype), _dtype_code(out_dtype), flags)
    dev = q.device
    if o is None:
        o = torch.empty(T_tot, H, dv, dtype=out_dtype, device=dev)
    if S_T is None:
        S_T = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(split_varlen_workspace_size(dims, cu_seqlens_host), 256), dtype=torch.uint8,
                                device=dev)
    host_cu = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
    _check(lib.gdn2_chunk_fwd_split_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(b), _ptr(w), _ptr(S0),
                                           _ptr(cu_seqlens), host_cu, _ptr(o), _ptr(S_T), ctypes.byref(dims),
                                           _ptr(workspace), workspace.numel(), _stream(dev)))
    return o, S_T


def _segment_dims(q, v, flags, out_dtype):
    N, L, H, dk = q.shape
    return make_dims(N, L, H, dk, v.shape[-1], 64, _dtype_code(q.dtype), _dtype_code(out_dtype), flags)


def segment_maps(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_a: torch.Tensor, b: torch.Tensor,
                 w: Optional[torch.Tensor] = None, S0: Optional[torch.Tensor] = None, *,
                 scalar_decay: bool = False, scalar_gates: bool = False, tied_gates: bool = False,
                 gate_form_p3: bool = False, fused_prologue: bool = False,
                 out_dtype: Optional[torch.dtype] = None, workspace: Optional[torch.Tensor] = None):
    """One rank's segment [N, L, H, d] of N sequences through ``gdn2_segment_maps``.
    Returns (o from the start S0 or 0, F, G): the segment maps a start state S to F S + G
    (F, G fp32 [N, H, d_k, d_v])."""
    N, L, H, dk = q.shape
    dv = v.shape[-1]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    dims = _segment_dims(q, v, flags_of(scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue),
                         out_dtype)
    dev = q.device
    o = torch.empty(N, L, H, dv, dtype=out_dtype, device=dev)
    F = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    G = torch.empty_like(F)
    if workspace is None:
        workspace = torch.empty(max(int(lib.gdn2_segment_maps_workspace_size(ctypes.byref(dims))), 256),
                                dtype=torch.uint8, device=dev)
    _check(lib.gdn2_segment_maps(_ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(b), _ptr(w), _ptr(S0), _ptr(o), _ptr(F),
                                 _ptr(G), ctypes.byref(dims), _ptr(workspace), workspace.numel(), _stream(dev)))
    return o, F, G


def affine_prefix(F_all: torch.Tensor, G_all: torch.Tensor, seg: int, *, want_S_T: bool = True):
    """``gdn2_affine_prefix``: F_all, G_all [R, N, H, d_k, d_v] (segment r = rank r).
    Returns (the start state of segment ``seg`` [N, H, d_k, d_v], the end state after all R
    segments or None)."""
    R, N, H, dk, dv = F_all.shape
    start = torch.empty(N, H, dk, dv, dtype=torch.float32, device=F_all.device)
    S_T = torch.empty_like(start) if want_S_T else None
    _check(lib.gdn2_affine_prefix(_ptr(F_all), _ptr(G_all), _ptr(start), _ptr(S_T), N, H, R, int(seg),
                                  _stream(F_all.device)))
    return start, S_T


def segment_correct(q: torch.Tensor, k: torch.Tensor, log_a: torch.Tensor, b: torch.Tensor,
                    w: Optional[torch.Tensor], start: torch.Tensor, o: torch.Tensor, *,
                    scalar_decay: bool = False, scalar_gates: bool = False, tied_gates: bool = False,
                    gate_form_p3: bool = False, fused_prologue: bool = False,
                    workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """``gdn2_segment_correct``: o += the segment's outputs from ``start`` with v = 0 (in place)."""
    dims = _segment_dims(q, o, flags_of(scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue),
                         o.dtype)
    if workspace is None:
        workspace = torch.empty(max(int(lib.gdn2_segment_correct_workspace_size(ctypes.byref(dims))), 256),
                                dtype=torch.uint8, device=q.device)
    _check(lib.gdn2_segment_correct(_ptr(q), _ptr(k), _ptr(log_a), _ptr(b), _ptr(w), _ptr(start), _ptr(o),
                                    ctypes.byref(dims), _ptr(workspace), workspace.numel(), _stream(q.device)))
    return o


class SegmentOps:
    """The three per-rank calls of the sequence-parallel forward (the library's kernels)."""
    segment_maps = staticmethod(segment_maps)
    affine_prefix = staticmethod(affine_prefix)
    segment_correct = staticmethod(segment_correct)


def chunk_fwd_seq_ranks(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_a: torch.Tensor, b: torch.Tensor,
                        w: Optional[torch.Tensor] = None, S0: Optional[torch.Tensor] = None, *, group=None,
                        ops=SegmentOps, out_dtype: Optional[torch.dtype] = None, **flags):
    """Sequence-parallel chunked forward across the ranks of ``group`` (one process per
    GPU): rank r holds tokens [r L, (r + 1) L) of each of the N sequences as [N, L, H, d]
    tensors (S0 is read on rank 0 only).  Each rank computes its segment's outputs and
    affine map (F, G), the maps are all-gathered (the one collective: 2 x 64 KiB per
    (sequence, head) per rank), each rank folds the maps of the ranks before it into its
    true start state and adds that start state's contribution to its outputs.
    Returns (o [N, L, H, d_v] of this rank's tokens, S_T [N, H, d_k, d_v] of the whole
    sequences, on every rank)."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    maps_kw = dict(flags) if out_dtype is None else dict(flags, out_dtype=out_dtype)
    o, F, G = ops.segment_maps(q, k, v, log_a, b, w, S0 if rank == 0 else None, **maps_kw)
    F_all = torch.empty((world,) + tuple(F.shape), dtype=F.dtype, device=F.device)
    G_all = torch.empty_like(F_all)
    dist.all_gather(list(F_all.unbind(0)), F.contiguous(), group=group)
    dist.all_gather(list(G_all.unbind(0)), G.contiguous(), group=group)
    start, S_T = ops.affine_prefix(F_all, G_all, rank)
    if rank > 0:
        ops.segment_correct(q, k, log_a, b, w, start, o, **flags)
    return o, S_T


def check_status(workspace: torch.Tensor) -> int:
    """Synchronise and read the device status left in ``workspace`` by chunk_fwd."""
    return int(lib.gdn2_check_status(_ptr(workspace), _stream(workspace.device)))


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_a: torch.Tensor, b: torch.Tensor,
                w: Optional[torch.Tensor], S: torch.Tensor, *, scalar_decay: bool = False,
                scalar_gates: bool = False, tied_gates: bool = False, gate_form_p3: bool = False,
              fused_prologue: bool = False,
                out_dtype: torch.dtype = torch.float32, o: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One recurrent step through ``gdn2_decode_step``; ``S`` [N, H, d_k, d_v] fp32 is updated in place.

    q, k, log_a, b, w: [N, H, d_k] (or [N, H] with the scalar flags; w is [N, H, d_v]
    with ``gate_form_p3``); v: [N, H, d_v].
    Returns o [N, H, d_v].
    """
    N, H, dk = q.shape
    dv = v.shape[-1]
    flags = flags_of(scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue)
    dims = make_dims(N, 1, H, dk, dv, 0, _dtype_code(q.dtype), _dtype_code(out_dtype), flags)
    if o is None:
        o = torch.empty(N, H, dv, dtype=out_dtype, device=q.device)
    rc = lib.gdn2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(b), _ptr(w), _ptr(S), _ptr(o),
                              ctypes.byref(dims), _stream(q.device))
    _check(rc)
    return o


def decode_step_indexed(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_a: torch.Tensor, b: torch.Tensor,
                        w: Optional[torch.Tensor], S_pool: torch.Tensor, state_idx: torch.Tensor, *,
                        scalar_decay: bool = False, scalar_gates: bool = False, tied_gates: bool = False,
                        gate_form_p3: bool = False, fused_prologue: bool = False,
                        out_dtype: torch.dtype = torch.float32,
                        o: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One recurrent step through ``gdn2_decode_step_indexed``: row n uses slot
    ``state_idx[n]`` (int32 on the device) of ``S_pool`` [P, H, d_k, d_v] fp32, updated in
    place; an index outside [0, P) is a padding row (o row zero, no state touched)."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    if state_idx.dtype != torch.int32 or state_idx.numel() != N:
        raise TypeError("state_idx must be int32 with one entry per row")
    flags = flags_of(scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue)
    dims = make_dims(N, 1, H, dk, dv, 0, _dtype_code(q.dtype), _dtype_code(out_dtype), flags)
    if o is None:
        o = torch.empty(N, H, dv, dtype=out_dtype, device=q.device)
    rc = lib.gdn2_decode_step_indexed(_ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(b), _ptr(w), _ptr(S_pool),
                                      int(S_pool.shape[0]), _ptr(state_idx), _ptr(o), ctypes.byref(dims),
                                      _stream(q.device))
    _check(rc)
    return o


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_a: torch.Tensor, b: torch.Tensor,
        w: Optional[torch.Tensor], dO: torch.Tensor, S0: Optional[torch.Tensor] = None,
        dS_T: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None, *,
        scalar_decay: bool = False, scalar_gates: bool = False, tied_gates: bool = False,
        gate_form_p3: bool = False, fused_prologue: bool = False, need_dS0: bool = True,
        workspace: Optional[torch.Tensor] = None) -> dict:
    """Gradients through ``gdn2_bwd`` of  sum <dO, o> + <dS_T, S_T>  for the forward with the
    same inputs (layouts as ``chunk_fwd``).  Gradients take dO's dtype.  Returns a dict with
    dq, dk, dv, dlog_a, db, dw (None with ``tied_gates``: its gradient is added into db) and
    dS0 (fp32, None unless ``need_dS0``)."""
    return _bwd_call(lib.gdn2_bwd, lib.gdn2_bwd_workspace_size, q, k, v, log_a, b, w, dO, S0, dS_T, cu_seqlens,
                     scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue, need_dS0, workspace)


def chunk_bwd_workspace_size(dims: Dims, packed: bool = False) -> int:
    """Workspace bytes of ``gdn2_chunk_bwd`` (0: dims unsupported)."""
    return int(lib.gdn2_chunk_bwd_workspace_size(ctypes.byref(dims), 1 if packed else 0))


def chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_a: torch.Tensor, b: torch.Tensor,
              w: Optional[torch.Tensor], dO: torch.Tensor, S0: Optional[torch.Tensor] = None,
              dS_T: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None, *,
              scalar_decay: bool = False, scalar_gates: bool = False, tied_gates: bool = False,
              gate_form_p3: bool = False, fused_prologue: bool = False, need_dS0: bool = True,
              workspace: Optional[torch.Tensor] = None) -> dict:
    """The gradients of ``bwd`` through ``gdn2_chunk_bwd``: the chunked tensor-core backward
    (d_k = d_v = 128, bf16 inputs; any mix of the scalar flags; either gate placement; with
    or without the fused prologue).  Same arguments and result as ``bwd``;
    ``gdn2_check_status(workspace)`` reports a chunk whose decay range is beyond the
    factored form (ERR_RANGE)."""
    return _bwd_call(lib.gdn2_chunk_bwd, lib.gdn2_chunk_bwd_workspace_size, q, k, v, log_a, b, w, dO, S0, dS_T,
                     cu_seqlens, scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue, need_dS0,
                     workspace)


def _bwd_call(fn, ws_fn, q, k, v, log_a, b, w, dO, S0, dS_T, cu_seqlens, scalar_decay, scalar_gates, tied_gates,
              gate_form_p3, fused_prologue, need_dS0, workspace) -> dict:
    if q.dim() == 4:
        N, T, H, dk = q.shape
        seq_len = T
    elif cu_seqlens is None:
        N, (T, H, dk) = 1, q.shape
        seq_len = T
    else:
        N = cu_seqlens.numel() - 1
        seq_len, H, dk = q.shape
    dv = v.shape[-1]
    flags = flags_of(scalar_decay, scalar_gates, tied_gates, gate_form_p3, fused_prologue)
    dims = make_dims(N, seq_len, H, dk, dv, 0, _dtype_code(q.dtype), _dtype_code(dO.dtype), flags)
    dev = q.device
    g = dict(dq=torch.empty_like(q, dtype=dO.dtype), dk=torch.empty_like(k, dtype=dO.dtype),
             dv=torch.empty_like(v, dtype=dO.dtype), dlog_a=torch.empty_like(log_a, dtype=dO.dtype),
             db=torch.empty_like(b, dtype=dO.dtype),
             dw=None if tied_gates else torch.empty_like(w, dtype=dO.dtype),
             dS0=torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev) if need_dS0 else None)
    if workspace is None:
        nbytes = int(ws_fn(ctypes.byref(dims), 1 if cu_seqlens is not None else 0))
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(b), _ptr(w), _ptr(S0), _ptr(cu_seqlens),
            _ptr(dO), _ptr(dS_T), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_a"]),
            _ptr(g["db"]), _ptr(g["dw"]), _ptr(g["dS0"]), ctypes.byref(dims), _ptr(workspace),
            workspace.numel(), _stream(dev))
    _check(rc)
    g["workspace"] = workspace
    return g


def version() -> int:
    return int(lib.gdn2_version())
