"""CPU-side checks of the C ABI: the library loads, exports every entry point
include/gdn2.h declares, and rejects bad arguments before touching a GPU.

Every call below fails validation on the host, so no CUDA call is ever made
with the placeholder pointers used here.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn2.h")


@pytest.fixture(scope="module")
def g():
    from gated_delta_rule_159_b200 import build
    build.build()
    from gated_delta_rule_159_b200 import gdn2
    return gdn2


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(gdn2_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("gdn2_chunk_fwd", "gdn2_chunk_fwd_workspace_size", "gdn2_decode_step", "gdn2_last_error"):
        assert must in names


def test_library_exports_every_declared_symbol(g):
    lib = ctypes.CDLL(g.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in gdn2.h but not exported"
    assert set(declared_functions()) <= set(g.EXPORTED) | set(declared_functions())
    assert g.version() == 100


def _dims(g, **kw):
    base = dict(n_seqs=2, seq_len=128, n_heads=4, d_k=128, d_v=128, chunk=64, dtype_in=g.BF16, dtype_out=g.BF16,
                flags=0)
    base.update(kw)
    return g.make_dims(**base)


P = ctypes.c_void_p(1 << 20)       # 16-byte-aligned placeholders, never dereferenced
WS = ctypes.c_void_p(1 << 21)


def _chunk(g, dims, **ptrs):
    a = dict(q=P, k=P, v=P, log_a=P, b=P, w=P, S0=None, cu=None, cu_host=None, o=P, S_T=None, ws=WS,
             ws_bytes=1 << 20)
    a.update(ptrs)
    rc = g.lib.gdn2_chunk_fwd(a["q"], a["k"], a["v"], a["log_a"], a["b"], a["w"], a["S0"], a["cu"], a["cu_host"],
                              a["o"], a["S_T"], ctypes.byref(dims), a["ws"], a["ws_bytes"], None)
    return rc, g.lib.gdn2_last_error().decode()


def test_workspace_size(g):
    d = _dims(g, n_seqs=8, n_heads=16)
    assert g.workspace_size(d) == 256 + 512
    assert g.workspace_size(_dims(g, n_seqs=0)) == 0


@pytest.mark.parametrize("bad,code", [
    (dict(n_seqs=0), -1), (dict(n_heads=0), -1), (dict(seq_len=-1), -1), (dict(dtype_in=7), -1),
    (dict(flags=1 << 10), -1), (dict(flags=8 | 4, d_k=64, d_v=32), -1), (dict(d_k=96, d_v=96), -2), (dict(chunk=48, d_k=32, d_v=32), -2),
    (dict(dtype_in=1), -2),  # fp32 input with d = 128 has no kernel
])
def test_chunk_rejects_bad_dims(g, bad, code):
    rc, msg = _chunk(g, _dims(g, **bad))
    assert rc == code and msg


def test_chunk_rejects_bad_pointers(g):
    d = _dims(g)
    assert _chunk(g, d, q=None)[0] == g.ERR_INVALID_ARG
    assert _chunk(g, d, w=None)[0] == g.ERR_INVALID_ARG
    assert _chunk(g, d, k=ctypes.c_void_p((1 << 20) + 2))[0] == g.ERR_INVALID_ARG
    assert _chunk(g, d, o=None)[0] == g.ERR_INVALID_ARG
    assert _chunk(g, d, S_T=ctypes.c_void_p((1 << 20) + 8))[0] == g.ERR_INVALID_ARG
    assert _chunk(g, d, ws=None)[0] == g.ERR_WORKSPACE
    assert _chunk(g, d, ws=ctypes.c_void_p((1 << 21) + 64))[0] == g.ERR_WORKSPACE
    assert _chunk(g, d, ws_bytes=16)[0] == g.ERR_WORKSPACE


def test_chunk_rejects_bad_host_cu_seqlens(g):
    d = _dims(g, n_seqs=3, seq_len=100)
    bad = [(0, 60, 50, 100), (1, 20, 50, 100), (0, 20, 50, 99)]
    for cu in bad:
        host = (ctypes.c_int32 * 4)(*cu)
        rc, msg = _chunk(g, d, cu=P, cu_host=host)
        assert rc == g.ERR_INVALID_ARG, (cu, msg)
    host = (ctypes.c_int32 * 4)(0, 20, 50, 100)
    assert _chunk(g, d, cu=None, cu_host=host)[0] == g.ERR_INVALID_ARG


def test_decode_rejects_bad_arguments(g):
    def call(dims, **kw):
        a = dict(q=P, k=P, v=P, log_a=P, b=P, w=P, S=P, o=P)
        a.update(kw)
        return g.lib.gdn2_decode_step(a["q"], a["k"], a["v"], a["log_a"], a["b"], a["w"], a["S"], a["o"],
                                      ctypes.byref(dims), None)
    assert call(_dims(g, seq_len=1, d_v=96)) == g.ERR_UNSUPPORTED
    assert call(_dims(g, seq_len=1, d_k=256)) == g.ERR_UNSUPPORTED
    assert call(_dims(g, seq_len=2)) == g.ERR_INVALID_ARG
    assert call(_dims(g, seq_len=1), S=None) == g.ERR_INVALID_ARG
    assert call(_dims(g, seq_len=1), w=None) == g.ERR_INVALID_ARG
    assert call(_dims(g, seq_len=1, flags=g.TIED_GATES), w=None, o=ctypes.c_void_p(3)) == g.ERR_INVALID_ARG


def test_decode_indexed_rejects_bad_arguments(g):
    def call(dims, n_slots=4, **kw):
        a = dict(q=P, k=P, v=P, log_a=P, b=P, w=P, S=P, idx=P, o=P)
        a.update(kw)
        return g.lib.gdn2_decode_step_indexed(a["q"], a["k"], a["v"], a["log_a"], a["b"], a["w"], a["S"], n_slots,
                                              a["idx"], a["o"], ctypes.byref(dims), None)
    assert call(_dims(g, seq_len=1), idx=None) == g.ERR_INVALID_ARG
    assert call(_dims(g, seq_len=1), idx=ctypes.c_void_p((1 << 20) + 2)) == g.ERR_INVALID_ARG
    assert call(_dims(g, seq_len=1), n_slots=0) == g.ERR_INVALID_ARG
    assert call(_dims(g, seq_len=1), S=None) == g.ERR_INVALID_ARG
    assert call(_dims(g, seq_len=3)) == g.ERR_INVALID_ARG
    assert call(_dims(g, seq_len=1, d_v=96)) == g.ERR_UNSUPPORTED


def test_last_error_is_cleared(g):
    _chunk(g, _dims(g, n_seqs=0))
    assert g.lib.gdn2_last_error().decode()
    assert g.lib.gdn2_chunk_fwd_workspace_size(ctypes.byref(_dims(g))) > 0


def test_bwd_workspace_size(g):
    lib = g.lib
    d = _dims(g, n_seqs=2, seq_len=100, n_heads=3, d_k=128, d_v=128)
    eq = lib.gdn2_bwd_workspace_size(ctypes.byref(d), 0)          # 2 x 100 tokens
    d2 = _dims(g, n_seqs=2, seq_len=200, n_heads=3, d_k=128, d_v=128)
    packed = lib.gdn2_bwd_workspace_size(ctypes.byref(d2), 1)     # 200 tokens packed
    assert eq == packed > 0
    ckpt = (200 // 4 + 2) * 3 * 128 * 128 * 4
    part = 4 * 200 * 3 * 5 * 128 * 4
    dz = 200 * 3 * 128 * 4
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert eq == up(ckpt) + up(part) + up(dz)
    assert lib.gdn2_bwd_workspace_size(ctypes.byref(_dims(g, d_v=96)), 0) == 0


def test_bwd_rejects_bad_arguments(g):
    def call(dims, **kw):
        a = dict(q=P, k=P, v=P, log_a=P, b=P, w=P, S0=None, cu=None, dO=P, dS_T=None, dq=P, dk=P, dv=P, dg=P,
                 db=P, dw=P, dS0=None, ws=WS, ws_bytes=1 << 20)
        a.update(kw)
        return g.lib.gdn2_bwd(a["q"], a["k"], a["v"], a["log_a"], a["b"], a["w"], a["S0"], a["cu"], a["dO"],
                              a["dS_T"], a["dq"], a["dk"], a["dv"], a["dg"], a["db"], a["dw"], a["dS0"],
                              ctypes.byref(dims), a["ws"], a["ws_bytes"], None)
    d = _dims(g, seq_len=16)
    assert call(d, dO=None) == g.ERR_INVALID_ARG
    assert call(d, dw=None) == g.ERR_INVALID_ARG
    assert call(d, dS0=ctypes.c_void_p((1 << 20) + 4)) == g.ERR_INVALID_ARG
    assert call(d, ws=None) == g.ERR_WORKSPACE
    assert call(d, ws_bytes=1024) == g.ERR_WORKSPACE
    assert call(_dims(g, seq_len=16, d_v=48)) == g.ERR_UNSUPPORTED
    assert call(_dims(g, seq_len=16, d_k=256)) == g.ERR_UNSUPPORTED


def test_split_forward_rejects_bad_arguments(g):
    lib = g.lib

    def call(dims, n_split=4, ws_bytes=4096, **kw):  # too small: no call below can reach a launch
        a = dict(q=P, k=P, v=P, log_a=P, b=P, w=P, S0=None, o=P, S_T=None, ws=WS)
        a.update(kw)
        return lib.gdn2_chunk_fwd_split(a["q"], a["k"], a["v"], a["log_a"], a["b"], a["w"], a["S0"], a["o"],
                                        a["S_T"], ctypes.byref(dims), n_split, a["ws"], ws_bytes, None)
    d = _dims(g, n_seqs=1, seq_len=4096, n_heads=2)
    assert lib.gdn2_chunk_fwd_split_workspace_size(ctypes.byref(d), 4) > lib.gdn2_chunk_fwd_split_workspace_size(
        ctypes.byref(d), 1) > 0
    assert lib.gdn2_chunk_fwd_split_workspace_size(ctypes.byref(d), 0) == 0
    assert call(d, n_split=0) == g.ERR_INVALID_ARG
    assert call(_dims(g, n_seqs=1, seq_len=4096, d_k=64, d_v=64)) == g.ERR_UNSUPPORTED
    assert call(_dims(g, n_seqs=1, seq_len=4096, dtype_in=1)) == g.ERR_UNSUPPORTED
    assert call(d, q=None) == g.ERR_INVALID_ARG
    assert call(d, ws=None) == g.ERR_WORKSPACE
    assert call(d, ws_bytes=4096) == g.ERR_WORKSPACE


def test_segment_calls_reject_bad_arguments(g):
    """The per-rank sequence-parallel calls validate everything before their first launch."""
    lib = g.lib
    d = _dims(g, n_seqs=2, seq_len=256, n_heads=2)
    need = lib.gdn2_segment_maps_workspace_size(ctypes.byref(d))
    assert need > lib.gdn2_segment_correct_workspace_size(ctypes.byref(d)) > 0
    assert lib.gdn2_segment_maps_workspace_size(None) == 0

    def maps(dims, ws_bytes=None, **kw):
        a = dict(q=P, k=P, v=P, log_a=P, b=P, w=P, S0=None, o=P, F=P, G=P, ws=WS)
        a.update(kw)
        return lib.gdn2_segment_maps(a["q"], a["k"], a["v"], a["log_a"], a["b"], a["w"], a["S0"], a["o"], a["F"],
                                     a["G"], ctypes.byref(dims), a["ws"], need if ws_bytes is None else ws_bytes, None)
    assert maps(d, q=None) == g.ERR_INVALID_ARG
    assert maps(d, F=None) == g.ERR_INVALID_ARG
    assert maps(d, o=ctypes.c_void_p((1 << 20) + 4)) == g.ERR_INVALID_ARG
    assert maps(d, ws=None) == g.ERR_WORKSPACE
    assert maps(d, ws_bytes=need - 1) == g.ERR_WORKSPACE
    assert maps(_dims(g, n_seqs=2, seq_len=256, d_k=64, d_v=64)) == g.ERR_UNSUPPORTED

    def correct(dims, **kw):
        a = dict(q=P, k=P, log_a=P, b=P, w=P, start=P, o=P, ws=WS)
        a.update(kw)
        return lib.gdn2_segment_correct(a["q"], a["k"], a["log_a"], a["b"], a["w"], a["start"], a["o"],
                                        ctypes.byref(dims), a["ws"], 1 << 30, None)
    assert correct(d, start=None) == g.ERR_INVALID_ARG
    assert correct(d, k=None) == g.ERR_INVALID_ARG
    assert correct(d, o=None) == g.ERR_INVALID_ARG
    # affine prefix: the segment index must name one of the n_segs segments
    assert lib.gdn2_affine_prefix(P, P, P, None, 2, 2, 3, 3, None) == g.ERR_INVALID_ARG
    assert lib.gdn2_affine_prefix(P, P, P, None, 2, 2, 3, -1, None) == g.ERR_INVALID_ARG
    assert lib.gdn2_affine_prefix(None, P, P, None, 2, 2, 3, 0, None) == g.ERR_INVALID_ARG
    assert lib.gdn2_affine_prefix(P, P, None, None, 2, 2, 3, 0, None) == g.OK  # nothing requested: no launch


def test_debug_timeout_hook_rejects_bad_arguments(g):
    """The timeout test hook validates its site and wait limit on the host (invalid calls arm nothing)."""
    assert g.lib.gdn2_debug_timeout_once(0, 1_000_000) == g.ERR_INVALID_ARG
    assert "site" in g.lib.gdn2_last_error().decode()
    assert g.lib.gdn2_debug_timeout_once(4, 1_000_000) == g.ERR_INVALID_ARG
    assert g.lib.gdn2_debug_timeout_once(g.DEBUG_CHUNK, 10) == g.ERR_INVALID_ARG
    assert g.lib.gdn2_debug_timeout_once(g.DEBUG_BWD, 500) == g.ERR_INVALID_ARG
    assert g.lib.gdn2_debug_timeout_once(g.DEBUG_DECODE, 20_000_000_000) == g.ERR_INVALID_ARG
    assert "wait_ns" in g.lib.gdn2_last_error().decode()


def test_split_varlen_rejects_bad_arguments(g):
    import ctypes as C
    dims = _dims(g, n_seqs=3, seq_len=300)
    cu_ok = (C.c_int32 * 4)(0, 100, 100, 300)
    cu_bad = (C.c_int32 * 4)(0, 200, 100, 300)
    assert g.lib.gdn2_chunk_fwd_split_varlen_workspace_size(C.byref(dims), cu_ok) > 0
    assert g.lib.gdn2_chunk_fwd_split_varlen_workspace_size(C.byref(dims), cu_bad) == 0
    assert g.lib.gdn2_chunk_fwd_split_varlen_workspace_size(C.byref(dims), None) == 0
    fn = g.lib.gdn2_chunk_fwd_split_varlen

    def call(cu_dev=P, cu_host=cu_ok, ws=WS, ws_bytes=1 << 30, d=dims):
        return fn(P, P, P, P, P, P, None, cu_dev, cu_host, P, None, C.byref(d), ws, ws_bytes, None)

    assert call(cu_host=None) == g.ERR_INVALID_ARG
    assert "cu_seqlens_host" in g.lib.gdn2_last_error().decode()
    assert call(cu_host=cu_bad) == g.ERR_INVALID_ARG
    assert call(cu_dev=None) == g.ERR_INVALID_ARG
    assert call(ws_bytes=16) == g.ERR_WORKSPACE
    assert call(d=_dims(g, n_seqs=3, seq_len=300, d_k=64)) == g.ERR_UNSUPPORTED


def test_chunk_bwd_workspace_size_covers_its_flags(g):
    """gdn2_chunk_bwd takes either placement, tied gates, scalar decay and scalar gates (each alone
    or both) and the fused prologue; other head sizes and fp32 inputs are gdn2_bwd's (size 0)."""
    def size(flags=0, dk=128, dtype_in=None):
        dims = g.make_dims(2, 300, 4, dk, 128, 64, g.BF16 if dtype_in is None else dtype_in, g.BF16, flags)
        return g.chunk_bwd_workspace_size(dims)
    for flags in (0, g.TIED_GATES, g.GATE_FORM_P3, g.GATE_FORM_P3 | g.TIED_GATES,
                  g.SCALAR_DECAY | g.SCALAR_GATES | g.TIED_GATES, g.SCALAR_DECAY | g.SCALAR_GATES | g.GATE_FORM_P3,
                  g.SCALAR_DECAY, g.SCALAR_GATES, g.SCALAR_GATES | g.TIED_GATES | g.GATE_FORM_P3,
                  g.FUSED_PROLOGUE, g.FUSED_PROLOGUE | g.SCALAR_DECAY | g.SCALAR_GATES | g.TIED_GATES,
                  g.FUSED_PROLOGUE | g.SCALAR_DECAY, g.FUSED_PROLOGUE | g.SCALAR_GATES):
        assert size(flags) > 0, flags
    # the prologue's activated copies: q, k and three per-channel gate tensors (bf16) + inverse norms
    assert size(g.FUSED_PROLOGUE) - size() >= 2 * 300 * 4 * (5 * 128 * 2 + 8)
    # scalar decay keeps one log_a copy per row instead of d_k, scalar gates one b and one w
    rows = 2 * 300 * 4
    assert size(g.FUSED_PROLOGUE) - size(g.FUSED_PROLOGUE | g.SCALAR_DECAY) >= rows * 127 * 2 - 512
    assert size(g.FUSED_PROLOGUE) - size(g.FUSED_PROLOGUE | g.SCALAR_GATES) >= 2 * (rows * 127 * 2 - 512)
    assert size(dk=64) == 0 and size(dtype_in=g.F32) == 0
    # 2 sequences x 5 chunks x 4 heads slots of 40 KB, plus the fp32 final states and the header
    assert size() >= 2 * 5 * 4 * 40960 + 2 * 4 * 128 * 128 * 4
