"""gdn2_chunk_fwd_noalloc: the chunked forward for callers that cannot allocate
device memory (for instance a plugin inside a framework whose allocator owns
all of HBM).  It uses a fixed scratch array compiled into libgdn2.so instead
of a caller-allocated workspace.

The test calls the new entry point through the C ABI twice in a row and checks
each result against the ordinary gdn2_chunk_fwd (with a workspace) on the same
inputs, within the chunked path's tolerance.  It lives in a file of its own
that pytest collects last, and it passes both alone in a fresh process and
after the other tests.
"""
import ctypes

import pytest
import torch

from parity_utils import TOL_CHUNK_BF16, rel_err, to_f64

pytestmark = pytest.mark.gpu


def _noalloc(g):
    fn = g.lib.gdn2_chunk_fwd_noalloc
    vp = ctypes.c_void_p
    fn.restype = ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(g.Dims), vp]
    return fn


@pytest.mark.parametrize("packed", [False, True])
def test_noalloc_matches_workspace_entry_twice(packed):
    assert torch.cuda.is_available(), "GPU test"
    from gated_delta_rule_159_b200 import gdn2, inputs
    dev = torch.device("cuda:0")
    w = inputs.Workload("noalloc", 3, 200, 4, 128, 128, 64, torch.bfloat16, 0.05, False, 0.02)
    lengths = [70, 0, 257, 130] if packed else None
    inp = inputs.make_inputs(w, dev, lengths=lengths)
    names = ("q", "k", "v", "log_a", "b", "w")
    N, T_tot, H = inp["n_seqs"], inp["T_tot"], 4
    cu = torch.tensor(inp["cu_host"], dtype=torch.int32, device=dev) if packed else None
    host_cu = (ctypes.c_int32 * (N + 1))(*inp["cu_host"]) if packed else None
    seq_len = T_tot if packed else T_tot // N

    # the existing entry point, with a caller-allocated workspace
    o_ref, S_ref = gdn2.chunk_fwd(*(inp[n] for n in names), inp["S0"], cu if packed else None,
                                  cu_seqlens_host=inp["cu_host"] if packed else None) if packed else \
        gdn2.chunk_fwd(*(inp[n].view(N, seq_len, *inp[n].shape[1:]) for n in names), inp["S0"])
    o_ref = o_ref.reshape(T_tot, H, 128)

    fn = _noalloc(gdn2)
    dims = gdn2.make_dims(N, seq_len, H, 128, 128, 64, gdn2.BF16, gdn2.BF16, 0)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    for call in range(2):
        o = torch.full((T_tot, H, 128), float("nan"), dtype=torch.bfloat16, device=dev)
        S_T = torch.full((N, H, 128, 128), float("nan"), dtype=torch.float32, device=dev)
        rc = fn(*(ctypes.c_void_p(inp[n].data_ptr()) for n in names), ctypes.c_void_p(inp["S0"].data_ptr()),
                ctypes.c_void_p(cu.data_ptr()) if packed else None, host_cu, ctypes.c_void_p(o.data_ptr()),
                ctypes.c_void_p(S_T.data_ptr()), ctypes.byref(dims), stream)
        assert rc == gdn2.OK, gdn2.lib.gdn2_last_error().decode()
        torch.cuda.synchronize()
        assert torch.isfinite(o).all() and torch.isfinite(S_T).all(), f"call {call}"
        assert rel_err(to_f64(o), to_f64(o_ref)) <= TOL_CHUNK_BF16, f"call {call}"
        assert rel_err(to_f64(S_T), to_f64(S_ref)) <= TOL_CHUNK_BF16, f"call {call}"


def test_noalloc_rejects_more_units_than_its_scratch_holds():
    from gated_delta_rule_159_b200 import gdn2
    fn = _noalloc(gdn2)
    limit = 16384  # GDN2_NOALLOC_MAX_UNITS in include/gdn2.h
    dims = gdn2.make_dims(limit // 16 + 1, 64, 16, 128, 128, 64, gdn2.BF16, gdn2.BF16, 0)
    P = ctypes.c_void_p(1 << 20)  # placeholder; the size check fails before any pointer is used
    rc = fn(P, P, P, P, P, P, None, None, None, P, None, ctypes.byref(dims), None)
    assert rc == gdn2.ERR_UNSUPPORTED
    assert "limit" in gdn2.lib.gdn2_last_error().decode()
