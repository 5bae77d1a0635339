"""Failure detection on the GPU: the bounded device-side waits give up, report a
timeout and leave the context usable.

gdn2_debug_timeout_once arms a one-shot fault for the next launch of a kernel:
its first CTA announces the bytes of its first load group to the mbarrier but
issues none of the copies, and every wait of that launch has a 1 ms limit.  The
wait for that group therefore runs out (a flag that nothing sets; no copy is in
flight and no address is faulted).  The tests check that the host then reads
GDN2_ERR_TIMEOUT from the kernel's status word, and that an ordinary call right
after, on the same GPU and in the same process, matches the float64 oracle.
"""
import pytest
import torch

from parity_utils import TOL_CHUNK_BF16, TOL_DECODE, all_units, compare_units, rel_err, run_chunk, to_f64

pytestmark = pytest.mark.gpu

WAIT_NS = 1_000_000  # 1 ms


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from gated_delta_rule_159_b200 import gdn2  # noqa: F401  (fails loudly without libgdn2.so)
    return torch.device("cuda:0")


def _small(dev, **kw):
    from gated_delta_rule_159_b200 import inputs
    w = inputs.Workload("failure", kw.pop("n_seqs", 3), kw.pop("seq_len", 200), kw.pop("n_heads", 4), 128, 128, 64,
                        torch.bfloat16, 0.05, False, 0.02)
    return inputs.make_inputs(w, dev, **kw)


def test_chunk_wait_times_out_then_recovers(dev):
    from gated_delta_rule_159_b200 import gdn2
    inp = _small(dev)
    names = ("q", "k", "v", "log_a", "b", "w")
    N, T = inp["n_seqs"], inp["T_tot"] // inp["n_seqs"]
    args = [inp[n].view(N, T, *inp[n].shape[1:]) for n in names]
    dims = gdn2.make_dims(N, T, 4, 128, 128, 64, gdn2.BF16, gdn2.BF16, 0)
    ws = torch.empty(gdn2.workspace_size(dims), dtype=torch.uint8, device=dev)
    gdn2.debug_timeout_once(gdn2.DEBUG_CHUNK, WAIT_NS)
    gdn2.chunk_fwd(*args, inp["S0"], None, workspace=ws)
    assert gdn2.check_status(ws) == gdn2.ERR_TIMEOUT
    # the next call, same workspace: clean status and the oracle's result
    o, S_T = gdn2.chunk_fwd(*args, inp["S0"], None, out_dtype=torch.float32, workspace=ws)
    assert gdn2.check_status(ws) == gdn2.OK
    eo, es = compare_units(inp, o.reshape(inp["T_tot"], 4, 128), S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


def test_chunk_hook_is_one_shot(dev):
    """The hook is consumed by one launch: the launch after it reports no timeout."""
    from gated_delta_rule_159_b200 import gdn2
    inp = _small(dev, n_seqs=2, seq_len=130, n_heads=2)
    gdn2.debug_timeout_once(gdn2.DEBUG_CHUNK, WAIT_NS)
    ws = torch.empty(4096, dtype=torch.uint8, device=dev)
    names = ("q", "k", "v", "log_a", "b", "w")
    args = [inp[n].view(2, 130, *inp[n].shape[1:]) for n in names]
    gdn2.chunk_fwd(*args, inp["S0"], None, workspace=ws)
    assert gdn2.check_status(ws) == gdn2.ERR_TIMEOUT
    gdn2.chunk_fwd(*args, inp["S0"], None, workspace=ws)
    assert gdn2.check_status(ws) == gdn2.OK


def test_bwd_wait_times_out_then_recovers(dev):
    """The chunked backward's reverse kernel: its first load group never lands."""
    from gated_delta_rule_159_b200 import gdn2
    from parity_utils import compare_bwd_units
    inp = _small(dev, n_seqs=2, seq_len=200, n_heads=2)
    names = ("q", "k", "v", "log_a", "b", "w")
    args = [inp[n].view(2, 200, *inp[n].shape[1:]) for n in names]
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    dO = torch.randn(400, 2, 128, generator=g, device=dev)
    gdn2.debug_timeout_once(gdn2.DEBUG_BWD, WAIT_NS)
    res = gdn2.chunk_bwd(*args, dO.view(2, 200, 2, 128), S0=inp["S0"])
    ws = res["workspace"]
    assert gdn2.check_status(ws) == gdn2.ERR_TIMEOUT
    res = gdn2.chunk_bwd(*args, dO.view(2, 200, 2, 128), S0=inp["S0"], workspace=ws)
    assert gdn2.check_status(ws) == gdn2.OK
    grads = {k: (v.reshape(400, *v.shape[2:]) if k not in ("dS0", "workspace") and v is not None else v)
             for k, v in res.items()}
    errs = compare_bwd_units(inp, grads, dO, None, all_units(inp))
    assert max(errs.values()) <= TOL_CHUNK_BF16, errs


def test_decode_wait_times_out_then_recovers(dev):
    from gated_delta_rule_159_b200 import gdn2, inputs
    import oracle
    N, H, d = 200, 4, 128
    di = inputs.make_decode_inputs(N, H, d, 1, dev, seed=5)
    g = torch.Generator(device=dev)
    g.manual_seed(6)
    S0 = torch.randn(N, H, d, d, generator=g, device=dev) * 0.05
    names = ("q", "k", "v", "log_a", "b", "w")
    S = S0.clone()
    gdn2.debug_timeout_once(gdn2.DEBUG_DECODE, WAIT_NS)
    gdn2.decode_step(*(di[n][0] for n in names), S)
    assert gdn2.decode_status() == gdn2.ERR_TIMEOUT
    assert gdn2.decode_status() == gdn2.OK  # reading clears the record
    # the next step from the original states matches the oracle
    S = S0.clone()
    o = torch.empty(N, H, d, dtype=torch.float32, device=dev)
    gdn2.decode_step(*(di[n][0] for n in names), S, o=o)
    assert gdn2.decode_status() == gdn2.OK
    o_r, S_r = oracle.gdn2_decode_step(*(to_f64(di[n][0]) for n in names), to_f64(S0))
    for n in range(0, N, 37):
        for h in range(H):
            assert rel_err(to_f64(o[n, h]), o_r[n, h]) <= TOL_DECODE
            assert rel_err(to_f64(S[n, h]), S_r[n, h]) <= TOL_DECODE
