"""GPU parity of gdn2_chunk_bwd (the chunked tensor-core backward) against the float64
oracle backward.

The products take bf16 operands, as the bf16-input chunked forward's do, so the bound is
that path's tolerance TOL_CHUNK_BF16 (max error over max |reference| per unit and
gradient).  Small cases compare every element of every (sequence, head) across ragged
lengths (empty, one token, chunk-aligned and ragged tails over several chunks); the
full-size case runs the bench workload and compares sampled units.  A chunk whose decay
range is beyond the factored form must be reported through gdn2_check_status.
"""
import pytest
import torch

from parity_utils import TOL_CHUNK_BF16, all_units, compare_bwd_units

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from gated_delta_rule_159_b200 import gdn2  # noqa: F401  (fails loudly without libgdn2.so)
    return torch.device("cuda:0")


def _case(dev, lengths, tied=None, n_heads=2, seed=0, do_dtype=torch.float32, with_S0=True, with_dST=True,
          batch=None, scalar=False, p3=False, prolog=False, mix=None):
    """Inputs of the bwd tests.  scalar: one alpha and one beta per token and head (and, unless
    tied is False, b = w); p3: the gist.science placement (w gates the d_v value channels);
    mix "decay" / "gates": only log_a, or only b and w, one value per token and head (the
    first channel of the per-channel draw)."""
    from gated_delta_rule_159_b200 import inputs
    if batch is None:
        w = inputs.Workload("cbwd", len(lengths), 0, n_heads, 128, 128, 64, torch.bfloat16, 0.05, scalar, 0.05)
        inp = inputs.make_inputs(w, dev, seed=seed, lengths=lengths, gate_form_p3=p3, fused_prologue=prolog)
    else:
        n, T = batch
        w = inputs.Workload("cbwd", n, T, n_heads, 128, 128, 64, torch.bfloat16, 0.05, scalar, 0.05)
        inp = inputs.make_inputs(w, dev, seed=seed, gate_form_p3=p3)
    if mix == "decay":
        inp["log_a"] = inp["log_a"][..., 0].contiguous()
        inp["scalar_decay"] = True
    elif mix == "gates":
        inp["b"] = inp["b"][..., 0].contiguous()
        inp["w"] = inp["w"][..., 0].contiguous()
        inp["scalar_gates"] = True
    if tied is not None:
        inp["tied_gates"] = tied
        if tied:
            inp["w"] = None
        elif inp["w"] is None:  # scalar but untied: an independent w per token and head
            g = torch.Generator(device=dev)
            g.manual_seed(seed + 77)
            inp["w"] = torch.sigmoid(torch.randn(inp["b"].shape, generator=g, device=dev)).to(inp["b"].dtype)
    if not with_S0:
        inp["S0"] = None
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 1)
    T_tot = inp["T_tot"]
    dO = torch.randn(T_tot, n_heads, 128, generator=g, device=dev).to(do_dtype)
    dS_T = (torch.randn(inp["n_seqs"], n_heads, 128, 128, generator=g, device=dev) * 0.1) if with_dST else None
    return inp, dO, dS_T


def _run(inp, dO, dS_T, batch=None):
    """gdn2.chunk_bwd on a workload dict; ``batch`` = (B, T) passes [B, T, H, d] tensors (no
    cu_seqlens).  Returns the gradients with token-major [T_tot, H, ...] shapes."""
    from gated_delta_rule_159_b200 import gdn2
    flags = dict(tied_gates=inp["tied_gates"], scalar_decay=inp["scalar_decay"], scalar_gates=inp["scalar_gates"],
                 gate_form_p3=inp.get("gate_form_p3", False), fused_prologue=inp.get("fused_prologue", False))
    if batch is None:
        return gdn2.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_a"], inp["b"], inp["w"], dO, S0=inp["S0"],
                              dS_T=dS_T, cu_seqlens=inp["cu_seqlens"], **flags)
    B, T = batch
    r4 = lambda t: None if t is None else t.reshape(B, T, *t.shape[1:])  # noqa: E731
    g = gdn2.chunk_bwd(r4(inp["q"]), r4(inp["k"]), r4(inp["v"]), r4(inp["log_a"]), r4(inp["b"]), r4(inp["w"]),
                       r4(dO), S0=inp["S0"], dS_T=dS_T, **flags)
    for name in ("dq", "dk", "dv", "dlog_a", "db", "dw"):
        if g[name] is not None:
            g[name] = g[name].reshape(B * T, *g[name].shape[2:])
    return g


def _status(grads):
    from gated_delta_rule_159_b200 import gdn2
    return gdn2.lib.gdn2_check_status(gdn2._ptr(grads["workspace"]), gdn2._stream(grads["workspace"].device))


LENS = [1, 7, 64, 0, 65, 130, 200]


@pytest.mark.parametrize("variant", ["default", "tied", "bf16_grads", "no_state", "scalar_tied", "scalar_untied",
                                     "p3", "p3_tied", "p3_scalar", "p3_scalar_tied", "prolog", "prolog_scalar_tied",
                                     "prolog_p3", "scalar_decay_only", "scalar_gates_only", "scalar_gates_only_tied",
                                     "p3_scalar_gates_only", "prolog_scalar_decay_only", "prolog_scalar_gates_only"])
def test_chunk_bwd_varlen(dev, variant):
    kw = dict(default={}, tied=dict(tied=True), bf16_grads=dict(do_dtype=torch.bfloat16),
              no_state=dict(with_S0=False, with_dST=False), scalar_tied=dict(scalar=True),
              scalar_untied=dict(scalar=True, tied=False), p3=dict(p3=True), p3_tied=dict(p3=True, tied=True),
              p3_scalar=dict(p3=True, scalar=True, tied=False), p3_scalar_tied=dict(p3=True, scalar=True),
              prolog=dict(prolog=True), prolog_scalar_tied=dict(prolog=True, scalar=True),
              prolog_p3=dict(prolog=True, p3=True), scalar_decay_only=dict(mix="decay"),
              scalar_gates_only=dict(mix="gates"), scalar_gates_only_tied=dict(mix="gates", tied=True),
              p3_scalar_gates_only=dict(mix="gates", p3=True), prolog_scalar_decay_only=dict(mix="decay", prolog=True),
              prolog_scalar_gates_only=dict(mix="gates", prolog=True))[variant]
    inp, dO, dS_T = _case(dev, LENS, **kw)
    grads = _run(inp, dO, dS_T)
    assert _status(grads) == 0
    errs = compare_bwd_units(inp, grads, dO, dS_T, all_units(inp))
    assert max(errs.values()) <= TOL_CHUNK_BF16, errs


def test_chunk_bwd_equal_lengths(dev):
    """[B, T, H, d] inputs (no cu_seqlens), 3 sequences of 300 tokens (a ragged last chunk)."""
    inp, dO, dS_T = _case(dev, None, batch=(3, 300), n_heads=3, seed=4)
    grads = _run(inp, dO, dS_T, batch=(3, 300))
    assert _status(grads) == 0
    errs = compare_bwd_units(inp, grads, dO, dS_T, all_units(inp))
    assert max(errs.values()) <= TOL_CHUNK_BF16, errs


def test_chunk_bwd_matches_token_serial(dev):
    """The chunked backward against the fp32 token-serial gdn2_bwd on the same inputs."""
    from gated_delta_rule_159_b200 import gdn2
    inp, dO, dS_T = _case(dev, [300, 129], seed=9)
    cb = _run(inp, dO, dS_T)
    cu = inp["cu_seqlens"]
    ts = gdn2.bwd(inp["q"], inp["k"], inp["v"], inp["log_a"], inp["b"], inp["w"], dO, S0=inp["S0"], dS_T=dS_T,
                  cu_seqlens=cu)
    for name in ("dq", "dk", "dv", "dlog_a", "db", "dw", "dS0"):
        a, b = cb[name].double(), ts[name].double()
        err = float((a - b).abs().max() / b.abs().max())
        assert err <= TOL_CHUNK_BF16, (name, err)


def test_chunk_bwd_range_reported(dev):
    """A chunk with a decay range beyond the factored form is reported, not computed."""
    from gated_delta_rule_159_b200 import gdn2
    inp, dO, dS_T = _case(dev, [130], seed=2)
    la = inp["log_a"].clone()
    la[70:80, :, 5] = -30.0  # 300 nats inside chunk 1 on channel 5
    inp["log_a"] = la
    grads = _run(inp, dO, dS_T)
    assert _status(grads) == gdn2.ERR_RANGE


def test_chunk_bwd_full_size_sampled(dev):
    """The bench workload (8 x 4096 tokens, 16 heads, bf16 gradients): sampled units."""
    inp, dO, dS_T = _case(dev, None, batch=(8, 4096), n_heads=16, seed=5, do_dtype=torch.bfloat16)
    grads = _run(inp, dO, dS_T, batch=(8, 4096))
    assert _status(grads) == 0
    errs = compare_bwd_units(inp, grads, dO, dS_T, [(0, 0), (7, 15)])
    assert max(errs.values()) <= TOL_CHUNK_BF16, errs


def test_chunk_bwd_full_size_scalar_sampled(dev):
    """The tied scalar-gate shape of the bench (4 x 4096 tokens, 16 heads, bf16 gradients):
    sampled units; every chunk after a unit's first takes its scalar gates from the values
    requested a chunk ahead."""
    inp, dO, dS_T = _case(dev, None, batch=(4, 4096), n_heads=16, seed=6, do_dtype=torch.bfloat16, scalar=True)
    grads = _run(inp, dO, dS_T, batch=(4, 4096))
    assert _status(grads) == 0
    errs = compare_bwd_units(inp, grads, dO, dS_T, [(0, 0), (3, 15)])
    assert max(errs.values()) <= TOL_CHUNK_BF16, errs
