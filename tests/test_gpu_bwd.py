"""GPU parity of gdn2_bwd (gradients) against the float64 oracle backward.

Small cases compare every gradient element of every (sequence, head), across
ragged lengths that straddle the 8-token checkpoint blocks; the full-size case
runs the bench workload and compares sampled units.  Tolerance TOL_BWD
(parity_utils).
"""
import pytest
import torch

from parity_utils import TOL_BWD, all_units, compare_bwd_units

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from gated_delta_rule_159_b200 import gdn2  # noqa: F401  (fails loudly without libgdn2.so)
    return torch.device("cuda:0")


def _case(dev, dk, dv, dtype, lengths, scalar=False, p3=False, tied=None, n_heads=2, seed=0, prolog=False):
    from gated_delta_rule_159_b200 import inputs
    w = inputs.Workload("bwd", len(lengths), 0, n_heads, dk, dv, 64, dtype, 0.05, scalar, 0.05)
    inp = inputs.make_inputs(w, dev, seed=seed, lengths=lengths, gate_form_p3=p3, fused_prologue=prolog)
    if tied is not None:
        inp["tied_gates"] = tied
        if tied:
            inp["w"] = None
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 1)
    dO = torch.randn(inp["T_tot"], n_heads, dv, generator=g, device=dev)
    dS_T = torch.randn(inp["n_seqs"], n_heads, dk, dv, generator=g, device=dev) * 0.1
    return inp, dO, dS_T


def _run(inp, dO, dS_T):
    from gated_delta_rule_159_b200 import gdn2
    cu = inp["cu_seqlens"]
    if cu is None:
        cu = torch.tensor(inp["cu_host"], dtype=torch.int32, device=inp["q"].device)
    return gdn2.bwd(inp["q"], inp["k"], inp["v"], inp["log_a"], inp["b"], inp["w"], dO, S0=inp["S0"], dS_T=dS_T,
                    cu_seqlens=cu, scalar_decay=inp["scalar_decay"], scalar_gates=inp["scalar_gates"],
                    tied_gates=inp["tied_gates"], gate_form_p3=inp.get("gate_form_p3", False),
                    fused_prologue=inp.get("fused_prologue", False))


LENS = [1, 7, 8, 9, 0, 70]


@pytest.mark.parametrize("variant", ["default", "scalar_tied", "p3", "p3_tied", "p3_scalar"])
def test_bwd_d128(dev, variant):
    kw = dict(default={}, scalar_tied=dict(scalar=True), p3=dict(p3=True), p3_tied=dict(p3=True, tied=True),
              p3_scalar=dict(p3=True, scalar=True, tied=False))[variant]
    inp, dO, dS_T = _case(dev, 128, 128, torch.bfloat16, LENS, **kw)
    if variant == "p3_scalar":
        g = torch.Generator(device=dev)
        g.manual_seed(77)
        inp["w"] = torch.sigmoid(torch.randn(inp["b"].shape, generator=g, device=dev)).to(inp["b"].dtype)
    grads = _run(inp, dO, dS_T)
    errs = compare_bwd_units(inp, grads, dO, dS_T, all_units(inp))
    assert max(errs.values()) <= TOL_BWD, errs


@pytest.mark.parametrize("dk,dv,dtype", [(64, 32, torch.float32), (16, 16, torch.bfloat16), (32, 64, torch.float32)])
def test_bwd_small_heads(dev, dk, dv, dtype):
    inp, dO, dS_T = _case(dev, dk, dv, dtype, LENS + [33])
    grads = _run(inp, dO, dS_T)
    errs = compare_bwd_units(inp, grads, dO, dS_T, all_units(inp))
    assert max(errs.values()) <= TOL_BWD, errs


@pytest.mark.parametrize("variant", ["d128", "d128_scalar_tied", "d128_p3", "small_f32"])
def test_bwd_fused_prologue(dev, variant):
    """Gradients with respect to the pre-activations (q, k L2 norm; sigmoid gates)."""
    kw = dict(d128=(128, 128, torch.bfloat16, {}), d128_scalar_tied=(128, 128, torch.bfloat16, dict(scalar=True)),
              d128_p3=(128, 128, torch.bfloat16, dict(p3=True)), small_f32=(32, 64, torch.float32, {}))[variant]
    dk, dv, dtype, extra = kw
    inp, dO, dS_T = _case(dev, dk, dv, dtype, LENS, prolog=True, **extra)
    grads = _run(inp, dO, dS_T)
    errs = compare_bwd_units(inp, grads, dO, dS_T, all_units(inp))
    assert max(errs.values()) <= TOL_BWD, errs


def test_bwd_without_final_state_gradient(dev):
    """dS_T = NULL means a zero final-state gradient; dS0 of a zero-length sequence is then 0."""
    inp, dO, _ = _case(dev, 128, 128, torch.bfloat16, [5, 0, 17], n_heads=1)
    grads = _run(inp, dO, None)
    errs = compare_bwd_units(inp, grads, dO, None, all_units(inp))
    assert max(errs.values()) <= TOL_BWD, errs
    assert float(grads["dS0"][1].abs().max()) == 0.0


def test_bwd_full_size_sampled(dev):
    """The prefill workload (8 x 4096 tokens, 16 heads, d = 128): sampled units."""
    from gated_delta_rule_159_b200 import inputs
    inp = inputs.make_inputs("gdn2_b8_t4k", dev)
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    dO = torch.randn(inp["T_tot"], 16, 128, generator=g, device=dev)
    dS_T = torch.randn(inp["n_seqs"], 16, 128, 128, generator=g, device=dev) * 0.1
    grads = _run(inp, dO, dS_T)
    errs = compare_bwd_units(inp, grads, dO, dS_T, [(0, 0), (5, 11)])
    assert max(errs.values()) <= TOL_BWD, errs
