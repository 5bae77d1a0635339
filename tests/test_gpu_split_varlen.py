"""GPU parity of gdn2_chunk_fwd_split_varlen: packed varlen batches in which a few
sequences are far longer than the balanced per-SM share (so they are cut into
segments joined through their affine maps), with empty, one-token and ragged
sequences beside them, against the float64 oracle (2e-2), and the same batch
through the plain gdn2_chunk_fwd.  A balanced batch takes the plain path and
must match gdn2_chunk_fwd bit for bit.
"""
import pytest
import torch

from parity_utils import TOL_CHUNK_BF16, all_units, compare_units, rel_err, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from gated_delta_rule_159_b200 import gdn2  # noqa: F401  (fails loudly without libgdn2.so)
    return torch.device("cuda:0")


def _inputs(dev, lengths, s0=0.02, **kw):
    from gated_delta_rule_159_b200 import inputs
    w = inputs.Workload("split_varlen", len(lengths), 0, kw.pop("n_heads", 2), 128, 128, 64, torch.bfloat16, 0.05,
                        kw.pop("scalar", False), s0)
    return inputs.make_inputs(w, dev, lengths=lengths, **kw)


def _run(inp, out_dtype=torch.float32, split=True):
    from gated_delta_rule_159_b200 import gdn2
    names = ("q", "k", "v", "log_a", "b", "w")
    kw = dict(scalar_decay=inp["scalar_decay"], scalar_gates=inp["scalar_gates"], tied_gates=inp["tied_gates"],
              gate_form_p3=inp["gate_form_p3"], out_dtype=out_dtype)
    if split:
        return gdn2.chunk_fwd_split_varlen(*(inp[n] for n in names), inp["S0"], inp["cu_seqlens"], inp["cu_host"],
                                           **kw)
    return gdn2.chunk_fwd(*(inp[n] for n in names), inp["S0"], inp["cu_seqlens"], cu_seqlens_host=inp["cu_host"],
                          **kw)


SKEWED = [20000, 300, 1, 0, 4100, 64, 129]


@pytest.mark.parametrize("variant", ["default", "no_s0", "p3", "scalar"])
def test_skewed_batch_matches_oracle(dev, variant):
    inp = _inputs(dev, SKEWED, s0=0.0 if variant == "no_s0" else 0.02, gate_form_p3=(variant == "p3"),
                  scalar=(variant == "scalar"))
    o, S_T = _run(inp)
    assert torch.isfinite(o).all() and torch.isfinite(S_T).all()
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


def test_skewed_batch_matches_plain_forward(dev):
    inp = _inputs(dev, SKEWED, n_heads=3)
    o, S_T = _run(inp, out_dtype=torch.bfloat16)
    o_p, S_p = _run(inp, out_dtype=torch.bfloat16, split=False)
    for h in range(3):
        assert rel_err(to_f64(o[:, h]), to_f64(o_p[:, h])) <= TOL_CHUNK_BF16
    assert rel_err(to_f64(S_T), to_f64(S_p)) <= TOL_CHUNK_BF16


def test_balanced_batch_takes_the_plain_path(dev):
    """Lengths within 3x of the balanced share: no sequence is split, and the result is
    gdn2_chunk_fwd's, bit for bit."""
    inp = _inputs(dev, [700, 650, 0, 1, 640, 513], n_heads=16)
    o, S_T = _run(inp)
    o_p, S_p = _run(inp, split=False)
    assert torch.equal(o, o_p) and torch.equal(S_T, S_p)


def test_workspace_status_clean(dev):
    from gated_delta_rule_159_b200 import gdn2
    inp = _inputs(dev, SKEWED)
    dims = gdn2.make_dims(len(SKEWED), inp["T_tot"], 2, 128, 128, 64, gdn2.BF16, gdn2.F32, 0)
    ws = torch.empty(gdn2.split_varlen_workspace_size(dims, inp["cu_host"]), dtype=torch.uint8, device=dev)
    names = ("q", "k", "v", "log_a", "b", "w")
    gdn2.chunk_fwd_split_varlen(*(inp[n] for n in names), inp["S0"], inp["cu_seqlens"], inp["cu_host"],
                                out_dtype=torch.float32, workspace=ws)
    assert gdn2.check_status(ws) == gdn2.OK


@pytest.mark.parametrize("variant", ["prologue", "p3_prologue"])
def test_skewed_batch_fused_prologue(dev, variant):
    """The varlen split with pre-activations (GDN2_FUSED_PROLOGUE) in both gate forms."""
    inp = _inputs(dev, [9000, 70, 0, 1, 200], gate_form_p3=(variant == "p3_prologue"), fused_prologue=True)
    from gated_delta_rule_159_b200 import gdn2
    names = ("q", "k", "v", "log_a", "b", "w")
    o, S_T = gdn2.chunk_fwd_split_varlen(*(inp[n] for n in names), inp["S0"], inp["cu_seqlens"], inp["cu_host"],
                                         gate_form_p3=inp["gate_form_p3"], fused_prologue=True,
                                         out_dtype=torch.float32)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)
