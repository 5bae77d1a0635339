"""GPU parity of the tensor-core chunked path over the whole decay domain.

The chunk kernel factors the in-chunk decay e^{L_i - L_j} into per-row factors
around a per-channel reference; a chunk in which some channel decays by more
than 128 nats between its first and last row runs the recurrence token by token
instead.  These cases put chunks on both sides of that line -- uniform strong
decay (-20 per step), strong and weak channels side by side, the fused
prologue with decay pre-activations drawn from N(-6, 2), and bursts of strong
decay between weak stretches so that factored and token-serial chunks alternate
inside one sequence -- and compare every element with the float64 oracle
(max relative error per unit <= 2e-2, finite o and S_T).
"""
import pytest
import torch

from parity_utils import TOL_CHUNK_BF16, all_units, compare_units, run_chunk

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from gated_delta_rule_159_b200 import gdn2  # noqa: F401  (fails loudly without libgdn2.so)
    return torch.device("cuda:0")


def _small(dev, scalar=False, **kw):
    from gated_delta_rule_159_b200 import inputs
    w = inputs.Workload("range", kw.pop("n_seqs", 2), kw.pop("seq_len", 200), kw.pop("n_heads", 2), 128, 128, 64,
                        torch.bfloat16, 0.05, scalar, 0.02)
    return inputs.make_inputs(w, dev, **kw)


def _check(inp, out_dtype=None):
    o, S_T = run_chunk(inp, out_dtype=out_dtype)
    assert torch.isfinite(o).all() and torch.isfinite(S_T).all()
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


LENGTHS = [1, 63, 64, 65, 200, 0, 130]


@pytest.mark.parametrize("variant", ["default", "p3", "scalar"])
def test_uniform_strong_decay(dev, variant):
    """log_a = -20 on every channel of every token: every chunk runs token by token."""
    inp = _small(dev, lengths=LENGTHS, scalar=(variant == "scalar"), gate_form_p3=(variant == "p3"))
    inp["log_a"] = torch.full_like(inp["log_a"], -20.0)
    _check(inp, out_dtype=torch.float32)


def test_strong_and_weak_channels(dev):
    """Half the channels decay at -20 per step, the other half at -0.01."""
    inp = _small(dev, lengths=LENGTHS)
    la = torch.full_like(inp["log_a"], -0.01)
    la[..., :64] = -20.0
    inp["log_a"] = la
    _check(inp)


def test_moderate_decay_over_the_span(dev):
    """-2.4 per step: a chunk's decay range is 151 nats, just past the factored form."""
    inp = _small(dev, lengths=LENGTHS)
    inp["log_a"] = torch.full_like(inp["log_a"], -2.4)
    _check(inp, out_dtype=torch.float32)


def test_just_inside_the_span(dev):
    """-2.0 per step: a chunk's decay range is 126 nats, the factored form at its widest."""
    inp = _small(dev, lengths=LENGTHS)
    inp["log_a"] = torch.full_like(inp["log_a"], -2.0)
    _check(inp, out_dtype=torch.float32)


@pytest.mark.parametrize("variant", ["default", "p3", "scalar"])
def test_bursts_alternate_the_two_forms(dev, variant):
    """Weak decay with bursts of -12 per step on some channels: within one sequence chunks
    switch between the factored and the token-serial form (first chunk, middle chunks,
    ragged last chunk), and single reset tokens (-1000) appear mid-chunk."""
    inp = _small(dev, n_heads=3, lengths=[300, 64, 129, 17, 250], scalar=(variant == "scalar"),
                 gate_form_p3=(variant == "p3"))
    la = inp["log_a"].float().clone()
    cu = inp["cu_host"]
    bursts = [(cu[0] + 70, cu[0] + 100), (cu[0] + 250, cu[0] + 290), (cu[1] + 0, cu[1] + 10),
              (cu[2] + 120, cu[2] + 129), (cu[4] + 5, cu[4] + 6)]
    for a0, a1 in bursts:
        if la.dim() == 2:
            la[a0:a1] = -12.0
        else:
            la[a0:a1, :, ::3] = -12.0
    la[cu[4] + 180] = -1000.0  # a reset token in the middle of a chunk
    inp["log_a"] = la.to(inp["log_a"].dtype)
    _check(inp, out_dtype=torch.float32)


@pytest.mark.parametrize("variant", ["channel", "p3"])
def test_fused_prologue_strong_decay_preactivations(dev, variant):
    """GDN2_FUSED_PROLOGUE with decay pre-activations ~ N(-6, 2): log sigmoid(x) is about x,
    a decay of several nats per step on every channel."""
    inp = _small(dev, lengths=LENGTHS, gate_form_p3=(variant == "p3"), fused_prologue=True)
    g = torch.Generator(device=dev)
    g.manual_seed(77)
    x = torch.randn(inp["log_a"].shape, generator=g, device=dev) * 2.0 - 6.0
    inp["log_a"] = x.to(inp["log_a"].dtype)
    _check(inp)


def test_split_forward_strong_decay(dev):
    """The sequence-parallel forward (three passes of the chunk kernel and the affine
    combine) with token-serial chunks in every segment."""
    from gated_delta_rule_159_b200 import gdn2
    from parity_utils import oracle_on_units, rel_err, to_f64
    inp = _small(dev, n_seqs=1, seq_len=640, n_heads=2)
    la = inp["log_a"].float().clone()
    la[100:140] = -8.0
    la[400:410, :, :32] = -30.0
    inp["log_a"] = la.to(inp["log_a"].dtype)
    names = ("q", "k", "v", "log_a", "b", "w")
    o, S_T = gdn2.chunk_fwd_split(*(inp[n][None] for n in names), inp["S0"], n_split=4, out_dtype=torch.float32)
    ref = oracle_on_units(inp, all_units(inp))
    for h in range(2):
        o_r, S_r = ref[(0, h)]
        assert rel_err(to_f64(o[0, :, h]), o_r) <= TOL_CHUNK_BF16
        assert rel_err(to_f64(S_T[0, h]), S_r) <= TOL_CHUNK_BF16
