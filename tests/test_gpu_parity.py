"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Small cases compare every element of every (sequence, head); they span
several chunks and ragged tails.  Full-size workloads run in the launch
configuration bench.py times and compare sampled units one by one.
Tolerances: 2e-2 (bf16-input chunked path), 1e-4 (fp32 decode and the fp32
small-head chunk path); metric in parity_utils.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from parity_utils import (TOL_CHUNK_BF16, TOL_CHUNK_F32, TOL_DECODE, all_units, compare_units, oracle_on_units,
                          rel_err, run_chunk, to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from gated_delta_rule_159_b200 import gdn2  # noqa: F401  (fails loudly without libgdn2.so)
    return torch.device("cuda:0")


def _inputs(name, dev, **kw):
    from gated_delta_rule_159_b200 import inputs
    return inputs.make_inputs(name, dev, **kw)


def _small(dev, dk=128, dv=128, chunk=64, dtype=torch.bfloat16, scalar=False, s0=0.02, decay=0.05, **kw):
    from gated_delta_rule_159_b200 import inputs
    w = inputs.Workload("small", kw.pop("n_seqs", 2), kw.pop("seq_len", 200), kw.pop("n_heads", 3), dk, dv, chunk,
                        dtype, decay, scalar, s0)
    return inputs.make_inputs(w, dev, **kw)


# ----------------------------------------------------------------- small-head fp32 path
def test_tiny_fp32_config(dev):
    inp = _inputs("tiny_fp32", dev)
    o, S_T = run_chunk(inp)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_F32 and es <= TOL_CHUNK_F32, (eo, es)


@pytest.mark.parametrize("variant", ["gdn", "deltanet"])
def test_tiny_fp32_reductions(dev, variant):
    """Gated DeltaNet (a = alpha 1, b = w = beta 1) and DeltaNet (alpha = 1) special cases."""
    from gated_delta_rule_159_b200 import inputs
    w = inputs.Workload("tiny_gdn", 1, 256, 1, 16, 16, 16, torch.float32, 0.1, True, 0.0)
    inp = inputs.make_inputs(w, dev)
    if variant == "deltanet":
        inp["log_a"] = torch.zeros_like(inp["log_a"])
    o, S_T = run_chunk(inp)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_F32 and es <= TOL_CHUNK_F32, (eo, es)


@pytest.mark.parametrize("dk,chunk,dtype", [(64, 64, torch.bfloat16), (32, 32, torch.float32), (16, 16, torch.bfloat16)])
def test_simt_path_varlen(dev, dk, chunk, dtype):
    inp = _small(dev, dk=dk, dv=dk, chunk=chunk, dtype=dtype, lengths=[1, chunk - 1, chunk, chunk + 1, 0, 3 * chunk + 5])
    o, S_T = run_chunk(inp, out_dtype=torch.float32)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_F32 and es <= TOL_CHUNK_F32, (eo, es)


# ----------------------------------------------------------------- tensor-core path, small
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_tc_equal_lengths(dev, out_dtype):
    inp = _small(dev, n_seqs=2, seq_len=200, n_heads=3)
    o, S_T = run_chunk(inp, out_dtype=out_dtype)
    assert o.dtype == out_dtype
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


def test_tc_varlen_ragged(dev):
    lens = [1, 63, 64, 65, 130, 0, 257, 5]
    inp = _small(dev, n_heads=2, lengths=lens)
    o, S_T = run_chunk(inp)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)
    # the zero-length sequence returns its initial state exactly
    torch.testing.assert_close(S_T[5], inp["S0"][5], rtol=0, atol=0)


def test_tc_packed_equals_batched_form(dev):
    inp = _small(dev, n_seqs=3, seq_len=150, n_heads=2)
    o1, S1 = run_chunk(inp, packed=False)
    o2, S2 = run_chunk(inp, packed=True)
    torch.testing.assert_close(o1, o2, rtol=0, atol=0)
    torch.testing.assert_close(S1, S2, rtol=0, atol=0)


def test_tc_scalar_gates(dev):
    inp = _small(dev, scalar=True, s0=0.0, n_seqs=2, seq_len=300, n_heads=2)
    o, S_T = run_chunk(inp)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


# gist.science gate placement: S = (I - k (b.k)^T) D S + k (w.v)^T, w on the d_v axis
@pytest.mark.parametrize("variant", ["channel", "scalar", "tied"])
def test_tc_gate_form_p3(dev, variant):
    lens = [1, 63, 64, 65, 200, 0, 130]
    inp = _small(dev, n_heads=2, lengths=lens, scalar=(variant == "scalar"), gate_form_p3=True)
    if variant == "scalar":
        inp["tied_gates"] = False
        gen = torch.Generator(device=dev)
        gen.manual_seed(31)
        inp["w"] = torch.sigmoid(torch.randn(inp["b"].shape, generator=gen, device=dev)).to(inp["b"].dtype)
    if variant == "tied":
        inp["tied_gates"] = True
        inp["w"] = None
    o, S_T = run_chunk(inp)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


def test_tc_gate_forms_differ(dev):
    """With channel-wise b != w the two gate placements give different results: the
    flag reaches the kernel (each side is checked against its own oracle above)."""
    inp = _small(dev, n_seqs=1, seq_len=130, n_heads=2, gate_form_p3=True)
    o3, S3 = run_chunk(inp)
    inp["gate_form_p3"] = False
    o0, S0_ = run_chunk(inp)
    ref = max(float(o3.abs().max()), 1e-30)
    assert float((o3.float() - o0.float()).abs().max()) / ref > 10 * TOL_CHUNK_BF16


@pytest.mark.parametrize("dk,dv,chunk,dtype", [(32, 64, 32, torch.float32), (64, 16, 64, torch.bfloat16)])
def test_simt_gate_form_p3(dev, dk, dv, chunk, dtype):
    inp = _small(dev, dk=dk, dv=dv, chunk=chunk, dtype=dtype, n_heads=2,
                 lengths=[1, chunk - 1, chunk + 1, 0, 3 * chunk + 5], gate_form_p3=True)
    assert inp["w"].shape[-1] == dv
    o, S_T = run_chunk(inp, out_dtype=torch.float32)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_F32 and es <= TOL_CHUNK_F32, (eo, es)


# fused prologue: pre-activations in, q/k L2 norm and sigmoid gates inside the kernels
@pytest.mark.parametrize("variant", ["channel", "scalar", "p3"])
def test_tc_fused_prologue(dev, variant):
    inp = _small(dev, n_heads=2, lengths=[1, 63, 64, 65, 200, 0, 130], scalar=(variant == "scalar"),
                 gate_form_p3=(variant == "p3"), fused_prologue=True)
    o, S_T = run_chunk(inp)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


@pytest.mark.parametrize("dk,dv,chunk,dtype,p3", [(32, 64, 32, torch.float32, False), (64, 16, 64, torch.float32, True)])
def test_simt_fused_prologue(dev, dk, dv, chunk, dtype, p3):
    inp = _small(dev, dk=dk, dv=dv, chunk=chunk, dtype=dtype, n_heads=2,
                 lengths=[1, chunk - 1, chunk + 1, 0, 3 * chunk + 5], gate_form_p3=p3, fused_prologue=True)
    o, S_T = run_chunk(inp, out_dtype=torch.float32)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_F32 and es <= TOL_CHUNK_F32, (eo, es)


@pytest.mark.parametrize("dk,dv,p3", [(128, 128, False), (64, 32, True)])
def test_decode_fused_prologue(dev, dk, dv, p3):
    from gated_delta_rule_159_b200 import gdn2
    from oracle import prologue
    N, H, steps = 3, 2, 5
    g = torch.Generator(device=dev)
    g.manual_seed(41)
    rn = lambda *s: torch.randn(*s, generator=g, device=dev)  # noqa: E731
    raw = dict(q=rn(steps, N, H, dk) * 2, k=rn(steps, N, H, dk) * 2, v=rn(steps, N, H, dv), log_a=rn(steps, N, H, dk) + 3,
               b=rn(steps, N, H, dk), w=rn(steps, N, H, dv if p3 else dk))
    raw = {n: t.to(torch.bfloat16) for n, t in raw.items()}
    S = torch.randn(N, H, dk, dv, generator=g, device=dev) * 0.1
    S_start = to_f64(S)
    names = ("q", "k", "v", "log_a", "b", "w")
    outs = [gdn2.decode_step(*(raw[n][t] for n in names), S, gate_form_p3=p3, fused_prologue=True).clone()
            for t in range(steps)]
    o_gpu = to_f64(torch.stack(outs))
    flags = oracle.GATE_FORM_P3 if p3 else 0
    for n in range(N):
        r = {m: to_f64(raw[m][:, n]) for m in names}
        q, k, la, b, w = prologue.apply(r["q"], r["k"], r["log_a"], r["b"], r["w"])
        o_r, S_r = oracle.gdn2_fwd(q, k, r["v"], la, b, w, S0=S_start[n][None], flags=flags)
        for h in range(H):
            assert rel_err(o_gpu[:, n, h], o_r[:, h]) <= TOL_DECODE
            assert rel_err(to_f64(S[n, h]), S_r[0, h]) <= TOL_DECODE


# sequence-parallel forward: segments of whole chunks combined through their affine maps
@pytest.mark.parametrize("n_split,seq_len,variant", [(1, 300, "channel"), (3, 1000, "channel"), (8, 1000, "channel"),
                                                     (64, 200, "channel"), (4, 700, "scalar"), (5, 640, "p3")])
def test_tc_split_forward(dev, n_split, seq_len, variant):
    from gated_delta_rule_159_b200 import gdn2
    inp = _small(dev, n_seqs=2, seq_len=seq_len, n_heads=2, scalar=(variant == "scalar"),
                 gate_form_p3=(variant == "p3"))
    N, T = inp["n_seqs"], inp["T_tot"] // inp["n_seqs"]
    names = ("q", "k", "v", "log_a", "b", "w")
    v4 = lambda t: None if t is None else t.view(N, T, *t.shape[1:])  # noqa: E731
    dims = gdn2.make_dims(N, T, 2, 128, 128, 64, gdn2.BF16, gdn2.F32,
                          gdn2.flags_of(inp["scalar_decay"], inp["scalar_gates"], inp["tied_gates"], variant == "p3"))
    ws = torch.empty(gdn2.split_workspace_size(dims, n_split), dtype=torch.uint8, device=dev)
    o, S_T = gdn2.chunk_fwd_split(*(v4(inp[n]) for n in names), inp["S0"], n_split=n_split,
                                  scalar_decay=inp["scalar_decay"], scalar_gates=inp["scalar_gates"],
                                  tied_gates=inp["tied_gates"], gate_form_p3=(variant == "p3"),
                                  out_dtype=torch.float32, workspace=ws)
    assert gdn2.check_status(ws) == gdn2.OK
    eo, es = compare_units(inp, o.view(inp["T_tot"], 2, 128), S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


def test_tc_split_forward_default_split(dev):
    """chunk_fwd_split with its default segment count (from the SM count) equals the oracle."""
    from gated_delta_rule_159_b200 import gdn2
    inp = _small(dev, n_seqs=1, seq_len=1500, n_heads=2)
    N, T = inp["n_seqs"], inp["T_tot"] // inp["n_seqs"]
    names = ("q", "k", "v", "log_a", "b", "w")
    o, S_T = gdn2.chunk_fwd_split(*(inp[n].view(N, T, *inp[n].shape[1:]) for n in names), inp["S0"],
                                  out_dtype=torch.float32)
    eo, es = compare_units(inp, o.view(inp["T_tot"], 2, 128), S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


# sequence parallelism across ranks: the per-rank calls, with the ranks emulated in one process
# (the all-gather of the maps becomes a stack); bounds need not fall on chunk boundaries
@pytest.mark.parametrize("bounds,variant", [((0, 200, 400), "channel"), ((0, 64, 317, 580, 704), "channel"),
                                            ((0, 333, 333, 700), "channel"), ((0, 256, 640), "scalar"),
                                            ((0, 150, 512), "p3")])
def test_segment_calls_emulated_ranks(dev, bounds, variant):
    from gated_delta_rule_159_b200 import gdn2
    T = bounds[-1]
    inp = _small(dev, n_seqs=2, seq_len=T, n_heads=2, scalar=(variant == "scalar"), gate_form_p3=(variant == "p3"))
    N = inp["n_seqs"]
    names = ("q", "k", "v", "log_a", "b", "w")
    v4 = lambda t: None if t is None else t.view(N, T, *t.shape[1:])  # noqa: E731
    flags = dict(scalar_decay=inp["scalar_decay"], scalar_gates=inp["scalar_gates"], tied_gates=inp["tied_gates"],
                 gate_form_p3=(variant == "p3"))
    full = {n: v4(inp[n]) for n in names}
    R = len(bounds) - 1
    pieces = []
    for r in range(R):  # step 1 on every rank
        lo, hi = bounds[r], bounds[r + 1]
        loc = {n: None if full[n] is None else full[n][:, lo:hi].contiguous() for n in names}
        o, F, G = gdn2.segment_maps(*(loc[n] for n in names), inp["S0"] if r == 0 else None, out_dtype=torch.float32,
                                    **flags)
        pieces.append((loc, o, F, G))
    F_all = torch.stack([pc[2] for pc in pieces])  # step 2: the all-gather
    G_all = torch.stack([pc[3] for pc in pieces])
    outs, S_T = [], None
    for r in range(R):  # steps 3 and 4
        loc, o, _, _ = pieces[r]
        start, S_T = gdn2.affine_prefix(F_all, G_all, r)
        if r > 0:
            gdn2.segment_correct(*(loc[n] for n in ("q", "k", "log_a", "b", "w")), start, o, **flags)
        outs.append(o)
    torch.cuda.synchronize()
    o = torch.cat(outs, dim=1)
    eo, es = compare_units(inp, o.reshape(inp["T_tot"], 2, 128), S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


def test_seq_ranks_one_rank_nccl(dev):
    """gdn2.chunk_fwd_seq_ranks over a one-rank NCCL group: the collective path of the
    sequence-parallel forward on one GPU (the all-gather has one participant)."""
    import datetime
    import socket
    import torch.distributed as dist
    from gated_delta_rule_159_b200 import gdn2
    inp = _small(dev, n_seqs=2, seq_len=300, n_heads=2)
    N, T = inp["n_seqs"], inp["T_tot"] // inp["n_seqs"]
    names = ("q", "k", "v", "log_a", "b", "w")
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        o, S_T = gdn2.chunk_fwd_seq_ranks(*(inp[n].view(N, T, *inp[n].shape[1:]) for n in names), inp["S0"],
                                          out_dtype=torch.float32)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    eo, es = compare_units(inp, o.reshape(inp["T_tot"], 2, 128), S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)


@pytest.mark.parametrize("case", ["deltanet", "pure_decay", "zero_key", "strong_decay", "no_decay_no_gates"])
def test_tc_degenerate_cases(dev, case):
    inp = _small(dev, n_seqs=1, seq_len=192, n_heads=2)
    if case == "deltanet":            # alpha = 1
        inp["log_a"] = torch.zeros_like(inp["log_a"])
    elif case == "pure_decay":        # b = w = 0: S_T = Diag(exp(sum log_a)) S0
        inp["b"] = torch.zeros_like(inp["b"])
        inp["w"] = torch.zeros_like(inp["w"])
    elif case == "zero_key":
        inp["k"] = torch.zeros_like(inp["k"])
    elif case == "strong_decay":      # -2.4 per step: a 151-nat range per chunk, run token by token
        inp["log_a"] = torch.full_like(inp["log_a"], -2.4)
    elif case == "no_decay_no_gates":  # alpha = 1, b = w = 0: the state holds
        inp["log_a"] = torch.zeros_like(inp["log_a"])
        inp["b"] = torch.zeros_like(inp["b"])
        inp["w"] = torch.zeros_like(inp["w"])
    o, S_T = run_chunk(inp, out_dtype=torch.float32)
    eo, es = compare_units(inp, o, S_T, all_units(inp))
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (eo, es)
    if case == "pure_decay":
        L = inp["log_a"].float().sum(0)  # [H, d_k]
        want = torch.exp(L)[:, :, None] * inp["S0"][0]
        torch.testing.assert_close(S_T[0], want, rtol=1e-5, atol=1e-7)


def test_tc_split_resume(dev):
    """Prefill in two calls (S_T fed back as S0) equals one call."""
    from gated_delta_rule_159_b200 import gdn2
    inp = _small(dev, n_seqs=1, seq_len=320, n_heads=2)
    names = ("q", "k", "v", "log_a", "b", "w")
    o_full, S_full = gdn2.chunk_fwd(*(inp[n][None] for n in names), inp["S0"], out_dtype=torch.float32)
    cut = 130
    oa, Sa = gdn2.chunk_fwd(*(inp[n][None, :cut] for n in names), inp["S0"], out_dtype=torch.float32)
    ob, Sb = gdn2.chunk_fwd(*(inp[n][None, cut:].contiguous() for n in names), Sa, out_dtype=torch.float32)
    ref = oracle_on_units(inp, all_units(inp))
    for h in range(2):
        o_r, S_r = ref[(0, h)]
        assert rel_err(to_f64(torch.cat([oa[0, :, h], ob[0, :, h]])), o_r) <= TOL_CHUNK_BF16
        assert rel_err(to_f64(Sb[0, h]), S_r) <= TOL_CHUNK_BF16
    assert rel_err(to_f64(Sb), to_f64(S_full)) <= TOL_CHUNK_BF16


def test_tc_S0_aliases_S_T(dev):
    from gated_delta_rule_159_b200 import gdn2
    inp = _small(dev, n_seqs=2, seq_len=100, n_heads=2)
    names = ("q", "k", "v", "log_a", "b", "w")
    N, T = 2, 100
    args = [inp[n].view(N, T, *inp[n].shape[1:]) for n in names]
    o1, S1 = gdn2.chunk_fwd(*args, inp["S0"])
    S = inp["S0"].clone()
    o2, S2 = gdn2.chunk_fwd(*args, S, S_T=S)
    assert S2.data_ptr() == S.data_ptr()
    torch.testing.assert_close(S2, S1, rtol=0, atol=0)
    torch.testing.assert_close(o2, o1, rtol=0, atol=0)


def test_tc_status_word_ok(dev):
    from gated_delta_rule_159_b200 import gdn2
    inp = _small(dev, n_seqs=1, seq_len=64, n_heads=1)
    ws = torch.empty(4096, dtype=torch.uint8, device=dev)
    names = ("q", "k", "v", "log_a", "b", "w")
    gdn2.chunk_fwd(*(inp[n][None] for n in names), inp["S0"], workspace=ws)
    assert gdn2.check_status(ws) == gdn2.OK


# ----------------------------------------------------------------- full-size workloads, sampled units
def _sample_units(inp, k, seed, extra=()):
    rng = np.random.default_rng(seed)
    H = inp["q"].shape[1]
    units = set(extra)
    while len(units) < k + len(extra):
        units.add((int(rng.integers(inp["n_seqs"])), int(rng.integers(H))))
    return sorted(units)


@pytest.mark.parametrize("name", ["gdn_scalar_b4_t4k", "gdn2_b8_t4k", "gdn2_varlen_16x4k-64k"])
def test_full_size_sampled(dev, name):
    inp = _inputs(name, dev)
    o, S_T = run_chunk(inp)
    torch.cuda.synchronize()
    extra = ()
    if not inp["equal_lengths"]:
        lens = np.diff(inp["cu_host"])
        extra = ((int(np.argmax(lens)), 0), (int(np.argmin(lens)), 15))
    units = _sample_units(inp, 4, seed=7, extra=extra)
    eo, es = compare_units(inp, o, S_T, units)
    assert eo <= TOL_CHUNK_BF16 and es <= TOL_CHUNK_BF16, (name, eo, es)
    # every output is finite across the whole workload
    assert torch.isfinite(o).all() and torch.isfinite(S_T).all()


# ----------------------------------------------------------------- decode
@pytest.mark.parametrize("d,scalar", [(128, False), (64, False), (128, True)])
def test_decode_small(dev, d, scalar):
    from gated_delta_rule_159_b200 import gdn2, inputs
    N, H, steps = 5, 3, 7
    di = inputs.make_decode_inputs(N, H, d, steps, dev, seed=3)
    if scalar:
        for n in ("log_a", "b"):
            di[n] = di[n][..., 0].contiguous()
        di["w"] = None
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    S = torch.randn(N, H, d, d, generator=g, device=dev) * 0.1
    S_start = to_f64(S)
    outs = []
    for t in range(steps):
        outs.append(gdn2.decode_step(di["q"][t], di["k"][t], di["v"][t], di["log_a"][t], di["b"][t],
                                     None if di["w"] is None else di["w"][t], S,
                                     scalar_decay=scalar, scalar_gates=scalar, tied_gates=scalar))
    o_gpu = to_f64(torch.stack(outs))  # [steps, N, H, d]
    assert gdn2.decode_status() == gdn2.OK
    flags = (oracle.SCALAR_DECAY | oracle.SCALAR_GATES | oracle.TIED_GATES) if scalar else 0
    # the decode steps of one (n, h) are one sequence of the recurrence
    for n in range(N):
        sl = lambda t: None if t is None else to_f64(t[:, n])  # noqa: E731
        o_r, S_r = oracle.gdn2_fwd(sl(di["q"]), sl(di["k"]), sl(di["v"]), sl(di["log_a"]), sl(di["b"]),
                                   sl(di["w"]), S0=S_start[n][None], flags=flags)
        for h in range(H):
            assert rel_err(o_gpu[:, n, h], o_r[:, h]) <= TOL_DECODE
            assert rel_err(to_f64(S[n, h]), S_r[0, h]) <= TOL_DECODE


@pytest.mark.parametrize("dk,dv,scalar", [(128, 128, False), (64, 32, False), (128, 64, True)])
def test_decode_gate_form_p3(dev, dk, dv, scalar):
    from gated_delta_rule_159_b200 import gdn2, inputs
    N, H, steps = 3, 2, 6
    di = inputs.make_decode_inputs(N, H, dk, steps, dev, seed=9, d_v=dv, gate_form_p3=True)
    if scalar:
        for n in ("log_a", "b", "w"):
            di[n] = di[n][..., 0].contiguous()
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    S = torch.randn(N, H, dk, dv, generator=g, device=dev) * 0.1
    S_start = to_f64(S)
    outs = []
    for t in range(steps):
        outs.append(gdn2.decode_step(*(di[n][t] for n in ("q", "k", "v", "log_a", "b", "w")), S,
                                     scalar_decay=scalar, scalar_gates=scalar, gate_form_p3=True))
    o_gpu = to_f64(torch.stack(outs))
    flags = oracle.GATE_FORM_P3 | ((oracle.SCALAR_DECAY | oracle.SCALAR_GATES) if scalar else 0)
    for n in range(N):
        sl = lambda t: to_f64(t[:, n])  # noqa: E731
        o_r, S_r = oracle.gdn2_fwd(*(sl(di[m]) for m in ("q", "k", "v", "log_a", "b", "w")),
                                   S0=S_start[n][None], flags=flags)
        for h in range(H):
            assert rel_err(o_gpu[:, n, h], o_r[:, h]) <= TOL_DECODE
            assert rel_err(to_f64(S[n, h]), S_r[0, h]) <= TOL_DECODE


@pytest.mark.parametrize("variant", ["channel", "scalar", "p3"])
def test_decode_indexed_matches_gathered_states(dev, variant):
    """Continuous batching: row n updates pool slot state_idx[n]; padding rows (index
    outside the pool) give zero output; slots no row names stay bit-identical.  With
    channel-wise gates, one alpha and one tied beta per row, and the gist.science form."""
    from gated_delta_rule_159_b200 import gdn2, inputs
    P, N, H, d, steps = 7, 5, 3, 128, 3
    idx = torch.tensor([3, 0, -1, 6, 9], dtype=torch.int32, device=dev)
    live = [0, 1, 3]
    di = inputs.make_decode_inputs(N, H, d, steps, dev, seed=13, gate_form_p3=(variant == "p3"))
    kw = {}
    flags = 0
    if variant == "scalar":
        for n in ("log_a", "b"):
            di[n] = di[n][..., 0].contiguous()
        di["w"] = None
        kw = dict(scalar_decay=True, scalar_gates=True, tied_gates=True)
        flags = oracle.SCALAR_DECAY | oracle.SCALAR_GATES | oracle.TIED_GATES
    elif variant == "p3":
        kw = dict(gate_form_p3=True)
        flags = oracle.GATE_FORM_P3
    g = torch.Generator(device=dev)
    g.manual_seed(17)
    pool = torch.randn(P, H, d, d, generator=g, device=dev) * 0.1
    pool_start = pool.clone()
    names = ("q", "k", "v", "log_a", "b", "w")
    outs = [gdn2.decode_step_indexed(*(None if di[n] is None else di[n][t] for n in names), pool, idx, **kw).clone()
            for t in range(steps)]
    assert gdn2.decode_status() == gdn2.OK
    o_gpu = to_f64(torch.stack(outs))
    assert np.all(o_gpu[:, [2, 4]] == 0.0)
    for s in (1, 2, 4, 5):
        torch.testing.assert_close(pool[s], pool_start[s], rtol=0, atol=0)
    for n in live:
        slot = int(idx[n])
        sl = lambda t: None if t is None else to_f64(t[:, n])  # noqa: E731
        o_r, S_r = oracle.gdn2_fwd(*(sl(di[m]) for m in names), S0=to_f64(pool_start[slot])[None], flags=flags)
        for h in range(H):
            assert rel_err(o_gpu[:, n, h], o_r[:, h]) <= TOL_DECODE
            assert rel_err(to_f64(pool[slot, h]), S_r[0, h]) <= TOL_DECODE


def test_decode_graph_replay_matches_eager(dev):
    """Decode steps captured in a CUDA graph and replayed give the eager results bit for bit."""
    from gated_delta_rule_159_b200 import gdn2, inputs
    N, H, d, steps = 8, 4, 128, 5
    names = ("q", "k", "v", "log_a", "b", "w")
    di = inputs.make_decode_inputs(N, H, d, steps, dev, seed=21)
    g = torch.Generator(device=dev)
    g.manual_seed(23)
    S_init = torch.randn(N, H, d, d, generator=g, device=dev) * 0.1
    S_eager = S_init.clone()
    o_eager = [gdn2.decode_step(*(di[n][t] for n in names), S_eager).clone() for t in range(steps)]
    S_graph = S_init.clone()
    o_buf = torch.empty(steps, N, H, d, device=dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for t in range(steps):
            gdn2.decode_step(*(di[n][t] for n in names), S_graph, o=o_buf[t])
    S_graph.copy_(S_init)  # capture records the launches without running them
    graph.replay()
    torch.cuda.synchronize()
    del graph
    torch.testing.assert_close(S_graph, S_eager, rtol=0, atol=0)
    torch.testing.assert_close(o_buf, torch.stack(o_eager), rtol=0, atol=0)


def test_decode_full_size_sampled(dev):
    """256 sequences x 16 heads x 128x128 state from a 2048-token chunked prefill,
    then 1024 decode steps; the oracle starts from the GPU prefill state."""
    from gated_delta_rule_159_b200 import gdn2, inputs
    cfg = inputs.DECODE
    N, H, d, steps = cfg["n_seqs"], cfg["n_heads"], cfg["d"], cfg["steps"]
    w = inputs.Workload("decode_prefill", N, cfg["prefill_len"], H, d, d, 64, torch.bfloat16, 0.05, False, 0.0)
    pre = inputs.make_inputs(w, dev)
    _, S = run_chunk(pre)
    del pre
    di = inputs.make_decode_inputs(N, H, d, steps, dev, seed=1)
    units = [(0, 0), (17, 5), (128, 9), (255, 15)]
    S_start = {u: to_f64(S[u]) for u in units}
    o = torch.empty(N, H, d, device=dev)
    idx_n = torch.tensor([u[0] for u in units], device=dev)
    idx_h = torch.tensor([u[1] for u in units], device=dev)
    rec = []
    for t in range(steps):
        gdn2.decode_step(di["q"][t], di["k"][t], di["v"][t], di["log_a"][t], di["b"][t], di["w"][t], S, o=o)
        rec.append(o[idx_n, idx_h].clone())
    rec = to_f64(torch.stack(rec))  # [steps, len(units), d]
    assert gdn2.decode_status() == gdn2.OK
    for i, (n, h) in enumerate(units):
        sl = lambda t: to_f64(t[:, n, h:h + 1])  # noqa: E731
        o_r, S_r = oracle.gdn2_fwd(sl(di["q"]), sl(di["k"]), sl(di["v"]), sl(di["log_a"]), sl(di["b"]),
                                   sl(di["w"]), S0=S_start[(n, h)][None, None])
        assert rel_err(rec[:, i], o_r[:, 0]) <= TOL_DECODE
        assert rel_err(to_f64(S[n, h]), S_r[0, 0]) <= TOL_DECODE
