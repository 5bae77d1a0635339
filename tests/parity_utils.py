"""Helpers shared by the parity tests: run the float64 oracle on selected
(sequence, head) units of a packed problem and compare against the GPU.

Error metric (per output tensor): for every (sequence, head) unit,
err = max|gpu - oracle| / max|oracle| over that unit's elements; the test
takes the maximum over units and compares it with the tolerance.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle import prologue

# The chunked path consumes bf16 inputs and runs bf16 tensor-core GEMMs with
# fp32 accumulation; the decode path and the fp32 small-head path are fp32.
TOL_CHUNK_BF16 = 2e-2
TOL_DECODE = 1e-4
# fp32 small-head chunk path: fp32 rounding (~6e-8) accumulated over dot
# products of <= 64 terms and a few hundred sequential steps stays far below
# this; 1e-4 keeps two orders of margin.
TOL_CHUNK_F32 = 1e-4


def to_f64(t):
    if t is None:
        return None
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_flags(inp) -> int:
    f = 0
    if inp["scalar_decay"]:
        f |= oracle.SCALAR_DECAY
    if inp["scalar_gates"]:
        f |= oracle.SCALAR_GATES
    if inp["tied_gates"]:
        f |= oracle.TIED_GATES
    if inp.get("gate_form_p3", False):
        f |= oracle.GATE_FORM_P3
    return f


def oracle_on_units(inp, units, n_threads: int = 0):
    """Run the oracle on the listed (n, h) units only.  Returns {(n, h): (o [len, d_v], S_T [d_k, d_v])}."""
    cu = inp["cu_host"]
    pieces = {name: [] for name in ("q", "k", "v", "log_a", "b", "w")}
    S0s, lens = [], []
    for (n, h) in units:
        a0, a1 = cu[n], cu[n + 1]
        lens.append(a1 - a0)
        for name in pieces:
            t = inp[name]
            if t is None:
                continue
            pieces[name].append(to_f64(t[a0:a1, h:h + 1]))
        S0s.append(np.zeros((1, inp["q"].shape[-1], inp["v"].shape[-1])) if inp["S0"] is None
                   else to_f64(inp["S0"][n, h:h + 1]))
    cat = {k: (np.concatenate(v) if v else None) for k, v in pieces.items()}
    if inp.get("fused_prologue", False):
        cat["q"], cat["k"], cat["log_a"], cat["b"], cat["w"] = prologue.apply(cat["q"], cat["k"], cat["log_a"],
                                                                               cat["b"], cat["w"])
    cu_sub = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    o, S = oracle.gdn2_fwd(cat["q"], cat["k"], cat["v"], cat["log_a"], cat["b"], cat["w"],
                           S0=np.stack(S0s), cu_seqlens=cu_sub, flags=oracle_flags(inp), n_threads=n_threads)
    out = {}
    for i, u in enumerate(units):
        out[u] = (o[cu_sub[i]:cu_sub[i + 1], 0], S[i, 0])
    return out


def rel_err(g: np.ndarray, r: np.ndarray) -> float:
    scale = np.abs(r).max() if r.size else 0.0
    if scale == 0.0:
        return float(np.abs(g).max()) if g.size else 0.0
    return float(np.abs(g - r).max() / scale)


def compare_units(inp, o_gpu, S_T_gpu, units, n_threads: int = 0):
    """Max over units of the per-unit relative errors of o and S_T."""
    ref = oracle_on_units(inp, units, n_threads)
    cu = inp["cu_host"]
    eo, es = 0.0, 0.0
    for (n, h), (o_r, S_r) in ref.items():
        a0, a1 = cu[n], cu[n + 1]
        g = to_f64(o_gpu[a0:a1, h])
        assert np.isfinite(g).all(), f"non-finite o in unit {(n, h)}"
        eo = max(eo, rel_err(g, o_r))
        if S_T_gpu is not None:
            gs = to_f64(S_T_gpu[n, h])
            assert np.isfinite(gs).all(), f"non-finite S_T in unit {(n, h)}"
            es = max(es, rel_err(gs, S_r))
    return eo, es


def all_units(inp):
    H = inp["q"].shape[1]
    return [(n, h) for n in range(inp["n_seqs"]) for h in range(H)]


def run_chunk(inp, out_dtype=None, S0="inp", packed=None):
    """Call gdn2.chunk_fwd on a workload dict.  Equal-length batches go through
    the [B, T, H, d] form unless ``packed`` forces the cu_seqlens form.
    Returns (o as [T_tot, H, d_v], S_T)."""
    from gated_delta_rule_159_b200 import gdn2
    w = inp["workload"]
    S0t = inp["S0"] if S0 == "inp" else S0
    kw = dict(chunk=w.chunk, scalar_decay=inp["scalar_decay"], scalar_gates=inp["scalar_gates"],
              tied_gates=inp["tied_gates"], gate_form_p3=inp.get("gate_form_p3", False),
              fused_prologue=inp.get("fused_prologue", False), out_dtype=out_dtype)
    names = ("q", "k", "v", "log_a", "b", "w")
    if packed is None:
        packed = not inp["equal_lengths"]
    if packed:
        cu = inp["cu_seqlens"]
        if cu is None:
            cu = torch.tensor(inp["cu_host"], dtype=torch.int32, device=inp["q"].device)
        o, S_T = gdn2.chunk_fwd(*(inp[n] for n in names), S0t, cu, cu_seqlens_host=inp["cu_host"], **kw)
        return o, S_T
    N = inp["n_seqs"]
    T = inp["T_tot"] // N

    def v4(t):
        return None if t is None else t.view(N, T, *t.shape[1:])

    o, S_T = gdn2.chunk_fwd(*(v4(inp[n]) for n in names), S0t, None, **kw)
    return o.view(inp["T_tot"], *o.shape[2:]), S_T


# Backward (fp32 token-serial reverse mode on the GPU).  Every gradient is a
# sum of fp32 products over one token's d_k x d_v state, carried backward over
# the sequence; dlog_a and db are dot products of mixed-sign terms whose size
# can be far below the largest term, so the metric (max error / max |ref| per
# unit) gets 1e-3: ten times the fp32 forward's bound.
TOL_BWD = 1e-3

GRADS = ("dq", "dk", "dv", "dlog_a", "db", "dw")
GRAD_INPUT = dict(dq="q", dk="k", dv="v", dlog_a="log_a", db="b", dw="w")


def oracle_bwd_on_units(inp, dO, dS_T, units, n_threads: int = 0):
    """Oracle gradients for the listed (n, h) units, each as its own problem.
    Returns {(n, h): dict of float64 arrays with the unit's token rows}."""
    cu = inp["cu_host"]
    out = {}
    for (n, h) in units:
        a0, a1 = cu[n], cu[n + 1]
        sl = lambda t: None if t is None else to_f64(t[a0:a1, h:h + 1])  # noqa: E731
        S0 = None if inp["S0"] is None else to_f64(inp["S0"][n, h:h + 1])[None]
        dST = None if dS_T is None else to_f64(dS_T[n, h:h + 1])[None]
        raw = [sl(inp[m]) for m in ("q", "k", "log_a", "b", "w")]
        act = prologue.apply(*raw) if inp.get("fused_prologue", False) else raw
        g = oracle.gdn2_bwd(act[0], act[1], sl(inp["v"]), act[2], act[3], act[4], sl(dO), S0=S0, dS_T=dST,
                            flags=oracle_flags(inp), n_threads=n_threads)
        if inp.get("fused_prologue", False):
            g.update({k: v for k, v in prologue.vjp(*raw, g["dq"], g["dk"], g["dlog_a"], g["db"], g["dw"]).items()
                      if v is not None})
        out[(n, h)] = g
    return out


def compare_bwd_units(inp, g_gpu, dO, dS_T, units, n_threads: int = 0):
    """Max over units of the per-unit relative error of every gradient (dict by name)."""
    ref = oracle_bwd_on_units(inp, dO, dS_T, units, n_threads)
    cu = inp["cu_host"]
    errs = {name: 0.0 for name in GRADS + ("dS0",)}
    for (n, h), r in ref.items():
        a0, a1 = cu[n], cu[n + 1]
        for name in GRADS:
            if r[name] is None or g_gpu[name] is None:
                continue
            g = to_f64(g_gpu[name][a0:a1, h])
            assert np.isfinite(g).all(), f"non-finite {name} in unit {(n, h)}"
            errs[name] = max(errs[name], rel_err(g, r[name][:, 0]))
        if g_gpu["dS0"] is not None:
            errs["dS0"] = max(errs["dS0"], rel_err(to_f64(g_gpu["dS0"][n, h]), r["dS0"][0, 0]))
    return errs
