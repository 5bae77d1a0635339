"""Seeded synthetic workloads for the GDN-2 forward (shared by tests and bench).

This module only draws random inputs with the shapes and distributions of the
workloads; it holds none of the recurrence's arithmetic.  Recipe (all draws in
float32 from one ``torch.Generator`` on the target device, in the order q, k,
v, log_a, b, w, S0, then cast to the input dtype):

* q, k ~ N(0, 1), each [d_k] vector L2-normalised per token and head;
* v ~ N(0, 1);
* log_a = -softplus(N(0, 1)) * decay_scale (per channel, or one per token and
  head for the scalar-gate workload, where a = alpha * 1);
* b, w = sigmoid(N(0, 1)), independent per channel; the scalar-gate workload
  draws one beta per token and head and uses b = w = beta (tied);
* S0 ~ N(0, 1) * s0_std (0.02 for the full GDN-2 workload, else zeros).

The pages train a 1.3B-parameter model on FineWeb-Edu; no dataset or weights
are used here.  These inputs take the head shape of such a model (16 heads x
128) and stand in for its activations.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_seqs: int
    seq_len: int          # per sequence (equal lengths); ignored for varlen
    n_heads: int
    d_k: int
    d_v: int
    chunk: int
    dtype: torch.dtype
    decay_scale: float
    scalar_gates: bool    # one alpha and one beta per token and head, b = w = beta
    s0_std: float         # 0 -> zero initial state
    varlen_total: int = 0  # > 0: packed varlen batch with this many tokens
    varlen_min: int = 0
    varlen_max: int = 0

    @property
    def varlen(self) -> bool:
        return self.varlen_total > 0


WORKLOADS: Dict[str, Workload] = {
    # Tiny GDN-2 forward in fp32, chunk 16 (correctness only).
    "tiny_fp32": Workload("tiny_fp32", 1, 256, 1, 16, 16, 16, torch.float32, 0.1, False, 0.0),
    # Scalar-gate Gated DeltaNet special case (a = alpha 1, b = w = beta 1).
    "gdn_scalar_b4_t4k": Workload("gdn_scalar_b4_t4k", 4, 4096, 16, 128, 128, 64, torch.bfloat16, 0.05, True, 0.0),
    # Full GDN-2 with channel-wise decay and decoupled channel-wise gates.
    "gdn2_b8_t4k": Workload("gdn2_b8_t4k", 8, 4096, 16, 128, 128, 64, torch.bfloat16, 0.05, False, 0.02),
    # Packed varlen long context: 16 sequences of 4k-64k tokens, 524288 in total.
    "gdn2_varlen_16x4k-64k": Workload("gdn2_varlen_16x4k-64k", 16, 0, 16, 128, 128, 64, torch.bfloat16, 0.05,
                                      False, 0.0, 524288, 4096, 65536),
}

# Recurrent decode: 256 sequences x 16 heads x 128 x 128 fp32 state, 1024 steps,
# state from a chunked prefill of 2048 tokens.
DECODE = dict(n_seqs=256, n_heads=16, d=128, steps=1024, prefill_len=2048)


def varlen_lengths(total: int, n: int, lo: int, hi: int, seed: int = 0) -> List[int]:
    """n lengths drawn uniformly from [lo, hi], rescaled to sum to `total`,
    rounded, clamped to [lo, hi], with the residual spread by +-1 over the
    largest (or smallest) entries."""
    rng = np.random.default_rng(seed)
    raw = rng.uniform(lo, hi, n)
    lens = np.clip(np.round(raw * total / raw.sum()), lo, hi).astype(np.int64)
    order = np.argsort(-lens, kind="stable")
    i = 0
    while lens.sum() != total:
        j = order[i % n]
        step = 1 if lens.sum() < total else -1
        if lo <= lens[j] + step <= hi:
            lens[j] += step
        i += 1
    return [int(x) for x in lens]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device):
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32)


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_inputs(workload, device="cuda", seed: int = 0, seq_len: Optional[int] = None,
                n_seqs: Optional[int] = None, lengths: Optional[List[int]] = None,
                gate_form_p3: bool = False, fused_prologue: bool = False) -> dict:
    """Inputs of a workload (by name or ``Workload``).  ``seq_len``/``n_seqs``/``lengths``
    override the sizes (smaller parity cases with the same distributions).  With
    ``gate_form_p3`` the write gate w has d_v channels (the gist.science placement).
    With ``fused_prologue`` q, k, log_a, b, w are pre-activations: q, k ~ 2 N(0, 1)
    (not normalised), the decay pre-activation ~ N(3, 1) (sigmoid about 0.95) and the
    gate pre-activations ~ N(0, 1); draws keep the same order."""
    w = WORKLOADS[workload] if isinstance(workload, str) else workload
    device = torch.device(device)
    H, dk, dv = w.n_heads, w.d_k, w.d_v
    if lengths is None and w.varlen and seq_len is None:
        lengths = varlen_lengths(w.varlen_total, w.n_seqs, w.varlen_min, w.varlen_max, seed)
    if lengths is not None:
        N = len(lengths)
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
        T_tot = int(cu[-1])
    else:
        N = n_seqs if n_seqs is not None else w.n_seqs
        T = seq_len if seq_len is not None else w.seq_len
        cu = np.arange(N + 1, dtype=np.int64) * T
        T_tot = N * T
    g = _gen(device, seed)
    gshape = (T_tot, H) if w.scalar_gates else (T_tot, H, dk)
    wshape = (T_tot, H, dv) if gate_form_p3 else gshape
    if fused_prologue:
        q = (_randn((T_tot, H, dk), g, device) * 2).to(w.dtype)
        k = (_randn((T_tot, H, dk), g, device) * 2).to(w.dtype)
        v = _randn((T_tot, H, dv), g, device).to(w.dtype)
        log_a = (_randn(gshape, g, device) + 3.0).to(w.dtype)
        b = _randn(gshape, g, device).to(w.dtype)
        wg = None if w.scalar_gates else _randn(wshape, g, device).to(w.dtype)
    else:
        q = _l2n(_randn((T_tot, H, dk), g, device)).to(w.dtype)
        k = _l2n(_randn((T_tot, H, dk), g, device)).to(w.dtype)
        v = _randn((T_tot, H, dv), g, device).to(w.dtype)
        log_a = (-torch.nn.functional.softplus(_randn(gshape, g, device)) * w.decay_scale).to(w.dtype)
        b = torch.sigmoid(_randn(gshape, g, device)).to(w.dtype)
        wg = None if w.scalar_gates else torch.sigmoid(_randn(wshape, g, device)).to(w.dtype)
    S0 = (_randn((N, H, dk, dv), g, device) * w.s0_std) if w.s0_std > 0 else None
    equal = lengths is None
    return dict(
        workload=w, q=q, k=k, v=v, log_a=log_a, b=b, w=wg, S0=S0,
        cu_seqlens=None if equal else torch.tensor(cu, dtype=torch.int32, device=device),
        cu_host=cu.tolist(), n_seqs=N, T_tot=T_tot, equal_lengths=equal,
        scalar_decay=w.scalar_gates, scalar_gates=w.scalar_gates, tied_gates=w.scalar_gates,
        gate_form_p3=gate_form_p3, fused_prologue=fused_prologue,
    )


def make_decode_inputs(n_seqs: int, n_heads: int, d: int, steps: int, device="cuda", seed: int = 1,
                       dtype=torch.bfloat16, decay_scale: float = 0.05, d_v: Optional[int] = None,
                       gate_form_p3: bool = False) -> dict:
    """Per-step decode inputs [steps, N, H, d] (v: d_v, default d) with the full GDN-2
    gate distributions; w has d_v channels with ``gate_form_p3``."""
    device = torch.device(device)
    g = _gen(device, seed)
    dv = d if d_v is None else d_v
    shp = (steps, n_seqs, n_heads, d)
    shv = (steps, n_seqs, n_heads, dv)
    q = _l2n(_randn(shp, g, device)).to(dtype)
    k = _l2n(_randn(shp, g, device)).to(dtype)
    v = _randn(shv, g, device).to(dtype)
    log_a = (-torch.nn.functional.softplus(_randn(shp, g, device)) * decay_scale).to(dtype)
    b = torch.sigmoid(_randn(shp, g, device)).to(dtype)
    w = torch.sigmoid(_randn(shv if gate_form_p3 else shp, g, device)).to(dtype)
    return dict(q=q, k=k, v=v, log_a=log_a, b=b, w=w)
