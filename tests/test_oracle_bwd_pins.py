"""Pins for the float64 oracle backward (CPU only).

The oracle backward is hand-written reverse mode; it is pinned here against
things that do not share its arithmetic:

* central finite differences of the oracle FORWARD (every input element of a
  tiny problem, every flag combination, several packed sequences);
* the same across the 64-token recompute segments of the backward;
* closed forms: with b = w = 0 the state only decays, S_T = Diag(e^{sum log_a}) S0,
  so dS0 = Diag(e^{sum log_a}) dS_T and every token's d log_a equals
  sum_j dS_T[i, j] S_T[i, j]; and o_t = S_t^T q_t gives dq_t = S_t dO_t, with
  S_t read off a forward run cut at token t.
"""
import numpy as np
import pytest

import oracle

SD, SG, TIED, P3 = oracle.SCALAR_DECAY, oracle.SCALAR_GATES, oracle.TIED_GATES, oracle.GATE_FORM_P3


def _problem(rng, lens, H, dk, dv, flags):
    T = int(sum(lens))
    N = len(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    gshape = (T, H) if flags & SD else (T, H, dk)
    bshape = (T, H) if flags & SG else (T, H, dk)
    wshape = (T, H) if flags & SG else ((T, H, dv) if flags & P3 else (T, H, dk))
    q = rng.standard_normal((T, H, dk)) * 0.7
    k = rng.standard_normal((T, H, dk)) * 0.7
    inp = dict(q=q, k=k, v=rng.standard_normal((T, H, dv)),
               log_a=-rng.uniform(0.05, 0.6, gshape), b=rng.uniform(0.1, 0.9, bshape),
               w=None if flags & TIED else rng.uniform(0.1, 0.9, wshape),
               S0=rng.standard_normal((N, H, dk, dv)) * 0.5)
    cot = dict(dO=rng.standard_normal((T, H, dv)), dS_T=rng.standard_normal((N, H, dk, dv)))
    return inp, cot, cu


def _loss(inp, cot, cu, flags):
    o, S_T = oracle.gdn2_fwd(inp["q"], inp["k"], inp["v"], inp["log_a"], inp["b"], inp["w"], S0=inp["S0"],
                             cu_seqlens=cu, flags=flags)
    return float((o * cot["dO"]).sum() + (S_T * cot["dS_T"]).sum())


def _fd(inp, cot, cu, flags, name, idx, h=1e-6):
    def at(delta):
        x = {k: (None if v is None else v.copy()) for k, v in inp.items()}
        x[name][idx] += delta
        return _loss(x, cot, cu, flags)
    return (at(h) - at(-h)) / (2 * h)


GRAD_OF = dict(q="dq", k="dk", v="dv", log_a="dlog_a", b="db", w="dw", S0="dS0")


@pytest.mark.parametrize("flags,dk,dv", [
    (0, 3, 2), (SD, 3, 2), (SD | SG, 3, 2), (TIED, 3, 2), (SD | SG | TIED, 2, 3),
    (P3, 3, 2), (P3 | SG, 2, 3), (P3 | TIED, 3, 3), (P3 | SD | SG | TIED, 3, 2),
])
def test_backward_matches_finite_differences(flags, dk, dv):
    rng = np.random.default_rng(7 + flags)
    inp, cot, cu = _problem(rng, [5, 0, 3], 2, dk, dv, flags)
    g = oracle.gdn2_bwd(inp["q"], inp["k"], inp["v"], inp["log_a"], inp["b"], inp["w"], cot["dO"],
                        S0=inp["S0"], dS_T=cot["dS_T"], cu_seqlens=cu, flags=flags)
    if flags & TIED:
        assert g["dw"] is None
    for name, gname in GRAD_OF.items():
        if inp[name] is None:
            continue
        grad = g[gname]
        assert grad.shape == inp[name].shape
        scale = max(1.0, float(np.abs(grad).max()))
        for idx in np.ndindex(*inp[name].shape):
            fd = _fd(inp, cot, cu, flags, name, idx)
            assert abs(fd - grad[idx]) <= 2e-7 * scale, (name, idx, fd, grad[idx])


def test_backward_across_recompute_segments():
    """Tokens on both sides of the 64-token segment boundaries of the backward."""
    rng = np.random.default_rng(3)
    inp, cot, cu = _problem(rng, [150], 1, 2, 2, 0)
    inp["log_a"] *= 0.1  # keep the state alive over 150 tokens
    g = oracle.gdn2_bwd(inp["q"], inp["k"], inp["v"], inp["log_a"], inp["b"], inp["w"], cot["dO"],
                        S0=inp["S0"], dS_T=cot["dS_T"], cu_seqlens=cu)
    for t in (0, 62, 63, 64, 65, 127, 128, 149):
        for name in ("q", "k", "v", "log_a", "b", "w"):
            idx = (t, 0, 1)
            fd = _fd(inp, cot, cu, 0, name, idx)
            assert abs(fd - g[GRAD_OF[name]][idx]) <= 2e-7 * max(1.0, abs(fd)), (name, t)
    for idx in np.ndindex(1, 1, 2, 2):
        fd = _fd(inp, cot, cu, 0, "S0", idx)
        assert abs(fd - g["dS0"][idx]) <= 2e-7 * max(1.0, abs(fd))


def test_backward_pure_decay_closed_form():
    rng = np.random.default_rng(5)
    T, H, dk, dv = 9, 2, 4, 3
    inp, cot, cu = _problem(rng, [T], H, dk, dv, 0)
    inp["b"][:] = 0.0
    inp["w"][:] = 0.0
    cot["dO"][:] = 0.0
    g = oracle.gdn2_bwd(inp["q"], inp["k"], inp["v"], inp["log_a"], inp["b"], inp["w"], cot["dO"],
                        S0=inp["S0"], dS_T=cot["dS_T"], cu_seqlens=cu)
    decay = np.exp(inp["log_a"].sum(axis=0))                 # [H, dk]
    S_T = decay[..., None] * inp["S0"][0]                    # [H, dk, dv]
    np.testing.assert_allclose(g["dS0"][0], decay[..., None] * cot["dS_T"][0], rtol=1e-13, atol=1e-15)
    per_token = (cot["dS_T"][0] * S_T).sum(-1)               # [H, dk]
    for t in range(T):
        np.testing.assert_allclose(g["dlog_a"][t], per_token, rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(g["dq"], 0.0)
    np.testing.assert_array_equal(g["dv"], 0.0)


def test_backward_dq_is_state_times_dO():
    rng = np.random.default_rng(9)
    T, H, dk, dv = 7, 1, 3, 4
    inp, cot, cu = _problem(rng, [T], H, dk, dv, 0)
    g = oracle.gdn2_bwd(inp["q"], inp["k"], inp["v"], inp["log_a"], inp["b"], inp["w"], cot["dO"],
                        S0=inp["S0"], dS_T=cot["dS_T"], cu_seqlens=cu)
    for t in range(T):
        cut = {k: (None if v is None else (v[:t + 1] if k != "S0" else v)) for k, v in inp.items()}
        _, S_t = oracle.gdn2_fwd(cut["q"], cut["k"], cut["v"], cut["log_a"], cut["b"], cut["w"], S0=cut["S0"])
        np.testing.assert_allclose(g["dq"][t, 0], S_t[0, 0] @ cot["dO"][t, 0], rtol=1e-12, atol=1e-14)
