"""Pins of the float64 oracle to what the pages and the mathematics fix.

Each test checks ``oracle.gdn2_fwd`` (the C recurrence) against something other
than itself: the pages' printed examples (tests/golden, each cited there),
closed forms derived by hand from the defining recurrence, independently
written textbook special cases (Gated DeltaNet, DeltaNet, KDA), brute-force
agreement with the chunkwise form, and structural invariants.  The set is
chosen so that a plausible slip in the oracle -- wrong step order, reading
before the update, a transposed state, erase and write gates swapped or put on
the wrong side, a dropped decay, a sign error -- fails at least one test.
"""
import math

import numpy as np
import pytest

import oracle
from oracle.chunked import gdn2_chunked_fwd


def _run_2x2(S0, alpha, k, v, beta, q, b=None, w=None):
    """One token through the oracle on a 2x2 state (d_k = d_v = 2, one head)."""
    dk = len(k)
    b = np.full(dk, beta) if b is None else np.asarray(b, float)
    w = np.full(dk, beta) if w is None else np.asarray(w, float)
    o, S = oracle.gdn2_fwd(
        np.array(q, float).reshape(1, 1, dk), np.array(k, float).reshape(1, 1, dk),
        np.array(v, float).reshape(1, 1, -1), np.full((1, 1, dk), math.log(alpha)),
        b.reshape(1, 1, dk), w.reshape(1, 1, dk),
        S0=np.array(S0, float).reshape(1, 1, dk, -1))
    return o[0, 0], S[0, 0]


# --------------------------------------------------------------------------
# Printed worked examples
# --------------------------------------------------------------------------

def test_scalar_gdn_step(golden):
    g = golden("scalar_gdn_step.txt")
    o, S = _run_2x2(np.array(g["S0"]).reshape(1, 1), g["alpha"][0], g["k"], g["v"],
                    g["beta"][0], q=[1.0])
    assert S[0, 0] == pytest.approx(g["S1"][0], abs=1e-12)
    assert abs(S[0, 0] - g["S1_error_on_old_state"][0]) > 0.4
    assert o[0] == pytest.approx(g["S1"][0], abs=1e-12)  # read after the update


def test_trace_2x2_decay_then_correct(golden):
    g = golden("trace_2x2.txt")
    o, S = _run_2x2(np.reshape(g["S0"], (2, 2)), g["alpha"][0], g["k"], g["v"],
                    g["beta"][0], q=g["q"])
    np.testing.assert_allclose(S.ravel(), g["S1"], atol=1e-12)
    np.testing.assert_allclose(o, g["read"], atol=1e-12)
    # residual error left by a beta = 0.5 write is exactly (1 - beta) e
    residual = np.array(g["v"]) - S.T @ np.array(g["k"])
    np.testing.assert_allclose(residual, g["residual"], atol=1e-12)
    np.testing.assert_allclose(residual, (1 - g["beta"][0]) * np.array(g["e"]), atol=1e-12)


def test_trace_2x2_intermediates(golden):
    """The decayed state and the erase read printed in the trace: with b = w = 0
    the oracle returns the decayed state; v_hat = S_decayed^T k."""
    g = golden("trace_2x2.txt")
    _, Sd = _run_2x2(np.reshape(g["S0"], (2, 2)), g["alpha"][0], g["k"], g["v"], 0.0, q=g["q"])
    np.testing.assert_allclose(Sd.ravel(), g["S_decayed"], atol=1e-12)
    np.testing.assert_allclose(Sd.T @ np.array(g["k"]), g["v_hat"], atol=1e-12)
    np.testing.assert_allclose(np.array(g["v"]) - Sd.T @ np.array(g["k"]), g["e"], atol=1e-12)


def test_trace_2x2_negative_control(golden):
    """The correct-then-decay order must NOT be what the oracle computes."""
    g = golden("trace_2x2.txt")
    _, S = _run_2x2(np.reshape(g["S0"], (2, 2)), g["alpha"][0], g["k"], g["v"],
                    g["beta"][0], q=g["q"])
    assert np.max(np.abs(S.ravel() - np.array(g["S1_correct_then_decay"]))) > 0.5


def test_trace_2x2_beta_limits(golden):
    g = golden("trace_2x2.txt")
    S0 = np.reshape(g["S0"], (2, 2))
    _, S = _run_2x2(S0, g["alpha"][0], g["k"], g["v"], 0.0, q=g["q"])
    np.testing.assert_allclose(S.ravel(), g["S1_beta0"], atol=1e-12)
    _, S = _run_2x2(S0, g["alpha"][0], g["k"], g["v"], 1.0, q=g["q"])
    np.testing.assert_allclose(S[0], g["S1_beta1_row1"], atol=1e-12)
    np.testing.assert_allclose(S[1], np.array(g["S_decayed"])[2:], atol=1e-12)


# --------------------------------------------------------------------------
# Decay, retention, half-life
# --------------------------------------------------------------------------

def _pure_decay(S0, log_a_per_step, steps):
    dk, dv = S0.shape
    T = steps
    la = np.broadcast_to(np.asarray(log_a_per_step, float), (T, dk)).reshape(T, 1, dk)
    z = np.zeros((T, 1, dk))
    rng = np.random.default_rng(1)
    q = rng.standard_normal((T, 1, dk))
    k = rng.standard_normal((T, 1, dk))
    v = rng.standard_normal((T, 1, dv))
    o, S = oracle.gdn2_fwd(q, k, v, la, z, z, S0=S0.reshape(1, 1, dk, dv))
    return o, S[0, 0], q


def test_decay_trace(golden):
    g = golden("decay_retention.txt")
    S0 = np.reshape(g["S0"], (2, 2))
    _, S1, _ = _pure_decay(S0, math.log(g["alpha"][0]), 1)
    _, S2, _ = _pure_decay(S0, math.log(g["alpha"][0]), 2)
    np.testing.assert_allclose(S1.ravel(), g["S_t1"], atol=1e-12)
    np.testing.assert_allclose(S2.ravel(), g["S_t2"], atol=1e-12)
    one = np.ones((1, 1))
    for t, want in enumerate(g["trace"]):
        _, St, _ = _pure_decay(one, math.log(0.8), t) if t else (None, one, None)
        assert St[0, 0] == pytest.approx(want, abs=1e-12)
    # first step below 0.1 is the 11th, at ~0.086
    vals = [_pure_decay(one, math.log(0.8), t)[1][0, 0] for t in (10, 11)]
    assert vals[0] > 0.1 > vals[1]
    assert int(g["below_0.1_at"][0]) == 11
    assert vals[1] == pytest.approx(g["value_at_11"][0], abs=5e-4)


def test_retention_and_half_lives(golden):
    g = golden("decay_retention.txt")
    one = np.ones((1, 1))
    _, S, _ = _pure_decay(one, math.log(0.9), 10)
    assert S[0, 0] == pytest.approx(g["retention_0.9_10"][0], abs=5e-4)
    # the half-life h = ln 0.5 / ln alpha: one step of log-decay h*ln(alpha) halves the state
    for alpha, key, tol in ((0.9, "half_life_0.9", 5e-3), (0.8, "half_life_0.8", 5e-4),
                            (0.99, "half_life_0.99", 0.5), (0.5, "half_life_0.5", 1e-12)):
        h = g[key][0]
        _, S, _ = _pure_decay(one, h * math.log(alpha), 1)
        assert S[0, 0] == pytest.approx(0.5, abs=tol * abs(math.log(alpha)))
    # alpha = 0.5: exactly one token halves the trace
    _, S, _ = _pure_decay(one, math.log(0.5), 1)
    assert S[0, 0] == 0.5
    # transfer challenge: alpha^2000 = 0.5.  alpha is printed to 5 decimals
    # (|error| <= 5e-6), which moves alpha^2000 by up to 2000 * 0.5 * 5e-6 = 5e-3.
    _, S, _ = _pure_decay(one, math.log(g["alpha_half_at_2000"][0]), 2000)
    assert S[0, 0] == pytest.approx(0.5, abs=5.1e-3)


def test_unbounded_gate_growth(golden):
    """log_a > 0 is outside the GPU path's preconditions, but the oracle must
    still apply a = exp(log_a) multiplicatively: 1.05^40 ~ 7.0, 1.05^100 ~ 131.5."""
    g = golden("decay_retention.txt")
    one = np.ones((1, 1))
    _, S40, _ = _pure_decay(one, math.log(1.05), 40)
    _, S100, _ = _pure_decay(one, math.log(1.05), 100)
    assert S40[0, 0] == pytest.approx(g["growth_1.05_40"][0], abs=0.05)
    assert S100[0, 0] == pytest.approx(g["growth_1.05_100"][0], abs=0.05)


def test_pure_decay_closed_form_per_channel():
    """b = w = 0: S_T = Diag(exp(sum_t log_a_t)) S0 and o_t = S_t^T q_t."""
    rng = np.random.default_rng(7)
    dk, dv, T = 5, 3, 9
    S0 = rng.standard_normal((dk, dv))
    la = -rng.uniform(0, 0.7, (T, dk))
    z = np.zeros((T, 1, dk))
    q = rng.standard_normal((T, 1, dk))
    o, S = oracle.gdn2_fwd(q, rng.standard_normal((T, 1, dk)), rng.standard_normal((T, 1, dv)),
                           la.reshape(T, 1, dk), z, z, S0=S0.reshape(1, 1, dk, dv))
    np.testing.assert_allclose(S[0, 0], np.exp(la.sum(0))[:, None] * S0, rtol=1e-13)
    for t in range(T):
        St = np.exp(la[: t + 1].sum(0))[:, None] * S0
        np.testing.assert_allclose(o[t, 0], St.T @ q[t, 0], rtol=1e-12, atol=1e-14)


def test_hold_when_alpha1_beta0():
    rng = np.random.default_rng(3)
    dk, dv, T = 4, 6, 12
    S0 = rng.standard_normal((dk, dv))
    z = np.zeros((T, 1, dk))
    _, S = oracle.gdn2_fwd(rng.standard_normal((T, 1, dk)), rng.standard_normal((T, 1, dk)),
                           rng.standard_normal((T, 1, dv)), z, z, z, S0=S0.reshape(1, 1, dk, dv))
    np.testing.assert_array_equal(S[0, 0], S0)


# --------------------------------------------------------------------------
# Gate decoupling: placement of b and w (no printed example distinguishes
# them, so closed forms derived from the defining recurrence pin them)
# --------------------------------------------------------------------------

def test_erase_gate_placement_closed_form():
    """k = (e1 + e2)/sqrt2, b = (1, 0), w = 0, no decay.  The default gate placement
    erases with the OUTER factor b.k = (1/sqrt2, 0) and reads with k:
        row1 -= (row1 + row2)/2,  row2 unchanged.
    Swapping the sides (read with b.k, erase along k) would instead give
        row1 -= row1/2, row2 -= row1/2."""
    S0 = np.array([[2.0, -1.0, 0.5], [4.0, 3.0, -2.0]])
    k = np.array([1.0, 1.0]) / math.sqrt(2)
    _, S = _run_2x2(S0, 1.0, k, [0.0, 0.0, 0.0], 0.0, q=[1, 0], b=[1.0, 0.0], w=[0.0, 0.0])
    want = S0.copy()
    want[0] -= (S0[0] + S0[1]) / 2
    np.testing.assert_allclose(S, want, atol=1e-14)
    swapped = S0.copy()
    swapped[0] -= S0[0] / 2
    swapped[1] -= S0[0] / 2
    assert np.max(np.abs(S - swapped)) > 0.5


def test_write_gate_placement_closed_form():
    """b = 0: S_T = Gamma_T S0 + sum_t Diag(gamma_T / gamma_t) (w_t . k_t) v_t^T.
    The write gate scales the key axis (rows), not the value axis."""
    rng = np.random.default_rng(11)
    dk, dv, T = 4, 3, 6
    S0 = rng.standard_normal((dk, dv))
    k = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    w = rng.uniform(0, 1, (T, dk))
    la = -rng.uniform(0, 0.5, (T, dk))
    _, S = oracle.gdn2_fwd(rng.standard_normal((T, 1, dk)), k.reshape(T, 1, dk), v.reshape(T, 1, dv),
                           la.reshape(T, 1, dk), np.zeros((T, 1, dk)), w.reshape(T, 1, dk),
                           S0=S0.reshape(1, 1, dk, dv))
    L = np.cumsum(la, axis=0)
    want = np.exp(L[-1])[:, None] * S0
    for t in range(T):
        want += np.outer(np.exp(L[-1] - L[t]) * w[t] * k[t], v[t])
    np.testing.assert_allclose(S[0, 0], want, rtol=1e-12, atol=1e-13)


def test_erase_only_projection():
    """w = 0, b = 1, unit key e_j, no decay: the erase removes exactly row j
    (S' = (I - k k^T) S with k k^T the projector on e_j)."""
    S0 = np.arange(12, dtype=float).reshape(4, 3) + 1
    for j in range(4):
        k = np.zeros(4)
        k[j] = 1.0
        _, S = _run_2x2(S0, 1.0, k, [5.0, 6.0, 7.0], 0.0, q=k, b=np.ones(4), w=np.zeros(4))
        want = S0.copy()
        want[j] = 0
        np.testing.assert_array_equal(S, want)


# --------------------------------------------------------------------------
# Reductions to textbook special cases
# --------------------------------------------------------------------------

def _gdn_textbook(S0, q, k, v, alpha, beta):
    """Gated DeltaNet as the neelmishra.github.io chapter states it: decay the
    state by alpha, take the error against the decayed read, write beta k err^T."""
    S = S0.copy()
    outs = []
    for t in range(len(k)):
        dec = alpha[t] * S
        err = v[t] - dec.T @ k[t]
        S = dec + beta[t] * np.outer(k[t], err)
        outs.append(S.T @ q[t])
    return np.array(outs), S


def _kda_textbook(S0, q, k, v, a, beta):
    """KDA: channel-wise decay Diag(a_t), single scalar beta for erase and write."""
    S = S0.copy()
    outs = []
    for t in range(len(k)):
        dec = a[t][:, None] * S
        S = dec + beta[t] * np.outer(k[t], v[t] - dec.T @ k[t])
        outs.append(S.T @ q[t])
    return np.array(outs), S


@pytest.mark.parametrize("alpha_one", [False, True])
def test_reduces_to_gated_deltanet_and_deltanet(alpha_one):
    rng = np.random.default_rng(5)
    dk, dv, T = 6, 5, 30
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    alpha = np.ones(T) if alpha_one else np.exp(-rng.uniform(0, 0.3, T))
    beta = rng.uniform(0, 1, T)
    S0 = rng.standard_normal((dk, dv))
    want_o, want_S = _gdn_textbook(S0, q, k, v, alpha, beta)
    ones = np.ones((T, 1, dk))
    o, S = oracle.gdn2_fwd(q.reshape(T, 1, dk), k.reshape(T, 1, dk), v.reshape(T, 1, dv),
                           np.log(alpha)[:, None, None] * ones, beta[:, None, None] * ones,
                           beta[:, None, None] * ones, S0=S0.reshape(1, 1, dk, dv))
    np.testing.assert_allclose(o[:, 0], want_o, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], want_S, rtol=1e-11, atol=1e-12)
    # the scalar-gate flags give the same numbers from [T, H] gates
    o2, S2 = oracle.gdn2_fwd(q.reshape(T, 1, dk), k.reshape(T, 1, dk), v.reshape(T, 1, dv),
                             np.log(alpha)[:, None], beta[:, None], None,
                             S0=S0.reshape(1, 1, dk, dv),
                             flags=oracle.SCALAR_DECAY | oracle.SCALAR_GATES | oracle.TIED_GATES)
    np.testing.assert_allclose(o2, o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S2, S, rtol=1e-13, atol=1e-14)


def test_reduces_to_kda_and_p3_agrees_when_tied():
    rng = np.random.default_rng(9)
    dk = dv = 6
    T = 25
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    a = np.exp(-rng.uniform(0, 0.4, (T, dk)))
    beta = rng.uniform(0, 1, T)
    S0 = rng.standard_normal((dk, dv))
    want_o, want_S = _kda_textbook(S0, q, k, v, a, beta)
    bb = beta[:, None, None] * np.ones((T, 1, dk))
    args = (q.reshape(T, 1, dk), k.reshape(T, 1, dk), v.reshape(T, 1, dv), np.log(a).reshape(T, 1, dk), bb, bb)
    for flags in (0, oracle.GATE_FORM_P3):
        o, S = oracle.gdn2_fwd(*args, S0=S0.reshape(1, 1, dk, dv), flags=flags)
        np.testing.assert_allclose(o[:, 0], want_o, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(S[0, 0], want_S, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# The gist.science gate placement (Methodologie 1, the printed update
# S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1} + k_t (w_t . v_t)^T) with
# channel-wise b != w: hand-derived closed forms in which the erase read side,
# the erase outer side and the write axis each change the answer.
# --------------------------------------------------------------------------

def _p3_run(S0, log_a, k, v, b, w, q=None):
    """Tokens through the oracle in the gist.science form: k, log_a, b [T, d_k];
    v, w [T, d_v]; S0 [d_k, d_v]."""
    k = np.atleast_2d(np.asarray(k, float))
    T, dk = k.shape
    v = np.atleast_2d(np.asarray(v, float))
    dv = v.shape[1]
    q = k if q is None else np.atleast_2d(np.asarray(q, float))
    return oracle.gdn2_fwd(q.reshape(T, 1, dk), k.reshape(T, 1, dk), v.reshape(T, 1, dv),
                           np.broadcast_to(np.asarray(log_a, float), (T, dk)).reshape(T, 1, dk),
                           np.atleast_2d(np.asarray(b, float)).reshape(T, 1, dk),
                           np.atleast_2d(np.asarray(w, float)).reshape(T, 1, dv),
                           S0=np.asarray(S0, float).reshape(1, 1, dk, dv), flags=oracle.GATE_FORM_P3)


def test_p3_erase_side_closed_form():
    """No decay, w = 0, k = (e1 + e2)/sqrt2, b = (1, 0).  In the gist.science form
    the erase READS with b.k = (1/sqrt2, 0) and erases ALONG k:
        (b.k)^T S = row1 / sqrt2,   S' = S - k (row1 / sqrt2)  ->  row1 -= row1/2, row2 -= row1/2.
    Reading with k and erasing along b.k (the other placement) instead gives
        row1 -= (row1 + row2)/2, row2 unchanged."""
    S0 = np.array([[2.0, -1.0, 0.5], [4.0, 3.0, -2.0]])
    k = np.array([1.0, 1.0]) / math.sqrt(2)
    _, S = _p3_run(S0, 0.0, k, np.zeros(3), [1.0, 0.0], np.zeros(3))
    want = S0.copy()
    want[0] -= S0[0] / 2
    want[1] -= S0[0] / 2
    np.testing.assert_allclose(S[0, 0], want, atol=1e-14)
    other = S0.copy()
    other[0] -= (S0[0] + S0[1]) / 2
    assert np.max(np.abs(S[0, 0] - other)) > 0.5


def test_p3_erase_with_decay_two_channels():
    """One token, d_k = d_v = 2, decay a = (0.5, 0.8), k = (0.6, 0.8), b = (0.25, 1), w = 0.
    By hand: Sbar = Diag(a) S; (b.k) = (0.15, 0.8); e^T Sbar = 0.15 Sbar_1 + 0.8 Sbar_2;
    S' = Sbar - k (e^T Sbar).  With S = [[4, -2], [1, 3]]: Sbar = [[2, -1], [0.8, 2.4]],
    e^T Sbar = (0.3 + 0.64, -0.15 + 1.92) = (0.94, 1.77),
    S' = [[2 - 0.564, -1 - 1.062], [0.8 - 0.752, 2.4 - 1.416]]."""
    S0 = np.array([[4.0, -2.0], [1.0, 3.0]])
    _, S = _p3_run(S0, np.log([0.5, 0.8]), [0.6, 0.8], [0.0, 0.0], [0.25, 1.0], [0.0, 0.0])
    want = np.array([[2 - 0.564, -1 - 1.062], [0.8 - 0.752, 2.4 - 1.416]])
    np.testing.assert_allclose(S[0, 0], want, atol=1e-13)


def test_p3_write_axis_closed_form():
    """b = 0 in the gist.science form: S_T = Gamma_T S0 + sum_t Diag(gamma_T / gamma_t) k_t (w_t . v_t)^T,
    with w on the VALUE axis (d_v = 4 channels, d_k = 3): the write gate scales columns, not rows."""
    rng = np.random.default_rng(31)
    dk, dv, T = 3, 4, 6
    S0 = rng.standard_normal((dk, dv))
    k = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    w = rng.uniform(0, 1, (T, dv))
    la = -rng.uniform(0, 0.5, (T, dk))
    _, S = oracle.gdn2_fwd(rng.standard_normal((T, 1, dk)), k.reshape(T, 1, dk), v.reshape(T, 1, dv),
                           la.reshape(T, 1, dk), np.zeros((T, 1, dk)), w.reshape(T, 1, dv),
                           S0=S0.reshape(1, 1, dk, dv), flags=oracle.GATE_FORM_P3)
    L = np.cumsum(la, axis=0)
    want = np.exp(L[-1])[:, None] * S0
    for t in range(T):
        want += np.outer(np.exp(L[-1] - L[t]) * k[t], w[t] * v[t])
    np.testing.assert_allclose(S[0, 0], want, rtol=1e-12, atol=1e-13)


def test_p3_erase_only_rank_one_projection():
    """w = 0, no decay, unit key e_j, b = e_j: (I - e_j e_j^T) S removes exactly row j;
    with b = 0 nothing is erased (the read side carries the gate)."""
    S0 = np.arange(12, dtype=float).reshape(4, 3) + 1
    for j in range(4):
        k = np.zeros(4)
        k[j] = 1.0
        _, S = _p3_run(S0, 0.0, k, [5.0, 6.0, 7.0], k, np.zeros(3))
        want = S0.copy()
        want[j] = 0
        np.testing.assert_array_equal(S[0, 0], want)
        _, S = _p3_run(S0, 0.0, k, [5.0, 6.0, 7.0], np.zeros(4), np.zeros(3))
        np.testing.assert_array_equal(S[0, 0], S0)


def test_p3_printed_update_matrix_form():
    """Several tokens with channel-wise b != w and d_k != d_v against the update as the
    gist.science page prints it, applied as whole matrices (I - k (b.k)^T) Diag(a) S + k (w.v)^T,
    with the read o_t = S_t^T q_t after the update."""
    rng = np.random.default_rng(33)
    dk, dv, T = 5, 3, 7
    S = rng.standard_normal((dk, dv))
    S0 = S.copy()
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    la = -rng.uniform(0, 0.6, (T, dk))
    b = rng.uniform(0, 1, (T, dk))
    w = rng.uniform(0, 1, (T, dv))
    o_want = []
    for t in range(T):
        S = (np.eye(dk) - np.outer(k[t], b[t] * k[t])) @ np.diag(np.exp(la[t])) @ S + np.outer(k[t], w[t] * v[t])
        o_want.append(S.T @ q[t])
    o, Sg = oracle.gdn2_fwd(q.reshape(T, 1, dk), k.reshape(T, 1, dk), v.reshape(T, 1, dv), la.reshape(T, 1, dk),
                            b.reshape(T, 1, dk), w.reshape(T, 1, dv), S0=S0.reshape(1, 1, dk, dv),
                            flags=oracle.GATE_FORM_P3)
    np.testing.assert_allclose(Sg[0, 0], S, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o[:, 0], np.array(o_want), rtol=1e-12, atol=1e-13)


def test_p3_form_differs_when_gates_are_channelwise():
    """With channel-wise b != w the two gate placements are different models."""
    rng = np.random.default_rng(13)
    dk = dv = 4
    T = 8
    args = [rng.standard_normal((T, 1, dk)) for _ in range(3)]
    la = -rng.uniform(0, 0.3, (T, 1, dk))
    b = rng.uniform(0, 1, (T, 1, dk))
    w = rng.uniform(0, 1, (T, 1, dk))
    o1, S1 = oracle.gdn2_fwd(*args, la, b, w)
    o2, S2 = oracle.gdn2_fwd(*args, la, b, w, flags=oracle.GATE_FORM_P3)
    assert np.max(np.abs(S1 - S2)) > 1e-3


# --------------------------------------------------------------------------
# Chunkwise form == recurrence (brute force on tiny inputs)
# --------------------------------------------------------------------------

def _rand_problem(rng, T, H, dk, dv, strong=False, N=1):
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    la = -rng.uniform(0, 2.0 if strong else 0.2, (T, H, dk))
    b = rng.uniform(0, 1, (T, H, dk))
    w = rng.uniform(0, 1, (T, H, dk))
    S0 = 0.5 * rng.standard_normal((N, H, dk, dv))
    return q, k, v, la, b, w, S0


@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
@pytest.mark.parametrize("strong", [False, True])
def test_chunked_equals_recurrence(chunk, strong):
    rng = np.random.default_rng(100 + chunk)
    T = 77
    q, k, v, la, b, w, S0 = _rand_problem(rng, T, 2, 8, 6, strong)
    o_r, S_r = oracle.gdn2_fwd(q, k, v, la, b, w, S0=S0)
    o_c, S_c = gdn2_chunked_fwd(q, k, v, la, b, w, S0=S0, chunk=chunk)
    scale = max(1.0, np.abs(o_r).max())
    assert np.abs(o_c - o_r).max() <= 1e-12 * scale
    assert np.abs(S_c - S_r).max() <= 1e-12 * max(1.0, np.abs(S_r).max())


# --------------------------------------------------------------------------
# Structure
# --------------------------------------------------------------------------

def test_column_independence():
    rng = np.random.default_rng(21)
    q, k, v, la, b, w, S0 = _rand_problem(rng, 40, 2, 8, 6)
    o, S = oracle.gdn2_fwd(q, k, v, la, b, w, S0=S0)
    o1, S1 = oracle.gdn2_fwd(q, k, v[..., :2], la, b, w, S0=S0[..., :2])
    o2, S2 = oracle.gdn2_fwd(q, k, v[..., 2:], la, b, w, S0=S0[..., 2:])
    np.testing.assert_array_equal(np.concatenate([o1, o2], -1), o)
    np.testing.assert_array_equal(np.concatenate([S1, S2], -1), S)


def test_split_resume():
    rng = np.random.default_rng(22)
    q, k, v, la, b, w, S0 = _rand_problem(rng, 50, 2, 8, 6)
    o, S = oracle.gdn2_fwd(q, k, v, la, b, w, S0=S0)
    cut = 23
    oa, Sa = oracle.gdn2_fwd(*(t[:cut] for t in (q, k, v, la, b, w)), S0=S0)
    ob, Sb = oracle.gdn2_fwd(*(t[cut:] for t in (q, k, v, la, b, w)), S0=Sa)
    np.testing.assert_array_equal(np.concatenate([oa, ob]), o)
    np.testing.assert_array_equal(Sb, S)


def test_varlen_equals_per_sequence():
    rng = np.random.default_rng(23)
    lens = [5, 0, 17, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, la, b, w, S0 = _rand_problem(rng, int(cu[-1]), 3, 4, 5, N=len(lens))
    o, S = oracle.gdn2_fwd(q, k, v, la, b, w, S0=S0, cu_seqlens=cu)
    for n in range(len(lens)):
        sl = slice(cu[n], cu[n + 1])
        on, Sn = oracle.gdn2_fwd(*(t[sl] for t in (q, k, v, la, b, w)), S0=S0[n:n + 1])
        np.testing.assert_array_equal(o[sl], on)
        np.testing.assert_array_equal(S[n], Sn[0])
    # a zero-length sequence returns its initial state
    np.testing.assert_array_equal(S[1], S0[1])


def test_linearity_in_v_and_S0():
    rng = np.random.default_rng(24)
    q, k, v, la, b, w, S0 = _rand_problem(rng, 30, 1, 6, 4)
    v2 = rng.standard_normal(v.shape)
    S02 = rng.standard_normal(S0.shape)
    o1, S1 = oracle.gdn2_fwd(q, k, v, la, b, w, S0=S0)
    o2, S2 = oracle.gdn2_fwd(q, k, v2, la, b, w, S0=S02)
    o3, S3 = oracle.gdn2_fwd(q, k, 2 * v - 3 * v2, la, b, w, S0=2 * S0 - 3 * S02)
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, atol=1e-11)
    np.testing.assert_allclose(S3, 2 * S1 - 3 * S2, atol=1e-11)


def test_zero_key_is_pure_decay():
    rng = np.random.default_rng(25)
    q, k, v, la, b, w, S0 = _rand_problem(rng, 20, 1, 5, 4)
    o, S = oracle.gdn2_fwd(q, np.zeros_like(k), v, la, b, w, S0=S0)
    L = np.cumsum(la[:, 0], axis=0)
    np.testing.assert_allclose(S[0, 0], np.exp(L[-1])[:, None] * S0[0, 0], rtol=1e-13)
    for t in range(20):
        np.testing.assert_allclose(o[t, 0], (np.exp(L[t])[:, None] * S0[0, 0]).T @ q[t, 0],
                                   rtol=1e-12, atol=1e-14)


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(26)
    q, k, v, la, b, w, S0 = _rand_problem(rng, 33, 4, 8, 8)
    o1, S1 = oracle.gdn2_fwd(q, k, v, la, b, w, S0=S0, n_threads=1)
    o2, S2 = oracle.gdn2_fwd(q, k, v, la, b, w, S0=S0, n_threads=4)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)


def test_decode_step_is_one_token_of_the_recurrence():
    rng = np.random.default_rng(27)
    N, H, dk, dv = 3, 2, 4, 5
    q, k, v, la, b, w, _ = _rand_problem(rng, N, H, dk, dv)
    S = rng.standard_normal((N, H, dk, dv))
    o, Sn = oracle.gdn2_decode_step(q, k, v, la, b, w, S)
    for n in range(N):
        on, Snn = oracle.gdn2_fwd(q[n:n + 1], k[n:n + 1], v[n:n + 1], la[n:n + 1], b[n:n + 1],
                                  w[n:n + 1], S0=S[n:n + 1])
        np.testing.assert_array_equal(o[n], on[0])
        np.testing.assert_array_equal(Sn[n], Snn[0])


def test_rejects_bad_arguments():
    rng = np.random.default_rng(28)
    q, k, v, la, b, w, S0 = _rand_problem(rng, 10, 1, 4, 4)
    with pytest.raises(ValueError):
        oracle.gdn2_fwd(q, k, v, la, b, w, cu_seqlens=[0, 6, 4, 10])
    with pytest.raises(ValueError):
        oracle.gdn2_fwd(q, k, v, la, b, None)
