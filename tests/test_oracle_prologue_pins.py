"""Pins for the float64 prologue (CPU only): library routines and closed forms."""
import numpy as np
import scipy.special

from oracle import prologue


def test_sigmoid_and_log_sigmoid_match_scipy():
    x = np.concatenate([np.linspace(-40, 40, 801), [0.0, -1e-3, 1e-3, 700.0, -700.0]])
    np.testing.assert_allclose(prologue.sigmoid(x), scipy.special.expit(x), rtol=1e-15, atol=0)
    np.testing.assert_allclose(prologue.log_sigmoid(x), scipy.special.log_expit(x), rtol=1e-14, atol=1e-300)


def test_closed_forms():
    assert prologue.sigmoid(0.0) == 0.5
    np.testing.assert_allclose(prologue.log_sigmoid(0.0), -np.log(2.0), rtol=1e-16)
    np.testing.assert_allclose(prologue.sigmoid(np.log(3.0)), 0.75, rtol=1e-15)
    np.testing.assert_allclose(prologue.log_sigmoid(-50.0), -50.0 - np.exp(-50.0), rtol=1e-15)


def test_l2norm():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 3, 16)) * 4
    y = prologue.l2norm(x)
    n2 = (x * x).sum(-1, keepdims=True)
    np.testing.assert_allclose((y * y).sum(-1), (n2 / (n2 + prologue.EPS))[..., 0], rtol=1e-14)
    np.testing.assert_allclose(y, x / np.linalg.norm(x, axis=-1, keepdims=True), rtol=1e-7)
    np.testing.assert_array_equal(prologue.l2norm(np.zeros(4)), np.zeros(4))
    np.testing.assert_allclose(prologue.l2norm(np.array([3.0, 4.0])), [3 / np.sqrt(25 + 1e-6), 4 / np.sqrt(25 + 1e-6)],
                               rtol=1e-16)


def test_vjp_matches_finite_differences_through_the_recurrence():
    """Gradients of <dO, o> + <dS_T, S_T> with respect to the pre-activations, from
    the oracle backward composed with prologue.vjp, against central differences of
    the composed forward (prologue then recurrence)."""
    import oracle
    rng = np.random.default_rng(4)
    T, H, dk, dv = 6, 1, 3, 2
    raw = dict(q=rng.standard_normal((T, H, dk)), k=rng.standard_normal((T, H, dk)),
               a=rng.standard_normal((T, H, dk)) + 2.0, b=rng.standard_normal((T, H, dk)),
               w=rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    S0 = rng.standard_normal((1, H, dk, dv)) * 0.5
    dO = rng.standard_normal((T, H, dv))
    dS_T = rng.standard_normal((1, H, dk, dv))

    def loss(r):
        q, k, la, b, w = prologue.apply(r["q"], r["k"], r["a"], r["b"], r["w"])
        o, S_T = oracle.gdn2_fwd(q, k, v, la, b, w, S0=S0)
        return float((o * dO).sum() + (S_T * dS_T).sum())

    q, k, la, b, w = prologue.apply(raw["q"], raw["k"], raw["a"], raw["b"], raw["w"])
    g = oracle.gdn2_bwd(q, k, v, la, b, w, dO, S0=S0, dS_T=dS_T)
    gr = prologue.vjp(raw["q"], raw["k"], raw["a"], raw["b"], raw["w"], g["dq"], g["dk"], g["dlog_a"], g["db"],
                      g["dw"])
    names = dict(q="dq", k="dk", a="dlog_a", b="db", w="dw")
    h = 1e-6
    for name, gname in names.items():
        for idx in np.ndindex(*raw[name].shape):
            rp = {n: x.copy() for n, x in raw.items()}
            rm = {n: x.copy() for n, x in raw.items()}
            rp[name][idx] += h
            rm[name][idx] -= h
            fd = (loss(rp) - loss(rm)) / (2 * h)
            assert abs(fd - gr[gname][idx]) <= 2e-7 * max(1.0, abs(fd)), (name, idx, fd, gr[gname][idx])
