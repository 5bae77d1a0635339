"""Float64 token-mixer prologue: the activations that turn pre-activations into
the recurrence inputs.  TEST INFRASTRUCTURE ONLY (same rule as the package).

The pages say the mixer builds q, k, v and the gates from the residual stream
with normalisation (neelmishra.github.io, "What makes the architecture more
than a recurrence"), that gates are commonly parameterised with sigmoid-like
functions (same page, "Read the limiting cases"), and that the gate domains are
alpha in (0, 1) (same page, "Decay first, then compute the write error") and
b, w in [0, 1] (gist.science, Methodologie 1).  The plainest reading, used here:

    q = q_raw / sqrt(|q_raw|^2 + eps),   k = k_raw / sqrt(|k_raw|^2 + eps)   (over d_k)
    a = sigmoid(x_a)  ->  log_a = log sigmoid(x_a)
    b = sigmoid(x_b),   w = sigmoid(x_w)

with eps = 1e-6.  v passes through unchanged.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def l2norm(x, eps: float = EPS):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps)


def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def log_sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def apply(q_raw, k_raw, a_raw, b_raw, w_raw):
    """(q, k, log_a, b, w) from the pre-activations; w_raw may be None (tied gates)."""
    return (l2norm(q_raw), l2norm(k_raw), log_sigmoid(a_raw), sigmoid(b_raw),
            None if w_raw is None else sigmoid(w_raw))


def vjp(q_raw, k_raw, a_raw, b_raw, w_raw, dq, dk, dlog_a, db, dw):
    """Gradients with respect to the pre-activations, given those with respect to
    the activated inputs.  For y = x / s with s = sqrt(|x|^2 + eps):
    dx = (dy - y (y . dy)) / s;  d/dx log sigmoid(x) = 1 - sigmoid(x);
    d/dx sigmoid(x) = sigmoid(x) (1 - sigmoid(x))."""
    def norm_vjp(x, dy):
        x = np.asarray(x, dtype=np.float64)
        s = np.sqrt((x * x).sum(axis=-1, keepdims=True) + EPS)
        y = x / s
        return (dy - y * (y * dy).sum(axis=-1, keepdims=True)) / s

    sb = sigmoid(b_raw)
    out = dict(dq=norm_vjp(q_raw, dq), dk=norm_vjp(k_raw, dk), dlog_a=dlog_a * (1.0 - sigmoid(a_raw)),
               db=db * sb * (1.0 - sb), dw=None)
    if w_raw is not None and dw is not None:
        sw = sigmoid(w_raw)
        out["dw"] = dw * sw * (1.0 - sw)
    return out
