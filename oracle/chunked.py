"""Float64 chunkwise (WY) form of the Gated DeltaNet-2 recurrence.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Used to prove that the
chunk algebra the GPU path implements equals the token-by-token recurrence; it
is never the parity reference for the GPU (that is ``oracle.gdn2_fwd``).

The pages describe the chunkwise algorithm only in outline: the cumulative
channel-wise decay is absorbed into asymmetric rank-one erase factors and write
factors (gist.science, Methodologie 3 "Vervalabsorptie"), and a lower-triangular
system (I + T)^-1 yields auxiliary matrices on the erase side and the write
side (same section, "Driehoekig oplossen"); alanhou.org ("Core Mechanism")
names it a WY representation.  Written out for one chunk of rows i = 1..C
starting from state S (d_k x d_v), with x = b.k (erase outer), y = k (erase
read), p = w.k (write outer), z = v, and gamma_i = exp(sum_{j<=i} log_a_j):

    Yh = y * gamma,  Qh = q * gamma,  Xh = x / gamma,  Ph = p / gamma
    A  = strict_lower(Yh Xh^T),  B  = strict_lower(Yh Ph^T)
    QX = lower(Qh Xh^T),         QP = lower(Qh Ph^T)
    M  = (I + A)^-1 (Yh S + B Z)            -- the erase reads r_i of all rows
    O  = Qh S + QP Z - QX M
    S' = Diag(gamma_C) S + (P * gamma_C/gamma)^T Z - (X * gamma_C/gamma)^T M

Row i of M is the erase read r_i = Sbar_i^T k_i of the recurrence; unrolling
S_i = D_i S_{i-1} - x_i r_i^T + p_i z_i^T inside the chunk gives the three
lines above directly.  A library solve stands in for (I + A)^-1.
"""
from __future__ import annotations

import numpy as np


def gdn2_chunked_unit(q, k, v, log_a, b, w, S0, chunk: int):
    """One (sequence, head): q, k, log_a, b, w [T, d_k], v [T, d_v], S0 [d_k, d_v]."""
    q, k, v, log_a, b, w = (np.asarray(t, dtype=np.float64) for t in (q, k, v, log_a, b, w))
    T, dk = k.shape
    dv = v.shape[1]
    S = np.array(S0, dtype=np.float64, copy=True)
    o = np.zeros((T, dv))
    for c0 in range(0, T, chunk):
        sl = slice(c0, min(c0 + chunk, T))
        n = sl.stop - sl.start
        L = np.cumsum(log_a[sl], axis=0)
        gam = np.exp(L)
        gC = gam[-1]
        x = b[sl] * k[sl]
        y = k[sl]
        p = w[sl] * k[sl]
        z = v[sl]
        Yh, Qh, Xh, Ph = y * gam, q[sl] * gam, x / gam, p / gam
        A = np.tril(Yh @ Xh.T, -1)
        B = np.tril(Yh @ Ph.T, -1)
        QX = np.tril(Qh @ Xh.T)
        QP = np.tril(Qh @ Ph.T)
        M = np.linalg.solve(np.eye(n) + A, Yh @ S + B @ z)
        o[sl] = Qh @ S + QP @ z - QX @ M
        S = gC[:, None] * S + (p * (gC / gam)).T @ z - (x * (gC / gam)).T @ M
    return o, S


def gdn2_chunked_fwd(q, k, v, log_a, b, w, S0=None, cu_seqlens=None, chunk: int = 64):
    """Packed layout as ``oracle.gdn2_fwd`` (per-channel gates only)."""
    q = np.asarray(q, dtype=np.float64)
    T_tot, H, dk = q.shape
    dv = np.asarray(v).shape[2]
    cu = np.array([0, T_tot]) if cu_seqlens is None else np.asarray(cu_seqlens)
    N = len(cu) - 1
    o = np.zeros((T_tot, H, dv))
    S_T = np.zeros((N, H, dk, dv))
    for n in range(N):
        a0, a1 = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            s0 = np.zeros((dk, dv)) if S0 is None else np.asarray(S0)[n, h]
            o[a0:a1, h], S_T[n, h] = gdn2_chunked_unit(
                q[a0:a1, h], np.asarray(k)[a0:a1, h], np.asarray(v)[a0:a1, h],
                np.asarray(log_a)[a0:a1, h], np.asarray(b)[a0:a1, h], np.asarray(w)[a0:a1, h],
                s0, chunk)
    return o, S_T
