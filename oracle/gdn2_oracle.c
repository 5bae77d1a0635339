/*
 * gdn2_oracle.c -- float64 CPU oracle for the Gated DeltaNet-2 recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The GPU
 * product path never calls it, and it shares no code with the CUDA sources.
 *
 * What it computes (the plain sequential recurrence, one token at a time):
 *
 *   Gated DeltaNet-2 (gist.science, "Gated DeltaNet-2: Decoupling Erase and
 *   Write in Linear Attention", Methodologie 1 "Gated Delta-regel-2"; alanhou.org,
 *   "Core Mechanism" and "Key Concepts / Erase-Write Decoupling"), in the
 *   key-by-value state orientation of neelmishra.github.io, "Gated DeltaNet",
 *   section "Decay first, then compute the write error".  Per head the state
 *   S is d_k x d_v.  For every token t, in this order:
 *
 *     1. decay        Sbar = Diag(a_t) S,        a_t = exp(log_a_t)
 *                     (the channel-wise decay D_t = Diag(alpha_t) inherited
 *                      from Kimi Delta Attention)
 *     2. erase read   r    = Sbar^T k_t          (read of the DECAYED state:
 *                      neelmishra.github.io says the subtraction must use the
 *                      decayed state; spawnkit session 16 "Stability" fixes the
 *                      order decay, read, correct)
 *     3. erase        S'   = Sbar - (b_t . k_t) r^T        (erase gate b_t)
 *     4. write        S    = S'   + (w_t . k_t) v_t^T      (write gate w_t)
 *     5. read         o_t  = S^T q_t             (read AFTER the update, as the
 *                      spawnkit worked trace reads q=[1,0] off the updated S_1)
 *
 *   With GATE_FORM_P3 set, steps 2-4 follow the equation printed on the
 *   gist.science page instead:  S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1}
 *   + k_t (w_t . v_t)^T, i.e. the erase read uses (b . k), the erase outer
 *   factor is k, and the write gate w_t (length d_v) multiplies the value.
 *
 * Layouts (all row-major, float64):
 *   q, k        [T_tot][H][d_k]          v   [T_tot][H][d_v]
 *   log_a       [T_tot][H][d_k]  or [T_tot][H] with OR_SCALAR_DECAY
 *   b           [T_tot][H][d_k]  or [T_tot][H] with OR_SCALAR_GATES
 *   w           [T_tot][H][d_k]  ([T_tot][H][d_v] in the P3 form),
 *               or [T_tot][H] with OR_SCALAR_GATES; ignored with OR_TIED_GATES
 *               (then w = b)
 *   S0, S_T     [N][H][d_k][d_v]; S0 may be NULL (zero initial state)
 *   o           [T_tot][H][d_v]
 *   cu_seqlens  [N+1] token offsets of the N packed sequences
 *
 * Parallel only across independent (sequence, head) units; inside a unit the
 * tokens run strictly in order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum {
    OR_SCALAR_DECAY = 1,
    OR_SCALAR_GATES = 2,
    OR_TIED_GATES = 4,
    OR_GATE_FORM_P3 = 8,
};

/* One (sequence, head) unit.  Vectors of token t sit at base + t * tok_stride. */
static void unit_fwd(int64_t T, int64_t dk, int64_t dv, int64_t flags,
                     const double *q, const double *k, const double *v,
                     const double *log_a, const double *b, const double *w,
                     int64_t tok_stride_k, int64_t tok_stride_v, int64_t tok_stride_s,
                     const double *S0, double *o, double *S,
                     double *a, double *r, double *x, double *p)
{
    const int scalar_decay = (flags & OR_SCALAR_DECAY) != 0;
    const int scalar_gates = (flags & OR_SCALAR_GATES) != 0;
    const int tied = (flags & OR_TIED_GATES) != 0;
    const int p3 = (flags & OR_GATE_FORM_P3) != 0;
    const int64_t w_stride = scalar_gates ? tok_stride_s : (p3 ? tok_stride_v : tok_stride_k);

    if (S0) memcpy(S, S0, sizeof(double) * dk * dv);
    else memset(S, 0, sizeof(double) * dk * dv);

    for (int64_t t = 0; t < T; ++t) {
        const double *qt = q + t * tok_stride_k;
        const double *kt = k + t * tok_stride_k;
        const double *vt = v + t * tok_stride_v;
        const double *gt = log_a + t * (scalar_decay ? tok_stride_s : tok_stride_k);
        const double *bt = b + t * (scalar_gates ? tok_stride_s : tok_stride_k);
        const double *wt = tied ? bt : (w + t * w_stride);
        double *ot = o + t * tok_stride_v;

        /* 1. decay: Sbar = Diag(exp(log_a_t)) S */
        for (int64_t i = 0; i < dk; ++i) a[i] = exp(scalar_decay ? gt[0] : gt[i]);
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= a[i];

        if (!p3) {
            /* 2. erase read r = Sbar^T k_t */
            for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * kt[i];
            /* 3. erase: S' = Sbar - (b_t . k_t) r^T */
            for (int64_t i = 0; i < dk; ++i) x[i] = (scalar_gates ? bt[0] : bt[i]) * kt[i];
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) S[i * dv + j] -= x[i] * r[j];
            /* 4. write: S = S' + (w_t . k_t) v_t^T */
            for (int64_t i = 0; i < dk; ++i) p[i] = (scalar_gates ? wt[0] : wt[i]) * kt[i];
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) S[i * dv + j] += p[i] * vt[j];
        } else {
            /* gist.science form: erase read with (b_t . k_t), erase along k_t */
            for (int64_t i = 0; i < dk; ++i) x[i] = (scalar_gates ? bt[0] : bt[i]) * kt[i];
            for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) r[j] += S[i * dv + j] * x[i];
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) S[i * dv + j] -= kt[i] * r[j];
            /* write k_t (w_t . v_t)^T, w_t of length d_v (or the tied / scalar gate) */
            /* (tied gates in this form need d_k == d_v, checked by the caller) */
            for (int64_t j = 0; j < dv; ++j) p[j] = (scalar_gates ? wt[0] : wt[j]) * vt[j];
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * p[j];
        }

        /* 5. read after the update: o_t = S^T q_t */
        for (int64_t j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * qt[i];
    }
}

/*
 * Full forward over N packed sequences and H heads.  Returns 0, or -1 on a bad
 * argument.  n_threads <= 0 leaves the OpenMP default.
 */
int oracle_gdn2_fwd(int64_t n_seqs, int64_t n_heads, int64_t dk, int64_t dv, int64_t flags,
                    const int64_t *cu_seqlens,
                    const double *q, const double *k, const double *v,
                    const double *log_a, const double *b, const double *w,
                    const double *S0, double *o, double *S_T, int64_t n_threads)
{
    if (n_seqs < 0 || n_heads <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens || !S_T) return -1;
    if ((flags & OR_GATE_FORM_P3) && (flags & OR_TIED_GATES) && !(flags & OR_SCALAR_GATES) && dk != dv)
        return -1;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    const int64_t n_units = n_seqs * n_heads;
    const int64_t scratch_len = (dk > dv ? dk : dv);
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads((int)n_threads);
#else
    (void)n_threads;
#endif
    int status = 0;
#pragma omp parallel
    {
        double *buf = (double *)malloc(sizeof(double) * (4 * scratch_len + dk * dv));
        if (!buf) {
#pragma omp atomic write
            status = -1;
        } else {
            double *a = buf, *r = buf + scratch_len, *x = buf + 2 * scratch_len, *p = buf + 3 * scratch_len;
            double *S = buf + 4 * scratch_len;
#pragma omp for schedule(dynamic, 1)
            for (int64_t u = 0; u < n_units; ++u) {
                const int64_t n = u / n_heads, h = u % n_heads;
                const int64_t bos = cu_seqlens[n], T = cu_seqlens[n + 1] - cu_seqlens[n];
                const int64_t sk = n_heads * dk, sv = n_heads * dv, ss = n_heads;
                const int p3 = (flags & OR_GATE_FORM_P3) != 0;
                const int64_t w_head = (flags & OR_SCALAR_GATES) ? 1 : (p3 ? dv : dk);
                const int64_t g_head = (flags & OR_SCALAR_DECAY) ? 1 : dk;
                const int64_t b_head = (flags & OR_SCALAR_GATES) ? 1 : dk;
                const double *wb = w ? w + bos * n_heads * w_head + h * w_head : NULL;
                unit_fwd(T, dk, dv, flags,
                         q + bos * sk + h * dk, k + bos * sk + h * dk, v + bos * sv + h * dv,
                         log_a + bos * n_heads * g_head + h * g_head,
                         b + bos * n_heads * b_head + h * b_head, wb,
                         sk, sv, ss,
                         S0 ? S0 + u * dk * dv : NULL,
                         o + bos * sv + h * dv, S, a, r, x, p);
                memcpy(S_T + u * dk * dv, S, sizeof(double) * dk * dv);
            }
            free(buf);
        }
    }
    return status;
}

/*
 * Backward (reverse mode) of the same recurrence.  The pages name a gate-aware
 * backward of the chunked form as part of the method (gist.science,
 * Methodologie 3: the per-channel gates b and w are folded into the gradient
 * accumulation of the auxiliary matrices; alanhou.org, "Core Mechanism": the
 * chunkwise algorithm is what training runs) but print no formula for it; the
 * gradient of a function is fixed by the function, so this is the plain
 * reverse-mode differentiation of steps 1-5 above, token by token in reverse.
 *
 * Write each token in the general form (erase read vector y, erase outer
 * factor x, write outer factor p, written value z):
 *     Sbar = Diag(a) S_prev,  r = Sbar^T y,  S = Sbar - x r^T + p z^T,  o = S^T q
 * with (y, x, p, z) = (k, b.k, w.k, v) by default and (b.k, k, k, w.v) in the
 * gist.science form.  Given the gradient G of the loss with respect to S_t
 * (starting from dS_T) and do_t:
 *     G  += q do^T                  dq = S do
 *     dp  = G z      dz = G^T p     dx = -G r      dr = -G^T x
 *     Gbar = G + y dr^T             dy = Sbar dr
 *     dlog_a_i = sum_j Gbar_ij Sbar_ij          (d/dlog_a of a_i S_prev_ij)
 *     G  <- Diag(a) Gbar            (the gradient with respect to S_prev)
 * and dS0 is the last G.  The chain rule through (y, x, p, z) gives
 *     default: dk = dy + b.dx + w.dp,  db = k.dx,  dw = k.dp,  dv = dz
 *     P3:      dk = b.dy + dx + dp,    db = k.dy,  dw = v.dz,  dv = w.dz
 * summed over channels for the scalar flags, and db += dw with tied gates.
 *
 * States are kept at every 64th token and each 64-token segment is recomputed
 * forward before it is walked backward, so the memory is O(64 d_k d_v) per
 * unit.  Output layouts equal the input layouts (dw has w's layout, and with
 * OR_TIED_GATES the w gradient is added into db and dw is not written).
 */
enum { OR_SEG = 64 };

static void token_vectors(int64_t dk, int64_t dv, int64_t flags, const double *kt, const double *vt,
                          const double *gt, const double *bt, const double *wt,
                          double *a, double *y, double *x, double *p, double *z)
{
    const int scalar_decay = (flags & OR_SCALAR_DECAY) != 0;
    const int scalar_gates = (flags & OR_SCALAR_GATES) != 0;
    const int p3 = (flags & OR_GATE_FORM_P3) != 0;
    for (int64_t i = 0; i < dk; ++i) {
        const double bi = scalar_gates ? bt[0] : bt[i];
        a[i] = exp(scalar_decay ? gt[0] : gt[i]);
        if (p3) {
            y[i] = bi * kt[i];
            x[i] = kt[i];
            p[i] = kt[i];
        } else {
            y[i] = kt[i];
            x[i] = bi * kt[i];
            p[i] = (scalar_gates ? wt[0] : wt[i]) * kt[i];
        }
    }
    for (int64_t j = 0; j < dv; ++j) z[j] = p3 ? (scalar_gates ? wt[0] : wt[j]) * vt[j] : vt[j];
}

/* One forward token from S_prev into S (separate buffers); r receives Sbar^T y. */
static void token_step(int64_t dk, int64_t dv, const double *a, const double *y, const double *x,
                       const double *p, const double *z, const double *S_prev, double *S, double *r)
{
    for (int64_t j = 0; j < dv; ++j) r[j] = 0.0;
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) r[j] += a[i] * S_prev[i * dv + j] * y[i];
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j)
            S[i * dv + j] = a[i] * S_prev[i * dv + j] - x[i] * r[j] + p[i] * z[j];
}

typedef struct {
    const double *q, *k, *v, *g, *b, *w, *dO;
    double *dq, *dk, *dv, *dg, *db, *dw;
    int64_t sk, sv, sg, sb, sw;   /* per-token strides of the k-like, v-like, log_a, b and w arrays */
} unit_io;

static void unit_bwd(int64_t T, int64_t dk, int64_t dv, int64_t flags, const unit_io *u,
                     const double *S0, const double *dS_T, double *dS0, double *ws)
{
    const int scalar_decay = (flags & OR_SCALAR_DECAY) != 0;
    const int scalar_gates = (flags & OR_SCALAR_GATES) != 0;
    const int tied = (flags & OR_TIED_GATES) != 0;
    const int p3 = (flags & OR_GATE_FORM_P3) != 0;
    const int64_t D = dk * dv, m = dk > dv ? dk : dv;
    const int64_t n_seg = (T + OR_SEG - 1) / OR_SEG;
    double *ckpt = ws;                      /* [n_seg][D]: state before each segment */
    double *seg = ckpt + (n_seg > 0 ? n_seg : 1) * D;  /* [OR_SEG + 1][D]: states inside a segment */
    double *rs = seg + (OR_SEG + 1) * D;    /* [OR_SEG][dv]: r of each token */
    double *G = rs + OR_SEG * dv;           /* [D] gradient with respect to the current state */
    double *Gbar = G + D;                   /* [D] */
    double *a = Gbar + D, *y = a + m, *x = y + m, *p = x + m, *z = p + m;
    double *dp = z + m, *dz = dp + m, *dx = dz + m, *dr = dx + m, *dy = dr + m;

    /* forward sweep: checkpoints */
    if (S0) memcpy(seg, S0, sizeof(double) * D);
    else memset(seg, 0, sizeof(double) * D);
    for (int64_t t = 0; t < T; ++t) {
        if (t % OR_SEG == 0) memcpy(ckpt + (t / OR_SEG) * D, seg, sizeof(double) * D);
        token_vectors(dk, dv, flags, u->k + t * u->sk, u->v + t * u->sv, u->g + t * u->sg, u->b + t * u->sb,
                      tied ? u->b + t * u->sb : u->w + t * u->sw, a, y, x, p, z);
        token_step(dk, dv, a, y, x, p, z, seg, seg + D, rs);
        memcpy(seg, seg + D, sizeof(double) * D);
    }

    if (dS_T) memcpy(G, dS_T, sizeof(double) * D);
    else memset(G, 0, sizeof(double) * D);
    for (int64_t sgi = n_seg - 1; sgi >= 0; --sgi) {
        const int64_t t0 = sgi * OR_SEG, t1 = (t0 + OR_SEG < T) ? t0 + OR_SEG : T;
        /* recompute the segment: seg[s] = state before token t0 + s, seg[s + 1] after it */
        memcpy(seg, ckpt + sgi * D, sizeof(double) * D);
        for (int64_t t = t0; t < t1; ++t) {
            token_vectors(dk, dv, flags, u->k + t * u->sk, u->v + t * u->sv, u->g + t * u->sg, u->b + t * u->sb,
                          tied ? u->b + t * u->sb : u->w + t * u->sw, a, y, x, p, z);
            token_step(dk, dv, a, y, x, p, z, seg + (t - t0) * D, seg + (t - t0 + 1) * D, rs + (t - t0) * dv);
        }
        for (int64_t t = t1 - 1; t >= t0; --t) {
            const double *kt = u->k + t * u->sk, *vt = u->v + t * u->sv, *gt = u->g + t * u->sg;
            const double *bt = u->b + t * u->sb, *wt = tied ? bt : u->w + t * u->sw;
            const double *qt = u->q + t * u->sk, *dot = u->dO + t * u->sv;
            const double *S_prev = seg + (t - t0) * D, *S = seg + (t - t0 + 1) * D, *r = rs + (t - t0) * dv;
            token_vectors(dk, dv, flags, kt, vt, gt, bt, wt, a, y, x, p, z);
            double *dqt = u->dq + t * u->sk, *dkt = u->dk + t * u->sk, *dvt = u->dv + t * u->sv;
            double *dgt = u->dg + t * u->sg, *dbt = u->db + t * u->sb;
            double *dwt = tied ? NULL : u->dw + t * u->sw;

            /* read: o = S^T q */
            for (int64_t i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < dv; ++j) acc += S[i * dv + j] * dot[j];
                dqt[i] = acc;
                for (int64_t j = 0; j < dv; ++j) G[i * dv + j] += qt[i] * dot[j];
            }
            /* write and erase: S = Sbar - x r^T + p z^T */
            for (int64_t i = 0; i < dk; ++i) {
                double ap = 0.0, ax = 0.0;
                for (int64_t j = 0; j < dv; ++j) {
                    ap += G[i * dv + j] * z[j];
                    ax -= G[i * dv + j] * r[j];
                }
                dp[i] = ap;
                dx[i] = ax;
            }
            for (int64_t j = 0; j < dv; ++j) {
                double az = 0.0, ar = 0.0;
                for (int64_t i = 0; i < dk; ++i) {
                    az += G[i * dv + j] * p[i];
                    ar -= G[i * dv + j] * x[i];
                }
                dz[j] = az;
                dr[j] = ar;
            }
            /* erase read: r = Sbar^T y */
            for (int64_t i = 0; i < dk; ++i) {
                double ay = 0.0, ag = 0.0;
                for (int64_t j = 0; j < dv; ++j) {
                    const double sbar = a[i] * S_prev[i * dv + j];
                    const double gb = G[i * dv + j] + y[i] * dr[j];
                    Gbar[i * dv + j] = gb;
                    ay += sbar * dr[j];
                    ag += gb * sbar;
                }
                dy[i] = ay;
                /* decay: Sbar = Diag(exp(log_a)) S_prev */
                if (scalar_decay) {
                    if (i == 0) dgt[0] = 0.0;
                    dgt[0] += ag;
                } else {
                    dgt[i] = ag;
                }
            }
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) G[i * dv + j] = a[i] * Gbar[i * dv + j];

            /* chain rule to (k, v, b, w) */
            if (scalar_gates) {
                dbt[0] = 0.0;
                if (dwt) dwt[0] = 0.0;
            }
            double wsum = 0.0;
            for (int64_t i = 0; i < dk; ++i) {
                const double bi = scalar_gates ? bt[0] : bt[i];
                double gb_i, gw_i = 0.0;
                if (p3) {
                    dkt[i] = bi * dy[i] + dx[i] + dp[i];
                    gb_i = kt[i] * dy[i];
                } else {
                    const double wi = scalar_gates ? wt[0] : wt[i];
                    dkt[i] = dy[i] + bi * dx[i] + wi * dp[i];
                    gb_i = kt[i] * dx[i];
                    gw_i = kt[i] * dp[i];
                }
                if (scalar_gates) {
                    dbt[0] += gb_i;
                    wsum += gw_i;
                } else {
                    dbt[i] = gb_i;
                    if (!p3) {
                        if (tied) dbt[i] += gw_i;
                        else dwt[i] = gw_i;
                    }
                }
            }
            for (int64_t j = 0; j < dv; ++j) {
                if (p3) {
                    const double wj = scalar_gates ? wt[0] : wt[j];
                    dvt[j] = wj * dz[j];
                    const double gw_j = vt[j] * dz[j];
                    if (scalar_gates) wsum += gw_j;
                    else if (tied) dbt[j] += gw_j;  /* tied per-channel P3 needs d_k == d_v */
                    else dwt[j] = gw_j;
                } else {
                    dvt[j] = dz[j];
                }
            }
            if (scalar_gates) {
                if (tied) dbt[0] += wsum;
                else dwt[0] = wsum;
            }
        }
    }
    memcpy(dS0, G, sizeof(double) * D);
}

/*
 * Gradients of  sum_t <do_t, o_t> + <dS_T, S_T>  for the forward above.
 * dO [T_tot][H][d_v]; dS_T [N][H][d_k][d_v] or NULL (zero).  Outputs have the
 * layouts of the corresponding inputs; dw may be NULL with OR_TIED_GATES; dS0
 * [N][H][d_k][d_v] is always written.  Returns 0, or -1 on a bad argument or
 * an allocation failure.
 */
int oracle_gdn2_bwd(int64_t n_seqs, int64_t n_heads, int64_t dk, int64_t dv, int64_t flags,
                    const int64_t *cu_seqlens,
                    const double *q, const double *k, const double *v,
                    const double *log_a, const double *b, const double *w,
                    const double *S0, const double *dO, const double *dS_T,
                    double *dq, double *dk_out, double *dv_out, double *dlog_a, double *db, double *dw,
                    double *dS0, int64_t n_threads)
{
    if (n_seqs < 0 || n_heads <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens || !dO || !dS0) return -1;
    if (!(flags & OR_TIED_GATES) && (!w || !dw)) return -1;
    if ((flags & OR_GATE_FORM_P3) && (flags & OR_TIED_GATES) && !(flags & OR_SCALAR_GATES) && dk != dv)
        return -1;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    const int64_t n_units = n_seqs * n_heads;
    const int64_t D = dk * dv, m = dk > dv ? dk : dv;
    int64_t max_T = 0;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] - cu_seqlens[n] > max_T) max_T = cu_seqlens[n + 1] - cu_seqlens[n];
    const int64_t max_seg = (max_T + OR_SEG - 1) / OR_SEG;
    const size_t ws_len = (size_t)((max_seg > 0 ? max_seg : 1) * D + (OR_SEG + 1) * D + OR_SEG * dv + 2 * D + 10 * m);
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads((int)n_threads);
#else
    (void)n_threads;
#endif
    const int p3 = (flags & OR_GATE_FORM_P3) != 0;
    const int64_t g_head = (flags & OR_SCALAR_DECAY) ? 1 : dk;
    const int64_t b_head = (flags & OR_SCALAR_GATES) ? 1 : dk;
    const int64_t w_head = (flags & OR_SCALAR_GATES) ? 1 : (p3 ? dv : dk);
    int status = 0;
#pragma omp parallel
    {
        double *ws = (double *)malloc(sizeof(double) * ws_len);
        if (!ws) {
#pragma omp atomic write
            status = -1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t un = 0; un < n_units; ++un) {
                const int64_t n = un / n_heads, h = un % n_heads;
                const int64_t bos = cu_seqlens[n], T = cu_seqlens[n + 1] - cu_seqlens[n];
                unit_io io;
                io.sk = n_heads * dk;
                io.sv = n_heads * dv;
                io.sg = n_heads * g_head;
                io.sb = n_heads * b_head;
                io.sw = n_heads * w_head;
                io.q = q + bos * io.sk + h * dk;
                io.k = k + bos * io.sk + h * dk;
                io.v = v + bos * io.sv + h * dv;
                io.g = log_a + bos * io.sg + h * g_head;
                io.b = b + bos * io.sb + h * b_head;
                io.w = w ? w + bos * io.sw + h * w_head : NULL;
                io.dO = dO + bos * io.sv + h * dv;
                io.dq = dq + bos * io.sk + h * dk;
                io.dk = dk_out + bos * io.sk + h * dk;
                io.dv = dv_out + bos * io.sv + h * dv;
                io.dg = dlog_a + bos * io.sg + h * g_head;
                io.db = db + bos * io.sb + h * b_head;
                io.dw = dw ? dw + bos * io.sw + h * w_head : NULL;
                unit_bwd(T, dk, dv, flags, &io, S0 ? S0 + un * D : NULL, dS_T ? dS_T + un * D : NULL,
                         dS0 + un * D, ws);
            }
            free(ws);
        }
    }
    return status;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
