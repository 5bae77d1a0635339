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

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
