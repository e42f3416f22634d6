/*
 * Attention forward + JVP oracle: plain, slow, fp64, on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the parity reference for the CUDA
 * path.  Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may load it.  The CUDA library never includes, links or calls it, and it
 * shares no code, header or constant with the CUDA sources.
 *
 * What it computes (the plain definition, two passes, no online softmax, no
 * blocking):  the FlashAttention-2 JVP kernel of rCM ("Large Scale Diffusion
 * Distillation via Score-Regularized Continuous-Time Consistency", ai.info AI
 * summary, Key Contributions 1 and Methodology in Plain English; papernotes.org
 * notes, 关键设计 1) returns, for one attention call, the forward output and its
 * exact Jacobian-vector product along the tangents (Q', K', V').  Per (b, h)
 * and query row i, over the valid keys j < n_b:
 *
 *   S_ij   = s * <q_i, k_j>
 *   P_ij   = exp(S_ij - m_i) / l_i,   m_i = max_j S_ij,  l_i = sum_j exp(S_ij - m_i)
 *   lse_i  = m_i + ln l_i
 *   O_i    = sum_j P_ij v_j
 *   S'_ij  = s * (<q'_i, k_j> + <q_i, k'_j>)
 *   mu_i   = sum_j P_ij S'_ij
 *   O'_i   = sum_j P_ij (S'_ij - mu_i) v_j + sum_j P_ij v'_j
 *
 * (P' = P (S' - mu) is the derivative of the row softmax; O' = P' V + P V'.)
 * mu_i is also the tangent of lse_i (d lse = sum_j P_ij dS_ij) and is
 * returned as lse' when asked for.
 *
 * Readings where the pages say nothing:
 *   - n_b = min(Lk, kv_len[b]) clamped at 0; kv_len == NULL means n_b = Lk.
 *     Keys j >= n_b take no part: their k, k', v, v' are never read.
 *   - n_b == 0: O = O' = 0, lse = -inf and lse' = 0 (a constant has no
 *     tangent).
 *   - lse is the natural logarithm, in units of the scaled logits.
 *   - Inputs are either bf16 bit patterns (widened exactly to fp64) or fp64.
 *
 * Layout: q, q', o, o' are [B, H, Lq, d]; k, k', v, v' are [B, H, Lk, d];
 * lse and lse' are [B, H, Lq]; all dense row-major.  With a row subset, output r holds
 * flat query row rows[r] (row = (b*H + h)*Lq + i).
 *
 * Built with -O2 -ffp-contract=off and no fast-math, so every sum is the
 * sequential IEEE fp64 sum in index order.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_IN_BF16 0
#define ORACLE_IN_F64 1

static double bf16_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Copy one length-d row of an input tensor into fp64. */
static void widen_row(const void *base, int dtype, size_t off, int d, double *dst)
{
    if (dtype == ORACLE_IN_BF16) {
        const uint16_t *p = (const uint16_t *)base + off;
        for (int c = 0; c < d; ++c) dst[c] = bf16_to_f64(p[c]);
    } else {
        const double *p = (const double *)base + off;
        for (int c = 0; c < d; ++c) dst[c] = p[c];
    }
}

static double dot(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += a[c] * b[c];
    return s;
}

/* One query row: the definition above, written out. */
static void one_row(int dtype, const void *q, const void *k, const void *v,
                    const void *qd, const void *kd, const void *vd,
                    int H, int Lq, int Lk, int d, double scale, const int32_t *kv_len,
                    int64_t row, double *o, double *od, double *lse, double *lse_dot,
                    double *S, double *P, double *Sd, double *qi, double *qdi,
                    double *kj, double *kdj, double *vj, double *vdj)
{
    int64_t bh = row / Lq;
    int64_t i = row % Lq;
    int64_t b = bh / H;
    int n = Lk;
    if (kv_len) {
        n = kv_len[b];
        if (n < 0) n = 0;
        if (n > Lk) n = Lk;
    }
    if (n == 0) {
        for (int c = 0; c < d; ++c) { o[c] = 0.0; od[c] = 0.0; }
        *lse = -INFINITY;
        if (lse_dot) *lse_dot = 0.0;
        return;
    }
    size_t qoff = (size_t)(bh * Lq + i) * (size_t)d;
    size_t kbase = (size_t)bh * (size_t)Lk * (size_t)d;
    widen_row(q, dtype, qoff, d, qi);
    widen_row(qd, dtype, qoff, d, qdi);

    /* logits and their tangent */
    for (int j = 0; j < n; ++j) {
        widen_row(k, dtype, kbase + (size_t)j * d, d, kj);
        widen_row(kd, dtype, kbase + (size_t)j * d, d, kdj);
        S[j] = scale * dot(qi, kj, d);
        Sd[j] = scale * (dot(qdi, kj, d) + dot(qi, kdj, d));
    }

    /* softmax over the valid keys */
    double m = S[0];
    for (int j = 1; j < n; ++j) if (S[j] > m) m = S[j];
    double l = 0.0;
    for (int j = 0; j < n; ++j) { P[j] = exp(S[j] - m); l += P[j]; }
    for (int j = 0; j < n; ++j) P[j] = P[j] / l;
    *lse = m + log(l);

    /* mu = sum_j P_j S'_j */
    double mu = 0.0;
    for (int j = 0; j < n; ++j) mu += P[j] * Sd[j];
    if (lse_dot) *lse_dot = mu;

    /* O = P V ;  O' = sum_j P_j (S'_j - mu) v_j + sum_j P_j v'_j */
    for (int c = 0; c < d; ++c) { o[c] = 0.0; od[c] = 0.0; }
    for (int j = 0; j < n; ++j) {
        widen_row(v, dtype, kbase + (size_t)j * d, d, vj);
        for (int c = 0; c < d; ++c) o[c] += P[j] * vj[c];
    }
    double *tv = qi; /* reuse: accumulates sum_j P_j (S'_j - mu) v_j */
    double *tvd = qdi; /* reuse: accumulates sum_j P_j v'_j */
    for (int c = 0; c < d; ++c) { tv[c] = 0.0; tvd[c] = 0.0; }
    for (int j = 0; j < n; ++j) {
        widen_row(v, dtype, kbase + (size_t)j * d, d, vj);
        widen_row(vd, dtype, kbase + (size_t)j * d, d, vdj);
        double w = P[j] * (Sd[j] - mu);
        for (int c = 0; c < d; ++c) {
            tv[c] += w * vj[c];
            tvd[c] += P[j] * vdj[c];
        }
    }
    for (int c = 0; c < d; ++c) od[c] = tv[c] + tvd[c];
}

/*
 * Returns 0 on success, -1 on a bad argument, -2 if scratch could not be
 * allocated.  lse_dot may be NULL (not computed).  n_threads <= 0 lets OpenMP
 * choose.
 */
int oracle_attn_jvp(int dtype, const void *q, const void *k, const void *v,
                    const void *qd, const void *kd, const void *vd,
                    int B, int H, int Lq, int Lk, int d, double scale,
                    const int32_t *kv_len, const int64_t *rows, int64_t n_rows,
                    double *o, double *od, double *lse, double *lse_dot, int n_threads)
{
    if (!q || !k || !v || !qd || !kd || !vd || !o || !od || !lse) return -1;
    if (B < 1 || H < 1 || Lq < 1 || Lk < 1 || d < 1) return -1;
    if (dtype != ORACLE_IN_BF16 && dtype != ORACLE_IN_F64) return -1;
    int64_t total = (int64_t)B * H * Lq;
    int64_t n_out = rows ? n_rows : total;
    if (rows) {
        for (int64_t r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= total) return -1;
    }
    int nt = 1;
#ifdef _OPENMP
    nt = n_threads > 0 ? n_threads : omp_get_max_threads();
#endif
    /* per-thread scratch: S, P, S' (Lk each) and six rows of length d */
    size_t per = 3 * (size_t)Lk + 6 * (size_t)d;
    double *scratch = malloc(sizeof(double) * per * (size_t)nt);
    if (!scratch) return -2;
#ifdef _OPENMP
#pragma omp parallel for num_threads(nt) schedule(dynamic, 4)
#endif
    for (int64_t r = 0; r < n_out; ++r) {
        int t = 0;
#ifdef _OPENMP
        t = omp_get_thread_num();
#endif
        double *S = scratch + per * (size_t)t;
        double *P = S + Lk;
        double *Sd = P + Lk;
        double *rb = Sd + Lk;
        int64_t row = rows ? rows[r] : r;
        one_row(dtype, q, k, v, qd, kd, vd, H, Lq, Lk, d, scale, kv_len, row,
                o + (size_t)r * d, od + (size_t)r * d, lse + r, lse_dot ? lse_dot + r : NULL, S, P, Sd,
                rb, rb + d, rb + 2 * d, rb + 3 * d, rb + 4 * d, rb + 5 * d);
    }
    free(scratch);
    return 0;
}

/* Number of threads the OpenMP runtime would use by default. */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
