/*
 * attention_ref.c -- the fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain definition that the
 * CUDA library is checked against.  It shares no code, header or constant with
 * the GPU path, and the product never links or calls it.
 *
 * What it computes (FlashAttention-2 abstract, "FlashAttention-2: Faster
 * Attention with Better Parallelism and Work Partitioning": the method is exact,
 * "with no approximation"; the iplexlaw FlashAttention-2 blog, section "Tiling
 * preserves the attention calculation": the tiled result equals the globally
 * normalised softmax, and output and gradient comparisons use tolerances).
 * Because the method reaches the plain definition exactly, this oracle is that
 * definition written out, not the tiled algorithm:
 *
 *   s_ij   = scale * <q_i, k_j>                 j in J(i)
 *   J(i)   = {0..N-1}, or {0..i} when causal (N_q = N_k = N, mask j > i)
 *   m_i    = max_j s_ij,   Z_i = sum_j exp(s_ij - m_i)
 *   P_ij   = exp(s_ij - m_i) / Z_i
 *   O_i    = sum_j P_ij v_j
 *   LSE_i  = m_i + ln Z_i                       (natural log)
 *
 * and its gradient for an upstream dO (textbook softmax calculus; the pages
 * name gradients and training but print no formula):
 *
 *   dV_j  = sum_{i: j in J(i)} P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 *
 * Layout: every [B,H,N,d] tensor is contiguous, row (b,h,n) at
 * ((b*H + h)*N + n)*d.  LSE and D are [B,H,N].  All arithmetic is double.
 * One row of scores is materialised at a time (N doubles per thread); the
 * N x N matrix is never held.  OpenMP spreads independent rows (forward) or
 * heads (backward) over host cores.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double dot(const double *a, const double *b, int d) {
    double acc = 0.0;
    for (int t = 0; t < d; ++t) acc += a[t] * b[t];
    return acc;
}

/* Number of keys row i attends to: N, or i+1 under the causal mask. */
static int row_extent(int i, int N, int causal) { return causal ? i + 1 : N; }

/*
 * One forward row: fills s[0..n) with scaled scores, turns them into the
 * normalised probabilities P_i. (two passes: max, then sum), writes O_i and
 * returns LSE_i.
 */
static double forward_row(const double *q_i, const double *k, const double *v,
                          int n, int d, double scale, double *p, double *o_i) {
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        p[j] = scale * dot(q_i, k + (size_t)j * d, d);
        if (p[j] > m) m = p[j];
    }
    double z = 0.0;
    for (int j = 0; j < n; ++j) {
        p[j] = exp(p[j] - m);
        z += p[j];
    }
    for (int j = 0; j < n; ++j) p[j] /= z;
    if (o_i) {
        for (int t = 0; t < d; ++t) o_i[t] = 0.0;
        for (int j = 0; j < n; ++j) {
            const double *v_j = v + (size_t)j * d;
            for (int t = 0; t < d; ++t) o_i[t] += p[j] * v_j[t];
        }
    }
    return m + log(z);
}

/*
 * Forward pass over all B*H heads.  q,k,v,o: [B,H,N,d]; lse: [B,H,N].
 * Returns 0, or -1 when a scratch row cannot be allocated.
 */
int ref_fwd(const double *q, const double *k, const double *v, double *o,
            double *lse, int B, int H, int N, int d, int causal, double scale) {
    const long long rows = (long long)B * H * N;
    int failed = 0;
#pragma omp parallel reduction(| : failed)
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        if (!p) failed = 1;
#pragma omp for schedule(dynamic, 16)
        for (long long r = 0; r < rows; ++r) {
            if (!p) continue;
            const long long bh = r / N;
            const int i = (int)(r % N);
            const size_t head = (size_t)bh * N * d;
            lse[r] = forward_row(q + (size_t)r * d, k + head, v + head,
                                 row_extent(i, N, causal), d, scale, p,
                                 o + (size_t)r * d);
        }
        free(p);
    }
    return failed ? -1 : 0;
}

/*
 * Backward pass of one head (pointers already offset to the head), from the
 * definition: P is recomputed row by row, then dV, dP, D, dS, dQ, dK follow the
 * formulas in the file header.  dq, dk, dv are overwritten; D (length N) too.
 */
static int backward_head(const double *q, const double *k, const double *v,
                         const double *dO, double *dq, double *dk, double *dv,
                         double *D, int N, int d, int causal, double scale) {
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    if (!p || !dp) {
        free(p);
        free(dp);
        return -1;
    }
    memset(dk, 0, sizeof(double) * (size_t)N * d);
    memset(dv, 0, sizeof(double) * (size_t)N * d);
    for (int i = 0; i < N; ++i) {
        const int n = row_extent(i, N, causal);
        const double *q_i = q + (size_t)i * d;
        const double *do_i = dO + (size_t)i * d;
        forward_row(q_i, k, v, n, d, scale, p, NULL);
        double Di = 0.0;
        for (int j = 0; j < n; ++j) {
            dp[j] = dot(do_i, v + (size_t)j * d, d);
            Di += p[j] * dp[j];
        }
        D[i] = Di;
        double *dq_i = dq + (size_t)i * d;
        for (int t = 0; t < d; ++t) dq_i[t] = 0.0;
        for (int j = 0; j < n; ++j) {
            const double ds = p[j] * (dp[j] - Di);
            const double *k_j = k + (size_t)j * d;
            double *dk_j = dk + (size_t)j * d;
            double *dv_j = dv + (size_t)j * d;
            for (int t = 0; t < d; ++t) {
                dq_i[t] += ds * k_j[t];
                dk_j[t] += ds * q_i[t];
                dv_j[t] += p[j] * do_i[t];
            }
        }
        for (int t = 0; t < d; ++t) dq_i[t] *= scale;
    }
    for (size_t e = 0; e < (size_t)N * d; ++e) dk[e] *= scale;
    free(p);
    free(dp);
    return 0;
}

/*
 * Backward pass over all heads.  dO, dq, dk, dv: [B,H,N,d]; D: [B,H,N]
 * (may be NULL).  Returns 0, or -1 on allocation failure.
 */
int ref_bwd(const double *q, const double *k, const double *v, const double *dO,
            double *dq, double *dk, double *dv, double *D, int B, int H, int N,
            int d, int causal, double scale) {
    const int heads = B * H;
    double *Dbuf = D;
    if (!Dbuf) {
        Dbuf = (double *)malloc(sizeof(double) * (size_t)heads * N);
        if (!Dbuf) return -1;
    }
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int bh = 0; bh < heads; ++bh) {
        const size_t off = (size_t)bh * N * d;
        if (backward_head(q + off, k + off, v + off, dO + off, dq + off,
                          dk + off, dv + off, Dbuf + (size_t)bh * N, N, d,
                          causal, scale))
            failed = 1;
    }
    if (!D) free(Dbuf);
    return failed ? -1 : 0;
}

/*
 * Forward for selected rows of one head (any N): the same row definition as
 * ref_fwd.  q,k,v point at the head's [N,d] slices; rows[0..nrows) are query
 * indices; o is [nrows,d], lse is [nrows].
 */
int ref_fwd_rows(const double *q, const double *k, const double *v, int N,
                 int d, int causal, double scale, const long long *rows,
                 int nrows, double *o, double *lse) {
    int failed = 0;
#pragma omp parallel reduction(| : failed)
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        if (!p) failed = 1;
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            if (!p) continue;
            const int i = (int)rows[r];
            lse[r] = forward_row(q + (size_t)i * d, k, v,
                                 row_extent(i, N, causal), d, scale, p,
                                 o + (size_t)r * d);
        }
        free(p);
    }
    return failed ? -1 : 0;
}

/*
 * Per-row softmax statistics of one head: LSE_i and D_i = sum_j P_ij dP_ij for
 * the query rows i in [first, N) (rows before `first` are left untouched).
 * Costs O((N - first) N d); used to sample dK/dV rows at large N.  Under the
 * causal mask, key row j only meets query rows i >= j, so the statistics of
 * the rows from `first` on are all that dK/dV rows j >= first need.
 */
int ref_head_stats(const double *q, const double *k, const double *v,
                   const double *dO, int N, int d, int causal, double scale,
                   int first, double *lse, double *D) {
    int failed = 0;
#pragma omp parallel reduction(| : failed)
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        if (!p) failed = 1;
#pragma omp for schedule(dynamic, 16)
        for (int i = first; i < N; ++i) {
            if (!p) continue;
            const int n = row_extent(i, N, causal);
            lse[i] = forward_row(q + (size_t)i * d, k, v, n, d, scale, p, NULL);
            double Di = 0.0;
            for (int j = 0; j < n; ++j)
                Di += p[j] * dot(dO + (size_t)i * d, v + (size_t)j * d, d);
            D[i] = Di;
        }
        free(p);
    }
    return failed ? -1 : 0;
}

/*
 * dQ for selected query rows of one head: recomputes row i's P and D_i from
 * the definition, then dQ_i = scale * sum_j dS_ij k_j.  dq is [nrows,d].
 */
int ref_dq_rows(const double *q, const double *k, const double *v,
                const double *dO, int N, int d, int causal, double scale,
                const long long *rows, int nrows, double *dq) {
    int failed = 0;
#pragma omp parallel reduction(| : failed)
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *dp = (double *)malloc(sizeof(double) * (size_t)N);
        if (!p || !dp) failed = 1;
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            if (!p || !dp) continue;
            const int i = (int)rows[r];
            const int n = row_extent(i, N, causal);
            const double *do_i = dO + (size_t)i * d;
            forward_row(q + (size_t)i * d, k, v, n, d, scale, p, NULL);
            double Di = 0.0;
            for (int j = 0; j < n; ++j) {
                dp[j] = dot(do_i, v + (size_t)j * d, d);
                Di += p[j] * dp[j];
            }
            double *dq_r = dq + (size_t)r * d;
            for (int t = 0; t < d; ++t) dq_r[t] = 0.0;
            for (int j = 0; j < n; ++j) {
                const double ds = p[j] * (dp[j] - Di);
                for (int t = 0; t < d; ++t) dq_r[t] += ds * k[(size_t)j * d + t];
            }
            for (int t = 0; t < d; ++t) dq_r[t] *= scale;
        }
        free(p);
        free(dp);
    }
    return failed ? -1 : 0;
}

/*
 * dK and dV for selected key rows j of one head, given every row's LSE_i and
 * D_i (from ref_head_stats): P_ij = exp(s_ij - LSE_i) is the normalised
 * probability, and the sums run over the query rows i that see key j.
 */
void ref_dkdv_rows(const double *q, const double *k, const double *v,
                   const double *dO, const double *lse, const double *D, int N,
                   int d, int causal, double scale, const long long *rows,
                   int nrows, double *dk, double *dv) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const int j = (int)rows[r];
        const double *k_j = k + (size_t)j * d;
        const double *v_j = v + (size_t)j * d;
        double *dk_r = dk + (size_t)r * d;
        double *dv_r = dv + (size_t)r * d;
        for (int t = 0; t < d; ++t) dk_r[t] = dv_r[t] = 0.0;
        for (int i = causal ? j : 0; i < N; ++i) {
            const double *q_i = q + (size_t)i * d;
            const double *do_i = dO + (size_t)i * d;
            const double p = exp(scale * dot(q_i, k_j, d) - lse[i]);
            const double ds = p * (dot(do_i, v_j, d) - D[i]);
            for (int t = 0; t < d; ++t) {
                dv_r[t] += p * do_i[t];
                dk_r[t] += ds * q_i[t];
            }
        }
        for (int t = 0; t < d; ++t) dk_r[t] *= scale;
    }
}

/*
 * Forward with different query and key counts (token-by-token decoding
 * against a key/value cache: the iplexlaw FlashAttention-2 blog, section
 * "Document the implementation difference", separates long-prompt
 * processing from token-by-token generation).  q, o: [BH, Nq, d];
 * k, v: [BH, Nk, d]; lse: [BH, Nq].  With causal != 0, query i sees key j iff
 * j <= i + (Nk - Nq): the last query sees every key and the diagonal ends at
 * the last key, the usual alignment when Nq new tokens extend a cache of
 * Nk - Nq.  Requires Nk >= Nq when causal (every row then sees >= 1 key).
 * Returns 0, -1 on allocation failure, -2 on an invalid size.
 */
int ref_fwd_decode(const double *q, const double *k, const double *v, double *o,
                   double *lse, int BH, int Nq, int Nk, int d, int causal,
                   double scale) {
    if (causal && Nk < Nq) return -2;
    const long long rows = (long long)BH * Nq;
    const int offset = Nk - Nq;
    int failed = 0;
#pragma omp parallel reduction(| : failed)
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        if (!p) failed = 1;
#pragma omp for schedule(dynamic, 4)
        for (long long r = 0; r < rows; ++r) {
            if (!p) continue;
            const long long bh = r / Nq;
            const int i = (int)(r % Nq);
            const int n = causal ? i + offset + 1 : Nk;
            const size_t kv = (size_t)bh * Nk * d;
            lse[r] = forward_row(q + (size_t)r * d, k + kv, v + kv, n, d, scale, p,
                                 o + (size_t)r * d);
        }
        free(p);
    }
    return failed ? -1 : 0;
}

/* Threads OpenMP will use (1 without OpenMP). */
int ref_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
