/*
 * Plain fp64 CPU attention: the oracle the CUDA path is checked against.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do. It shares no code, header or constant with the CUDA kernels.
 *
 * What it computes is the definition of scaled dot-product attention, one
 * query row at a time ("FlashAttention/zh", section "why standard attention
 * is slow"): a row of scores s_j = scale * <q_i, k_j> is materialised in
 * full, masked keys are set to -inf, and the safe softmax is taken in two
 * passes, max first and then exp and sum ("YOLOv12 ... Flash Attention v2",
 * section 2.2; "FlashAttention/zh", section "online softmax", first formula).
 * The output row is o_i = sum_j p_ij v_j and the log-sum-exp is
 * L_i = m_i + ln(l_i) ("FlashAttention/zh", the last step of the forward
 * algorithm). There is no tiling, no online recurrence and no reordering
 * beyond row independence: rows of a softmax are independent by definition.
 *
 * The backward pass is not written out on the pages; they only say that S
 * and P are recomputed from L and dO ("FlashAttention/zh", section
 * "backward pass and recomputation"). The oracle therefore takes the exact
 * gradient of the definition above:
 *     dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij,
 *     dS = P o (dP - D 1^T),  dQ = scale dS K,  dK = scale dS^T Q,
 * and with grouped KV heads the dK and dV of a KV head sum over the query
 * heads that share it.
 *
 * Layout (all row-major, float64): q [B,Nq,Hq,d], k and v [B,Nk,Hkv,d],
 * o and dO [B,Nq,Hq,d], lse [B,Hq,Nq]. Query head h reads KV head
 * h / (Hq/Hkv). Masking: with a = i + (Nk - Nq) (bottom-right alignment),
 * key j is visible to query i iff
 *     key_keep == NULL or key_keep[b*Nk + j] != 0, and
 *     wl < 0 or j >= a - wl or j < na (global anchor keys), and
 *     wr < 0 or j <= a + wr.
 * (wl, wr) is a sliding window of wl keys before and wr keys after the
 * aligned key; a negative side is unbounded. The causal mask is
 * (wl, wr) = (-1, 0), no mask (-1, -1).
 * A query row with no visible key has o_i = 0 and L_i = -inf.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static int visible(const unsigned char* key_keep, int b, int Nq, int Nk, int wl, int wr, int na, int i, int j) {
    if (key_keep && !key_keep[(long)b * Nk + j]) return 0;
    const long a = (long)i + (long)(Nk - Nq);
    if (wl >= 0 && (long)j < a - wl && j >= na) return 0;
    if (wr >= 0 && (long)j > a + wr) return 0;
    return 1;
}

static double dot(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += a[c] * b[c];
    return s;
}

/* Probabilities of one query row: fills p[0..Nk) and returns m and l through
 * pointers. Returns 0 if the row has no visible key (p is all zero then). */
static int softmax_row(const double* qi, const double* kbase, long kstride, int Nk, int d,
                       double scale, const unsigned char* key_keep, int b, int Nq, int wl, int wr, int na,
                       int i, double* s, double* p, double* m_out, double* l_out) {
    double m = -INFINITY;
    for (int j = 0; j < Nk; ++j) {
        if (visible(key_keep, b, Nq, Nk, wl, wr, na, i, j)) {
            s[j] = scale * dot(qi, kbase + (long)j * kstride, d);
            if (s[j] > m) m = s[j];
        } else {
            s[j] = -INFINITY;
        }
    }
    if (m == -INFINITY) {
        for (int j = 0; j < Nk; ++j) p[j] = 0.0;
        *m_out = -INFINITY;
        *l_out = 0.0;
        return 0;
    }
    double l = 0.0;
    for (int j = 0; j < Nk; ++j) {
        p[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
        l += p[j];
    }
    for (int j = 0; j < Nk; ++j) p[j] /= l;
    *m_out = m;
    *l_out = l;
    return 1;
}

int ora_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the parallel regions that follow (the CPU baseline times one core too). */
void ora_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Forward. rows == NULL computes every query row; otherwise only the nrows
 * listed query indices (for every batch and head) are written to o and lse. */
int ora_attn_fwd(const double* q, const double* k, const double* v, int B, int Hq, int Hkv,
                 int Nq, int Nk, int d, double scale, int wl, int wr, int na,
                 const unsigned char* key_keep, const int* rows, int nrows,
                 double* o, double* lse) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Nq < 0 || Nk < 0 || d <= 0) return 1;
    const int group = Hq / Hkv;
    const int nr = rows ? nrows : Nq;
    const long total = (long)B * Hq * nr;
    int err = 0;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
        double* p = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
        if (!s || !p) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 4)
        for (long t = 0; t < total; ++t) {
            if (!s || !p) continue;
            const int b = (int)(t / ((long)Hq * nr));
            const int h = (int)((t / nr) % Hq);
            const int i = rows ? rows[t % nr] : (int)(t % nr);
            const int hk = h / group;
            const double* qi = q + (((long)b * Nq + i) * Hq + h) * d;
            const double* kb = k + ((long)b * Nk * Hkv + hk) * d;
            const double* vb = v + ((long)b * Nk * Hkv + hk) * d;
            const long kvs = (long)Hkv * d;
            double m, l;
            double* oi = o + (((long)b * Nq + i) * Hq + h) * d;
            for (int c = 0; c < d; ++c) oi[c] = 0.0;
            if (softmax_row(qi, kb, kvs, Nk, d, scale, key_keep, b, Nq, wl, wr, na, i, s, p, &m, &l)) {
                for (int j = 0; j < Nk; ++j) {
                    if (p[j] == 0.0) continue;
                    const double* vj = vb + (long)j * kvs;
                    for (int c = 0; c < d; ++c) oi[c] += p[j] * vj[c];
                }
                lse[((long)b * Hq + h) * Nq + i] = m + log(l);
            } else {
                lse[((long)b * Hq + h) * Nq + i] = -INFINITY;
            }
        }
        free(s);
        free(p);
    }
    return err;
}

/* The probability matrix P of one (batch, query head), Nq x Nk, row-major. */
int ora_attn_probs(const double* q, const double* k, int B, int Hq, int Hkv, int Nq, int Nk,
                   int d, double scale, int wl, int wr, int na, const unsigned char* key_keep, int b, int h,
                   double* P) {
    if (b < 0 || b >= B || h < 0 || h >= Hq || Hq % Hkv) return 1;
    const int hk = h / (Hq / Hkv);
    double* s = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
    if (!s) return 2;
    for (int i = 0; i < Nq; ++i) {
        double m, l;
        softmax_row(q + (((long)b * Nq + i) * Hq + h) * d, k + ((long)b * Nk * Hkv + hk) * d,
                    (long)Hkv * d, Nk, d, scale, key_keep, b, Nq, wl, wr, na, i, s, P + (long)i * Nk,
                    &m, &l);
    }
    free(s);
    return 0;
}

/* Gradient terms of one query row i of query head h: recomputes the row's P and
 * dP = dO_i V^T, D = sum_j P_ij dP_ij and dS_ij = P_ij (dP_ij - D); writes
 * dq_i = scale sum_j dS_ij k_j when dqi != NULL, and adds scale dS_ij q_i into
 * the dK row and P_ij dO_i into the dV row of every listed key: key krows[t]
 * (every key t when krows == NULL) at dk_out + t * out_stride and
 * dv_out + t * out_stride. s, p, dp are scratch rows of Nk doubles. */
static void row_grads(const double* qi, const double* doi, const double* kb, const double* vb, long kvs,
                      int Nq, int Nk, int d, double scale, int wl, int wr, int na,
                      const unsigned char* key_keep, int b, int i, double* s, double* p, double* dp,
                      double* dqi, const int* krows, int nkeys, double* dk_out, double* dv_out,
                      long out_stride) {
    double m, l;
    if (dqi)
        for (int c = 0; c < d; ++c) dqi[c] = 0.0;
    if (!softmax_row(qi, kb, kvs, Nk, d, scale, key_keep, b, Nq, wl, wr, na, i, s, p, &m, &l))
        return; /* no visible key: every gradient term of this row is 0 */
    double D = 0.0;
    for (int j = 0; j < Nk; ++j) {
        dp[j] = (p[j] == 0.0) ? 0.0 : dot(doi, vb + (long)j * kvs, d);
        D += p[j] * dp[j];
    }
    if (dqi) {
        for (int j = 0; j < Nk; ++j) {
            const double ds = p[j] * (dp[j] - D);
            if (ds == 0.0) continue;
            const double* kj = kb + (long)j * kvs;
            for (int c = 0; c < d; ++c) dqi[c] += scale * ds * kj[c];
        }
    }
    for (int t = 0; t < nkeys; ++t) {
        const int j = krows ? krows[t] : t;
        if (p[j] == 0.0) continue;
        const double ds = p[j] * (dp[j] - D);
        double* dkj = dk_out + (long)t * out_stride;
        double* dvj = dv_out + (long)t * out_stride;
        for (int c = 0; c < d; ++c) {
            dkj[c] += scale * ds * qi[c];
            dvj[c] += p[j] * doi[c];
        }
    }
}

/* Backward of one (batch, KV head) group over all its query heads: writes the dq
 * rows of those query heads and accumulates dk, dv of the KV head (every row and
 * key; serial, callers run groups in parallel). */
static int bwd_group(const double* q, const double* k, const double* v, const double* dout,
                     int Nq, int Nk, int Hq, int Hkv, int d, double scale, int wl, int wr, int na,
                     const unsigned char* key_keep, int b, int hk, double* dq, double* dk, double* dv) {
    const int group = Hq / Hkv;
    const long qs = (long)Hq * d, kvs = (long)Hkv * d;
    const double* kb = k + ((long)b * Nk * Hkv + hk) * d;
    const double* vb = v + ((long)b * Nk * Hkv + hk) * d;
    double* dkb = dk + ((long)b * Nk * Hkv + hk) * d;
    double* dvb = dv + ((long)b * Nk * Hkv + hk) * d;
    double* s = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
    double* p = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
    double* dp = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
    if (!s || !p || !dp) {
        free(s); free(p); free(dp);
        return 2;
    }
    for (int g = 0; g < group; ++g) {
        const int h = hk * group + g;
        for (int i = 0; i < Nq; ++i) {
            const long off = ((long)b * Nq + i) * qs + (long)h * d;
            row_grads(q + off, dout + off, kb, vb, kvs, Nq, Nk, d, scale, wl, wr, na, key_keep, b, i, s, p,
                      dp, dq + off, NULL, Nk, dkb, dvb, kvs);
        }
    }
    free(s); free(p); free(dp);
    return 0;
}

/* Full backward: dq [B,Nq,Hq,d], dk and dv [B,Nk,Hkv,d] (overwritten). */
int ora_attn_bwd(const double* q, const double* k, const double* v, const double* dout, int B,
                 int Hq, int Hkv, int Nq, int Nk, int d, double scale, int wl, int wr, int na,
                 const unsigned char* key_keep, double* dq, double* dk, double* dv) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Nq < 0 || Nk < 0 || d <= 0) return 1;
    memset(dq, 0, sizeof(double) * (size_t)B * Nq * Hq * d);
    memset(dk, 0, sizeof(double) * (size_t)B * Nk * Hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)B * Nk * Hkv * d);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < (long)B * Hkv; ++t) {
        int e = bwd_group(q, k, v, dout, Nq, Nk, Hq, Hkv, d, scale, wl, wr, na, key_keep,
                          (int)(t / Hkv), (int)(t % Hkv), dq, dk, dv);
        if (e) {
#pragma omp atomic write
            err = e;
        }
    }
    return err;
}

/* Sampled backward of one (batch b, KV head hk) group: dq for the nq query
 * rows in qrows (every query head of the group), dk and dv for the nk key
 * rows in krows. Outputs use the full tensor layouts; only the sampled rows
 * are written (dk/dv rows are overwritten, not accumulated). Query rows that
 * are not sampled and see none of the sampled keys are skipped: they add
 * nothing to those keys' gradients. The rows are spread over the OpenMP
 * threads; each thread adds its rows' dk/dv terms into partial sums of its
 * own, which are added together at the end (every row's arithmetic is that of
 * the full backward; only the order of the final sums differs). */
int ora_attn_bwd_sampled(const double* q, const double* k, const double* v, const double* dout,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d, double scale, int wl, int wr, int na,
                         const unsigned char* key_keep, int b, int hk, const int* qrows, int nq,
                         const int* krows, int nk, double* dq, double* dk, double* dv) {
    if (b < 0 || b >= B || hk < 0 || hk >= Hkv || Hq % Hkv || nk < 0 || nq < 0) return 1;
    const int group = Hq / Hkv;
    const long qs = (long)Hq * d, kvs = (long)Hkv * d;
    const double* kb = k + ((long)b * Nk * Hkv + hk) * d;
    const double* vb = v + ((long)b * Nk * Hkv + hk) * d;
    unsigned char* want_q = (unsigned char*)calloc(Nq > 0 ? Nq : 1, 1);
    double* sum_k = (double*)calloc((size_t)(nk > 0 ? nk : 1) * d, sizeof(double));
    double* sum_v = (double*)calloc((size_t)(nk > 0 ? nk : 1) * d, sizeof(double));
    int* rows = (int*)malloc(sizeof(int) * (Nq > 0 ? Nq : 1));
    int err = 0;
    if (!want_q || !sum_k || !sum_v || !rows) {
        free(want_q); free(sum_k); free(sum_v); free(rows);
        return 2;
    }
    for (int t = 0; t < nq; ++t) want_q[qrows[t]] = 1;
    /* the query rows that take part: sampled, or seeing a sampled key */
    int nrows = 0;
    for (int i = 0; i < Nq; ++i) {
        int needed = want_q[i];
        for (int t = 0; t < nk && !needed; ++t) needed = visible(key_keep, b, Nq, Nk, wl, wr, na, i, krows[t]);
        if (needed) rows[nrows++] = i;
    }
    const long work = (long)group * nrows;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
        double* p = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
        double* dp = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
        double* part_k = (double*)calloc((size_t)(nk > 0 ? nk : 1) * d, sizeof(double));
        double* part_v = (double*)calloc((size_t)(nk > 0 ? nk : 1) * d, sizeof(double));
        const int have = s && p && dp && part_k && part_v;
        if (!have) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 8)
        for (long w = 0; w < work; ++w) {
            if (!have) continue;
            const int h = hk * group + (int)(w / nrows);
            const int i = rows[w % nrows];
            const long off = ((long)b * Nq + i) * qs + (long)h * d;
            row_grads(q + off, dout + off, kb, vb, kvs, Nq, Nk, d, scale, wl, wr, na, key_keep, b, i, s, p, dp,
                      want_q[i] ? dq + off : NULL, krows, nk, part_k, part_v, d);
        }
        if (have) {
#pragma omp critical
            for (long x = 0; x < (long)nk * d; ++x) {
                sum_k[x] += part_k[x];
                sum_v[x] += part_v[x];
            }
        }
        free(s); free(p); free(dp); free(part_k); free(part_v);
    }
    for (int t = 0; t < nk; ++t) {
        double* dkj = dk + ((long)b * Nk + krows[t]) * kvs + (long)hk * d;
        double* dvj = dv + ((long)b * Nk + krows[t]) * kvs + (long)hk * d;
        for (int c = 0; c < d; ++c) {
            dkj[c] = sum_k[(long)t * d + c];
            dvj[c] = sum_v[(long)t * d + c];
        }
    }
    free(want_q); free(sum_k); free(sum_v); free(rows);
    return err;
}
