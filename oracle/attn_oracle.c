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

/* Backward of one (batch, KV head) group over all its query heads. Writes dq
 * rows of those query heads and accumulates dk, dv of the KV head. When
 * krows != NULL only the listed key rows of dk/dv are produced and only the
 * query rows listed in qrows (may be NULL with nq == 0) get dq; query rows
 * that can see none of the listed keys are skipped, which is exact because
 * they add nothing to those keys' gradients. */
static int bwd_group(const double* q, const double* k, const double* v, const double* dout,
                     int Nq, int Nk, int Hq, int Hkv, int d, double scale, int wl, int wr, int na,
                     const unsigned char* key_keep, int b, int hk, const int* qrows, int nq,
                     const int* krows, int nk, double* dq, double* dk, double* dv) {
    const int group = Hq / Hkv;
    const long qs = (long)Hq * d, kvs = (long)Hkv * d;
    const double* kb = k + ((long)b * Nk * Hkv + hk) * d;
    const double* vb = v + ((long)b * Nk * Hkv + hk) * d;
    double* s = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
    double* p = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
    double* dp = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
    unsigned char* want_q = (unsigned char*)calloc(Nq > 0 ? Nq : 1, 1);
    if (!s || !p || !dp || !want_q) {
        free(s); free(p); free(dp); free(want_q);
        return 2;
    }
    if (krows) {
        for (int t = 0; t < nq; ++t) want_q[qrows[t]] = 1;
    }
    for (int g = 0; g < group; ++g) {
        const int h = hk * group + g;
        for (int i = 0; i < Nq; ++i) {
            int needed = 1;
            if (krows) {
                needed = want_q[i];
                for (int t = 0; t < nk && !needed; ++t)
                    needed = visible(key_keep, b, Nq, Nk, wl, wr, na, i, krows[t]);
            }
            if (!needed) continue;
            const double* qi = q + ((long)b * Nq + i) * qs + (long)h * d;
            const double* doi = dout + ((long)b * Nq + i) * qs + (long)h * d;
            double m, l;
            if (!softmax_row(qi, kb, kvs, Nk, d, scale, key_keep, b, Nq, wl, wr, na, i, s, p, &m, &l))
                continue; /* no visible key: every gradient term of this row is 0 */
            double D = 0.0;
            for (int j = 0; j < Nk; ++j) {
                dp[j] = (p[j] == 0.0) ? 0.0 : dot(doi, vb + (long)j * kvs, d);
                D += p[j] * dp[j];
            }
            if (!krows || want_q[i]) {
                double* dqi = dq + ((long)b * Nq + i) * qs + (long)h * d;
                for (int c = 0; c < d; ++c) dqi[c] = 0.0;
                for (int j = 0; j < Nk; ++j) {
                    const double ds = p[j] * (dp[j] - D);
                    if (ds == 0.0) continue;
                    const double* kj = kb + (long)j * kvs;
                    for (int c = 0; c < d; ++c) dqi[c] += scale * ds * kj[c];
                }
            }
            const int nkeys = krows ? nk : Nk;
            for (int t = 0; t < nkeys; ++t) {
                const int j = krows ? krows[t] : t;
                if (p[j] == 0.0) continue;
                const double ds = p[j] * (dp[j] - D);
                double* dkj = dk + ((long)b * Nk + j) * kvs + (long)hk * d;
                double* dvj = dv + ((long)b * Nk + j) * kvs + (long)hk * d;
                for (int c = 0; c < d; ++c) {
                    dkj[c] += scale * ds * qi[c];
                    dvj[c] += p[j] * doi[c];
                }
            }
        }
    }
    free(s); free(p); free(dp); free(want_q);
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
                          (int)(t / Hkv), (int)(t % Hkv), NULL, 0, NULL, 0, dq, dk, dv);
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
 * are written (dk/dv rows are overwritten, not accumulated). Parallel over
 * the sampled key rows is not needed: one call is one group. */
int ora_attn_bwd_sampled(const double* q, const double* k, const double* v, const double* dout,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d, double scale, int wl, int wr, int na,
                         const unsigned char* key_keep, int b, int hk, const int* qrows, int nq,
                         const int* krows, int nk, double* dq, double* dk, double* dv) {
    if (b < 0 || b >= B || hk < 0 || hk >= Hkv || Hq % Hkv) return 1;
    for (int t = 0; t < nk; ++t) {
        double* dkj = dk + ((long)b * Nk + krows[t]) * Hkv * d + (long)hk * d;
        double* dvj = dv + ((long)b * Nk + krows[t]) * Hkv * d + (long)hk * d;
        for (int c = 0; c < d; ++c) dkj[c] = dvj[c] = 0.0;
    }
    /* Split the group's query heads across threads would race on dk/dv; the
     * speed comes from the caller sampling few rows, so this runs serially
     * per group and callers may run several groups in parallel processes. */
    return bwd_group(q, k, v, dout, Nq, Nk, Hq, Hkv, d, scale, wl, wr, na, key_keep, b, hk, qrows,
                     nq, krows, nk ? nk : 0, dq, dk, dv);
}
