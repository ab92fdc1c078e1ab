/* fp64 CPU oracle for exact GQA forward.  TEST INFRASTRUCTURE ONLY; see ref_attn.h
 * for what is computed and which passages of the pages each step follows. */
#include "ref_attn.h"

#include <math.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* key j allowed for query row i (causal mask aligned bottom-right when Sq != Sk) */
static int key_allowed(int causal, int i, int j, int Sq, int Sk) {
    return !causal || (long)j <= (long)i + (long)(Sk - Sq);
}

void gqa_oracle_row(const double* q, const double* k, const double* v, long kv_row_stride,
                    int d, int Sq, int Sk, int i, double scale, int causal, int key_lo,
                    int key_hi, double* o, double* lse) {
    if (key_lo < 0) key_lo = 0;
    if (key_hi > Sk) key_hi = Sk;
    for (int c = 0; c < d; ++c) o[c] = 0.0;

    /* pass 1: scores s_j = scale * q . k_j over the allowed keys, and their max */
    double* s = (double*)malloc(sizeof(double) * (size_t)(key_hi > key_lo ? key_hi - key_lo : 1));
    double m = -INFINITY;
    int n_allowed = 0;
    for (int j = key_lo; j < key_hi; ++j) {
        if (!key_allowed(causal, i, j, Sq, Sk)) continue;
        const double* kj = k + (long)j * kv_row_stride;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q[c] * kj[c];
        s[j - key_lo] = scale * dot;
        if (s[j - key_lo] > m) m = s[j - key_lo];
        ++n_allowed;
    }
    if (n_allowed == 0) {
        *lse = -INFINITY;
        free(s);
        return;
    }

    /* pass 2: l = sum_j exp(s_j - m);  o = sum_j exp(s_j - m) v_j / l */
    double l = 0.0;
    for (int j = key_lo; j < key_hi; ++j) {
        if (!key_allowed(causal, i, j, Sq, Sk)) continue;
        double p = exp(s[j - key_lo] - m);
        l += p;
        const double* vj = v + (long)j * kv_row_stride;
        for (int c = 0; c < d; ++c) o[c] += p * vj[c];
    }
    for (int c = 0; c < d; ++c) o[c] /= l;
    *lse = m + log(l);
    free(s);
}

int gqa_oracle_fwd_range(const double* q, const double* k, const double* v, int B, int Sq,
                         int Sk, int Hq, int Hk, int d, double scale, int causal, int key_lo,
                         int key_hi, double* o, double* lse) {
    const int g = Hq / Hk; /* q-heads per kv-head */
    int threads = 1;
    long nbh = (long)B * Hq;
#pragma omp parallel
    {
#ifdef _OPENMP
#pragma omp single
        threads = omp_get_num_threads();
#endif
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < nbh; ++bh) {
            int b = (int)(bh / Hq), h = (int)(bh % Hq);
            int kvh = h / g;
            const double* kb = k + ((long)b * Sk * Hk + kvh) * d;
            const double* vb = v + ((long)b * Sk * Hk + kvh) * d;
            for (int i = 0; i < Sq; ++i) {
                const double* qi = q + (((long)b * Sq + i) * Hq + h) * d;
                double* oi = o + (((long)b * Sq + i) * Hq + h) * d;
                gqa_oracle_row(qi, kb, vb, (long)Hk * d, d, Sq, Sk, i, scale, causal, key_lo,
                               key_hi, oi, &lse[((long)b * Hq + h) * Sq + i]);
            }
        }
    }
    return threads;
}

int gqa_oracle_fwd(const double* q, const double* k, const double* v, int B, int Sq, int Sk,
                   int Hq, int Hk, int d, double scale, int causal, double* o, double* lse) {
    return gqa_oracle_fwd_range(q, k, v, B, Sq, Sk, Hq, Hk, d, scale, causal, 0, Sk, o, lse);
}

void gqa_oracle_combine(int nsplit, long rows, int d, const double* o_parts,
                        const double* lse_parts, double* out, double* lse) {
    for (long r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int s = 0; s < nsplit; ++s)
            if (lse_parts[(long)s * rows + r] > M) M = lse_parts[(long)s * rows + r];
        double* orow = out + r * d;
        for (int c = 0; c < d; ++c) orow[c] = 0.0;
        if (M == -INFINITY) { /* no split saw an allowed key */
            lse[r] = -INFINITY;
            continue;
        }
        double wsum = 0.0;
        for (int s = 0; s < nsplit; ++s) {
            double w = exp(lse_parts[(long)s * rows + r] - M); /* exp(-inf) = 0 */
            wsum += w;
            const double* op = o_parts + ((long)s * rows + r) * d;
            for (int c = 0; c < d; ++c) orow[c] += w * op[c];
        }
        for (int c = 0; c < d; ++c) orow[c] /= wsum;
        lse[r] = M + log(wsum);
    }
}
