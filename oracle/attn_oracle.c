/*
 * attn_oracle.c -- fp64 CPU oracle for causal (GQA-capable) softmax attention,
 * forward and analytic backward.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain definition that the
 * CUDA kernels are checked against.  Only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or constant with the CUDA library, and it includes nothing from it.
 *
 * What it computes (the pages name the operation but never write its formula,
 * so this is the textbook scaled-dot-product attention they describe):
 *   - Axis (zyoralabs.com/axis), feature list: "fused flash attention, forward
 *     and backward"; bf16 storage with fp32 accumulation.  Here: inputs are the
 *     bf16-rounded values widened to double; all arithmetic is double.
 *   - Axis, second code sample (n_heads=24, n_kv_heads=8) and the shape-fuzz
 *     bullet ("KV groups"); axiomlm (PyPI), Key Features ("Grouped-Query
 *     Attention"): query head h reads key/value head h / G, G = Hq / Hkv.
 *   - axiomlm, Quick Start section 8 (q of shape (2,1024,12,64)): tensors are
 *     laid out [B, S, H, D], contiguous.
 *   - furkanhaney/axis README, "Training building blocks" table (causal
 *     attention, central differences): key j is visible to query i iff j <= i.
 *
 * Definition, for batch b, query head h, kv = h / G, query row i:
 *   s_ij  = scale * sum_d Q[b,i,h,d] K[b,j,kv,d]      (s_ij = -inf if causal, j > i)
 *   m_i   = max_j s_ij,  l_i = sum_j exp(s_ij - m_i),  P_ij = exp(s_ij - m_i) / l_i
 *   O[b,i,h,:] = sum_j P_ij V[b,j,kv,:]               LSE[b,h,i] = m_i + ln l_i
 *   Dr_i  = sum_d dO[b,i,h,d] O[b,i,h,d]               (O is the fp64 O)
 *   dP_ij = sum_d dO[b,i,h,d] V[b,j,kv,d]
 *   dS_ij = P_ij (dP_ij - Dr_i)
 *   dQ[b,i,h,:]  = scale * sum_j dS_ij K[b,j,kv,:]
 *   dK[b,j,kv,:] = scale * sum_{h in group(kv)} sum_i dS_ij Q[b,i,h,:]
 *   dV[b,j,kv,:] =         sum_{h in group(kv)} sum_i P_ij  dO[b,i,h,:]
 *
 * Every row is computed on its own, over the full key range with the mask
 * applied explicitly, so memory is O(S) per thread and no S x S matrix exists.
 * OpenMP parallelises over independent rows or over (b, kv) units, which own
 * their dK/dV rows, so no reduction races exist.
 *
 * A row whose keys are all masked cannot occur for causal attention with one
 * sequence length for queries and keys (row i always sees key 0).  If it ever
 * did, m_i = -inf and the row would come out NaN; nothing here guards it.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, Hq, Hkv, S, D;
    double scale;
    int causal;
} dims_t;

static size_t at(const dims_t* z, int b, int s, int h, int H, int d) {
    return (((size_t)b * z->S + s) * H + h) * z->D + d;
}

static double dot(const double* x, const double* y, int n) {
    double acc = 0.0;
    for (int d = 0; d < n; ++d) acc += x[d] * y[d];
    return acc;
}

/* Scores, mask, softmax for one query row: p[0..S) receives P_i., *lse the
 * row's log-sum-exp (natural log, scale included). */
static void softmax_row(const dims_t* z, const double* q, const double* k,
                        int b, int h, int i, double* p, double* lse) {
    const int kv = h / (z->Hq / z->Hkv);
    const double* qi = q + at(z, b, i, h, z->Hq, 0);
    double m = -INFINITY;
    for (int j = 0; j < z->S; ++j) {
        if (z->causal && j > i) {
            p[j] = -INFINITY;
        } else {
            p[j] = z->scale * dot(qi, k + at(z, b, j, kv, z->Hkv, 0), z->D);
        }
        if (p[j] > m) m = p[j];
    }
    double l = 0.0;
    for (int j = 0; j < z->S; ++j) {
        p[j] = exp(p[j] - m);
        l += p[j];
    }
    for (int j = 0; j < z->S; ++j) p[j] /= l;
    *lse = m + log(l);
}

/* O row from a probability row. */
static void out_row(const dims_t* z, const double* v, int b, int kv,
                    const double* p, double* o) {
    for (int d = 0; d < z->D; ++d) o[d] = 0.0;
    for (int j = 0; j < z->S; ++j) {
        if (p[j] == 0.0) continue;
        const double* vj = v + at(z, b, j, kv, z->Hkv, 0);
        for (int d = 0; d < z->D; ++d) o[d] += p[j] * vj[d];
    }
}

/* Rows of the backward that depend only on query row i: dS_i. into ds,
 * plus Dr_i.  p holds P_i. on entry. */
static double dscore_row(const dims_t* z, const double* v, const double* dout,
                         const double* o_row, int b, int h, int i,
                         const double* p, double* ds) {
    const int kv = h / (z->Hq / z->Hkv);
    const double* doi = dout + at(z, b, i, h, z->Hq, 0);
    const double dr = dot(doi, o_row, z->D);
    for (int j = 0; j < z->S; ++j) {
        if (p[j] == 0.0) { ds[j] = 0.0; continue; }
        const double dp = dot(doi, v + at(z, b, j, kv, z->Hkv, 0), z->D);
        ds[j] = p[j] * (dp - dr);
    }
    return dr;
}

static dims_t mk(int B, int Hq, int Hkv, int S, int D, double scale, int causal) {
    dims_t z = {B, Hq, Hkv, S, D, scale, causal};
    return z;
}

static int bad_dims(const dims_t* z) {
    return z->B < 1 || z->Hq < 1 || z->Hkv < 1 || z->S < 1 || z->D < 1 ||
           z->Hq % z->Hkv != 0;
}

/* ---------------------------------------------------------------- forward */

/* Full forward.  o: [B,S,Hq,D], lse: [B,Hq,S].  Returns 0, or -1 on bad dims. */
int oracle_attn_fwd(const double* q, const double* k, const double* v,
                    double* o, double* lse, int B, int Hq, int Hkv, int S, int D,
                    double scale, int causal) {
    dims_t z = mk(B, Hq, Hkv, S, D, scale, causal);
    if (bad_dims(&z)) return -1;
    const long rows = (long)B * Hq * S;
#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(dynamic, 16)
        for (long r = 0; r < rows; ++r) {
            const int i = (int)(r % S);
            const int h = (int)((r / S) % Hq);
            const int b = (int)(r / ((long)S * Hq));
            double l;
            softmax_row(&z, q, k, b, h, i, p, &l);
            out_row(&z, v, b, h / (Hq / Hkv), p, o + at(&z, b, i, h, Hq, 0));
            lse[((size_t)b * Hq + h) * S + i] = l;
        }
        free(p);
    }
    return 0;
}

/* Forward for selected rows only.  rows: n triples (b, h, i).
 * o_out: [n, D], lse_out: [n]. */
int oracle_attn_fwd_rows(const double* q, const double* k, const double* v,
                         int B, int Hq, int Hkv, int S, int D, double scale,
                         int causal, int n, const int* rows, double* o_out,
                         double* lse_out) {
    dims_t z = mk(B, Hq, Hkv, S, D, scale, causal);
    if (bad_dims(&z)) return -1;
#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < n; ++r) {
            const int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            softmax_row(&z, q, k, b, h, i, p, &lse_out[r]);
            out_row(&z, v, b, h / (Hq / Hkv), p, o_out + (size_t)r * D);
        }
        free(p);
    }
    return 0;
}

/* The probability row P[b,h,i,:] (length S), for the invariant checks. */
int oracle_attn_probs_row(const double* q, const double* k, int B, int Hq,
                          int Hkv, int S, int D, double scale, int causal,
                          int b, int h, int i, double* p_out) {
    dims_t z = mk(B, Hq, Hkv, S, D, scale, causal);
    if (bad_dims(&z)) return -1;
    double l;
    softmax_row(&z, q, k, b, h, i, p_out, &l);
    return 0;
}

/* --------------------------------------------------------------- backward */

/* Full backward.  dq: [B,S,Hq,D]; dk, dv: [B,S,Hkv,D]; dr_out (optional,
 * may be NULL): [B,Hq,S] = rowsum(dO * O).  One OpenMP task per (b, kv) unit,
 * which owns its dK/dV rows. */
int oracle_attn_bwd(const double* q, const double* k, const double* v,
                    const double* dout, double* dq, double* dk, double* dv,
                    double* dr_out, int B, int Hq, int Hkv, int S, int D,
                    double scale, int causal) {
    dims_t z = mk(B, Hq, Hkv, S, D, scale, causal);
    if (bad_dims(&z)) return -1;
    const int G = Hq / Hkv;
    const int units = B * Hkv;
#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)S);
        double* ds = (double*)malloc(sizeof(double) * (size_t)S);
        double* o_row = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int u = 0; u < units; ++u) {
            const int b = u / Hkv, kv = u % Hkv;
            for (int j = 0; j < S; ++j)
                for (int d = 0; d < D; ++d) {
                    dk[at(&z, b, j, kv, Hkv, d)] = 0.0;
                    dv[at(&z, b, j, kv, Hkv, d)] = 0.0;
                }
            for (int h = kv * G; h < (kv + 1) * G; ++h) {
                for (int i = 0; i < S; ++i) {
                    double l;
                    softmax_row(&z, q, k, b, h, i, p, &l);
                    out_row(&z, v, b, kv, p, o_row);
                    const double dr = dscore_row(&z, v, dout, o_row, b, h, i, p, ds);
                    if (dr_out) dr_out[((size_t)b * Hq + h) * S + i] = dr;
                    const double* qi = q + at(&z, b, i, h, Hq, 0);
                    const double* doi = dout + at(&z, b, i, h, Hq, 0);
                    double* dqi = dq + at(&z, b, i, h, Hq, 0);
                    for (int d = 0; d < D; ++d) dqi[d] = 0.0;
                    for (int j = 0; j < S; ++j) {
                        if (p[j] == 0.0) continue;
                        const double* kj = k + at(&z, b, j, kv, Hkv, 0);
                        double* dkj = dk + at(&z, b, j, kv, Hkv, 0);
                        double* dvj = dv + at(&z, b, j, kv, Hkv, 0);
                        for (int d = 0; d < D; ++d) {
                            dqi[d] += ds[j] * kj[d];
                            dkj[d] += ds[j] * qi[d];
                            dvj[d] += p[j] * doi[d];
                        }
                    }
                    for (int d = 0; d < D; ++d) dqi[d] *= scale;
                }
            }
            for (int j = 0; j < S; ++j)
                for (int d = 0; d < D; ++d) dk[at(&z, b, j, kv, Hkv, d)] *= scale;
        }
        free(p);
        free(ds);
        free(o_row);
    }
    return 0;
}

/* dQ for selected query rows.  rows: n triples (b, h, i); dq_out: [n, D];
 * dr_out (optional): [n]. */
int oracle_attn_bwd_dq_rows(const double* q, const double* k, const double* v,
                            const double* dout, int B, int Hq, int Hkv, int S,
                            int D, double scale, int causal, int n,
                            const int* rows, double* dq_out, double* dr_out) {
    dims_t z = mk(B, Hq, Hkv, S, D, scale, causal);
    if (bad_dims(&z)) return -1;
#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)S);
        double* ds = (double*)malloc(sizeof(double) * (size_t)S);
        double* o_row = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < n; ++r) {
            const int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            const int kv = h / (Hq / Hkv);
            double l;
            softmax_row(&z, q, k, b, h, i, p, &l);
            out_row(&z, v, b, kv, p, o_row);
            const double dr = dscore_row(&z, v, dout, o_row, b, h, i, p, ds);
            if (dr_out) dr_out[r] = dr;
            double* out = dq_out + (size_t)r * D;
            for (int d = 0; d < D; ++d) out[d] = 0.0;
            for (int j = 0; j < S; ++j) {
                if (ds[j] == 0.0) continue;
                const double* kj = k + at(&z, b, j, kv, Hkv, 0);
                for (int d = 0; d < D; ++d) out[d] += ds[j] * kj[d];
            }
            for (int d = 0; d < D; ++d) out[d] *= scale;
        }
        free(p);
        free(ds);
        free(o_row);
    }
    return 0;
}

/* dK and dV for selected key rows.  rows: n triples (b, kv, j);
 * dk_out, dv_out: [n, D].  For every query row i that can see key j (and every
 * query head h of the group) it needs LSE_i and Dr_i, which are per-row
 * quantities of the forward; they are computed here first, for each (b, kv)
 * unit that the sample touches, then P_ij and dS_ij follow from them:
 *   P_ij = exp(s_ij - LSE_i),  dS_ij = P_ij (dP_ij - Dr_i). */
int oracle_attn_bwd_dkdv_rows(const double* q, const double* k, const double* v,
                              const double* dout, int B, int Hq, int Hkv, int S,
                              int D, double scale, int causal, int n,
                              const int* rows, double* dk_out, double* dv_out) {
    dims_t z = mk(B, Hq, Hkv, S, D, scale, causal);
    if (bad_dims(&z)) return -1;
    const int G = Hq / Hkv;
    /* Distinct units touched by the sample. */
    int* unit_of = (int*)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
    int* units = (int*)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
    int nu = 0;
    for (int r = 0; r < n; ++r) {
        const int u = rows[3 * r] * Hkv + rows[3 * r + 1];
        int f = -1;
        for (int t = 0; t < nu; ++t)
            if (units[t] == u) f = t;
        if (f < 0) { units[nu] = u; f = nu++; }
        unit_of[r] = f;
    }
    /* Under the causal mask only query rows i >= j see key j, so each unit
     * needs the per-row statistics from its smallest sampled key row on. */
    int* first = (int*)malloc(sizeof(int) * (size_t)(nu > 0 ? nu : 1));
    for (int t = 0; t < nu; ++t) first[t] = causal ? S : 0;
    if (causal)
        for (int r = 0; r < n; ++r)
            if (rows[3 * r + 2] < first[unit_of[r]]) first[unit_of[r]] = rows[3 * r + 2];
    double* lse = (double*)malloc(sizeof(double) * (size_t)(nu > 0 ? nu : 1) * G * S);
    double* dr = (double*)malloc(sizeof(double) * (size_t)(nu > 0 ? nu : 1) * G * S);
    const long stat_rows = (long)nu * G * S;
#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)S);
        double* o_row = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 16)
        for (long t = 0; t < stat_rows; ++t) {
            const int i = (int)(t % S);
            const int g = (int)((t / S) % G);
            const int un = (int)(t / ((long)S * G));
            const int b = units[un] / Hkv, kv = units[un] % Hkv, h = kv * G + g;
            if (i < first[un]) { lse[t] = 0.0; dr[t] = 0.0; continue; }
            double l;
            softmax_row(&z, q, k, b, h, i, p, &l);
            out_row(&z, v, b, kv, p, o_row);
            lse[t] = l;
            dr[t] = dot(dout + at(&z, b, i, h, Hq, 0), o_row, D);
        }
        free(p);
        free(o_row);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n; ++r) {
        const int b = rows[3 * r], kv = rows[3 * r + 1], j = rows[3 * r + 2];
        const double* kj = k + at(&z, b, j, kv, Hkv, 0);
        const double* vj = v + at(&z, b, j, kv, Hkv, 0);
        double* dko = dk_out + (size_t)r * D;
        double* dvo = dv_out + (size_t)r * D;
        for (int d = 0; d < D; ++d) { dko[d] = 0.0; dvo[d] = 0.0; }
        for (int g = 0; g < G; ++g) {
            const int h = kv * G + g;
            const double* lse_u = lse + ((size_t)unit_of[r] * G + g) * S;
            const double* dr_u = dr + ((size_t)unit_of[r] * G + g) * S;
            for (int i = 0; i < S; ++i) {
                if (causal && j > i) continue;
                const double* qi = q + at(&z, b, i, h, Hq, 0);
                const double* doi = dout + at(&z, b, i, h, Hq, 0);
                const double pij = exp(scale * dot(qi, kj, D) - lse_u[i]);
                const double dsij = pij * (dot(doi, vj, D) - dr_u[i]);
                for (int d = 0; d < D; ++d) {
                    dko[d] += dsij * qi[d];
                    dvo[d] += pij * doi[d];
                }
            }
        }
        for (int d = 0; d < D; ++d) dko[d] *= scale;
    }
    free(unit_of);
    free(units);
    free(first);
    free(lse);
    free(dr);
    return 0;
}

/*
 * Rotary position embedding, the step the axiomlm models apply to Q and K
 * before attention: axiomlm (PyPI), Key Features ("Rotary Position Embeddings
 * (RoPE)") and Quick Start section 8 (precompute_rope_frequencies(dim, end),
 * then apply_rope(q, k, freqs_cis)).  The page names the calls, not the
 * formula; the reading taken is the complex-pair form that the name freqs_cis
 * points to: in a row at sequence position s, the pair (x[2p], x[2p+1]) is
 * turned by the angle s * base^(-2p/D) -- the complex number x[2p] + i x[2p+1]
 * times exp(i s base^(-2p/D)).  base is the caller's (the page gives none;
 * 10000 is the usual value).  inverse != 0 turns by minus the angle: the
 * transpose of the rotation, which carries dQ, dK back through it.
 * x is [B, S, H, D] (D even), rotated in place.  Returns 0, or -1 for bad sizes.
 */
int oracle_rope(double* x, int B, int S, int H, int D, double base, int inverse) {
    if (B < 1 || S < 1 || H < 1 || D < 2 || (D & 1) || !(base > 0.0)) return -1;
    const double sgn = inverse ? -1.0 : 1.0;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int s = 0; s < S; ++s)
            for (int h = 0; h < H; ++h) {
                double* row = x + (((size_t)b * S + s) * H + h) * D;
                for (int p = 0; p < D / 2; ++p) {
                    const double ang = sgn * (double)s * pow(base, -2.0 * p / D);
                    const double c = cos(ang), sn = sin(ang);
                    const double x0 = row[2 * p], x1 = row[2 * p + 1];
                    row[2 * p] = x0 * c - x1 * sn;
                    row[2 * p + 1] = x0 * sn + x1 * c;
                }
            }
    return 0;
}

/*
 * Decode step: one new query row per sequence against the keys and values
 * already cached for it -- the step the axiomlm inference engine repeats per
 * generated token: axiomlm (PyPI), Key Features ("State-cached Key-Value (KV)
 * decode engine achieving O(1) step latency") and Quick Start section 4 ("Use
 * the Paged KV-Cache engine for O(1) step decoding"), with the GQA heads of
 * Key Features ("4-head Grouped-Query Attention").  The new token is the last
 * position of its sequence, so the causal mask lets it see every cached key,
 * itself included:
 *   s_j  = scale * sum_d q[b,h,d] K[b,j,kv,d]       for j < lens[b], kv = h / G
 *   o[b,h,:] = sum_j softmax(s)_j V[b,j,kv,:]         lse[b,h] = ln sum_j exp(s_j)
 * q, o: [B, Hq, D]; k, v: [B, Smax, Hkv, D], of which sequence b uses its first
 * lens[b] rows (1 <= lens[b] <= Smax); lse: [B, Hq].  (The cache's layout in
 * device memory -- pages, a block table -- is the kernel's business; the
 * definition reads it as one row per position.)  Returns 0, or -1 for bad sizes.
 */
int oracle_attn_decode(const double* q, const double* k, const double* v, const int* lens,
                       double* o, double* lse, int B, int Hq, int Hkv, int Smax, int D,
                       double scale) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Smax < 1 || D < 1 || Hq % Hkv) return -1;
    for (int b = 0; b < B; ++b)
        if (lens[b] < 1 || lens[b] > Smax) return -1;
    const int G = Hq / Hkv;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)Smax);
#pragma omp for collapse(2) schedule(dynamic, 1)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < Hq; ++h) {
                const int kv = h / G, L = lens[b];
                const double* qh = q + ((size_t)b * Hq + h) * D;
                double m = -INFINITY;
                for (int j = 0; j < L; ++j) {
                    s[j] = scale * dot(qh, k + (((size_t)b * Smax + j) * Hkv + kv) * D, D);
                    if (s[j] > m) m = s[j];
                }
                double l = 0.0;
                for (int j = 0; j < L; ++j) l += exp(s[j] - m);
                double* oh = o + ((size_t)b * Hq + h) * D;
                for (int d = 0; d < D; ++d) oh[d] = 0.0;
                for (int j = 0; j < L; ++j) {
                    const double pj = exp(s[j] - m) / l;
                    const double* vj = v + (((size_t)b * Smax + j) * Hkv + kv) * D;
                    for (int d = 0; d < D; ++d) oh[d] += pj * vj[d];
                }
                lse[(size_t)b * Hq + h] = m + log(l);
            }
        free(s);
    }
    return 0;
}

/*
 * Decode step with q_len new tokens per sequence at once (q_len = 1 is
 * oracle_attn_decode): the decode engine of the axiomlm page (Key Features,
 * "State-cached Key-Value (KV) decode engine"; Quick Start section 4) advancing
 * several positions in one step -- a chunk of a prompt appended to the cache,
 * or several proposed tokens checked together.  The new tokens are the last
 * q_len positions of their sequence, so new token t of sequence b sits at
 * position p = lens[b] - q_len + t and, under the causal mask, sees the cached
 * keys j <= p (the earlier new tokens and itself included, the later ones
 * not):
 *   s_j = scale * sum_d q[b,t,h,d] K[b,j,kv,d]   for j <= p, kv = h / G
 *   o[b,t,h,:] = sum_j softmax(s)_j V[b,j,kv,:]   lse[b,h,t] = ln sum_j exp(s_j)
 * q, o: [B, q_len, Hq, D]; k, v: [B, Smax, Hkv, D], of which sequence b uses its
 * first lens[b] rows (q_len <= lens[b] <= Smax); lse: [B, Hq, q_len].  Returns
 * 0, or -1 for bad sizes.
 */
int oracle_attn_decode_q(const double* q, const double* k, const double* v, const int* lens,
                         double* o, double* lse, int B, int q_len, int Hq, int Hkv, int Smax, int D,
                         double scale) {
    if (B < 1 || q_len < 1 || Hq < 1 || Hkv < 1 || Smax < 1 || D < 1 || Hq % Hkv) return -1;
    for (int b = 0; b < B; ++b)
        if (lens[b] < q_len || lens[b] > Smax) return -1;
    const int G = Hq / Hkv;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)Smax);
#pragma omp for collapse(3) schedule(dynamic, 1)
        for (int b = 0; b < B; ++b)
            for (int t = 0; t < q_len; ++t)
                for (int h = 0; h < Hq; ++h) {
                    const int kv = h / G, p = lens[b] - q_len + t;  /* this token's position */
                    const double* qh = q + (((size_t)b * q_len + t) * Hq + h) * D;
                    double m = -INFINITY;
                    for (int j = 0; j <= p; ++j) {
                        s[j] = scale * dot(qh, k + (((size_t)b * Smax + j) * Hkv + kv) * D, D);
                        if (s[j] > m) m = s[j];
                    }
                    double l = 0.0;
                    for (int j = 0; j <= p; ++j) l += exp(s[j] - m);
                    double* oh = o + (((size_t)b * q_len + t) * Hq + h) * D;
                    for (int d = 0; d < D; ++d) oh[d] = 0.0;
                    for (int j = 0; j <= p; ++j) {
                        const double pj = exp(s[j] - m) / l;
                        const double* vj = v + (((size_t)b * Smax + j) * Hkv + kv) * D;
                        for (int d = 0; d < D; ++d) oh[d] += pj * vj[d];
                    }
                    lse[((size_t)b * Hq + h) * q_len + t] = m + log(l);
                }
        free(s);
    }
    return 0;
}

/* Threads OpenMP will use (1 when built without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
