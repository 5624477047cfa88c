/*
 * poem_oracle.c -- plain, slow, fp64 CPU oracle for POEM-style output-relative
 * block-sparse attention prefill.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file: it exists so that the tests, the smoke check and the CPU-baseline
 * leg of the benchmark can compare the CUDA library against an independent
 * statement of what the method computes.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Source of the definitions: "Attention deletion error" (jinlucs.github.io
 * reading note on Wu et al., POEM: Output-Relative Block-Sparse Attention for
 * Long-Context Prefilling), Section 4.1 and Equations (3) and (4).  For one
 * query and one head:
 *   m_b  = dense softmax mass of visible key block b, sum_b m_b = 1
 *   v_b  = attention-weighted mean value of block b  (sum_{u in b} p_u v_u / m_b)
 *   o    = sum_b m_b v_b, the dense output
 *   o~   = (o - sum_{b in D} m_b v_b) / (1 - delta), delta = sum_{b in D} m_b
 *   I_b  = m_b * || v_b - o ||                                   (Eq. 4 proxy)
 * and the triangle bound || o - o~ || <= sum_{b in D} I_b / (1 - delta).
 *
 * Choices the note leaves open (tile size, sampled queries, aggregation,
 * mandatory blocks, stopping rule) are fixed as in the CUDA library: 16 strided
 * queries per tile (rows i*B + j*(B/S)), max-aggregation of I_b and of m_b,
 * mandatory blocks {0, i-1, i}, and the stopping rule
 *     S_m < 1  and  S_I <= tau * (1 - S_m)
 * over the discarded candidate suffix, which is the triangle bound made
 * sufficient at every sampled query.  Ties in the ranking go to the smaller
 * block id and kept lists are emitted in ascending id order (the convention of
 * the "Block-Filtered Long-Context Attention" page, Appendix "Block ordering").
 *
 * Inputs are [n_tokens, n_heads, head_dim] row-major arrays, either fp64
 * (in_kind 0) or raw bf16 bit patterns (in_kind 1), widened exactly to fp64.
 * For a chunked prefill (q_offset > 0) q holds only the rows of the positions
 * q_offset .. n_tokens-1; every function takes global token positions and
 * global tiles and must only be asked about query positions >= q_offset.
 * All arithmetic is fp64.  Parallelism is OpenMP over independent
 * (head, query tile) units only; each unit is computed by the plain loops
 * below with no blocking or reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct oracle_shape {
    int n_tokens;
    int n_q_heads;
    int n_kv_heads;
    int head_dim;
    int block;     /* key block size == query tile size */
    int n_sample;  /* sampled queries per tile; must divide block */
    double scale;  /* softmax scale applied to q.k */
    int in_kind;   /* 0: double arrays, 1: bf16 bit patterns (uint16) */
    int q_offset;  /* position of the first query among the keys (chunked prefill):
                      q holds rows for positions q_offset .. n_tokens-1 only */
} oracle_shape;

/* ---- element access ------------------------------------------------------ */

static double bf16_bits_to_double(uint16_t b) {
    /* bf16 is the upper half of an IEEE binary32; widening is exact. */
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Element x[t, h, c] of a [n_tokens, n_heads, head_dim] array. */
static double elem(const oracle_shape* s, const void* x, int n_heads, int t, int h, int c) {
    size_t idx = ((size_t)t * (size_t)n_heads + (size_t)h) * (size_t)s->head_dim + (size_t)c;
    if (s->in_kind == 1) return bf16_bits_to_double(((const uint16_t*)x)[idx]);
    return ((const double*)x)[idx];
}

/* Query row at key position t (t >= q_offset). */
static double qelem(const oracle_shape* s, const void* q, int t, int h, int c) {
    return elem(s, q, s->n_q_heads, t - s->q_offset, h, c);
}

static int kv_head_of(const oracle_shape* s, int h) {
    int g = s->n_q_heads / s->n_kv_heads; /* query heads per KV head (GQA) */
    return h / g;
}

/* logit(h, t, u) = scale * <q_t, k_u> */
static double logit(const oracle_shape* s, const void* q, const void* k, int h, int t, int u) {
    int hk = kv_head_of(s, h);
    double acc = 0.0;
    for (int c = 0; c < s->head_dim; ++c)
        acc += qelem(s, q, t, h, c) * elem(s, k, s->n_kv_heads, u, hk, c);
    return s->scale * acc;
}

/* ---- softmax over an explicit key set ------------------------------------ */

/*
 * Softmax attention of query row t over the keys u <= t whose block is marked
 * in `visible_block` (NULL: every block).  Writes the normalised weights into
 * p[0..t] (0 for masked keys), the output into o[head_dim] and returns the
 * log-sum-exp of the scaled logits (-inf when no key is visible, o = 0 then).
 */
static double softmax_row(const oracle_shape* s, const void* q, const void* k, const void* v,
                          int h, int t, const unsigned char* visible_block, double* p, double* o) {
    const int B = s->block, d = s->head_dim, hk = kv_head_of(s, h);
    double mx = -INFINITY;
    for (int u = 0; u <= t; ++u) {
        if (visible_block && !visible_block[u / B]) { p[u] = -INFINITY; continue; }
        p[u] = logit(s, q, k, h, t, u);
        if (p[u] > mx) mx = p[u];
    }
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    if (mx == -INFINITY) {
        for (int u = 0; u <= t; ++u) p[u] = 0.0;
        return -INFINITY;
    }
    double denom = 0.0;
    for (int u = 0; u <= t; ++u) {
        p[u] = (p[u] == -INFINITY) ? 0.0 : exp(p[u] - mx);
        denom += p[u];
    }
    for (int u = 0; u <= t; ++u) {
        p[u] /= denom;
        if (p[u] == 0.0) continue;
        for (int c = 0; c < d; ++c) o[c] += p[u] * elem(s, v, s->n_kv_heads, u, hk, c);
    }
    return mx + log(denom);
}

/* ---- public: dense attention (Sec. 4.1 definition of o) ------------------- */

double oracle_dense_row(const oracle_shape* s, const void* q, const void* k, const void* v,
                        int h, int t, double* o) {
    double* p = (double*)malloc(sizeof(double) * (size_t)(t + 1));
    double lse = softmax_row(s, q, k, v, h, t, NULL, p, o);
    free(p);
    return lse;
}

/* ---- public: per-block statistics of one query row (Sec. 4.1, Eq. 4) ------ */

/*
 * For query row t of head h, and every visible block b = 0..t/B:
 *   m[b]          mass of block b
 *   vb[b*d + c]   attention-weighted mean value v_b (0 when m_b = 0)
 *   I[b]          I_b = m_b * ||v_b - o||  (0 when m_b = 0)
 * o[d] receives the dense output.
 */
void oracle_block_stats(const oracle_shape* s, const void* q, const void* k, const void* v,
                        int h, int t, double* m, double* vb, double* I, double* o) {
    const int B = s->block, d = s->head_dim, hk = kv_head_of(s, h);
    const int nb = t / B + 1;
    double* p = (double*)malloc(sizeof(double) * (size_t)(t + 1));
    softmax_row(s, q, k, v, h, t, NULL, p, o);
    for (int b = 0; b < nb; ++b) {
        double mb = 0.0;
        double* vbb = vb + (size_t)b * d;
        for (int c = 0; c < d; ++c) vbb[c] = 0.0;
        int u_end = (b + 1) * B - 1;
        if (u_end > t) u_end = t;
        for (int u = b * B; u <= u_end; ++u) {
            mb += p[u];
            for (int c = 0; c < d; ++c) vbb[c] += p[u] * elem(s, v, s->n_kv_heads, u, hk, c);
        }
        m[b] = mb;
        if (mb > 0.0) {
            double dev2 = 0.0;
            for (int c = 0; c < d; ++c) {
                vbb[c] /= mb;
                double e = vbb[c] - o[c];
                dev2 += e * e;
            }
            I[b] = mb * sqrt(dev2);
        } else {
            for (int c = 0; c < d; ++c) vbb[c] = 0.0;
            I[b] = 0.0;
        }
    }
    free(p);
}

/* ---- public: aggregated block scores per (head, tile) ----------------------- */
/* Eq. (4) scores of "Attention deletion error" Sec. 4.1, taken on 16 strided sampled
 * queries per tile and max-aggregated (the sampling and aggregation the note leaves
 * open, fixed in the file header). */

/* Offset of row (h, i) in the packed lower-triangular score arrays. */
static size_t tri_offset(int n_tiles, int h, int i) {
    return (size_t)h * ((size_t)n_tiles * (size_t)(n_tiles + 1) / 2) + (size_t)i * (size_t)(i + 1) / 2;
}

/*
 * For every listed unit (h = unit_h[u], i = unit_i[u]): over the sampled rows
 * t_j = i*B + j*(B/S), j = 0..S-1, take the max over j of I_b(t_j) and of
 * m_b(t_j) for b = 0..i, and store them at the packed offset of (h, i):
 *   Ihat[tri(h,i) + b], mhat[tri(h,i) + b].
 */
void oracle_score_units(const oracle_shape* s, const void* q, const void* k, const void* v,
                        int n_units, const int* unit_h, const int* unit_i,
                        double* Ihat, double* mhat) {
    const int B = s->block, d = s->head_dim, S = s->n_sample;
    const int T = s->n_tokens / B, stride = B / S;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < n_units; ++u) {
        const int h = unit_h[u], i = unit_i[u];
        const int nb = i + 1;
        double* m = (double*)malloc(sizeof(double) * (size_t)nb);
        double* I = (double*)malloc(sizeof(double) * (size_t)nb);
        double* vb = (double*)malloc(sizeof(double) * (size_t)nb * (size_t)d);
        double* o = (double*)malloc(sizeof(double) * (size_t)d);
        double* Ih = Ihat + tri_offset(T, h, i);
        double* mh = mhat + tri_offset(T, h, i);
        for (int b = 0; b < nb; ++b) { Ih[b] = 0.0; mh[b] = 0.0; }
        for (int j = 0; j < S; ++j) {
            int t = i * B + j * stride;
            oracle_block_stats(s, q, k, v, h, t, m, vb, I, o);
            for (int b = 0; b < nb; ++b) {
                if (I[b] > Ih[b]) Ih[b] = I[b];
                if (m[b] > mh[b]) mh[b] = m[b];
            }
        }
        free(m); free(I); free(vb); free(o);
    }
}

/* ---- public: selection ------------------------------------------------------ */
/* The Eq. (4) triangle bound of "Attention deletion error" Sec. 4.1 turned into a
 * stopping rule over the discarded candidates; ties and ascending order as in the
 * "Block-Filtered Long-Context Attention" page, Appendix "Block ordering". */

/* Ranking: larger score first, equal scores by smaller block id. */
typedef struct { double key; int id; } ranked;

static int ranked_cmp(const void* a, const void* b) {
    const ranked* x = (const ranked*)a;
    const ranked* y = (const ranked*)b;
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

static int mark_mandatory(int i, unsigned char* keep) {
    /* Sink block 0, the causal diagonal block i and the local block i-1. */
    keep[0] = 1;
    keep[i] = 1;
    if (i >= 1) keep[i - 1] = 1;
    return 0;
}

static int emit_ascending(int i, const unsigned char* keep, int* out) {
    int n = 0;
    for (int b = 0; b <= i; ++b)
        if (keep[b]) out[n++] = b;
    return n;
}

/*
 * Threshold selection for query tile i from its aggregated scores Ihat[0..i]
 * and masses mhat[0..i].  Candidates are blocks 1..i-2, ranked by
 * (Ihat desc, id asc).  With D_k the candidates ranked k, k+1, ... (those not
 * kept when the top k are kept), S_I(k) = sum_{D_k} Ihat and
 * S_m(k) = sum_{D_k} mhat, the number kept is the smallest k with
 *     S_m(k) < 1  and  S_I(k) <= tau * (1 - S_m(k)).
 * k = |Cand| always qualifies (D empty).  The kept list -- mandatory blocks and
 * the top k candidates -- is written to keep_out in ascending order; returns
 * its length.  *k_out (if non-NULL) receives k.
 */
int oracle_select_row(int i, const double* Ihat, const double* mhat, double tau,
                      int* keep_out, int* k_out) {
    unsigned char* keep = (unsigned char*)calloc((size_t)i + 1, 1);
    mark_mandatory(i, keep);
    int nc = i - 2; /* candidates 1..i-2 */
    if (nc < 0) nc = 0;
    ranked* r = (ranked*)malloc(sizeof(ranked) * (size_t)(nc > 0 ? nc : 1));
    for (int c = 0; c < nc; ++c) { r[c].key = Ihat[c + 1]; r[c].id = c + 1; }
    qsort(r, (size_t)nc, sizeof(ranked), ranked_cmp);
    /* Suffix sums over the ranked order: SI[k] = sum_{c >= k} Ihat, SM[k] likewise. */
    double* SI = (double*)malloc(sizeof(double) * (size_t)(nc + 1));
    double* SM = (double*)malloc(sizeof(double) * (size_t)(nc + 1));
    SI[nc] = 0.0; SM[nc] = 0.0;
    for (int c = nc - 1; c >= 0; --c) {
        SI[c] = SI[c + 1] + r[c].key;
        SM[c] = SM[c + 1] + mhat[r[c].id];
    }
    int kcut = nc;
    for (int kk = 0; kk <= nc; ++kk) {
        if (SM[kk] < 1.0 && SI[kk] <= tau * (1.0 - SM[kk])) { kcut = kk; break; }
    }
    for (int c = 0; c < kcut; ++c) keep[r[c].id] = 1;
    int n = emit_ascending(i, keep, keep_out);
    if (k_out) *k_out = kcut;
    free(SI); free(SM); free(r); free(keep);
    return n;
}

/*
 * Mass-only baseline (the comparison at a matched block budget in the last section
 * of "Attention deletion error"): keep the mandatory blocks and the k_free
 * candidates of largest mhat (equal masses by smaller id).  Returns the list length.
 */
int oracle_select_mass_only_row(int i, const double* mhat, int k_free, int* keep_out) {
    unsigned char* keep = (unsigned char*)calloc((size_t)i + 1, 1);
    mark_mandatory(i, keep);
    int nc = i - 2;
    if (nc < 0) nc = 0;
    if (k_free > nc) k_free = nc;
    if (k_free < 0) k_free = 0;
    ranked* r = (ranked*)malloc(sizeof(ranked) * (size_t)(nc > 0 ? nc : 1));
    for (int c = 0; c < nc; ++c) { r[c].key = mhat[c + 1]; r[c].id = c + 1; }
    qsort(r, (size_t)nc, sizeof(ranked), ranked_cmp);
    for (int c = 0; c < k_free; ++c) keep[r[c].id] = 1;
    int n = emit_ascending(i, keep, keep_out);
    free(r); free(keep);
    return n;
}

/*
 * Selection for many rows at once.  Row r = (h, i) with h = row_h[r],
 * i = row_i[r] reads Ihat/mhat at its packed offset; its list goes to
 * lists[r * n_tiles ...] (capacity n_tiles each), its length to counts[r] and
 * its k to kcut[r].
 */
void oracle_select_rows(int n_tiles, int n_rows, const int* row_h, const int* row_i,
                        const double* Ihat, const double* mhat, double tau,
                        int* lists, int* counts, int* kcut) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int r = 0; r < n_rows; ++r) {
        size_t off = tri_offset(n_tiles, row_h[r], row_i[r]);
        counts[r] = oracle_select_row(row_i[r], Ihat + off, mhat + off, tau,
                                      lists + (size_t)r * n_tiles, kcut ? kcut + r : NULL);
    }
}

/* ---- public: masked (block-sparse) attention (Sec. 4.1 definition of o~) --- */

/*
 * Softmax attention of query row t of head h restricted to the keys u <= t in
 * the listed blocks (o~ of "Attention deletion error" Sec. 4.1).  Writes o[d] and
 * returns the log-sum-exp (-inf, o = 0, when no key is visible).
 */
double oracle_masked_row(const oracle_shape* s, const void* q, const void* k, const void* v,
                         int h, int t, const int* blocks, int n_blocks, double* o) {
    const int nb = s->n_tokens / s->block;
    unsigned char* vis = (unsigned char*)calloc((size_t)nb, 1);
    for (int j = 0; j < n_blocks; ++j)
        if (blocks[j] >= 0 && blocks[j] < nb) vis[blocks[j]] = 1;
    double* p = (double*)malloc(sizeof(double) * (size_t)(t + 1));
    double lse = softmax_row(s, q, k, v, h, t, vis, p, o);
    free(p); free(vis);
    return lse;
}

/*
 * Masked attention for every query row of the listed units: the renormalised
 * output o~ of "Attention deletion error" Sec. 4.1 over each row's kept blocks.  Unit u covers
 * tile i = unit_i[u] of head h = unit_h[u]; its block list is
 * col_idx[row_ptr[r] .. row_ptr[r+1]) with r = h * n_tiles + i.  Output rows
 * go to O[(u*B + j) * d + c] and lse[u*B + j], j = 0..B-1.
 */
void oracle_masked_units(const oracle_shape* s, const void* q, const void* k, const void* v,
                         int n_units, const int* unit_h, const int* unit_i,
                         const int* row_ptr, const int* col_idx, double* O, double* lse) {
    const int B = s->block, d = s->head_dim, T = s->n_tokens / B;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < n_units; ++u) {
        const int h = unit_h[u], i = unit_i[u];
        const int r = h * T + i;
        for (int j = 0; j < B; ++j) {
            int t = i * B + j;
            lse[(size_t)u * B + j] = oracle_masked_row(s, q, k, v, h, t, col_idx + row_ptr[r],
                                                       row_ptr[r + 1] - row_ptr[r],
                                                       O + ((size_t)u * B + j) * d);
        }
    }
}

/* Dense attention (o of "Attention deletion error" Sec. 4.1) for every row of the
 * listed units (same output layout). */
void oracle_dense_units(const oracle_shape* s, const void* q, const void* k, const void* v,
                        int n_units, const int* unit_h, const int* unit_i, double* O, double* lse) {
    const int B = s->block, d = s->head_dim;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < n_units; ++u) {
        for (int j = 0; j < B; ++j) {
            int t = unit_i[u] * B + j;
            lse[(size_t)u * B + j] = oracle_dense_row(s, q, k, v, unit_h[u], t, O + ((size_t)u * B + j) * d);
        }
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- practical (estimated) scoring: pooled block statistics ----------------- */

/*
 * Practical POEM (reading note, the paragraph on Equation (6) and Appendix B):
 * cheap estimates stand in for the exact dense output and block outputs; a
 * shortlist of candidates is taken by mass, re-ordered by log mass plus w times
 * log deviation, and blocks are kept in the new order until their pooled mass
 * reaches the threshold.  No estimator is printed; the reading taken here is
 * the plainest one:
 *   q~_i = mean of the B queries of tile i,   k~_b, v~_b = means of block b,
 *   m~_b = softmax over visible b <= i of scale * <q~_i, k~_b>,
 *   o~_i = sum_b m~_b v~_b,   d~_b = || v~_b - o~_i ||.
 * For each listed unit (h, i) this writes m~ and d~ of blocks 0..i at the packed
 * offset of (h, i).  With one token per block and one query per tile the pooled
 * quantities are the exact m_b, o and || v_b - o ||.
 */
void oracle_pooled_units(const oracle_shape* s, const void* q, const void* k, const void* v,
                         int n_units, const int* unit_h, const int* unit_i, double* m_pool, double* d_pool) {
    const int B = s->block, d = s->head_dim, T = s->n_tokens / B;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < n_units; ++u) {
        const int h = unit_h[u], i = unit_i[u], hk = kv_head_of(s, h);
        const int nb = i + 1;
        double* qm = (double*)calloc((size_t)d, sizeof(double));
        double* km = (double*)calloc((size_t)nb * d, sizeof(double));
        double* vm = (double*)calloc((size_t)nb * d, sizeof(double));
        double* lg = (double*)malloc(sizeof(double) * (size_t)nb);
        double* om = (double*)calloc((size_t)d, sizeof(double));
        for (int t = i * B; t < (i + 1) * B; ++t)
            for (int c = 0; c < d; ++c) qm[c] += qelem(s, q, t, h, c) / B;
        for (int b = 0; b < nb; ++b)
            for (int t = b * B; t < (b + 1) * B; ++t)
                for (int c = 0; c < d; ++c) {
                    km[(size_t)b * d + c] += elem(s, k, s->n_kv_heads, t, hk, c) / B;
                    vm[(size_t)b * d + c] += elem(s, v, s->n_kv_heads, t, hk, c) / B;
                }
        double mx = -INFINITY;
        for (int b = 0; b < nb; ++b) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += qm[c] * km[(size_t)b * d + c];
            lg[b] = s->scale * acc;
            if (lg[b] > mx) mx = lg[b];
        }
        double den = 0.0;
        for (int b = 0; b < nb; ++b) { lg[b] = exp(lg[b] - mx); den += lg[b]; }
        double* mo = m_pool + tri_offset(T, h, i);
        double* dv = d_pool + tri_offset(T, h, i);
        for (int b = 0; b < nb; ++b) {
            mo[b] = lg[b] / den;
            for (int c = 0; c < d; ++c) om[c] += mo[b] * vm[(size_t)b * d + c];
        }
        for (int b = 0; b < nb; ++b) {
            double dev2 = 0.0;
            for (int c = 0; c < d; ++c) {
                double e = vm[(size_t)b * d + c] - om[c];
                dev2 += e * e;
            }
            dv[b] = sqrt(dev2);
        }
        free(qm); free(km); free(vm); free(lg); free(om);
    }
}

/*
 * Practical selection of tile i from pooled masses m~[0..i] and deviations
 * d~[0..i]:
 *   mandatory {0, i-1, i};
 *   stage 1: candidates 1..i-2 ranked by (m~ desc, id asc), the first
 *            ceil(rho * |Cand|) kept (rho in [0, 1]);
 *   stage 2: that shortlist reranked by (log m~ + w log d~ desc, id asc)
 *            (Equation (6) form; log 0 = -inf);
 *   keep the shortest prefix of the reranked shortlist with
 *            sum_{mandatory} m~ + sum_{prefix} m~ >= gamma
 *            (the whole shortlist when the threshold is never reached).
 * Writes the kept ids ascending; returns the count, *k_out = prefix length.
 */
static double rank_key(double m, double dv, double w) {
    double lm = (m > 0.0) ? log(m) : -INFINITY;
    double ld = (dv > 0.0) ? log(dv) : -INFINITY;
    if (lm == -INFINITY || (w > 0.0 && ld == -INFINITY)) return -INFINITY;
    return lm + w * ((w == 0.0) ? 0.0 : ld);
}

int oracle_select_practical_row(int i, const double* m_pool, const double* d_pool, double w, double gamma,
                                double rho, int* keep_out, int* k_out) {
    unsigned char* keep = (unsigned char*)calloc((size_t)i + 1, 1);
    mark_mandatory(i, keep);
    int nc = i - 2;
    if (nc < 0) nc = 0;
    ranked* r = (ranked*)malloc(sizeof(ranked) * (size_t)(nc > 0 ? nc : 1));
    for (int c = 0; c < nc; ++c) { r[c].key = m_pool[c + 1]; r[c].id = c + 1; }
    qsort(r, (size_t)nc, sizeof(ranked), ranked_cmp);
    int n1 = (int)ceil(rho * (double)nc);
    if (n1 > nc) n1 = nc;
    if (n1 < 0) n1 = 0;
    for (int c = 0; c < n1; ++c) r[c].key = rank_key(m_pool[r[c].id], d_pool[r[c].id], w);
    qsort(r, (size_t)n1, sizeof(ranked), ranked_cmp);
    double acc = 0.0;
    for (int b = 0; b <= i; ++b)
        if (keep[b]) acc += m_pool[b];
    int kcut = 0;
    while (kcut < n1 && acc < gamma) {
        acc += m_pool[r[kcut].id];
        keep[r[kcut].id] = 1;
        ++kcut;
    }
    int n = emit_ascending(i, keep, keep_out);
    if (k_out) *k_out = kcut;
    free(r); free(keep);
    return n;
}

void oracle_select_practical_rows(int n_tiles, int n_rows, const int* row_h, const int* row_i, const double* m_pool,
                                  const double* d_pool, double w, double gamma, double rho, int* lists, int* counts,
                                  int* kcut) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int rr = 0; rr < n_rows; ++rr) {
        size_t off = tri_offset(n_tiles, row_h[rr], row_i[rr]);
        counts[rr] = oracle_select_practical_row(row_i[rr], m_pool + off, d_pool + off, w, gamma, rho,
                                                 lists + (size_t)rr * n_tiles, kcut ? kcut + rr : NULL);
    }
}
