/*
 * Plain FP64 CPU oracle for Inkling2 learned-relative grouped-query attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it. It shares no code, header, table or constant with the CUDA path.
 *
 * What it computes (sources: NVIDIA NeMo AutoModel API reference pages,
 * "nemo_automodel.components.models.inkling2.flex_attention" -- class
 * Inkling2FlexAttention and its forward() parameter list -- and
 * "nemo_automodel.components.models.inkling2.attention" -- the quadratic
 * reference Inkling2Attention._eager and the sink of Inkling2Attention.forward,
 * a virtual key whose value row is zero):
 *
 *   For every batch b, query head h (kv head g = h / (Hq/Hkv)) and local query
 *   row i (global column i_g = query_offset + i), over the keys j that are
 *   allowed:
 *     allowed(i,j) = valid[b,i] && key_valid[b,j] && j <= i_g
 *                    && pos_q[b,i] - pos_k[b,j] == i_g - j      (same document)
 *                    && (W == 0 || i_g - j < W)                   (sliding window)
 *     d      = pos_q[b,i] - pos_k[b,j]
 *     z_j    = scale * <q[b,i,h,:], k[b,j,g,:]> + (d < R ? profiles[b,h,i,d] : 0)
 *     lse    = log( exp(sink[b,i,h]) + sum_j exp(z_j) )
 *     out    = sum_j exp(z_j - lse) * v[b,j,g,:]
 *   with scale = head_dim^-0.5 (Inkling2FlexAttention.scale).
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes): the sink is a virtual key with logit sink[b,i,h] and a zero value
 * row; lse includes the sink; a query row with no allowed key has out = 0 and
 * lse = sink; positions restarting per document means two tokens share one exactly
 * when their logical-position difference equals their column difference; the
 * window admits i_g - j < W (W tokens including the query itself) unless the
 * caller asks for the generic FlexAttention docstring's inclusive reading through
 * window_inclusive (only a self-test uses that).
 *
 * The backward pass is the chain rule of the formulas above, written out
 * term by term (no blocking, no recomputation tricks):
 *   P_j   = exp(z_j - lse),  p_sink = exp(sink - lse)
 *   dP_j  = <dout, v_j>,     Dv = <dout, out> - dlse
 *   dz_j  = P_j * (dP_j - Dv)
 *   dsink = -p_sink * Dv
 *   dq    = scale * sum_j dz_j k_j
 *   dk_j  = scale * sum_{i,h in g} dz_ij q_i
 *   dv_j  = sum_{i,h in g} P_ij dout_i
 *   dprofiles[b,h,i,d] += dz_j for every allowed j with d < R.
 *
 * Everything is evaluated in double precision; BF16 inputs are decoded
 * exactly by a bit shift. OpenMP parallelises over independent rows.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/*
 * ORACLE_MUTANT selects one deliberately planted mistake. It is never defined
 * in the oracle that the tests trust; the mutation self-test compiles each
 * variant separately and checks that the pins reject it.
 */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

typedef struct {
    int64_t batch, seq_q, seq_k, heads_q, heads_kv, head_dim, rel_extent;
    int64_t window;           /* 0 = no sliding window */
    int64_t query_offset;     /* global column of local query row 0 */
    int64_t window_inclusive; /* 0: i_g - j < W ; 1: i_g - j <= W (self-test only) */
} oracle_dims;

/* Exact BF16 -> double: a bfloat16 is the upper half of an IEEE float. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OpenMP threads of the parallel loops below: set (n > 0) and query. */
void oracle_set_threads(int n) {
    if (n > 0) omp_set_num_threads(n);
}
int oracle_threads(void) { return omp_get_max_threads(); }

void oracle_decode_bf16(const uint16_t* src, double* dst, int64_t n) {
    for (int64_t t = 0; t < n; ++t) dst[t] = bf16_bits_to_double(src[t]);
}

/* --- indexing helpers: all tensors are dense row-major ------------------ */
static int64_t ix_q(const oracle_dims* m, int64_t b, int64_t i, int64_t h) {
    return ((b * m->seq_q + i) * m->heads_q + h) * m->head_dim;
}
static int64_t ix_kv(const oracle_dims* m, int64_t b, int64_t j, int64_t g) {
    return ((b * m->seq_k + j) * m->heads_kv + g) * m->head_dim;
}
static int64_t ix_prof(const oracle_dims* m, int64_t b, int64_t h, int64_t i) {
    return ((b * m->heads_q + h) * m->seq_q + i) * m->rel_extent;
}
static int64_t ix_row(const oracle_dims* m, int64_t b, int64_t i, int64_t h) {
    return (b * m->seq_q + i) * m->heads_q + h; /* sink / lse layout [B,S,Hq] */
}

static int is_allowed(const oracle_dims* m, const uint8_t* valid, const uint8_t* key_valid,
                      const int32_t* pos_q, const int32_t* pos_k, int64_t b, int64_t i, int64_t j) {
    const int64_t ig = m->query_offset + i;
    if (!valid[b * m->seq_q + i]) return 0;
    if (!key_valid[b * m->seq_k + j]) return 0;
#if ORACLE_MUTANT == 9
    if (j >= ig) return 0;                                  /* planted: self excluded */
#else
    if (j > ig) return 0;                                   /* causal */
#endif
    const int64_t d = (int64_t)pos_q[b * m->seq_q + i] - (int64_t)pos_k[b * m->seq_k + j];
    if (d != ig - j) return 0;                              /* same document */
    if (m->window > 0) {
#if ORACLE_MUTANT == 4
        if (ig - j > m->window) return 0;                   /* planted: inclusive bound */
#else
        if (m->window_inclusive ? (ig - j > m->window) : (ig - j >= m->window)) return 0;
#endif
    }
    return 1;
}

/* Logit z for an allowed pair (uses the relative bias when d < R). */
static double logit(const oracle_dims* m, const double* q, const double* k, const double* prof,
                    const int32_t* pos_q, const int32_t* pos_k,
                    int64_t b, int64_t h, int64_t i, int64_t j) {
    const int64_t G = m->heads_q / m->heads_kv;
#if ORACLE_MUTANT == 5
    const int64_t g = h % m->heads_kv;                      /* planted: interleaved head groups */
#else
    const int64_t g = h / G;
#endif
#if ORACLE_MUTANT == 6
    const double scale = 1.0 / (double)m->head_dim;         /* planted: 1/D scale */
#else
    const double scale = 1.0 / sqrt((double)m->head_dim);
#endif
    const double* qr = q + ix_q(m, b, i, h);
    const double* kr = k + ix_kv(m, b, j, g);
    double dot = 0.0;
    for (int64_t c = 0; c < m->head_dim; ++c) dot += qr[c] * kr[c];
    double z = scale * dot;
#if ORACLE_MUTANT == 2
    const int64_t d = (int64_t)pos_k[b * m->seq_k + j] - (int64_t)pos_q[b * m->seq_q + i]; /* planted: sign */
#else
    const int64_t d = (int64_t)pos_q[b * m->seq_q + i] - (int64_t)pos_k[b * m->seq_k + j];
#endif
#if ORACLE_MUTANT != 1
    if (d >= 0 && d < m->rel_extent) z += prof[ix_prof(m, b, h, i) + d];
#endif
    (void)G;
    return z;
}

/* Row statistics: lse (sink included) and lse over keys only. */
static void row_lse(const oracle_dims* m, const double* q, const double* k, const double* prof,
                    const double* sink, const uint8_t* valid, const uint8_t* key_valid,
                    const int32_t* pos_q, const int32_t* pos_k,
                    int64_t b, int64_t h, int64_t i, double* lse_out, double* lse_content_out) {
    const double sg = sink[ix_row(m, b, i, h)];
    double mx = -INFINITY;
    for (int64_t j = 0; j < m->seq_k; ++j) {
        if (!is_allowed(m, valid, key_valid, pos_q, pos_k, b, i, j)) continue;
        const double z = logit(m, q, k, prof, pos_q, pos_k, b, h, i, j);
        if (z > mx) mx = z;
    }
    double zsum = 0.0; /* sum_j exp(z_j - mx) */
    if (mx > -INFINITY) {
        for (int64_t j = 0; j < m->seq_k; ++j) {
            if (!is_allowed(m, valid, key_valid, pos_q, pos_k, b, i, j)) continue;
            zsum += exp(logit(m, q, k, prof, pos_q, pos_k, b, h, i, j) - mx);
        }
    }
    const double lc = (mx > -INFINITY) ? mx + log(zsum) : -INFINITY;
    /* lse = log(exp(sink) + exp(lc)), evaluated stably */
    double l;
#if ORACLE_MUTANT == 3
    l = (lc == -INFINITY) ? sg : lc;                        /* planted: sink left out */
#else
    if (lc == -INFINITY) l = sg;
    else if (sg == -INFINITY) l = lc;
    else if (sg == INFINITY || lc == INFINITY) l = INFINITY;
    else {
        const double hi = sg > lc ? sg : lc, lo = sg > lc ? lc : sg;
        l = hi + log1p(exp(lo - hi));
    }
#endif
    *lse_out = l;
    if (lse_content_out) *lse_content_out = lc;
}

/* Forward for one (b, h, i) row. */
static void fwd_row(const oracle_dims* m, const double* q, const double* k, const double* v,
                    const double* prof, const double* sink, const uint8_t* valid,
                    const uint8_t* key_valid, const int32_t* pos_q, const int32_t* pos_k,
                    int64_t b, int64_t h, int64_t i, double* out, double* lse, double* lse_content) {
    const int64_t G = m->heads_q / m->heads_kv;
    const int64_t g = h / G;
    double l, lc;
    row_lse(m, q, k, prof, sink, valid, key_valid, pos_q, pos_k, b, h, i, &l, &lc);
    double* o = out + ix_q(m, b, i, h);
    for (int64_t c = 0; c < m->head_dim; ++c) o[c] = 0.0;
    if (isfinite(l)) {
        for (int64_t j = 0; j < m->seq_k; ++j) {
            if (!is_allowed(m, valid, key_valid, pos_q, pos_k, b, i, j)) continue;
            const double p = exp(logit(m, q, k, prof, pos_q, pos_k, b, h, i, j) - l);
            const double* vr = v + ix_kv(m, b, j, g);
            for (int64_t c = 0; c < m->head_dim; ++c) o[c] += p * vr[c];
        }
    }
    lse[ix_row(m, b, i, h)] = l;
    if (lse_content) lse_content[ix_row(m, b, i, h)] = lc;
}

static int check_dims(const oracle_dims* m) {
    if (m->batch < 0 || m->seq_q < 0 || m->seq_k < 0 || m->head_dim <= 0) return 1;
    if (m->heads_q <= 0 || m->heads_kv <= 0 || m->heads_q % m->heads_kv != 0) return 2;
    if (m->rel_extent < 0 || m->window < 0 || m->query_offset < 0) return 3;
    return 0;
}

/*
 * Forward over all rows, or over a list of flattened row ids (b*S + i)*Hq + h
 * when rows != NULL (only those rows of out / lse / lse_content are written).
 * lse_content may be NULL.
 */
int oracle_fwd_f64(const oracle_dims* m, const double* q, const double* k, const double* v,
                   const double* prof, const double* sink, const uint8_t* valid,
                   const uint8_t* key_valid, const int32_t* pos_q, const int32_t* pos_k,
                   double* out, double* lse, double* lse_content,
                   const int64_t* rows, int64_t nrows) {
    const int rc = check_dims(m);
    if (rc) return rc;
    const int64_t total = rows ? nrows : m->batch * m->seq_q * m->heads_q;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < total; ++t) {
        const int64_t r = rows ? rows[t] : t;
        const int64_t h = r % m->heads_q;
        const int64_t i = (r / m->heads_q) % m->seq_q;
        const int64_t b = r / (m->heads_q * m->seq_q);
        fwd_row(m, q, k, v, prof, sink, valid, key_valid, pos_q, pos_k, b, h, i, out, lse, lse_content);
    }
    return 0;
}

/*
 * Per-row backward quantities for one (b, h, i): writes dq row, dprofiles row,
 * dsink entry, and the row's lse and Dv (= <dout,out> - dlse) for the key pass.
 */
static void bwd_row(const oracle_dims* m, const double* q, const double* k, const double* v,
                    const double* prof, const double* sink, const uint8_t* valid,
                    const uint8_t* key_valid, const int32_t* pos_q, const int32_t* pos_k,
                    const double* dout, const double* dlse,
                    int64_t b, int64_t h, int64_t i,
                    double* dq, double* dprof, double* dsink, double* row_l, double* row_dv) {
    const int64_t D = m->head_dim;
    const int64_t G = m->heads_q / m->heads_kv;
    const int64_t g = h / G;
    const double scale = 1.0 / sqrt((double)D);
    const int64_t rid = ix_row(m, b, i, h);
    double l;
    row_lse(m, q, k, prof, sink, valid, key_valid, pos_q, pos_k, b, h, i, &l, NULL);

    /* out for this row, recomputed from the definition */
    double* o = (double*)calloc((size_t)D, sizeof(double));
    const double* go = dout + ix_q(m, b, i, h);
    if (isfinite(l)) {
        for (int64_t j = 0; j < m->seq_k; ++j) {
            if (!is_allowed(m, valid, key_valid, pos_q, pos_k, b, i, j)) continue;
            const double p = exp(logit(m, q, k, prof, pos_q, pos_k, b, h, i, j) - l);
            const double* vr = v + ix_kv(m, b, j, g);
            for (int64_t c = 0; c < D; ++c) o[c] += p * vr[c];
        }
    }
    double dv_row = 0.0;
    for (int64_t c = 0; c < D; ++c) dv_row += go[c] * o[c];
    if (dlse) dv_row -= dlse[rid];
    free(o);

    double* dqr = dq ? dq + ix_q(m, b, i, h) : NULL;
    double* dpr = dprof ? dprof + ix_prof(m, b, h, i) : NULL;
    if (dqr) for (int64_t c = 0; c < D; ++c) dqr[c] = 0.0;
    if (dpr) for (int64_t d = 0; d < m->rel_extent; ++d) dpr[d] = 0.0;
    if (isfinite(l)) {
        for (int64_t j = 0; j < m->seq_k; ++j) {
            if (!is_allowed(m, valid, key_valid, pos_q, pos_k, b, i, j)) continue;
            const double p = exp(logit(m, q, k, prof, pos_q, pos_k, b, h, i, j) - l);
            const double* vr = v + ix_kv(m, b, j, g);
            const double* kr = k + ix_kv(m, b, j, g);
            double dp = 0.0;
            for (int64_t c = 0; c < D; ++c) dp += go[c] * vr[c];
#if ORACLE_MUTANT == 7
            const double dz = p * (dp + dv_row);            /* planted: sign of the softmax term */
#else
            const double dz = p * (dp - dv_row);
#endif
            if (dqr) for (int64_t c = 0; c < D; ++c) dqr[c] += scale * dz * kr[c];
            const int64_t d = (int64_t)pos_q[b * m->seq_q + i] - (int64_t)pos_k[b * m->seq_k + j];
#if ORACLE_MUTANT == 8
            if (dpr && d + 1 < m->rel_extent) dpr[d + 1] += dz;   /* planted: off-by-one index */
#else
            if (dpr && d >= 0 && d < m->rel_extent) dpr[d] += dz;
#endif
        }
    }
    /* sink probability; an infinite sink that dominates the row has p = 1 */
    double ps = 0.0;
    if (isfinite(l)) ps = exp(sink[rid] - l);
    else if (l == INFINITY && sink[rid] == INFINITY) ps = 1.0;
    if (dsink) dsink[rid] = -ps * dv_row;
    if (row_l) row_l[rid] = l;
    if (row_dv) row_dv[rid] = dv_row;
}

/* dk / dv for key column (b, j, g), given every row's lse and Dv. */
static void bwd_key(const oracle_dims* m, const double* q, const double* k, const double* v,
                    const double* prof, const uint8_t* valid, const uint8_t* key_valid,
                    const int32_t* pos_q, const int32_t* pos_k, const double* dout,
                    const double* row_l, const double* row_dv,
                    int64_t b, int64_t j, int64_t g, double* dk, double* dv) {
    const int64_t D = m->head_dim;
    const int64_t G = m->heads_q / m->heads_kv;
    const double scale = 1.0 / sqrt((double)D);
    double* dkr = dk + ix_kv(m, b, j, g);
    double* dvr = dv + ix_kv(m, b, j, g);
    const double* vr = v + ix_kv(m, b, j, g);
    for (int64_t c = 0; c < D; ++c) { dkr[c] = 0.0; dvr[c] = 0.0; }
    for (int64_t h = g * G; h < (g + 1) * G; ++h) {
        for (int64_t i = 0; i < m->seq_q; ++i) {
            if (!is_allowed(m, valid, key_valid, pos_q, pos_k, b, i, j)) continue;
            const int64_t rid = ix_row(m, b, i, h);
            const double l = row_l[rid];
            if (!isfinite(l)) continue;
            const double p = exp(logit(m, q, k, prof, pos_q, pos_k, b, h, i, j) - l);
            const double* go = dout + ix_q(m, b, i, h);
            const double* qr = q + ix_q(m, b, i, h);
            double dp = 0.0;
            for (int64_t c = 0; c < D; ++c) dp += go[c] * vr[c];
            const double dz = p * (dp - row_dv[rid]);
            for (int64_t c = 0; c < D; ++c) {
#if ORACLE_MUTANT == 10
                dkr[c] += dz * qr[c];                       /* planted: scale dropped in dk */
#else
                dkr[c] += scale * dz * qr[c];
#endif
                dvr[c] += p * go[c];
            }
        }
    }
}

/* Full backward: dq, dk, dv, dprofiles, dsink (all dense, all written). */
int oracle_bwd_f64(const oracle_dims* m, const double* q, const double* k, const double* v,
                   const double* prof, const double* sink, const uint8_t* valid,
                   const uint8_t* key_valid, const int32_t* pos_q, const int32_t* pos_k,
                   const double* dout, const double* dlse,
                   double* dq, double* dk, double* dv, double* dprof, double* dsink) {
    const int rc = check_dims(m);
    if (rc) return rc;
    const int64_t nrow = m->batch * m->seq_q * m->heads_q;
    double* row_l = (double*)malloc((size_t)(nrow > 0 ? nrow : 1) * sizeof(double));
    double* row_dv = (double*)malloc((size_t)(nrow > 0 ? nrow : 1) * sizeof(double));
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrow; ++r) {
        const int64_t h = r % m->heads_q;
        const int64_t i = (r / m->heads_q) % m->seq_q;
        const int64_t b = r / (m->heads_q * m->seq_q);
        bwd_row(m, q, k, v, prof, sink, valid, key_valid, pos_q, pos_k, dout, dlse,
                b, h, i, dq, dprof, dsink, row_l, row_dv);
    }
    const int64_t nkey = m->batch * m->seq_k * m->heads_kv;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nkey; ++r) {
        const int64_t g = r % m->heads_kv;
        const int64_t j = (r / m->heads_kv) % m->seq_k;
        const int64_t b = r / (m->heads_kv * m->seq_k);
        bwd_key(m, q, k, v, prof, valid, key_valid, pos_q, pos_k, dout, row_l, row_dv,
                b, j, g, dk, dv);
    }
    free(row_l);
    free(row_dv);
    return 0;
}

/*
 * Sampled backward for large shapes: the per-row outputs (dq, dprofiles,
 * dsink) for the listed query rows, and dk / dv for the listed key columns
 * (flattened (b*Skv + j)*Hkv + g). Row statistics needed by a key column are
 * computed for exactly the rows that can see it. Outputs are written only at
 * the listed rows / keys.
 */
int oracle_bwd_sampled_f64(const oracle_dims* m, const double* q, const double* k, const double* v,
                           const double* prof, const double* sink, const uint8_t* valid,
                           const uint8_t* key_valid, const int32_t* pos_q, const int32_t* pos_k,
                           const double* dout, const double* dlse,
                           const int64_t* rows, int64_t nrows, const int64_t* keys, int64_t nkeys,
                           double* dq, double* dprof, double* dsink, double* dk, double* dv) {
    const int rc = check_dims(m);
    if (rc) return rc;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < nrows; ++t) {
        const int64_t r = rows[t];
        const int64_t h = r % m->heads_q;
        const int64_t i = (r / m->heads_q) % m->seq_q;
        const int64_t b = r / (m->heads_q * m->seq_q);
        bwd_row(m, q, k, v, prof, sink, valid, key_valid, pos_q, pos_k, dout, dlse,
                b, h, i, dq, dprof, dsink, NULL, NULL);
    }
    if (nkeys == 0) return 0;
    const int64_t nrow = m->batch * m->seq_q * m->heads_q;
    double* row_l = (double*)malloc((size_t)nrow * sizeof(double));
    double* row_dv = (double*)malloc((size_t)nrow * sizeof(double));
    uint8_t* need = (uint8_t*)calloc((size_t)nrow, 1);
    for (int64_t t = 0; t < nkeys; ++t) {
        const int64_t r = keys[t];
        const int64_t g = r % m->heads_kv;
        const int64_t j = (r / m->heads_kv) % m->seq_k;
        const int64_t b = r / (m->heads_kv * m->seq_k);
        const int64_t G = m->heads_q / m->heads_kv;
        for (int64_t i = 0; i < m->seq_q; ++i) {
            if (!is_allowed(m, valid, key_valid, pos_q, pos_k, b, i, j)) continue;
            for (int64_t h = g * G; h < (g + 1) * G; ++h) need[ix_row(m, b, i, h)] = 1;
        }
    }
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrow; ++r) {
        if (!need[r]) continue;
        const int64_t h = r % m->heads_q;
        const int64_t i = (r / m->heads_q) % m->seq_q;
        const int64_t b = r / (m->heads_q * m->seq_q);
        bwd_row(m, q, k, v, prof, sink, valid, key_valid, pos_q, pos_k, dout, dlse,
                b, h, i, NULL, NULL, NULL, row_l, row_dv);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < nkeys; ++t) {
        const int64_t r = keys[t];
        const int64_t g = r % m->heads_kv;
        const int64_t j = (r / m->heads_kv) % m->seq_k;
        const int64_t b = r / (m->heads_kv * m->seq_k);
        bwd_key(m, q, k, v, prof, valid, key_valid, pos_q, pos_k, dout, row_l, row_dv,
                b, j, g, dk, dv);
    }
    free(row_l);
    free(row_dv);
    free(need);
    return 0;
}
