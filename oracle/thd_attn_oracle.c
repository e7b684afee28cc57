/*
 * CPU ORACLE -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 reference for the packed-THD sliding-window GQA attention
 * forward.  Only the tests, the smoke check and the benchmark's CPU-baseline /
 * reference arm may load it.  It shares no code with the CUDA path.
 *
 * What it computes (restated from the NeMo AutoModel API pages):
 *
 *   Packed THD tensors -- "muse_spark.magi_cp", MuseMagiPlan.attention
 *   (query/key/value parameters): q[T, Hq, D], k[T, Hkv, D], v[T, Hkv, D];
 *   documents delimited by cu_seqlens, "CPU int32 padded document boundaries
 *   [documents + 1]" (_build_magi_plan, cu_seqlens parameter).
 *
 *   Visible keys -- "flint.magi", FlintMagiPlan.attention, window parameter:
 *   the window counts the current token, zero means full causal.  For a query
 *   i of document [s, e):   V(i) = { j : s <= j <= i, and W == 0 or j > i - W }.
 *
 *   GQA -- "muse_glimmer.model", repeat_kv: each of the Hkv key/value heads is
 *   repeated Hq/Hkv times to reach the query-head count, so query head h reads
 *   kv head g = h / (Hq/Hkv).
 *
 *   Scores -- MuseMagiPlan.attention, scale parameter:
 *   s_ij = scale * sum_c q[i,h,c] * k[j,g,c].
 *
 *   Sink -- FlintMagiPlan.attention, sink parameter: one fp32 learned logit per
 *   query head that enters the softmax denominator only (it has no value row):
 *   Z = sum_{j in V(i)} exp(s_ij) + exp(sink_h);
 *   out[i,h,:] = sum_{j in V(i)} exp(s_ij) v[j,g,:] / Z;   lse[i,h] = ln Z.
 *
 * Readings where the pages leave a step open: the sink is compared unscaled
 * with the scaled scores; lse is the natural log and includes the sink term;
 * a row with an empty key set gives out = 0 and lse = -inf (or the sink).
 *
 * The max-shift below is only for range safety (the exponentials are taken
 * relative to the row maximum); it does not change the result in exact
 * arithmetic.  Parallelised over (token, head) rows with OpenMP; no other
 * reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F64 = 0, ORACLE_BF16 = 1 };

static double load_elem(const void *base, int64_t idx, int dtype) {
    if (dtype == ORACLE_F64) return ((const double *)base)[idx];
    uint32_t u = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Document containing token i: the d with cu[d] <= i < cu[d+1] (binary search). */
static int find_doc(const int32_t *cu, int n_docs, int64_t i) {
    int lo = 0, hi = n_docs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if ((int64_t)cu[mid] <= i) lo = mid; else hi = mid - 1;
    }
    while (lo < n_docs - 1 && (int64_t)cu[lo + 1] <= i) lo++; /* skip empty docs */
    return lo;
}

static int check_args(const int32_t *cu, int n_docs, int Hq, int Hkv, int D, int window) {
    if (n_docs < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || window < 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (cu == NULL) return -1;
    if (cu[0] != 0) return -1;
    for (int d = 0; d < n_docs; d++)
        if (cu[d + 1] < cu[d]) return -1;
    return 0;
}

/* One output row (token i, query head h).  out_row has D entries. */
static void attend_row(const void *q, const void *k, const void *v, int dtype,
                       const int32_t *cu, int n_docs, int Hq, int Hkv, int D,
                       int window, double scale, const float *sinks,
                       int64_t i, int h, double *out_row, double *lse_out) {
    const int G = Hq / Hkv;
    const int g = h / G;                       /* repeat_kv: contiguous repeats */
    const int d = find_doc(cu, n_docs, i);
    const int64_t s = cu[d];
    int64_t lo = s;                            /* j >= s */
    if (window > 0 && i - window + 1 > lo) lo = i - window + 1; /* j > i - W */
    const int64_t n = i - lo + 1;              /* keys lo..i inclusive */

    double *sc = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    double m = -INFINITY;
    for (int64_t j = lo; j <= i; j++) {
        double acc = 0.0;
        for (int c = 0; c < D; c++)
            acc += load_elem(q, (i * Hq + h) * (int64_t)D + c, dtype) *
                   load_elem(k, (j * Hkv + g) * (int64_t)D + c, dtype);
        sc[j - lo] = scale * acc;
        if (sc[j - lo] > m) m = sc[j - lo];
    }
    const int has_sink = sinks != NULL;
    const double sink = has_sink ? (double)sinks[h] : -INFINITY;
    if (has_sink && sink > m) m = sink;

    for (int c = 0; c < D; c++) out_row[c] = 0.0;
    if (m == -INFINITY) {                      /* empty key set, no sink */
        *lse_out = -INFINITY;
        free(sc);
        return;
    }
    double Z = has_sink ? exp(sink - m) : 0.0;
    for (int64_t j = lo; j <= i; j++) {
        const double w = exp(sc[j - lo] - m);
        Z += w;
        for (int c = 0; c < D; c++)
            out_row[c] += w * load_elem(v, (j * Hkv + g) * (int64_t)D + c, dtype);
    }
    for (int c = 0; c < D; c++) out_row[c] /= Z;
    *lse_out = m + log(Z);
    free(sc);
}

/*
 * Full forward: out[T, Hq, D] and lse[T, Hq] in fp64.
 * q/k/v are fp64 (dtype 0) or raw bf16 bit patterns (dtype 1).
 * sinks may be NULL.  Returns 0, or -1 on invalid arguments.
 */
int oracle_thd_attn(const void *q, const void *k, const void *v, int dtype,
                    const int32_t *cu_seqlens, int n_docs, int Hq, int Hkv, int D,
                    int window, double scale, const float *sinks,
                    double *out, double *lse) {
    if (check_args(cu_seqlens, n_docs, Hq, Hkv, D, window)) return -1;
    const int64_t T = n_docs > 0 ? cu_seqlens[n_docs] : 0;
    const int64_t rows = T * Hq;
#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t r = 0; r < rows; r++) {
        const int64_t i = r / Hq;
        const int h = (int)(r % Hq);
        attend_row(q, k, v, dtype, cu_seqlens, n_docs, Hq, Hkv, D, window, scale,
                   sinks, i, h, out + r * D, lse + r);
    }
    return 0;
}

/*
 * Selected rows only: rows[2*r] = token, rows[2*r+1] = query head.
 * out[n_rows, D], lse[n_rows].  Used for sampled checks of full-size packs.
 */
int oracle_thd_attn_rows(const void *q, const void *k, const void *v, int dtype,
                         const int32_t *cu_seqlens, int n_docs, int Hq, int Hkv, int D,
                         int window, double scale, const float *sinks,
                         const int64_t *rows, int64_t n_rows, double *out, double *lse) {
    if (check_args(cu_seqlens, n_docs, Hq, Hkv, D, window)) return -1;
    const int64_t T = n_docs > 0 ? cu_seqlens[n_docs] : 0;
    for (int64_t r = 0; r < n_rows; r++)
        if (rows[2 * r] < 0 || rows[2 * r] >= T || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= Hq)
            return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; r++)
        attend_row(q, k, v, dtype, cu_seqlens, n_docs, Hq, Hkv, D, window, scale, sinks,
                   rows[2 * r], (int)rows[2 * r + 1], out + r * D, lse + r);
    return 0;
}

/*
 * ------------------------------------------------------------------------
 * Backward.  The pages train through this attention (the Magi plans serve
 * activation-checkpointed layers, "muse_spark.magi_cp" and "flint.magi"), so
 * the adjacent step is its gradient.  It is the plain derivative of the
 * forward above; with P_ij = exp(s_ij - lse_i) (the sink's share is
 * P_sink,i = exp(sink_h - lse_i)) and dO = dL/d out:
 *
 *   D_i      = sum_c dO[i,h,c] * out[i,h,c]
 *   dP_ij    = sum_c dO[i,h,c] * v[j,g,c]
 *   dS_ij    = P_ij * (dP_ij - D_i)                (gradient of the score s_ij)
 *   dq[i,h]  = scale * sum_{j in V(i)} dS_ij * k[j,g]
 *   dk[j,g]  = scale * sum_{h in g} sum_{i : j in V(i)} dS_ij * q[i,h]
 *   dv[j,g]  = sum_{h in g} sum_{i : j in V(i)} P_ij * dO[i,h]
 *   dsink[h] = - sum_i P_sink,i * D_i              (the sink has no value row)
 *
 * The key heads collect the gradients of all Hq/Hkv query heads that read
 * them (the transpose of repeat_kv).
 * ------------------------------------------------------------------------
 */

/* Scores, lse and P for row (i, h); keys lo..i.  Returns the key count. */
static int64_t row_probs(const void *q, const void *k, int dtype, int Hq, int Hkv, int D,
                         double scale, const float *sinks, int64_t i, int h, int g,
                         int64_t lo, double *p, double *lse_out, double *psink_out) {
    const int64_t n = i - lo + 1;
    double m = -INFINITY;
    for (int64_t j = lo; j <= i; j++) {
        double acc = 0.0;
        for (int c = 0; c < D; c++)
            acc += load_elem(q, (i * Hq + h) * (int64_t)D + c, dtype) *
                   load_elem(k, (j * Hkv + g) * (int64_t)D + c, dtype);
        p[j - lo] = scale * acc;
        if (p[j - lo] > m) m = p[j - lo];
    }
    const double sink = sinks != NULL ? (double)sinks[h] : -INFINITY;
    if (sink > m) m = sink;
    double Z = sinks != NULL ? exp(sink - m) : 0.0;
    for (int64_t j = 0; j < n; j++) Z += exp(p[j] - m);
    const double lse = m + log(Z);
    for (int64_t j = 0; j < n; j++) p[j] = exp(p[j] - lse);
    *lse_out = lse;
    *psink_out = sinks != NULL ? exp(sink - lse) : 0.0;
    return n;
}

/* Lowest visible key of query i in a document starting at s. */
static int64_t first_key(int64_t i, int64_t s, int window) {
    const int64_t w_lo = i - window + 1;  /* j > i - W */
    return (window > 0 && w_lo > s) ? w_lo : s;
}

/* All gradients of document [s, e) for kv head g; dsink_part[G] collects the
 * sink gradients of the group's query heads. */
static void bwd_doc_group(const void *q, const void *k, const void *v, const void *dout,
                          int dtype, int Hq, int Hkv, int D, int window, double scale,
                          const float *sinks, int64_t s, int64_t e, int g,
                          double *dq, double *dk, double *dv, double *dsink_part) {
    const int G = Hq / Hkv;
    double *p = (double *)malloc((size_t)(e - s > 0 ? e - s : 1) * sizeof(double));
    double *o = (double *)malloc((size_t)D * sizeof(double));
    for (int hh = 0; hh < G; hh++) {
        const int h = g * G + hh;
        for (int64_t i = s; i < e; i++) {
            const int64_t lo = first_key(i, s, window);
            double lse, psink;
            const int64_t n = row_probs(q, k, dtype, Hq, Hkv, D, scale, sinks, i, h, g, lo,
                                        p, &lse, &psink);
            for (int c = 0; c < D; c++) o[c] = 0.0;
            for (int64_t j = lo; j <= i; j++)
                for (int c = 0; c < D; c++)
                    o[c] += p[j - lo] * load_elem(v, (j * Hkv + g) * (int64_t)D + c, dtype);
            double Di = 0.0;
            for (int c = 0; c < D; c++)
                Di += load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype) * o[c];
            dsink_part[hh] -= psink * Di;
            for (int64_t j = lo; j <= i; j++) {
                double dP = 0.0;
                for (int c = 0; c < D; c++)
                    dP += load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype) *
                          load_elem(v, (j * Hkv + g) * (int64_t)D + c, dtype);
                const double dS = p[j - lo] * (dP - Di);
                for (int c = 0; c < D; c++) {
                    dq[(i * Hq + h) * (int64_t)D + c] +=
                        scale * dS * load_elem(k, (j * Hkv + g) * (int64_t)D + c, dtype);
                    dk[(j * Hkv + g) * (int64_t)D + c] +=
                        scale * dS * load_elem(q, (i * Hq + h) * (int64_t)D + c, dtype);
                    dv[(j * Hkv + g) * (int64_t)D + c] +=
                        p[j - lo] * load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype);
                }
            }
            (void)n;
        }
    }
    free(o);
    free(p);
}

/*
 * Full backward in fp64: dq[T, Hq, D], dk/dv[T, Hkv, D], dsink[Hq] (dsink may
 * be NULL when sinks is NULL).  q/k/v/dout share one dtype (fp64 or bf16
 * bits).  Parallel over (document, kv head) pairs, whose dk/dv/dq rows are
 * disjoint.  Returns 0, or -1 on invalid arguments.
 */
int oracle_thd_attn_bwd(const void *q, const void *k, const void *v, const void *dout, int dtype,
                        const int32_t *cu_seqlens, int n_docs, int Hq, int Hkv, int D,
                        int window, double scale, const float *sinks,
                        double *dq, double *dk, double *dv, double *dsink) {
    if (check_args(cu_seqlens, n_docs, Hq, Hkv, D, window)) return -1;
    const int64_t T = n_docs > 0 ? cu_seqlens[n_docs] : 0;
    const int G = Hq / Hkv;
    memset(dq, 0, (size_t)(T * Hq * D) * sizeof(double));
    memset(dk, 0, (size_t)(T * Hkv * D) * sizeof(double));
    memset(dv, 0, (size_t)(T * Hkv * D) * sizeof(double));
    if (dsink) memset(dsink, 0, (size_t)Hq * sizeof(double));
    const int64_t units = (int64_t)n_docs * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; u++) {
        const int d = (int)(u / Hkv), g = (int)(u % Hkv);
        double *part = (double *)calloc((size_t)G, sizeof(double));
        bwd_doc_group(q, k, v, dout, dtype, Hq, Hkv, D, window, scale, sinks,
                      cu_seqlens[d], cu_seqlens[d + 1], g, dq, dk, dv, part);
        if (dsink) {
            for (int hh = 0; hh < G; hh++) {
#pragma omp atomic
                dsink[g * G + hh] += part[hh];
            }
        }
        free(part);
    }
    return 0;
}

/*
 * dq for selected (token, query head) rows only (rows[2r], rows[2r+1]):
 * each needs just its own row of P.  dq_rows[n_rows, D].
 */
int oracle_thd_attn_bwd_q_rows(const void *q, const void *k, const void *v, const void *dout,
                               int dtype, const int32_t *cu_seqlens, int n_docs, int Hq, int Hkv,
                               int D, int window, double scale, const float *sinks,
                               const int64_t *rows, int64_t n_rows, double *dq_rows) {
    if (check_args(cu_seqlens, n_docs, Hq, Hkv, D, window)) return -1;
    const int64_t T = n_docs > 0 ? cu_seqlens[n_docs] : 0;
    for (int64_t r = 0; r < n_rows; r++)
        if (rows[2 * r] < 0 || rows[2 * r] >= T || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= Hq)
            return -1;
    const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; r++) {
        const int64_t i = rows[2 * r];
        const int h = (int)rows[2 * r + 1], g = h / G;
        const int64_t s = cu_seqlens[find_doc(cu_seqlens, n_docs, i)];
        const int64_t lo = first_key(i, s, window);
        double *p = (double *)malloc((size_t)(i - lo + 1) * sizeof(double));
        double *o = (double *)calloc((size_t)D, sizeof(double));
        double lse, psink;
        row_probs(q, k, dtype, Hq, Hkv, D, scale, sinks, i, h, g, lo, p, &lse, &psink);
        for (int64_t j = lo; j <= i; j++)
            for (int c = 0; c < D; c++)
                o[c] += p[j - lo] * load_elem(v, (j * Hkv + g) * (int64_t)D + c, dtype);
        double Di = 0.0;
        for (int c = 0; c < D; c++) Di += load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype) * o[c];
        double *out = dq_rows + r * D;
        for (int c = 0; c < D; c++) out[c] = 0.0;
        for (int64_t j = lo; j <= i; j++) {
            double dP = 0.0;
            for (int c = 0; c < D; c++)
                dP += load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype) *
                      load_elem(v, (j * Hkv + g) * (int64_t)D + c, dtype);
            const double dS = p[j - lo] * (dP - Di);
            for (int c = 0; c < D; c++)
                out[c] += scale * dS * load_elem(k, (j * Hkv + g) * (int64_t)D + c, dtype);
        }
        free(o);
        free(p);
    }
    return 0;
}

/*
 * dk and dv for selected (key token, kv head) rows only: rows[2r] = key j,
 * rows[2r+1] = kv head g.  By the definition above,
 *   dk[j,g] = scale * sum_{h in g} sum_{i : j in V(i)} dS_ij q[i,h],
 *   dv[j,g] =         sum_{h in g} sum_{i : j in V(i)} P_ij dO[i,h],
 * and the queries that see key j of document [s, e) are i in [j, e) with
 * (W == 0 or i < j + W).  Each term needs the row quantities lse_i and D_i
 * of its query row (i, h), which depend on the whole row; they are computed
 * once per distinct row first (same formulas as row_probs and D_i above),
 * then the per-pair terms are summed.  dk_rows, dv_rows: [n_rows, D].
 */
static int64_t last_query(int64_t j, int64_t e, int window) {
    /* one past the last query that sees key j */
    return (window > 0 && j + window < e) ? j + window : e;
}

int oracle_thd_attn_bwd_kv_rows(const void *q, const void *k, const void *v, const void *dout,
                                int dtype, const int32_t *cu_seqlens, int n_docs, int Hq,
                                int Hkv, int D, int window, double scale, const float *sinks,
                                const int64_t *rows, int64_t n_rows, double *dk_rows,
                                double *dv_rows) {
    if (check_args(cu_seqlens, n_docs, Hq, Hkv, D, window)) return -1;
    const int64_t T = n_docs > 0 ? cu_seqlens[n_docs] : 0;
    for (int64_t r = 0; r < n_rows; r++)
        if (rows[2 * r] < 0 || rows[2 * r] >= T || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= Hkv)
            return -1;
    const int G = Hq / Hkv;
    /* 1. mark the query rows (i, h) the requested keys need */
    unsigned char *need = (unsigned char *)calloc((size_t)(T * Hq > 0 ? T * Hq : 1), 1);
    for (int64_t r = 0; r < n_rows; r++) {
        const int64_t j = rows[2 * r];
        const int g = (int)rows[2 * r + 1];
        const int d = find_doc(cu_seqlens, n_docs, j);
        const int64_t e = cu_seqlens[d + 1];
        for (int64_t i = j; i < last_query(j, e, window); i++)
            for (int hh = 0; hh < G; hh++) need[i * Hq + g * G + hh] = 1;
    }
    int64_t n_need = 0;
    for (int64_t x = 0; x < T * Hq; x++) n_need += need[x];
    int64_t *list = (int64_t *)malloc((size_t)(n_need > 0 ? n_need : 1) * sizeof(int64_t));
    int64_t *slot = (int64_t *)malloc((size_t)(T * Hq > 0 ? T * Hq : 1) * sizeof(int64_t));
    n_need = 0;
    for (int64_t x = 0; x < T * Hq; x++) {
        slot[x] = -1;
        if (need[x]) { slot[x] = n_need; list[n_need++] = x; }
    }
    /* 2. lse_i and D_i = sum_c dO[i,h,c] out[i,h,c] of every needed row */
    double *lse = (double *)malloc((size_t)(n_need > 0 ? n_need : 1) * sizeof(double));
    double *Dv = (double *)malloc((size_t)(n_need > 0 ? n_need : 1) * sizeof(double));
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t u = 0; u < n_need; u++) {
        const int64_t i = list[u] / Hq;
        const int h = (int)(list[u] % Hq), g = h / G;
        const int64_t s = cu_seqlens[find_doc(cu_seqlens, n_docs, i)];
        const int64_t lo = first_key(i, s, window);
        double *p = (double *)malloc((size_t)(i - lo + 1) * sizeof(double));
        double *o = (double *)calloc((size_t)D, sizeof(double));
        double psink;
        row_probs(q, k, dtype, Hq, Hkv, D, scale, sinks, i, h, g, lo, p, &lse[u], &psink);
        for (int64_t jj = lo; jj <= i; jj++)
            for (int c = 0; c < D; c++)
                o[c] += p[jj - lo] * load_elem(v, (jj * Hkv + g) * (int64_t)D + c, dtype);
        double Di = 0.0;
        for (int c = 0; c < D; c++) Di += load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype) * o[c];
        Dv[u] = Di;
        free(o);
        free(p);
    }
    /* 3. the sums over (h, i) for each requested key row */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; r++) {
        const int64_t j = rows[2 * r];
        const int g = (int)rows[2 * r + 1];
        const int d = find_doc(cu_seqlens, n_docs, j);
        const int64_t e = cu_seqlens[d + 1];
        double *dk_out = dk_rows + r * D, *dv_out = dv_rows + r * D;
        for (int c = 0; c < D; c++) { dk_out[c] = 0.0; dv_out[c] = 0.0; }
        for (int hh = 0; hh < G; hh++) {
            const int h = g * G + hh;
            for (int64_t i = j; i < last_query(j, e, window); i++) {
                const int64_t u = slot[i * Hq + h];
                double sc = 0.0, dP = 0.0;
                for (int c = 0; c < D; c++) {
                    sc += load_elem(q, (i * Hq + h) * (int64_t)D + c, dtype) *
                          load_elem(k, (j * Hkv + g) * (int64_t)D + c, dtype);
                    dP += load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype) *
                          load_elem(v, (j * Hkv + g) * (int64_t)D + c, dtype);
                }
                const double P = exp(scale * sc - lse[u]);
                const double dS = P * (dP - Dv[u]);
                for (int c = 0; c < D; c++) {
                    dk_out[c] += scale * dS * load_elem(q, (i * Hq + h) * (int64_t)D + c, dtype);
                    dv_out[c] += P * load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype);
                }
            }
        }
    }
    free(Dv);
    free(lse);
    free(slot);
    free(list);
    free(need);
    return 0;
}

/* Threads OpenMP would use for the calls above. */
int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
