/*
 * SOCKET oracle: a plain, slow, fp64 CPU statement of the decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library and must never be used as a
 * fallback for it.
 *
 * Sources (both pages summarise arXiv 2602.06283):
 *   [ES] "Resumen Técnico: SOCKET - Estimador de Núcleo de Colisión Suave para
 *        Atención Escasa" (gist.science/es/paper/2602.06283), section
 *        "Metodología: SOCKET", sub-section "Mecanismo Central: LSH Suave",
 *        steps 1-4.
 *   [DE] "SOCKET: SOft Collision Kernel EsTimator for Sparse Attention"
 *        (gist.science/de/paper/2602.06283), part "Technische Zusammenfassung",
 *        section "Methodik: SOCKET", sub-section "Kernmechanismus: Soft LSH".
 *
 * The pages leave the exact soft hash open ("a temperature-controlled softmax
 * over the query's projections on random hyperplanes").  The reading used here:
 * z_l = W_l q / ||q||, and p_l(b) = softmax over all 2^P sign patterns s_b of
 * <s_b, z_l> / tau, where s_{b,p} = +1 if bit p of b is set and -1 otherwise.
 * This file evaluates that softmax explicitly over all 2^P patterns; it never
 * uses the factorised product-of-sigmoids form.
 *
 * Everything is computed in double precision.  Stored inputs (fp32 or bf16)
 * are widened exactly before use.  Loops follow the definitions literally: no
 * blocking, no fusion, no reordering beyond what the definitions state.
 * Independent units (keys in the hash, (batch, kv-head) units in the decode)
 * run in parallel under OpenMP; the arithmetic inside a unit is sequential.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Element types of stored tensors. */
enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F64 = 2 };

/* Exact widening of one stored element to double. */
static double load_elem(const void* base, int dtype, int64_t i)
{
    if (dtype == ORACLE_F64) return ((const double*)base)[i];
    if (dtype == ORACLE_F32) return (double)((const float*)base)[i];
    /* bf16: the upper 16 bits of an IEEE binary32 value. */
    uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Step 1, prefill hashing ([ES] step 1 "Pre-cálculo (Prellenado)"; [DE]
 * "Vorverarbeitung (Prefill)"): every key goes into L independent tables by
 * random projection, one bucket id per table; the value-vector norm is cached.
 *
 *   y_{l,p}(k) = <W_{l,p}, k>                 (W: [L][P][d], doubles)
 *   id_l(k)    = sum_p [y_{l,p}(k) > 0] * 2^p (bit p <-> hyperplane p)
 *   vnorm(k)   = ||v||_2
 *   margin(k)  = min_{l,p} |y_{l,p}(k)| / ||k||  (0 when ||k|| = 0)
 *
 * K, V: n rows of d stored elements (dtype kv_dtype), row-major.
 * ids: [L][n] (table-major), vnorm: [n], margin: [n] (may be NULL).
 */
void oracle_hash(const void* K, const void* V, int kv_dtype, int64_t n, int d,
                 const double* W, int L, int P,
                 uint8_t* ids, double* vnorm, double* margin)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) {
        double kk = 0.0;
        for (int j = 0; j < d; ++j) {
            double kj = load_elem(K, kv_dtype, i * d + j);
            kk += kj * kj;
        }
        double knorm = sqrt(kk);
        double smallest = INFINITY;
        for (int l = 0; l < L; ++l) {
            unsigned id = 0;
            for (int p = 0; p < P; ++p) {
                const double* w = W + ((int64_t)l * P + p) * d;
                double y = 0.0;
                for (int j = 0; j < d; ++j) y += w[j] * load_elem(K, kv_dtype, i * d + j);
                if (y > 0.0) id |= 1u << p;
                if (fabs(y) < smallest) smallest = fabs(y);
            }
            ids[(int64_t)l * n + i] = (uint8_t)id;
        }
        double vv = 0.0;
        for (int j = 0; j < d; ++j) {
            double vj = load_elem(V, kv_dtype, i * d + j);
            vv += vj * vj;
        }
        vnorm[i] = sqrt(vv);
        if (margin) margin[i] = knorm > 0.0 ? smallest / knorm : 0.0;
    }
}

/*
 * Step 2, soft bucket assignment ([ES] step 2 "Asignación Suave
 * (Decodificación)"; [DE] "Weiche Zuweisung (Decoding)"): the query induces a
 * probability distribution over all buckets of each table, via a
 * temperature-controlled softmax of its projections on the hyperplanes.
 *
 *   z_{l,p}  = <W_{l,p}, q> / ||q||   (z = 0 when ||q|| = 0)
 *   logit(b) = sum_p s_{b,p} z_{l,p} / tau,  s_{b,p} = +1 if bit p of b else -1
 *   p_l(b)   = exp(logit(b) - max) / sum_b' exp(logit(b') - max)
 *
 * tau = 0 is hard LSH ([ES] "Enunciado del Problema" / "Fundamento Teórico",
 * the hard-hash collision count the soft score generalises): the query is
 * hashed like a key, bit p = [<W_{l,p}, q> > 0], and all mass sits on that
 * bucket, so the score counts the tables where key and query collide.
 *
 * q: d stored elements (dtype q_dtype).  prob: [L][2^P].
 */
void oracle_soft_assign(const void* q, int q_dtype, int d,
                        const double* W, int L, int P, double tau, double* prob)
{
    const int nb = 1 << P;
    double qq = 0.0;
    for (int j = 0; j < d; ++j) {
        double qj = load_elem(q, q_dtype, j);
        qq += qj * qj;
    }
    double qnorm = sqrt(qq);
    double z[8];
    if (tau == 0.0) {
        for (int l = 0; l < L; ++l) {
            int hb = 0;
            for (int p = 0; p < P; ++p) {
                const double* w = W + ((int64_t)l * P + p) * d;
                double y = 0.0;
                for (int j = 0; j < d; ++j) y += w[j] * load_elem(q, q_dtype, j);
                if (y > 0.0) hb |= 1 << p;
            }
            for (int b = 0; b < nb; ++b) prob[(int64_t)l * nb + b] = b == hb ? 1.0 : 0.0;
        }
        return;
    }
    double* logit = (double*)malloc(sizeof(double) * nb);
    for (int l = 0; l < L; ++l) {
        for (int p = 0; p < P; ++p) {
            const double* w = W + ((int64_t)l * P + p) * d;
            double y = 0.0;
            for (int j = 0; j < d; ++j) y += w[j] * load_elem(q, q_dtype, j);
            z[p] = qnorm > 0.0 ? y / qnorm : 0.0;
        }
        double mx = -INFINITY;
        for (int b = 0; b < nb; ++b) {
            double s = 0.0;
            for (int p = 0; p < P; ++p) s += (((b >> p) & 1) ? 1.0 : -1.0) * z[p];
            logit[b] = s / tau;
            if (logit[b] > mx) mx = logit[b];
        }
        double total = 0.0;
        for (int b = 0; b < nb; ++b) total += exp(logit[b] - mx);
        for (int b = 0; b < nb; ++b) prob[(int64_t)l * nb + b] = exp(logit[b] - mx) / total;
    }
    free(logit);
}

/*
 * Step 3, soft collision score ([ES] step 3 "Puntuación"; [DE] "Bewertung"):
 * for each key, the probability mass that the query puts on the key's own
 * bucket, summed over the L tables and weighted by the key's value norm.
 *
 * Grouped-query attention (the pages say nothing about it): the G query heads
 * that share a kv head share one selection, and their scores add up:
 *   score(k) = sum_h vnorm(k) * sum_l p_{h,l}(id_l(k)).
 *
 * ids: [L][n], vnorm: [n] (stored fp32, widened), prob: [G][L][2^P].
 */
void oracle_score(const uint8_t* ids, const float* vnorm, int64_t n, int L, int P,
                  const double* prob, int G, double* score)
{
    const int nb = 1 << P;
    for (int64_t i = 0; i < n; ++i) {
        double s = 0.0;
        for (int h = 0; h < G; ++h) {
            double mass = 0.0;
            for (int l = 0; l < L; ++l)
                mass += prob[((int64_t)h * L + l) * nb + ids[(int64_t)l * n + i]];
            s += (double)vnorm[i] * mass;
        }
        score[i] = s;
    }
}

/* Order for the selection: larger score first; equal scores, lower index first. */
typedef struct { double score; int64_t index; } ranked_t;

static int by_score_then_index(const void* a, const void* b)
{
    const ranked_t* x = (const ranked_t*)a;
    const ranked_t* y = (const ranked_t*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->index > y->index) - (x->index < y->index);
}

static int by_value(const void* a, const void* b)
{
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/*
 * Step 4, selection ([ES] step 4 "Selección"; [DE] "Auswahl"): the k keys with
 * the largest soft score, chosen deterministically: a full sort by (score
 * descending, index ascending), the first k taken, returned in ascending index
 * order.
 */
void oracle_topk(const double* score, int64_t n, int k, int32_t* idx)
{
    ranked_t* r = (ranked_t*)malloc(sizeof(ranked_t) * (size_t)n);
    for (int64_t i = 0; i < n; ++i) { r[i].score = score[i]; r[i].index = i; }
    qsort(r, (size_t)n, sizeof(ranked_t), by_score_then_index);
    for (int j = 0; j < k; ++j) idx[j] = (int32_t)r[j].index;
    qsort(idx, (size_t)k, sizeof(int32_t), by_value);
    free(r);
}

/*
 * Step 4 (second half), exact attention over the selected subset ([ES] step 4;
 * [DE] "Auswahl"): for each query head, softmax(q . K_i / sqrt(d)) over the
 * selected keys i only, then the weighted sum of their values.
 *
 * q: [G][d] (q_dtype), K, V: rows of d (kv_dtype), idx: k row indices,
 * out: [G][d] doubles.
 */
void oracle_attention(const void* q, int q_dtype, int G,
                      const void* K, const void* V, int kv_dtype, int d,
                      const int32_t* idx, int k, double* out)
{
    double* logit = (double*)malloc(sizeof(double) * (size_t)k);
    const double scale = 1.0 / sqrt((double)d);
    for (int h = 0; h < G; ++h) {
        double mx = -INFINITY;
        for (int i = 0; i < k; ++i) {
            double dot = 0.0;
            for (int j = 0; j < d; ++j)
                dot += load_elem(q, q_dtype, (int64_t)h * d + j) *
                       load_elem(K, kv_dtype, (int64_t)idx[i] * d + j);
            logit[i] = dot * scale;
            if (logit[i] > mx) mx = logit[i];
        }
        double total = 0.0;
        for (int i = 0; i < k; ++i) total += exp(logit[i] - mx);
        for (int j = 0; j < d; ++j) out[(int64_t)h * d + j] = 0.0;
        for (int i = 0; i < k; ++i) {
            double w = exp(logit[i] - mx) / total;
            for (int j = 0; j < d; ++j)
                out[(int64_t)h * d + j] += w * load_elem(V, kv_dtype, (int64_t)idx[i] * d + j);
        }
    }
    free(logit);
}

/*
 * One decode step for one (batch, kv-head) unit: steps 2-4 in the pages'
 * order.  q: [G][d]; ids: [L][ncap] (only the first n keys are live);
 * vnorm: [ncap]; K, V: [ncap][d].  Outputs: idx [k], out [G][d], and
 * optionally the scores [n] and the per-head probability tables [G][L][2^P].
 */
void oracle_decode_unit(const void* q, int q_dtype, int G, int d,
                        const double* W, int L, int P, double tau,
                        const uint8_t* ids, const float* vnorm, int64_t ncap, int64_t n,
                        const void* K, const void* V, int kv_dtype, int k,
                        int32_t* idx, double* out, double* score_out, double* prob_out)
{
    const int nb = 1 << P;
    double* prob = prob_out ? prob_out : (double*)malloc(sizeof(double) * (size_t)G * L * nb);
    for (int h = 0; h < G; ++h)
        oracle_soft_assign((const char*)q + (size_t)h * d * (q_dtype == ORACLE_F64 ? 8 : q_dtype == ORACLE_F32 ? 4 : 2),
                           q_dtype, d, W, L, P, tau, prob + (int64_t)h * L * nb);

    /* Gather the live prefix of each table row so that the score sees [L][n]. */
    uint8_t* live = (uint8_t*)malloc((size_t)L * (size_t)n);
    for (int l = 0; l < L; ++l) memcpy(live + (int64_t)l * n, ids + (int64_t)l * ncap, (size_t)n);

    double* score = score_out ? score_out : (double*)malloc(sizeof(double) * (size_t)n);
    oracle_score(live, vnorm, n, L, P, prob, G, score);
    oracle_topk(score, n, k, idx);
    oracle_attention(q, q_dtype, G, K, V, kv_dtype, d, idx, k, out);

    if (!score_out) free(score);
    if (!prob_out) free(prob);
    free(live);
}

/*
 * A batch of decode units, independent of one another, run in parallel.
 * q: [U][G][d]; ids: [U][L][ncap]; vnorm: [U][ncap]; K, V: [U][ncap][d];
 * idx: [U][k]; out: [U][G][d]; score_out: [U][n] or NULL.
 */
void oracle_decode(const void* q, int q_dtype, int64_t U, int G, int d,
                   const double* W, int L, int P, double tau,
                   const uint8_t* ids, const float* vnorm, int64_t ncap, int64_t n,
                   const void* K, const void* V, int kv_dtype, int k,
                   int32_t* idx, double* out, double* score_out)
{
    const size_t qsz = q_dtype == ORACLE_F64 ? 8 : q_dtype == ORACLE_F32 ? 4 : 2;
    const size_t kvsz = kv_dtype == ORACLE_F64 ? 8 : kv_dtype == ORACLE_F32 ? 4 : 2;
    int64_t u;
#pragma omp parallel for schedule(dynamic, 1)
    for (u = 0; u < U; ++u) {
        oracle_decode_unit((const char*)q + (size_t)u * G * d * qsz, q_dtype, G, d, W, L, P, tau,
                           ids + (size_t)u * L * ncap, vnorm + (size_t)u * ncap, ncap, n,
                           (const char*)K + (size_t)u * ncap * d * kvsz,
                           (const char*)V + (size_t)u * ncap * d * kvsz, kv_dtype, k,
                           idx + (size_t)u * k, out + (size_t)u * G * d,
                           score_out ? score_out + (size_t)u * n : NULL, NULL);
    }
}
