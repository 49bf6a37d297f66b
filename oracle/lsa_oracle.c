/*
 * CPU oracle of the Lookahead Sparse Attention indexer path -- TEST INFRASTRUCTURE.
 *
 * Plain, slow, scalar C in double precision.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this file; the CUDA library never does, and the two
 * share no code (no headers, helpers or tables).
 *
 * Sources (page title -- section):
 *   [MI]  "FlashMemory-DeepSeek-V4: 13.5% of the memory ..." blog review -- section 3.1
 *         "Memory Indexer math": c^Q_t = h_t W^DQ, q^l_t = c^Q_t W^IUQ, w^l_t = h_t W^w,
 *         I_{t,s} = sigmoid( sum_h w_{t,h} ReLU(q_{t,h} . K_s^IComp) ), fetch if I >= 0.5.
 *   [OR]  same review, section 4.2, and the hyper.ai summary, "Method": three independent
 *         indexers (layers 10, 12, 20) OR-combined -- fetched if any layer reaches 0.5.
 *   [C]   hyper.ai summary, "Method": the fetched set C_t^MemComp is loaded from the CPU
 *         cold pool into GPU memory.
 *   [LI]  blog review, sections 2.2 and 3.2: native Lightning Indexer, ReLU-weighted head
 *         sum followed by Top-k, run over C_t^MemComp only, giving C_i^CoreComp.
 *   [FP8] OCP 8-bit floating point specification, E4M3 encoding (bias 7, no infinities,
 *         S.1111.111 is NaN).  bf16 is the upper half of an IEEE-754 binary32.
 *   [TR]  hyper.ai summary, "Method"; blog review, section 3: the indexer is trained alone
 *         against frozen keys K^IComp, only W^DQ, W^IUQ and W^w being trained, with binary
 *         cross-entropy on the lookahead scores, and a focal loss in the final recipe.
 *   [GL]  blog review, section 4.1 "golden labels"; hyper.ai summary, "Dataset"; gist.science
 *         summary, section 2.2: per token of the future window and per CSA layer, softmax over
 *         the raw indexer logits, keep the top-p (p = 0.6) nucleus; an entry is golden for the
 *         token if at least theta = 3 layers keep it; the window's label set is the union of
 *         its tokens' golden sets.
 *
 * Readings where the pages are silent:
 *   - the threshold is inclusive, decided on the logit: I >= thr  <=>  x >= log(thr/(1-thr))
 *     (x >= 0 at thr = 0.5, so an exact-zero logit is fetched);
 *   - no softmax scale, norm or rotary embedding appears in the formulas, so none is applied;
 *   - intermediate c^Q and the queries q are stored in the storage dtype (bf16 or fp32) and
 *     w in fp32: the oracle rounds to nearest-even exactly at those points and nowhere else;
 *   - FP8 keys carry one fp32 scale per entry: K_s = scale_s * decode(code_s);
 *   - the fetched list is in ascending entry order; the Top-k output is ordered by score
 *     descending with ties broken toward the smaller entry index, padded with -1 / -inf
 *     when fewer than k entries were fetched.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_FP8_E4M3 = 2, ORC_F64 = 3 };  /* F64: inputs kept exact (pins only) */

/* ------------------------------------------------------------ stored-value decoding */

static double bf16_value(uint16_t u)
{
    uint32_t bits = (uint32_t)u << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* [FP8] E4M3: value = (-1)^S * 2^(E-7) * (1 + M/8) for E > 0, (-1)^S * 2^-6 * (M/8) for E = 0 */
static double e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(8.0 + (double)m, e - 10);
    return s ? -v : v;
}

static double elem(const void *base, int dt, size_t i)
{
    switch (dt) {
    case ORC_F32: return (double)((const float *)base)[i];
    case ORC_BF16: return bf16_value(((const uint16_t *)base)[i]);
    case ORC_FP8_E4M3: return e4m3_value(((const uint8_t *)base)[i]);
    case ORC_F64: return ((const double *)base)[i];
    }
    return NAN;
}

static size_t elem_bytes(int dt) { return dt == ORC_F32 ? 4 : (dt == ORC_BF16 ? 2 : 1); }

/* ------------------------------------------------------------ rounding to storage */

/* Nearest bf16 to a real number, ties to even, returned as the stored 16 bits.
 * bf16 keeps 8 significant bits; below 2^-126 the spacing stays 2^-133 (subnormals). */
uint16_t lsa_oracle_bf16_bits(double x)
{
    if (isnan(x))
        return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);                          /* a = f 2^e, f in [0.5, 1) */
    int qe = (e < -125 ? -125 : e) - 8;    /* exponent of one unit in the last place */
    double r = ldexp(nearbyint(ldexp(a, -qe)), qe);  /* nearbyint: ties to even */
    if (r > 0x1.fep127)
        return sign | 0x7F80;              /* overflow to infinity */
    float f = (float)r;                    /* exact: r has at most 8 significant bits */
    uint32_t bits;
    memcpy(&bits, &f, 4);
    return sign | (uint16_t)(bits >> 16);
}

void lsa_oracle_bf16_round_array(const double *x, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = lsa_oracle_bf16_bits(x[i]);
}

void lsa_oracle_e4m3_decode_array(const uint8_t *codes, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = e4m3_value(codes[i]);
}

/* the value a real number takes once stored in dtype dt (fp32 or bf16, nearest-even) */
static double round_to(int dt, double x)
{
    if (dt == ORC_F64)
        return x;
    if (dt == ORC_F32)
        return (double)(float)x;
    return bf16_value(lsa_oracle_bf16_bits(x));
}

/* store a real value in dtype dt at base[i] */
static void store(void *base, int dt, size_t i, double x)
{
    if (dt == ORC_F32)
        ((float *)base)[i] = (float)x;
    else
        ((uint16_t *)base)[i] = lsa_oracle_bf16_bits(x);
}

int lsa_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void lsa_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------ [MI] projections */

/*
 * For every layer l and sequence b:
 *   c[j]  = sum_i h[i] W^DQ[i][j]           stored in dt     (W^DQ kept as W_dq[j][i])
 *   q[o]  = sum_j c[j] W^IUQ[j][o]          stored in dt     (W^IUQ kept as W_iuq[o][j]), o = head*d_I + e
 *   w[hh] = sum_i h[i] W^w[i][hh]           stored in fp32   (W^w kept as W_w[hh][i])
 * Weights are stored transposed (row = one output), the layout of a linear layer.
 */
int lsa_oracle_project(const void *h, const void *W_dq, const void *W_iuq, const void *W_w, int dt,
                       int L, int B, int d, int r, int n_h, int d_I,
                       void *q_out, float *w_out, void *c_out)
{
    if (dt != ORC_F32 && dt != ORC_BF16)
        return 1;
    int nq = n_h * d_I;
    int status = 0;
#pragma omp parallel for schedule(dynamic) collapse(2)
    for (int l = 0; l < L; l++) {
        for (int b = 0; b < B; b++) {
            size_t hb = ((size_t)l * B + b) * d;
            double *c = (double *)malloc(sizeof(double) * (size_t)r);
            if (!c) { status = 2; continue; }
            for (int j = 0; j < r; j++) {
                double acc = 0.0;
                for (int i = 0; i < d; i++)
                    acc += elem(h, dt, hb + i) * elem(W_dq, dt, ((size_t)l * r + j) * d + i);
                c[j] = round_to(dt, acc);
                if (c_out)
                    store(c_out, dt, ((size_t)l * B + b) * r + j, c[j]);
            }
            for (int o = 0; o < nq; o++) {
                double acc = 0.0;
                for (int j = 0; j < r; j++)
                    acc += c[j] * elem(W_iuq, dt, ((size_t)l * nq + o) * r + j);
                store(q_out, dt, ((size_t)l * B + b) * nq + o, acc);
            }
            for (int hh = 0; hh < n_h; hh++) {
                double acc = 0.0;
                for (int i = 0; i < d; i++)
                    acc += elem(h, dt, hb + i) * elem(W_w, dt, ((size_t)l * n_h + hh) * d + i);
                w_out[((size_t)l * B + b) * n_h + hh] = (float)acc;
            }
            free(c);
        }
    }
    return status;
}

/* ------------------------------------------------------------ [MI] index score */

/* x = sum_h w_h * ReLU( scale * sum_e q_h[e] K[e] ): the logit inside the sigmoid */
static double index_logit(const void *q, int qdt, size_t q0, const float *w, size_t w0,
                          const void *K, int kdt, size_t k0, double scale, int n_h, int d_I)
{
    double x = 0.0;
    for (int hh = 0; hh < n_h; hh++) {
        double dot = 0.0;
        for (int e = 0; e < d_I; e++)
            dot += elem(q, qdt, q0 + (size_t)hh * d_I + e) * elem(K, kdt, k0 + e);
        dot *= scale;
        x += (double)w[w0 + hh] * (dot > 0.0 ? dot : 0.0);
    }
    return x;
}

double lsa_oracle_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/*
 * Memory-indexer fetch decision for every entry of every sequence ([MI], [OR]), then the
 * ascending list of fetched entries per sequence ([C]).
 *   q [L][B][n_h][d_I] qdt, w [L][B][n_h] f32, K [L][T][d_I] kdt, k_scale [L][T] f32 or NULL,
 *   seq_offsets [B+1] (T = seq_offsets[B]); entry s of sequence b is row seq_offsets[b]+s.
 * Outputs: x_out/I_out [L][T] (nullable), mask_out [T] (OR over layers), idx_out [T]
 * (segment b: ascending s, first count[b] slots), count_out [B].
 */
int lsa_oracle_score(const void *q, int qdt, const float *w, const void *K, const float *k_scale, int kdt,
                     const int64_t *seq_offsets, int L, int B, int n_h, int d_I, double threshold,
                     double *x_out, double *I_out, uint8_t *mask_out, int32_t *idx_out, int32_t *count_out)
{
    if (!(threshold > 0.0 && threshold < 1.0))
        return 1;
    const double t = log(threshold / (1.0 - threshold));
    const int64_t T = seq_offsets[B];
    uint8_t *fetched = (uint8_t *)malloc((size_t)(T > 0 ? T : 1));
    if (!fetched)
        return 2;
    /* every entry of every sequence: the OR over layers of (x >= t) */
#pragma omp parallel for schedule(dynamic, 256)
    for (int64_t row = 0; row < T; row++) {
        int b = 0;
        while (seq_offsets[b + 1] <= row)  /* the sequence that owns this row */
            b++;
        int f = 0;
        for (int l = 0; l < L; l++) {
            size_t lrow = (size_t)l * T + row;
            double scale = k_scale ? (double)k_scale[lrow] : 1.0;
            double x = index_logit(q, qdt, ((size_t)l * B + b) * n_h * d_I, w, ((size_t)l * B + b) * n_h,
                                   K, kdt, lrow * d_I, scale, n_h, d_I);
            if (x_out) x_out[lrow] = x;
            if (I_out) I_out[lrow] = lsa_oracle_sigmoid(x);
            if (x >= t)
                f = 1;
        }
        fetched[row] = (uint8_t)f;
    }
    /* the fetched set of each sequence, in ascending entry order */
    for (int b = 0; b < B; b++) {
        int64_t off = seq_offsets[b], S = seq_offsets[b + 1] - seq_offsets[b];
        int32_t n = 0;
        for (int64_t s = 0; s < S; s++) {
            if (mask_out) mask_out[off + s] = fetched[off + s];
            if (fetched[off + s]) {
                if (idx_out) idx_out[off + n] = (int32_t)s;
                n++;
            }
        }
        if (count_out) count_out[b] = n;
    }
    free(fetched);
    return 0;
}

/* Logits x for a sample of entries: entry i is (sequence eb[i], entry es[i]); out [L][n]. */
int lsa_oracle_score_entries(const void *q, int qdt, const float *w, const void *K, const float *k_scale,
                             int kdt, const int64_t *seq_offsets, int L, int B, int n_h, int d_I,
                             int64_t n, const int32_t *eb, const int64_t *es, double *x_out)
{
    const int64_t T = seq_offsets[B];
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; i++) {
        int b = eb[i];
        for (int l = 0; l < L; l++) {
            size_t row = (size_t)l * T + seq_offsets[b] + es[i];
            double scale = k_scale ? (double)k_scale[row] : 1.0;
            x_out[(size_t)l * n + i] = index_logit(q, qdt, ((size_t)l * B + b) * n_h * d_I, w,
                                                   ((size_t)l * B + b) * n_h, K, kdt, row * d_I, scale, n_h, d_I);
        }
    }
    return 0;
}

/* ------------------------------------------------------------ [C] fetch */

/*
 * Copy the fetched rows: hot_kv[off_b + j] = pool[off_b + idx_b[j]] (row_bytes each), and,
 * when K is given, hot_K[off_b + j] = K[off_b + idx_b[j]] (d_I elements of kdt) and
 * hot_scale likewise.  Byte copies; slots j >= count[b] are left untouched.
 */
int lsa_oracle_gather(const int32_t *idx, const int32_t *count, const int64_t *seq_offsets, int B,
                      const uint8_t *pool, int64_t row_bytes, uint8_t *hot_kv,
                      const void *K, const float *k_scale, int kdt, int d_I, void *hot_K, float *hot_scale)
{
    size_t kb = elem_bytes(kdt) * (size_t)d_I;
    for (int b = 0; b < B; b++) {
        int64_t off = seq_offsets[b];
        for (int32_t j = 0; j < count[b]; j++) {
            int64_t src = off + idx[off + j], dst = off + j;
            if (pool && hot_kv)
                memcpy(hot_kv + (size_t)dst * row_bytes, pool + (size_t)src * row_bytes, (size_t)row_bytes);
            if (K && hot_K)
                memcpy((char *)hot_K + (size_t)dst * kb, (const char *)K + (size_t)src * kb, kb);
            if (k_scale && hot_scale)
                hot_scale[dst] = k_scale[src];
        }
    }
    return 0;
}

/* ------------------------------------------------------------ [LI] Top-k over the fetched set */

typedef struct { double y; int32_t s; } scored_t;

/* score descending, then entry index ascending: a total order, so any sort is deterministic */
static int by_score_then_index(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (a->y > b->y) return -1;
    if (a->y < b->y) return 1;
    return (a->s > b->s) - (a->s < b->s);
}

/*
 * For each requested decode query (b = qb[n], i = qi[n]) -- or all B*tau queries when
 * nq < 0 -- score every fetched entry s = idx_b[j] (j < count[b]) with the native
 * Lightning-Indexer form y = sum_h w'_h ReLU(scale_s q'_h . K_s) using the keys of the
 * selected layer K_sel [T][d_I] (and k_scale_sel), sort by (y desc, s asc) and keep the
 * first min(k, count[b]); pad with -1 / -inf.
 *   q_dec [B][tau][n_h][d_I] qdt, w_dec [B][tau][n_h] f32.
 * Outputs per listed query n: topk_idx [n][k], topk_score [n][k] (nullable), y_out [n][T]
 * (nullable; scores of sequence b at columns seq_offsets[b] + j).
 */
int lsa_oracle_lightning_topk(const void *q_dec, int qdt, const float *w_dec, const void *K_sel,
                              const float *k_scale_sel, int kdt, const int32_t *idx, const int32_t *count,
                              const int64_t *seq_offsets, int B, int tau, int n_h, int d_I, int k,
                              int64_t nq, const int32_t *qb, const int32_t *qi,
                              int32_t *topk_idx, double *topk_score, double *y_out)
{
    const int64_t T = seq_offsets[B];
    const int64_t nall = nq < 0 ? (int64_t)B * tau : nq;
    int status = 0;
#pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < nall; n++) {
        int b = nq < 0 ? (int)(n / tau) : qb[n];
        int i = nq < 0 ? (int)(n % tau) : qi[n];
        int64_t off = seq_offsets[b];
        int32_t F = count[b];
        scored_t *v = (scored_t *)malloc(sizeof(scored_t) * (size_t)(F > 0 ? F : 1));
        if (!v) { status = 2; continue; }
        size_t q0 = (((size_t)b * tau + i) * n_h) * d_I, w0 = ((size_t)b * tau + i) * n_h;
        for (int32_t j = 0; j < F; j++) {
            int32_t s = idx[off + j];
            size_t row = (size_t)(off + s);
            double scale = k_scale_sel ? (double)k_scale_sel[row] : 1.0;
            double y = 0.0;
            for (int hh = 0; hh < n_h; hh++) {
                double dot = 0.0;
                for (int e = 0; e < d_I; e++)
                    dot += elem(q_dec, qdt, q0 + (size_t)hh * d_I + e) * elem(K_sel, kdt, row * d_I + e);
                dot *= scale;
                y += (double)w_dec[w0 + hh] * (dot > 0.0 ? dot : 0.0);
            }
            v[j].y = y;
            v[j].s = s;
            if (y_out) y_out[(size_t)n * T + off + j] = y;
        }
        qsort(v, (size_t)F, sizeof(scored_t), by_score_then_index);
        for (int j = 0; j < k; j++) {
            topk_idx[(size_t)n * k + j] = j < F ? v[j].s : -1;
            if (topk_score) topk_score[(size_t)n * k + j] = j < F ? v[j].y : -INFINITY;
        }
        free(v);
    }
    return status;
}

/* ----------------------------------------------------------------------------------------
 * [GL] Golden labels of one future window.
 *   z          [tau][Lc][T] fp32 raw indexer logits: token i, CSA layer l, entry offs[b] + s
 *   p          nucleus mass (the pages use 0.6), theta votes needed (the pages use 3)
 *   label_out  [T] uint8: 1 if entry s of sequence b is golden for some token of the window
 *   golden_out [tau][T] uint8 (nullable): the golden set of each token
 *   nsize_out  [B][tau][Lc] int32 (nullable): nucleus size of each (sequence, token, layer)
 * Per (b, i, l): softmax over the S_b entries, in double; entries taken by probability
 * descending (ties: smaller entry first) until the taken mass reaches p of the total (the
 * entry that reaches it is taken).  The comparison uses the unnormalised masses
 * e_s = exp(z_s - max z): taken while  sum e < p * sum_all e.
 * ---------------------------------------------------------------------------------------- */
typedef struct { double z; int32_t s; } logit_t;

static int by_logit_then_index(const void *pa, const void *pb)
{
    const logit_t *a = (const logit_t *)pa, *b = (const logit_t *)pb;
    if (a->z > b->z) return -1;
    if (a->z < b->z) return 1;
    return (a->s > b->s) - (a->s < b->s);
}

int lsa_oracle_golden_labels(const float *z, const int64_t *seq_offsets, int B, int tau, int Lc, double p,
                             int theta, uint8_t *label_out, uint8_t *golden_out, int32_t *nsize_out)
{
    const int64_t T = seq_offsets[B];
    int status = 0;
    uint8_t *kept = (uint8_t *)calloc((size_t)tau * Lc * (size_t)(T > 0 ? T : 1), 1);  /* nucleus membership */
    if (!kept) return 2;
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (int i = 0; i < tau; i++)
            for (int l = 0; l < Lc; l++) {
                const int64_t off = seq_offsets[b], S = seq_offsets[b + 1] - off;
                const float *row = z + ((size_t)i * Lc + l) * (size_t)T + off;
                uint8_t *krow = kept + ((size_t)i * Lc + l) * (size_t)T + off;
                int32_t taken = 0;
                if (S > 0) {
                    logit_t *v = (logit_t *)malloc(sizeof(logit_t) * (size_t)S);
                    if (!v) { status = 2; continue; }
                    double zmax = -INFINITY, total = 0.0;
                    for (int64_t s = 0; s < S; s++)
                        if ((double)row[s] > zmax) zmax = (double)row[s];
                    for (int64_t s = 0; s < S; s++) {
                        v[s].z = (double)row[s];
                        v[s].s = (int32_t)s;
                        total += exp((double)row[s] - zmax);
                    }
                    qsort(v, (size_t)S, sizeof(logit_t), by_logit_then_index);
                    const double target = p * total;
                    double mass = 0.0;
                    for (int64_t r = 0; r < S; r++) {
                        if (mass >= target) break;
                        mass += exp(v[r].z - zmax);
                        krow[v[r].s] = 1;
                        taken++;
                    }
                    free(v);
                }
                if (nsize_out) nsize_out[((size_t)b * tau + i) * Lc + l] = taken;
            }
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < T; e++) {
        uint8_t any = 0;
        for (int i = 0; i < tau; i++) {
            int votes = 0;
            for (int l = 0; l < Lc; l++) votes += kept[((size_t)i * Lc + l) * (size_t)T + e];
            const uint8_t g = votes >= theta;
            if (golden_out) golden_out[(size_t)i * T + e] = g;
            any |= g;
        }
        label_out[e] = any;
    }
    free(kept);
    return status;
}

/* ----------------------------------------------------------------------------------------
 * [TR] One training step of the indexer: loss and gradients of W^DQ, W^IUQ, W^w.
 *   h, W_dq, W_iuq, W_w as lsa_oracle_project (dt: F32, BF16, or F64 = exact inputs);
 *   K [L][T][d_I] kdt + k_scale [L][T] (nullable) frozen; labels [T] uint8 (the window's golden
 *   set, the same target for the L indexers).
 * Forward as the memory indexer ([MI]): c = round(h W^DQ), q = round(c W^IUQ), w = h W^w,
 *   a_h = scale_s q_h . K_s,  x = sum_h w_h ReLU(a_h),  p = sigmoid(x).
 * Loss: mean over the L*T (layer, entry) pairs of the focal loss
 *   l = -at (1 - pt)^gamma log(pt),  pt = y ? p : 1 - p,  at = alpha < 0 ? 1 : (y ? alpha : 1 - alpha),
 *   which is binary cross-entropy at gamma = 0, alpha < 0.
 * Backward: the rounding of c and q is passed straight through (d round(v) / dv = 1); the ReLU
 *   derivative is 1[a > 0].  Outputs loss_out [1] and the gradients g_* in the weights' layouts.
 * ---------------------------------------------------------------------------------------- */
static double focal_dx(double x, int y, double gamma, double alpha, double *loss)
{
    const double p = 1.0 / (1.0 + exp(-x));
    const double pt = y ? p : 1.0 - p;
    const double at = alpha < 0.0 ? 1.0 : (y ? alpha : 1.0 - alpha);
    /* log(pt) from the logit, stable: log sigmoid(+-x) */
    const double lpt = y ? -log1p(exp(-x)) : -log1p(exp(x));
    const double q1 = 1.0 - pt;
    *loss = -at * pow(q1, gamma) * lpt;
    /* dl/dpt = at (gamma (1-pt)^(gamma-1) log pt - (1-pt)^gamma / pt);  dpt/dx = +-p (1-p) */
    double dl_dx;
    if (gamma == 0.0)
        dl_dx = at * (y ? p - 1.0 : p);
    else
        dl_dx = at * (gamma * pow(q1, gamma - 1.0) * lpt * pt * q1 - pow(q1, gamma) * q1) * (y ? 1.0 : -1.0);
    return dl_dx;
}

int lsa_oracle_train_step(const void *h, const void *W_dq, const void *W_iuq, const void *W_w, int dt,
                          const void *K, const float *k_scale, int kdt, const uint8_t *labels,
                          const int64_t *seq_offsets, int L, int B, int d, int r, int n_h, int d_I,
                          double gamma, double alpha, double *loss_out, double *g_Wdq, double *g_Wiuq,
                          double *g_Ww)
{
    if (dt != ORC_F32 && dt != ORC_BF16 && dt != ORC_F64)
        return 1;
    const int nq = n_h * d_I;
    const int64_t T = seq_offsets[B];
    const double N = (double)L * (double)T;
    const size_t LB = (size_t)L * B;
    double *cs = (double *)calloc(LB * r, sizeof(double));
    double *dq = (double *)calloc(LB * nq, sizeof(double));
    double *dw = (double *)calloc(LB * n_h, sizeof(double));
    double *lossp = (double *)calloc(LB, sizeof(double));
    if (!cs || !dq || !dw || !lossp) { free(cs); free(dq); free(dw); free(lossp); return 2; }
    int status = 0;
    /* forward and the per-(layer, sequence) gradients of q and w */
#pragma omp parallel for schedule(dynamic) collapse(2)
    for (int l = 0; l < L; l++) {
        for (int b = 0; b < B; b++) {
            const size_t lb = (size_t)l * B + b, hb = lb * d;
            double *c = cs + lb * r;
            double *q = (double *)malloc(sizeof(double) * nq);
            double *w = (double *)malloc(sizeof(double) * n_h);
            double *a = (double *)malloc(sizeof(double) * n_h);
            if (!q || !w || !a) { status = 2; free(q); free(w); free(a); continue; }
            for (int j = 0; j < r; j++) {
                double acc = 0.0;
                for (int i = 0; i < d; i++) acc += elem(h, dt, hb + i) * elem(W_dq, dt, ((size_t)l * r + j) * d + i);
                c[j] = round_to(dt, acc);
            }
            for (int o = 0; o < nq; o++) {
                double acc = 0.0;
                for (int j = 0; j < r; j++) acc += c[j] * elem(W_iuq, dt, ((size_t)l * nq + o) * r + j);
                q[o] = round_to(dt, acc);
            }
            for (int hh = 0; hh < n_h; hh++) {
                double acc = 0.0;
                for (int i = 0; i < d; i++) acc += elem(h, dt, hb + i) * elem(W_w, dt, ((size_t)l * n_h + hh) * d + i);
                w[hh] = dt == ORC_F64 ? acc : (double)(float)acc;
            }
            const int64_t off = seq_offsets[b], S = seq_offsets[b + 1] - off;
            double lsum = 0.0;
            for (int64_t s = 0; s < S; s++) {
                const size_t row = (size_t)l * T + off + s;
                const double scale = k_scale ? (double)k_scale[row] : 1.0;
                double x = 0.0;
                for (int hh = 0; hh < n_h; hh++) {
                    double dot = 0.0;
                    for (int e = 0; e < d_I; e++) dot += q[(size_t)hh * d_I + e] * elem(K, kdt, row * d_I + e);
                    a[hh] = scale * dot;
                    x += w[hh] * (a[hh] > 0.0 ? a[hh] : 0.0);
                }
                double ls;
                const double g = focal_dx(x, labels[off + s] != 0, gamma, alpha, &ls) / N;
                lsum += ls;
                for (int hh = 0; hh < n_h; hh++) {
                    if (a[hh] > 0.0) {
                        dw[lb * n_h + hh] += g * a[hh];
                        const double gq = g * w[hh] * scale;
                        for (int e = 0; e < d_I; e++) dq[lb * nq + (size_t)hh * d_I + e] += gq * elem(K, kdt, row * d_I + e);
                    }
                }
            }
            lossp[lb] = lsum;
            free(q); free(w); free(a);
        }
    }
    double loss = 0.0;
    for (size_t lb = 0; lb < LB; lb++) loss += lossp[lb];
    *loss_out = loss / N;
    /* weight gradients: dc = dq W^IUQ (straight through the rounding), then outer products over b */
#pragma omp parallel for schedule(dynamic)
    for (int l = 0; l < L; l++) {
        double *dc = (double *)malloc(sizeof(double) * r);
        if (!dc) { status = 2; continue; }
        for (size_t o = 0; o < (size_t)nq * r; o++) g_Wiuq[(size_t)l * nq * r + o] = 0.0;
        for (size_t o = 0; o < (size_t)r * d; o++) g_Wdq[(size_t)l * r * d + o] = 0.0;
        for (size_t o = 0; o < (size_t)n_h * d; o++) g_Ww[(size_t)l * n_h * d + o] = 0.0;
        for (int b = 0; b < B; b++) {
            const size_t lb = (size_t)l * B + b, hb = lb * d;
            const double *c = cs + lb * r;
            for (int j = 0; j < r; j++) {
                double acc = 0.0;
                for (int o = 0; o < nq; o++) acc += dq[lb * nq + o] * elem(W_iuq, dt, ((size_t)l * nq + o) * r + j);
                dc[j] = acc;
            }
            for (int o = 0; o < nq; o++)
                for (int j = 0; j < r; j++) g_Wiuq[((size_t)l * nq + o) * r + j] += dq[lb * nq + o] * c[j];
            for (int j = 0; j < r; j++)
                for (int i = 0; i < d; i++) g_Wdq[((size_t)l * r + j) * d + i] += dc[j] * elem(h, dt, hb + i);
            for (int hh = 0; hh < n_h; hh++)
                for (int i = 0; i < d; i++) g_Ww[((size_t)l * n_h + hh) * d + i] += dw[lb * n_h + hh] * elem(h, dt, hb + i);
        }
        free(dc);
    }
    free(cs); free(dq); free(dw); free(lossp);
    return status;
}
