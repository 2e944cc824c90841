/*
 * oracle.c -- plain, slow, obviously-correct fp64 CPU oracle for RoPE +
 * grouped-query KV-cache attention and the lightning-indexer sparse path.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library never
 * calls it, includes nothing from it, and it includes nothing from the CUDA
 * library: the two are independent statements of the same method.
 *
 * Arithmetic: every floating-point step is IEEE double (no fast-math, no FMA
 * contraction).  bf16 inputs arrive as their 16-bit patterns and are widened
 * exactly (a bf16 value is the upper half of an fp32 value).  Where a result
 * has a plain definition (a softmax, a sort) this file writes the definition
 * out, with no blocking, splitting or reordering beyond it.
 *
 * Sources (pages of the mqa_kv_cache reading set, cited by title + section):
 *   [P1] "Agentic RL 入门3：transformer 架构"
 *   [P2] "注意力变体与 MoE"
 *   [P3] "attention" (MHA / MQA / GQA / DSA notes)
 *   [P4] "稀疏注意力：省了什么，没省什么" (C11 L05)
 *   [P5] "注意力机制进化史：从MHA、MQA、GQA、MLA到NSA、MoBA！"
 *
 * Readings where the pages are silent are documented next to the code that
 * takes them.  Every exported function returns 0 on success and a negative
 * number on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_PI 3.14159265358979323846

/* Frequency-scaling modes ([P1] §1.2 ①–④). */
enum { ORC_ROPE_NONE = 0, ORC_ROPE_PI = 1, ORC_ROPE_NTK = 2, ORC_ROPE_YARN = 3, ORC_ROPE_DYN_NTK = 4 };

/* Exact widening of a bf16 bit pattern. */
static double bf16_bits_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* An input array that is either bf16 bit patterns (f64 == 0) or doubles. */
typedef struct {
    const void* p;
    int f64;
} src_t;

static double ld(src_t s, int64_t i)
{
    return s.f64 ? ((const double*)s.p)[i] : bf16_bits_to_f64(((const uint16_t*)s.p)[i]);
}

static int set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
    return nthreads;
#else
    (void)nthreads;
    return 1;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* RoPE frequencies and tables                                              */
/* ------------------------------------------------------------------------ */

/* YaRN ramp gamma(r) ([P1] §1.2 ③(a) table): 1 above beta (many turns in
 * L_train), 0 at or below alpha (less than one turn), linear in between. */
static double yarn_ramp(double r, double alpha, double beta)
{
    if (r > beta) return 1.0;
    if (r <= alpha) return 0.0;
    return (r - alpha) / (beta - alpha);
}

/*
 * Effective angular frequency of every 2-D pair, the position scale and the
 * cos/sin magnitude.
 *
 *  plain  [P1] §1.1: theta_i = base^(-2i/d), i = 0 .. d/2-1 (so theta_0 = 1,
 *         the reading of "small i -> theta_i close to 1").
 *  PI     [P1] §1.2 ①: theta unchanged, position m -> m/s.
 *  NTK    [P1] §1.2 ②: base -> b' = b * s^(d/(d-2)), theta'_i = b'^(-2i/d).
 *  YaRN   [P1] §1.2 ③(a): r_i = L_train*theta_i/(2*pi); gamma = 1 when
 *         r_i > beta, 0 when r_i <= alpha, linear (r-alpha)/(beta-alpha) in
 *         between (the page only says "linear transition"); then
 *         theta^Y_i = (1-gamma)*theta_i/s + gamma*theta_i.
 *         ③(b): sqrt(1/t) = 0.1*ln(s) + 1 and cos/sin are both multiplied by
 *         it, so q.k picks up 1/t while the softmax scale stays 1/sqrt(d).
 *  DynNTK [P1] §1.2 ④: s = max(1, L_cur/L_train) fed to the NTK base formula.
 *
 * theta[d/2] receives the frequencies; *pos_div the divisor applied to the
 * position (s for PI, else 1); *mag the factor on cos and sin.
 */
int oracle_rope_freqs(int d, double base, int scaling, double s, double L_train, double alpha,
                      double beta, double L_cur, double* theta, double* pos_div, double* mag)
{
    if (d <= 2 || (d & 1) || base <= 0.0) return -1;
    int half = d / 2;
    double b = base;
    *pos_div = 1.0;
    *mag = 1.0;
    if (scaling == ORC_ROPE_NTK) {
        if (s < 1.0) return -1;
        b = base * pow(s, (double)d / (double)(d - 2));
    } else if (scaling == ORC_ROPE_DYN_NTK) {
        if (L_train <= 0.0) return -1;
        double sd = L_cur / L_train;
        if (sd < 1.0) sd = 1.0;
        b = base * pow(sd, (double)d / (double)(d - 2));
    } else if (scaling == ORC_ROPE_PI || scaling == ORC_ROPE_YARN) {
        if (s < 1.0) return -1;
    } else if (scaling != ORC_ROPE_NONE) {
        return -1;
    }
    for (int i = 0; i < half; ++i) theta[i] = pow(b, -2.0 * (double)i / (double)d);

    if (scaling == ORC_ROPE_PI) *pos_div = s;
    if (scaling == ORC_ROPE_YARN) {
        if (L_train <= 0.0 || !(beta > alpha)) return -1;
        for (int i = 0; i < half; ++i) {
            double gamma = yarn_ramp(L_train * theta[i] / (2.0 * ORACLE_PI), alpha, beta);
            theta[i] = (1.0 - gamma) * theta[i] / s + gamma * theta[i];
        }
        *mag = 0.1 * log(s) + 1.0;
    }
    return 0;
}

/* YaRN ramp value gamma(r_i) for every pair, exposed for the band-edge pins. */
int oracle_yarn_gamma(int d, double base, double L_train, double alpha, double beta, double* gamma)
{
    if (d <= 2 || (d & 1) || !(beta > alpha)) return -1;
    for (int i = 0; i < d / 2; ++i) {
        double th = pow(base, -2.0 * (double)i / (double)d);
        gamma[i] = yarn_ramp(L_train * th / (2.0 * ORACLE_PI), alpha, beta);
    }
    return 0;
}

/*
 * cos/sin table [max_pos][d/2]: entry (m, i) = mag * cos((m/pos_div) * theta_i)
 * and mag * sin(...), the rotation of [P1] §1.1 at position m with the
 * scaling's frequency, position and magnitude.
 */
int oracle_rope_table(int d, double base, int scaling, double s, double L_train, double alpha,
                      double beta, double L_cur, int max_pos, double* cos_out, double* sin_out)
{
    if (max_pos < 0) return -1;
    int half = d / 2;
    double* theta = (double*)malloc(sizeof(double) * (size_t)(half > 0 ? half : 1));
    double pos_div, mag;
    int rc = oracle_rope_freqs(d, base, scaling, s, L_train, alpha, beta, L_cur, theta, &pos_div, &mag);
    if (rc == 0) {
        for (int m = 0; m < max_pos; ++m) {
            double mm = (double)m / pos_div;
            for (int i = 0; i < half; ++i) {
                double ang = mm * theta[i];
                cos_out[(int64_t)m * half + i] = mag * cos(ang);
                sin_out[(int64_t)m * half + i] = mag * sin(ang);
            }
        }
    }
    free(theta);
    return rc;
}

/*
 * Rotate one head vector x (length d) with table row (c, s): pair i is
 * (x[2i], x[2i+1]) for pair_style 0 -- the plain reading of the
 * block-diagonal R of [P1] §1.1 -- or (x[i], x[i+d/2]) for pair_style 1.
 * y_a = x_a*c - x_b*s,  y_b = x_a*s + x_b*c  (R(m,theta_i) of [P1] §1.1).
 */
static void rotate_vec(src_t x, int64_t off, int d, int pair_style, const double* c, const double* s,
                       double* y)
{
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        int a = pair_style == 0 ? 2 * i : i;
        int b = pair_style == 0 ? 2 * i + 1 : i + half;
        double xa = ld(x, off + a), xb = ld(x, off + b);
        y[a] = xa * c[i] - xb * s[i];
        y[b] = xa * s[i] + xb * c[i];
    }
}

/*
 * Apply the rotation to a strided [n_b][n_t][n_h][d] array of head vectors
 * (element (b,t,h,j) at b*sb + t*st + h*sh + j).  pos[b*n_t + t] is the
 * position of token (b,t); the table rows (cos_tab/sin_tab, [max_pos][d/2],
 * fp64) come from oracle_rope_table.  Output y is dense [n_b][n_t][n_h][d].
 * Only q and k are ever passed here; v is never rotated ([P1] §1.1, last
 * paragraph).
 */
int oracle_rope_apply(int dtype, const void* x, int n_b, int n_t, int n_h, int64_t sb, int64_t st,
                      int64_t sh, const int32_t* pos, const double* cos_tab, const double* sin_tab,
                      int max_pos, int d, int pair_style, double* y)
{
    if (d <= 2 || (d & 1) || (pair_style != 0 && pair_style != 1)) return -1;
    src_t src = {x, dtype};
    int half = d / 2;
    for (int b = 0; b < n_b; ++b)
        for (int t = 0; t < n_t; ++t) {
            int m = pos[(int64_t)b * n_t + t];
            if (m < 0 || m >= max_pos) return -2;
            for (int h = 0; h < n_h; ++h) {
                int64_t off = (int64_t)b * sb + (int64_t)t * st + (int64_t)h * sh;
                double* out = y + (((int64_t)b * n_t + t) * n_h + h) * d;
                rotate_vec(src, off, d, pair_style, cos_tab + (int64_t)m * half,
                           sin_tab + (int64_t)m * half, out);
            }
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Attention                                                                */
/* ------------------------------------------------------------------------ */

/*
 * Softmax attention of one query over n key/value rows: the definition
 * softmax(q K^T * scale) V of [P2] "MQA 与 GQA" attention() and [P3]
 * MultiHeadAttention STEP 3-5, written as two passes:
 *   s_t = scale * sum_j q_j K[r_t][j];  m = max_t s_t;  p_t = exp(s_t - m);
 *   l = sum_t p_t;  out = sum_t p_t V[r_t] / l;  lse = m + ln l.
 * r_t = rows[t] when rows is given (a gathered set), else t.  An empty set
 * gives out = 0 and lse = -inf (the empty sum of exponentials is 0).
 * sbuf holds n doubles.
 */
static void attend_one(src_t q, int64_t q_off, int Dk, src_t K, int64_t k_off, int64_t k_row,
                       src_t V, int64_t v_off, int64_t v_row, int Dv, const int32_t* rows, int n,
                       double scale, double* sbuf, double* out, double* lse)
{
    for (int j = 0; j < Dv; ++j) out[j] = 0.0;
    if (n <= 0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
        int64_t r = rows ? rows[t] : t;
        double dot = 0.0;
        for (int j = 0; j < Dk; ++j) dot += ld(q, q_off + j) * ld(K, k_off + r * k_row + j);
        sbuf[t] = scale * dot;
        if (sbuf[t] > m) m = sbuf[t];
    }
    double l = 0.0;
    for (int t = 0; t < n; ++t) {
        sbuf[t] = exp(sbuf[t] - m);
        l += sbuf[t];
    }
    for (int t = 0; t < n; ++t) {
        int64_t r = rows ? rows[t] : t;
        for (int j = 0; j < Dv; ++j) out[j] += sbuf[t] * ld(V, v_off + r * v_row + j);
    }
    for (int j = 0; j < Dv; ++j) out[j] /= l;
    *lse = m + log(l);
}

/*
 * Decode: one new query per sequence over its KV cache.
 *   q [B][H][d], k,v [B][Hk][T_max][d] (cache rows 0 .. seq_lens[b]-1 valid).
 * Query head h reads KV head h / g with g = H / Hk: the repeat_interleave(g)
 * of [P2] "MQA 与 GQA" and the unsqueeze/expand/reshape of [P3]
 * GroupQueryAttention both give head h the group h // g.  Hk = H is MHA and
 * Hk = 1 is MQA ([P1] §2.1).  The new query attends to every cached row
 * ([P2] "生成时的瓶颈"; [P5] KV Cache, layer_past concatenation).
 * With sel == NULL every (b,h) is computed into out [B][H][d], lse [B][H];
 * otherwise only the n_sel pairs sel[2i], sel[2i+1] into out [n_sel][d],
 * lse [n_sel].
 */
int oracle_attn_decode(int dtype, const void* q, const void* k, const void* v,
                       const int32_t* seq_lens, int B, int H, int Hk, int d, int T_max,
                       double scale, int n_sel, const int32_t* sel, double* out, double* lse,
                       int nthreads)
{
    if (B < 0 || H <= 0 || Hk <= 0 || H % Hk || d <= 0 || T_max < 0) return -1;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] < 0 || seq_lens[b] > T_max) return -2;
    int g = H / Hk;
    int n_units = sel ? n_sel : B * H;
    src_t Q = {q, dtype}, K = {k, dtype}, V = {v, dtype};
    int nt = set_threads(nthreads);
#pragma omp parallel num_threads(nt)
    {
        double* sbuf = (double*)malloc(sizeof(double) * (size_t)(T_max > 0 ? T_max : 1));
#pragma omp for schedule(dynamic)
        for (int u = 0; u < n_units; ++u) {
            int b = sel ? sel[2 * u] : u / H;
            int h = sel ? sel[2 * u + 1] : u % H;
            int kvh = h / g;
            int64_t q_off = ((int64_t)b * H + h) * d;
            int64_t kv_off = ((int64_t)b * Hk + kvh) * T_max * d;
            attend_one(Q, q_off, d, K, kv_off, d, V, kv_off, d, d, NULL, seq_lens[b], scale, sbuf,
                       out + (int64_t)u * d, lse + u);
        }
        free(sbuf);
    }
    return 0;
}

/*
 * Causal prefill: q [B][T][H][d], k,v [B][Hk][T][d].  Query row i of head h
 * sees keys j <= i of KV head h / g: the lower-triangular mask of [P2]
 * attention() (masked_fill of triu(1) with -inf).  With sel == NULL all rows
 * go to out [B][T][H][d], lse [B][H][T]; otherwise the n_sel triples
 * (b, h, i) = sel[3u..3u+2] go to out [n_sel][d], lse [n_sel].
 */
int oracle_attn_prefill(int dtype, const void* q, const void* k, const void* v, int B, int T,
                        int H, int Hk, int d, double scale, int n_sel, const int32_t* sel,
                        double* out, double* lse, int nthreads)
{
    if (B < 0 || T < 0 || H <= 0 || Hk <= 0 || H % Hk || d <= 0) return -1;
    int g = H / Hk;
    int64_t n_units = sel ? (int64_t)n_sel : (int64_t)B * H * T;
    src_t Q = {q, dtype}, K = {k, dtype}, V = {v, dtype};
    if (sel)
        for (int64_t u = 0; u < n_units; ++u)
            if (sel[3 * u] < 0 || sel[3 * u] >= B || sel[3 * u + 1] < 0 || sel[3 * u + 1] >= H ||
                sel[3 * u + 2] < 0 || sel[3 * u + 2] >= T)
                return -2;
    int nt = set_threads(nthreads);
#pragma omp parallel num_threads(nt)
    {
        double* sbuf = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t u = 0; u < n_units; ++u) {
            int b, h, i;
            if (sel) {
                b = sel[3 * u];
                h = sel[3 * u + 1];
                i = sel[3 * u + 2];
            } else {
                b = (int)(u / ((int64_t)H * T));
                h = (int)((u / T) % H);
                i = (int)(u % T);
            }
            int kvh = h / g;
            int64_t q_off = (((int64_t)b * T + i) * H + h) * d;
            int64_t kv_off = ((int64_t)b * Hk + kvh) * T * d;
            double* o;
            double* l;
            if (sel) {
                o = out + u * d;
                l = lse + u;
            } else {
                o = out + (((int64_t)b * T + i) * H + h) * d;
                l = lse + ((int64_t)b * H + h) * T + i;
            }
            attend_one(Q, q_off, d, K, kv_off, d, V, kv_off, d, d, NULL, i + 1, scale, sbuf, o, l);
        }
        free(sbuf);
    }
    return 0;
}

/*
 * Merge attention results computed over disjoint key sets: given n pairs
 * (o_j, lse_j) of normalised outputs and log-sum-exps, the attention over
 * the union is  out = sum_j exp(lse_j - L) o_j  with  L = ln sum_j exp(lse_j).
 * This is the identity behind splitting a softmax along the keys (a softmax
 * over a union is the lse-weighted mix of the softmaxes over the parts).
 * Parts with lse = -inf (empty) contribute nothing.
 */
int oracle_softmax_merge(int n, int d, const double* o, const double* lse, double* out,
                         double* out_lse)
{
    if (n < 0 || d <= 0) return -1;
    double M = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (lse[j] > M) M = lse[j];
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    if (M == -INFINITY) {
        *out_lse = -INFINITY;
        return 0;
    }
    double Z = 0.0;
    for (int j = 0; j < n; ++j) Z += exp(lse[j] - M);
    for (int j = 0; j < n; ++j) {
        double wgt = exp(lse[j] - M) / Z;
        for (int i = 0; i < d; ++i) out[i] += wgt * o[(int64_t)j * d + i];
    }
    *out_lse = M + log(Z);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Lightning indexer, top-k and sparse latent attention                     */
/* ------------------------------------------------------------------------ */

/*
 * Indexer scores ([P1] §2.2 (1); [P3] DSA ① Lightning Indexer):
 *   s_{b,t} = sum_{j < H_I} w_{b,j} * ReLU(q^I_{b,j} . k^I_{b,t})
 * qI [B][H_I][d_I] bf16, w [B][H_I] fp32, kI [B][L_max][d_I] bf16 (one key
 * shared by all indexer heads).  No scale and no RoPE: the formula on the
 * pages has neither.  scores [B][L_max], -inf for t >= lens[b].
 */
int oracle_dsa_scores(const uint16_t* qI, const float* w, const uint16_t* kI, const int32_t* lens,
                      int B, int HI, int dI, int L_max, double* scores, int nthreads)
{
    if (B < 0 || HI <= 0 || dI <= 0 || L_max < 0) return -1;
    for (int b = 0; b < B; ++b)
        if (lens[b] < 0 || lens[b] > L_max) return -2;
    src_t Q = {qI, 0}, K = {kI, 0};
    int nt = set_threads(nthreads);
    int64_t n_units = (int64_t)B * L_max;
#pragma omp parallel for num_threads(nt) schedule(static)
    for (int64_t u = 0; u < n_units; ++u) {
        int b = (int)(u / L_max);
        int t = (int)(u % L_max);
        if (t >= lens[b]) {
            scores[u] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (int j = 0; j < HI; ++j) {
            double dot = 0.0;
            for (int i = 0; i < dI; ++i)
                dot += ld(Q, ((int64_t)b * HI + j) * dI + i) * ld(K, ((int64_t)b * L_max + t) * dI + i);
            double relu = dot > 0.0 ? dot : 0.0;
            acc += (double)w[(int64_t)b * HI + j] * relu;
        }
        scores[u] = acc;
    }
    return 0;
}

/* Total order for top-k: larger score first, then lower index first. */
typedef struct {
    double s;
    int32_t i;
} keyed_t;

static int cmp_desc_then_index(const void* pa, const void* pb)
{
    const keyed_t* a = (const keyed_t*)pa;
    const keyed_t* b = (const keyed_t*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

/*
 * Top-k ([P1] §2.2 (2): S_t = TopK_j(s_{t,j})): the k largest of
 * scores[0 .. len-1] under the total order (score descending, index
 * ascending), i.e. ties go to the lower index.  Written as a full sort of
 * all len candidates followed by taking the first k.  The pages do not fix an
 * output order; this one (the sort order) makes comparisons exact.  -0 and
 * +0 compare equal (so they tie by index).  Emits min(k, len) indices, then
 * -1 up to k.  NaN scores are rejected.
 */
int oracle_topk(const double* scores, int len, int k, int32_t* idx_out)
{
    if (len < 0 || k < 0) return -1;
    for (int t = 0; t < len; ++t)
        if (scores[t] != scores[t]) return -3;
    keyed_t* all = (keyed_t*)malloc(sizeof(keyed_t) * (size_t)(len > 0 ? len : 1));
    for (int t = 0; t < len; ++t) {
        all[t].s = scores[t];
        all[t].i = t;
    }
    qsort(all, (size_t)len, sizeof(keyed_t), cmp_desc_then_index);
    for (int r = 0; r < k; ++r) idx_out[r] = r < len ? all[r].i : -1;
    free(all);
    return 0;
}

/* Row-wise top-k over scores [B][L_max] with per-row lengths. */
int oracle_topk_rows(const double* scores, const int32_t* lens, int B, int L_max, int k,
                     int32_t* idx_out, int nthreads)
{
    if (B < 0 || L_max < 0 || k < 0) return -1;
    int rc = 0;
    int nt = set_threads(nthreads);
#pragma omp parallel for num_threads(nt) schedule(dynamic) reduction(min : rc)
    for (int b = 0; b < B; ++b) {
        int len = lens[b] < 0 ? 0 : (lens[b] > L_max ? L_max : lens[b]);
        int r = oracle_topk(scores + (int64_t)b * L_max, len, k, idx_out + (int64_t)b * k);
        if (r < rc) rc = r;
    }
    return rc;
}

/*
 * Sparse latent attention ([P1] §2.2 (2) o_t = MLA(q_t, {k_j, v_j : j in S_t});
 * [P3] DSA ② "MQA equivalent form" and "乘法结合律": after absorption every
 * query head scores the same single-head latent rows, so this is MQA over
 * the selected rows).  q [B][Hq][Dk], latent [B][L_max][Dk]; key row j is
 * latent[b][j][0 .. Dk-1] and value row j is latent[b][j][0 .. Dv-1] (K and
 * V share the latent c^KV, [P1] §2.3.5; 576 = 512 + 64, [P1] §2.3.3).
 * idx [B][k]: selected rows, -1 entries skipped.  out [B][Hq][Dv],
 * lse [B][Hq].
 */
int oracle_attn_sparse(int dtype, const void* q, const void* latent, const int32_t* idx, int B,
                       int Hq, int Dk, int Dv, int L_max, int k, double scale, double* out,
                       double* lse, int nthreads)
{
    if (B < 0 || Hq <= 0 || Dk <= 0 || Dv <= 0 || Dv > Dk || L_max < 0 || k < 0) return -1;
    for (int64_t u = 0; u < (int64_t)B * k; ++u)
        if (idx[u] >= L_max) return -2;
    src_t Q = {q, dtype}, C = {latent, dtype};
    int nt = set_threads(nthreads);
#pragma omp parallel num_threads(nt)
    {
        double* sbuf = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
        int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k > 0 ? k : 1));
#pragma omp for schedule(dynamic)
        for (int u = 0; u < B * Hq; ++u) {
            int b = u / Hq;
            int n = 0;
            for (int r = 0; r < k; ++r)
                if (idx[(int64_t)b * k + r] >= 0) rows[n++] = idx[(int64_t)b * k + r];
            int64_t c_off = (int64_t)b * L_max * Dk;
            attend_one(Q, (int64_t)u * Dk, Dk, C, c_off, Dk, C, c_off, Dk, Dv, rows, n, scale, sbuf,
                       out + (int64_t)u * Dv, lse + u);
        }
        free(sbuf);
        free(rows);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* KV-cache accounting                                                      */
/* ------------------------------------------------------------------------ */

/* Bytes per token of a K+V cache: 2 (K and V) * n_layer * n_kv_head * d_head
 * * bytes_per_elem ([P2] "生成时的瓶颈", the per-token byte formula). */
int64_t oracle_kv_cache_bytes_per_token(int n_layer, int n_kv_head, int d_head, int bytes_per_elem)
{
    return 2LL * n_layer * n_kv_head * d_head * bytes_per_elem;
}

/* Bytes per token of a latent cache: n_layer * (d_c + d_rope) * bytes, no
 * factor 2 because K and V share c^KV ([P1] §2.3.5; [P2] "MLA"). */
int64_t oracle_latent_cache_bytes_per_token(int n_layer, int d_c, int d_rope, int bytes_per_elem)
{
    return (int64_t)n_layer * (d_c + d_rope) * bytes_per_elem;
}

/* ------------------------------------------------------------------------ */
/* FP8 (E4M3) latent cache and indexer keys                                 */
/* ------------------------------------------------------------------------ */
/*
 * [P4] "改进一: DSA" (the paragraph after the selection chain): V3.2 stores,
 * per token and layer, 656 bytes -- the FP8 latent, its scales and the bf16
 * RoPE part -- plus an indexer key of about 132 bytes; [P1] §2.2 (1): the
 * indexer runs stably in fp8.  The pages give the byte budget but no rounding
 * rule.  Reading taken here (the plainest one the budget supports):
 *   - latent row (576 = 512 + 64): the 512 latent values in 4 groups of 128,
 *     each group one fp32 scale and 128 E4M3 codes; the 64 RoPE values kept as
 *     bf16: 4 * 128 * 1 + 4 * 4 + 64 * 2 = 656 bytes, stored in that order;
 *   - indexer key (128 values): one group: 128 codes + one fp32 scale = 132 B;
 *   - scale s = absmax / 448 (448 = the largest finite E4M3 value) in fp32,
 *     code = E4M3 round-to-nearest-even of x / s (fp32 division), saturating
 *     to +-448; an all-zero group has s = 0 and codes 0;
 *   - dequantised value = value(code) * s (exact in fp64).
 * E4M3 (the OCP 8-bit "E4M3FN" format): sign, 4 exponent bits (bias 7),
 * 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6); no infinities;
 * S.1111.111 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.
 */

/* Value of an E4M3 code (NaN for S.1111.111). */
static double e4m3_value(uint8_t c)
{
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sgn ? -v : v;
}

int oracle_e4m3_value(const uint8_t* codes, int64_t n, double* out)
{
    if (n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
    return 0;
}

/* Round an fp32 value to E4M3: the nearest of the 127 finite magnitudes
 * (codes 0x00 .. 0x7E, searched one by one), a tie going to the even code
 * (mantissa LSB 0); magnitudes above 448 saturate to 448; the sign (including
 * that of -0) is kept; NaN gives the NaN code. */
static uint8_t e4m3_round_sat(float y)
{
    if (y != y) return 0x7F;
    double a = fabs((double)y);
    uint8_t sgn = signbit(y) ? 0x80 : 0x00;
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(e4m3_value((uint8_t)c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    if (a > 448.0) best = 0x7E;
    return (uint8_t)(sgn | best);
}

int oracle_e4m3_round(const float* y, int64_t n, uint8_t* codes)
{
    if (n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) codes[i] = e4m3_round_sat(y[i]);
    return 0;
}

/* Quantise n_groups groups of `group` bf16 values (x: bf16 bits, group after
 * group) to E4M3 codes with one fp32 scale per group, as read above. */
int oracle_quant_fp8_groups(const uint16_t* x, int64_t n_groups, int group, uint8_t* codes, float* scales)
{
    if (n_groups < 0 || group <= 0) return -1;
    for (int64_t gi = 0; gi < n_groups; ++gi) {
        const uint16_t* xg = x + gi * group;
        float amax = 0.0f;
        for (int i = 0; i < group; ++i) {
            float a = fabsf((float)bf16_bits_to_f64(xg[i]));
            if (a > amax) amax = a;
        }
        volatile float s = amax / 448.0f; /* fp32 division, as stored */
        scales[gi] = s;
        for (int i = 0; i < group; ++i) {
            if (s == 0.0f) {
                codes[gi * group + i] = 0;
                continue;
            }
            volatile float yv = (float)bf16_bits_to_f64(xg[i]) / s; /* fp32 division */
            codes[gi * group + i] = e4m3_round_sat(yv);
        }
    }
    return 0;
}

/* value(code) * scale for n_groups groups of `group` codes. */
int oracle_dequant_fp8_groups(const uint8_t* codes, const float* scales, int64_t n_groups, int group, double* out)
{
    if (n_groups < 0 || group <= 0) return -1;
    for (int64_t gi = 0; gi < n_groups; ++gi)
        for (int i = 0; i < group; ++i)
            out[gi * group + i] = e4m3_value(codes[gi * group + i]) * (double)scales[gi];
    return 0;
}

#define ORC_LAT_DIM 576
#define ORC_LAT_NOPE 512
#define ORC_LAT_GROUP 128
#define ORC_LAT_ROW_BYTES 656

/* Latent rows [n][576] bf16 -> packed FP8 rows [n][656]: 512 codes, 4 fp32
 * scales (little-endian), 64 bf16 RoPE values. */
int oracle_latent_pack_fp8(const uint16_t* latent, int64_t n_rows, uint8_t* packed)
{
    if (n_rows < 0) return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint16_t* x = latent + r * ORC_LAT_DIM;
        uint8_t* p = packed + r * ORC_LAT_ROW_BYTES;
        float sc[ORC_LAT_NOPE / ORC_LAT_GROUP];
        oracle_quant_fp8_groups(x, ORC_LAT_NOPE / ORC_LAT_GROUP, ORC_LAT_GROUP, p, sc);
        memcpy(p + ORC_LAT_NOPE, sc, sizeof sc);
        memcpy(p + ORC_LAT_NOPE + sizeof sc, x + ORC_LAT_NOPE, (ORC_LAT_DIM - ORC_LAT_NOPE) * sizeof(uint16_t));
    }
    return 0;
}

/* Packed FP8 rows [n][656] -> dequantised latent rows [n][576] (fp64). */
int oracle_latent_unpack_fp8(const uint8_t* packed, int64_t n_rows, double* latent)
{
    if (n_rows < 0) return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint8_t* p = packed + r * ORC_LAT_ROW_BYTES;
        double* y = latent + r * ORC_LAT_DIM;
        float sc[ORC_LAT_NOPE / ORC_LAT_GROUP];
        uint16_t rope[ORC_LAT_DIM - ORC_LAT_NOPE];
        memcpy(sc, p + ORC_LAT_NOPE, sizeof sc);
        memcpy(rope, p + ORC_LAT_NOPE + sizeof sc, sizeof rope);
        oracle_dequant_fp8_groups(p, sc, ORC_LAT_NOPE / ORC_LAT_GROUP, ORC_LAT_GROUP, y);
        for (int i = 0; i < ORC_LAT_DIM - ORC_LAT_NOPE; ++i) y[ORC_LAT_NOPE + i] = bf16_bits_to_f64(rope[i]);
    }
    return 0;
}

/* Bytes of one packed latent row and of one FP8 indexer key (codes + scale). */
int oracle_latent_fp8_row_bytes(void) { return ORC_LAT_NOPE + (ORC_LAT_NOPE / ORC_LAT_GROUP) * 4 + (ORC_LAT_DIM - ORC_LAT_NOPE) * 2; }
int oracle_idx_key_fp8_bytes(int d_I) { return d_I + 4; }

/*
 * Indexer scores in fp8 ([P1] §2.2 (1): the indexer runs stably in fp8, read as its
 * product running on E4M3 operands): each indexer query head q^I_{b,j} (bf16, d_I
 * values, one group) and each key are quantised with the rule above, and
 *   s_{b,t} = sum_j w_{b,j} * ReLU(qhat_{b,j} . khat_{b,t}),  hat = value(code) * scale.
 * qI [B][H_I][d_I] bf16 (quantised here), codes [B][L_max][d_I], scales [B][L_max]
 * fp32; otherwise as oracle_dsa_scores.
 */
int oracle_dsa_scores_fp8(const uint16_t* qI, const float* w, const uint8_t* codes, const float* kscale,
                          const int32_t* lens, int B, int HI, int dI, int L_max, double* scores, int nthreads)
{
    if (B < 0 || HI <= 0 || dI <= 0 || L_max < 0) return -1;
    for (int b = 0; b < B; ++b)
        if (lens[b] < 0 || lens[b] > L_max) return -2;
    int64_t nq = (int64_t)B * HI;
    uint8_t* qc = (uint8_t*)malloc((size_t)(nq * dI > 0 ? nq * dI : 1));
    float* qs = (float*)malloc(sizeof(float) * (size_t)(nq > 0 ? nq : 1));
    double* qd = (double*)malloc(sizeof(double) * (size_t)(nq * dI > 0 ? nq * dI : 1));
    if (!qc || !qs || !qd) {
        free(qc);
        free(qs);
        free(qd);
        return -3;
    }
    oracle_quant_fp8_groups(qI, nq, dI, qc, qs);
    oracle_dequant_fp8_groups(qc, qs, nq, dI, qd);
    src_t Q = {qd, 1};
    int nt = set_threads(nthreads);
    int64_t n_units = (int64_t)B * L_max;
#pragma omp parallel for num_threads(nt) schedule(static)
    for (int64_t u = 0; u < n_units; ++u) {
        int b = (int)(u / L_max);
        int t = (int)(u % L_max);
        if (t >= lens[b]) {
            scores[u] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (int j = 0; j < HI; ++j) {
            double dot = 0.0;
            for (int i = 0; i < dI; ++i)
                dot += ld(Q, ((int64_t)b * HI + j) * dI + i) * (e4m3_value(codes[u * dI + i]) * (double)kscale[u]);
            double relu = dot > 0.0 ? dot : 0.0;
            acc += (double)w[(int64_t)b * HI + j] * relu;
        }
        scores[u] = acc;
    }
    free(qc);
    free(qs);
    free(qd);
    return 0;
}
