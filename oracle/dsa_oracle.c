/*
 * CPU oracle for the DeepSeek Sparse Attention (DSA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library. The CUDA
 * path never calls it and shares no code with it.
 *
 * Plain, slow, obviously correct: every quantity is the definition written
 * out, accumulated in fp64, one query row at a time. Rows are independent, so
 * the batched drivers run rows in parallel (OpenMP) without changing any
 * row's arithmetic.
 *
 * Sources (page titles and sections):
 *  - "Paper Breakdown: DeepSeek-V3.2", section 2 "Architecture: DSA (2.1)":
 *      index score  I_{t,s} = sum_{j=1..H^I} w^I_{t,j} * ReLU(q^I_{t,j} . k^I_s)
 *      selection    Top-k(I_{t,:})
 *      attention    u_t = Attn(h_t, {c_s : I_{t,s} in Top-k(I_{t,:})})
 *      "DSA under MLA (MQA Mode)": one latent entry c_s shared by all heads.
 *  - "DeepSeek V3.2: Sparse Attention and Reinforcement Learning Updates"
 *      (summary): the selector keeps high-scoring *past* tokens.
 *  - "DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models"
 *      (research summary), "Key points": 2048 selected tokens per query,
 *      few ReLU heads in FP8, MLA in MQA mode.
 *
 * Readings where the pages are silent:
 *  - candidates of row t are s = 0..pos[t] (the current token included);
 *  - equal scores: the lower s ranks first;
 *  - fewer than k candidates: all of them are selected, the rest is -1;
 *  - scores are accumulated in fp64 and rounded to fp32 before ranking;
 *  - the value vector of latent row c_s is its first d_v entries (the latent
 *    part); the trailing rope entries take part in q.c_s only;
 *  - no scale or softmax inside the index score: the formula as printed.
 *
 * Parity pins (tests/test_oracle.py): e4m3/bf16 decoding against the format
 * definition and torch's casts; a hand-derived worked example; int64 brute
 * force on integer inputs; ReLU/weight/head-permutation identities; Top-k
 * against a full lexicographic sort and against the rank definition; the
 * attention closed forms (one key, q = 0, two keys), torch SDPA on gathered
 * rows, order invariance, dense causal MQA equality when k >= L, and the
 * log-sum-exp merge of split sets.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- decoding */

/* OCP 8-bit floating point, E4M3: sign, 4 exponent bits (bias 7), 3 mantissa
 * bits. Exponent field 0 holds subnormals m/8 * 2^-6; S.1111.111 is NaN; there
 * are no infinities, so the largest finite magnitude is 1.75 * 2^8 = 448. */
static double e4m3_decode(unsigned code)
{
    const int sign = (code >> 7) & 1;
    const int e = (code >> 3) & 0xF;
    const int m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);            /* (m/8) * 2^(1-7) */
    else
        v = ldexp(8.0 + (double)m, e - 10);  /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

static double E4M3[256];
static int e4m3_ready = 0;

static void e4m3_init(void)
{
    if (e4m3_ready)
        return;
    for (unsigned c = 0; c < 256; ++c)
        E4M3[c] = e4m3_decode(c);
    e4m3_ready = 1;
}

/* bfloat16 is the upper half of an IEEE binary32. */
static double bf16_decode(uint16_t u)
{
    uint32_t bits = (uint32_t)u << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

void oracle_e4m3_table(double* out)
{
    e4m3_init();
    for (int c = 0; c < 256; ++c)
        out[c] = E4M3[c];
}

void oracle_bf16_decode(const uint16_t* in, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = bf16_decode(in[i]);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------ index score */

/* I_{t,s} for s = 0..n-1 of one query row ("Index score", section 2):
 *   q_row  e4m3 [H_I, d_I]   indexer query heads q^I_{t,j}
 *   w_row  fp32 [H_I]        head weights w^I_{t,j}
 *   keys   e4m3 rows k^I_s at keys + (k_base + s) * d_I
 * Sum over heads of w * ReLU(dot), accumulated in fp64, rounded to fp32. */
void oracle_indexer_row(const uint8_t* q_row, const float* w_row, const uint8_t* keys,
                        int64_t k_base, int64_t n, int H_I, int d_I, float* out)
{
    e4m3_init();
    double* q = (double*)malloc(sizeof(double) * (size_t)H_I * (size_t)d_I);
    for (int i = 0; i < H_I * d_I; ++i)
        q[i] = E4M3[q_row[i]];
    for (int64_t s = 0; s < n; ++s) {
        const uint8_t* kr = keys + (size_t)(k_base + s) * (size_t)d_I;
        double score = 0.0;
        for (int j = 0; j < H_I; ++j) {
            double dot = 0.0;
            for (int d = 0; d < d_I; ++d)
                dot += q[(size_t)j * d_I + d] * E4M3[kr[d]];
            const double relu = dot > 0.0 ? dot : 0.0;
            score += (double)w_row[j] * relu;
        }
        out[s] = (float)score;
    }
    free(q);
}

/* ------------------------------------------------------------ token select */

typedef struct {
    float v;
    int32_t s;
} ranked;

/* Total order: larger score first; equal scores, lower index first. */
static int rank_cmp(const void* a, const void* b)
{
    const ranked* x = (const ranked*)a;
    const ranked* y = (const ranked*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s > y->s) - (x->s < y->s);
}

/* Top-k(I_{t,:}) over candidates s = 0..n-1: the first min(k, n) entries of
 * the full ranking, in rank order, then -1 padding up to k. */
void oracle_topk_row(const float* scores, int64_t n, int k, int32_t* idx_out)
{
    ranked* r = (ranked*)malloc(sizeof(ranked) * (size_t)(n > 0 ? n : 1));
    for (int64_t s = 0; s < n; ++s) {
        r[s].v = scores[s];
        r[s].s = (int32_t)s;
    }
    qsort(r, (size_t)n, sizeof(ranked), rank_cmp);
    for (int i = 0; i < k; ++i)
        idx_out[i] = (i < n) ? r[i].s : -1;
    free(r);
}

/* Indexer + selector for a list of query rows (compact per-row arrays):
 *   q_rows [R, H_I, d_I] e4m3, w_rows [R, H_I], pos_rows [R], base_rows [R];
 *   keys: the whole key cache; idx_out [R, k]. */
void oracle_indexer_topk_rows(const uint8_t* q_rows, const float* w_rows, const uint8_t* keys,
                              const int32_t* pos_rows, const int32_t* base_rows, int R,
                              int H_I, int d_I, int k, int32_t* idx_out)
{
    e4m3_init();
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < R; ++r) {
        const int64_t n = (int64_t)pos_rows[r] + 1;
        float* sc = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
        oracle_indexer_row(q_rows + (size_t)r * H_I * d_I, w_rows + (size_t)r * H_I, keys,
                           base_rows[r], n, H_I, d_I, sc);
        oracle_topk_row(sc, n, k, idx_out + (size_t)r * k);
        free(sc);
    }
}

/* --------------------------------------------------- sparse MQA attention */

/* u_t = Attn(h_t, {c_s : s selected}) in MLA's MQA mode ("DSA under MLA (MQA
 * Mode)", section 2): every query head h attends to the same latent rows c_s.
 *   z_{h,s} = scale * q_{t,h} . c_s          (all d_qk entries)
 *   p_{h,s} = exp(z_{h,s} - m_h) / l_h       (softmax over the selected s)
 *   o_{t,h} = sum_s p_{h,s} * c_s[0:d_v]
 *   lse_h   = m_h + log l_h                  (natural log, scale included)
 * Entries of idx_row that are negative or beyond pos are not candidates and
 * are ignored. With no candidate left, o = 0 and lse = -inf. */
void oracle_sparse_attn_row(const uint16_t* q_row, const uint16_t* kv, int64_t k_base,
                            int64_t pos, const int32_t* idx_row, int k, int Hq, int d_qk,
                            int d_v, double scale, double* out, double* lse)
{
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k > 0 ? k : 1));
    int n = 0;
    for (int i = 0; i < k; ++i)
        if (idx_row[i] >= 0 && idx_row[i] <= pos)
            sel[n++] = idx_row[i];
    double* z = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double* qh = (double*)malloc(sizeof(double) * (size_t)d_qk);
    for (int h = 0; h < Hq; ++h) {
        double* o = out + (size_t)h * d_v;
        for (int c = 0; c < d_v; ++c)
            o[c] = 0.0;
        if (n == 0) {
            lse[h] = -INFINITY;
            continue;
        }
        for (int d = 0; d < d_qk; ++d)
            qh[d] = bf16_decode(q_row[(size_t)h * d_qk + d]);
        double m = -INFINITY;
        for (int i = 0; i < n; ++i) {
            const uint16_t* c_s = kv + (size_t)(k_base + sel[i]) * d_qk;
            double dot = 0.0;
            for (int d = 0; d < d_qk; ++d)
                dot += qh[d] * bf16_decode(c_s[d]);
            z[i] = scale * dot;
            if (z[i] > m)
                m = z[i];
        }
        double l = 0.0;
        for (int i = 0; i < n; ++i)
            l += exp(z[i] - m);
        for (int i = 0; i < n; ++i) {
            const double p = exp(z[i] - m) / l;
            const uint16_t* c_s = kv + (size_t)(k_base + sel[i]) * d_qk;
            for (int c = 0; c < d_v; ++c)
                o[c] += p * bf16_decode(c_s[c]);
        }
        lse[h] = m + log(l);
    }
    free(qh);
    free(z);
    free(sel);
}

/* Attention for a list of query rows: q_rows [R, Hq, d_qk], idx_rows [R, k],
 * pos_rows / base_rows [R]; out [R, Hq, d_v], lse [R, Hq]. */
void oracle_sparse_attn_rows(const uint16_t* q_rows, const uint16_t* kv, const int32_t* idx_rows,
                             const int32_t* pos_rows, const int32_t* base_rows, int R, int k,
                             int Hq, int d_qk, int d_v, double scale, double* out, double* lse)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < R; ++r)
        oracle_sparse_attn_row(q_rows + (size_t)r * Hq * d_qk, kv, base_rows[r], pos_rows[r],
                               idx_rows + (size_t)r * k, k, Hq, d_qk, d_v, scale,
                               out + (size_t)r * Hq * d_v, lse + (size_t)r * Hq);
}

/* Dense causal MQA over every s = 0..pos, written independently of the sparse
 * routine (keys in the outer loop, all logits kept, then per-head softmax).
 * With k >= pos + 1 the sparse path must reproduce it. */
void oracle_dense_attn_row(const uint16_t* q_row, const uint16_t* kv, int64_t k_base,
                           int64_t pos, int Hq, int d_qk, int d_v, double scale, double* out,
                           double* lse)
{
    const int64_t n = pos + 1;
    double* q = (double*)malloc(sizeof(double) * (size_t)Hq * d_qk);
    for (int64_t i = 0; i < (int64_t)Hq * d_qk; ++i)
        q[i] = bf16_decode(q_row[i]);
    double* logit = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * Hq);
    double* c = (double*)malloc(sizeof(double) * (size_t)d_qk);
    for (int64_t s = 0; s < n; ++s) {
        for (int d = 0; d < d_qk; ++d)
            c[d] = bf16_decode(kv[(size_t)(k_base + s) * d_qk + d]);
        for (int h = 0; h < Hq; ++h) {
            double acc = 0.0;
            for (int d = 0; d < d_qk; ++d)
                acc += q[(size_t)h * d_qk + d] * c[d];
            logit[(size_t)s * Hq + h] = acc * scale;
        }
    }
    for (int h = 0; h < Hq; ++h) {
        double m = -INFINITY;
        for (int64_t s = 0; s < n; ++s)
            if (logit[(size_t)s * Hq + h] > m)
                m = logit[(size_t)s * Hq + h];
        double l = 0.0;
        for (int64_t s = 0; s < n; ++s)
            l += exp(logit[(size_t)s * Hq + h] - m);
        for (int cc = 0; cc < d_v; ++cc) {
            double acc = 0.0;
            for (int64_t s = 0; s < n; ++s)
                acc += exp(logit[(size_t)s * Hq + h] - m) *
                       bf16_decode(kv[(size_t)(k_base + s) * d_qk + cc]);
            out[(size_t)h * d_v + cc] = acc / l;
        }
        lse[h] = n > 0 ? m + log(l) : -INFINITY;
    }
    free(c);
    free(logit);
    free(q);
}

/* Log-sum-exp merge of P partial results over disjoint parts of one selected
 * set: lse = log sum_p exp(lse_p), o = sum_p exp(lse_p - lse) o_p. Parts with
 * lse_p = -inf (no candidate) contribute nothing. */
void oracle_lse_merge(const double* o_parts, const double* lse_parts, int P, int Hq, int d_v,
                      double* out, double* lse)
{
    for (int h = 0; h < Hq; ++h) {
        double m = -INFINITY;
        for (int p = 0; p < P; ++p)
            if (lse_parts[(size_t)p * Hq + h] > m)
                m = lse_parts[(size_t)p * Hq + h];
        double* o = out + (size_t)h * d_v;
        for (int c = 0; c < d_v; ++c)
            o[c] = 0.0;
        if (m == -INFINITY) {
            lse[h] = -INFINITY;
            continue;
        }
        double l = 0.0;
        for (int p = 0; p < P; ++p)
            l += exp(lse_parts[(size_t)p * Hq + h] - m);
        const double total = m + log(l);
        for (int p = 0; p < P; ++p) {
            const double wgt = exp(lse_parts[(size_t)p * Hq + h] - total);
            const double* op = o_parts + ((size_t)p * Hq + h) * d_v;
            for (int c = 0; c < d_v; ++c)
                o[c] += wgt * op[c];
        }
        lse[h] = total;
    }
}

/* Backward of the sparse MQA attention: the sparse training stage trains the
 * main model with the LM loss through the selected entries only ("Paper
 * Breakdown: DeepSeek-V3.2", "Continued Pre-Training (2.1.1)" table, row
 * "Sparse Training"). The gradient is that of u_t = Attn(h_t, {c_s}) of the
 * forward above, by the chain rule through softmax.
 * For query row t with selected set sel and each head h (z_s = scale q_h.c_s,
 * p = softmax(z) over sel, o_h = sum_s p_s c_s[0:d_v]), given dout_h:
 *   dp_s = dout_h . c_s[0:d_v]
 *   D    = sum_s p_s dp_s                       (= dout_h . o_h)
 *   dz_s = p_s (dp_s - D)
 *   dq_h = scale sum_s dz_s c_s                 (all d_qk columns)
 *   dc_s += scale dz_s q_h  (all d_qk columns)  +  p_s dout_h  (first d_v)
 * dkv accumulates over rows and heads (a scatter-add over idx); the caller
 * zeroes it. Rows run one after another so the sums are deterministic. */
void oracle_sparse_attn_bwd_rows(const uint16_t* q_rows, const uint16_t* kv, const int32_t* idx_rows,
                                 const int32_t* pos_rows, const int32_t* base_rows, int R, int k,
                                 int Hq, int d_qk, int d_v, double scale, const uint16_t* dout_rows,
                                 double* dq, double* dkv)
{
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k > 0 ? k : 1));
    double* z = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    double* dp = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    double* qh = (double*)malloc(sizeof(double) * (size_t)d_qk);
    double* gh = (double*)malloc(sizeof(double) * (size_t)d_v);
    for (int r = 0; r < R; ++r) {
        const int32_t* idx_row = idx_rows + (size_t)r * k;
        const int64_t pos = pos_rows[r], k_base = base_rows[r];
        int n = 0;
        for (int i = 0; i < k; ++i)
            if (idx_row[i] >= 0 && idx_row[i] <= pos)
                sel[n++] = idx_row[i];
        for (int h = 0; h < Hq; ++h) {
            double* dqh = dq + ((size_t)r * Hq + h) * d_qk;
            for (int d = 0; d < d_qk; ++d)
                dqh[d] = 0.0;
            if (n == 0)
                continue;
            for (int d = 0; d < d_qk; ++d)
                qh[d] = bf16_decode(q_rows[((size_t)r * Hq + h) * d_qk + d]);
            for (int c = 0; c < d_v; ++c)
                gh[c] = bf16_decode(dout_rows[((size_t)r * Hq + h) * d_v + c]);
            double m = -INFINITY;
            for (int i = 0; i < n; ++i) {
                const uint16_t* c_s = kv + (size_t)(k_base + sel[i]) * d_qk;
                double dot = 0.0, dg = 0.0;
                for (int d = 0; d < d_qk; ++d)
                    dot += qh[d] * bf16_decode(c_s[d]);
                for (int c = 0; c < d_v; ++c)
                    dg += gh[c] * bf16_decode(c_s[c]);
                z[i] = scale * dot;
                dp[i] = dg;
                if (z[i] > m)
                    m = z[i];
            }
            double l = 0.0;
            for (int i = 0; i < n; ++i)
                l += exp(z[i] - m);
            double D = 0.0;
            for (int i = 0; i < n; ++i)
                D += exp(z[i] - m) / l * dp[i];
            for (int i = 0; i < n; ++i) {
                const double p = exp(z[i] - m) / l;
                const double dz = p * (dp[i] - D);
                const uint16_t* c_s = kv + (size_t)(k_base + sel[i]) * d_qk;
                double* dc = dkv + (size_t)(k_base + sel[i]) * d_qk;
                for (int d = 0; d < d_qk; ++d) {
                    dqh[d] += scale * dz * bf16_decode(c_s[d]);
                    dc[d] += scale * dz * qh[d];
                }
                for (int c = 0; c < d_v; ++c)
                    dc[c] += p * gh[c];
            }
        }
    }
    free(gh);
    free(qh);
    free(dp);
    free(z);
    free(sel);
}

/* Indexer KL loss and its gradient with respect to the indexer's inputs.
 * "Paper Breakdown: DeepSeek-V3.2", "Continued Pre-Training (2.1.1)" table:
 * the dense warm-up trains the indexer with L^I = sum_t D_KL(p_{t,:} || Softmax(I_{t,:}))
 * with the main model frozen; the sparse stage keeps the KL on the selected set
 * S_t, with the indexer's input detached (no gradient into the main model).
 * The pages leave p_{t,:} undefined; reading: the main attention distribution
 * of row t summed over the query heads and L1-normalised over the keys, so
 * over the set S_t (the dense stage is S_t = every s <= pos[t]):
 *   P_{h,s} = softmax over S_t of scale q_h.c_s        (one distribution per head)
 *   p_s     = sum_h P_{h,s} / sum_{s', h} P_{h,s'}
 *   u_{j,s} = q^I_j.k^I_s,  I_s = sum_j w_j ReLU(u_{j,s})   (index score, unrounded)
 *   L_t     = sum_s p_s (log p_s - log softmax_S(I)_s)     (0 log 0 = 0)
 * p is a constant (detached). With dI_s = softmax_S(I)_s - p_s:
 *   dw_j     = sum_s dI_s ReLU(u_{j,s})
 *   dq^I_j   = sum_s dI_s w_j [u_{j,s} > 0] k^I_s
 *   dk^I_s  += sum_j dI_s w_j [u_{j,s} > 0] q^I_j          (over rows; caller zeroes)
 * ReLU'(0) is taken as 0. S_t = the entries of idx_row that are >= 0 and <= pos.
 * Rows run one after another (dk accumulates deterministically). */
void oracle_indexer_kl_rows(const uint16_t* q_rows, const uint16_t* kv, const int32_t* idx_rows,
                            const int32_t* pos_rows, const int32_t* base_rows, int R, int k, int Hq,
                            int d_qk, double scale, const uint8_t* qi_rows, const float* w_rows,
                            const uint8_t* k_idx, int H_I, int d_I, double* loss, double* dw,
                            double* dqi, double* dki)
{
    e4m3_init();
    const size_t kk = (size_t)(k > 0 ? k : 1);
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * kk);
    double* z = (double*)malloc(sizeof(double) * kk);
    double* p = (double*)malloc(sizeof(double) * kk);
    double* I = (double*)malloc(sizeof(double) * kk);
    double* u = (double*)malloc(sizeof(double) * kk * (size_t)H_I);
    double* qh = (double*)malloc(sizeof(double) * (size_t)d_qk);
    for (int r = 0; r < R; ++r) {
        const int32_t* idx_row = idx_rows + (size_t)r * k;
        const int64_t pos = pos_rows[r], k_base = base_rows[r];
        const uint8_t* qi = qi_rows + (size_t)r * H_I * d_I;
        const float* w = w_rows + (size_t)r * H_I;
        double* dw_r = dw + (size_t)r * H_I;
        double* dq_r = dqi + (size_t)r * H_I * d_I;
        for (int j = 0; j < H_I; ++j)
            dw_r[j] = 0.0;
        for (int e = 0; e < H_I * d_I; ++e)
            dq_r[e] = 0.0;
        loss[r] = 0.0;
        int n = 0;
        for (int i = 0; i < k; ++i)
            if (idx_row[i] >= 0 && idx_row[i] <= pos)
                sel[n++] = idx_row[i];
        if (n == 0)
            continue;
        /* target: head-summed main attention over S_t, L1-normalised */
        for (int i = 0; i < n; ++i)
            p[i] = 0.0;
        for (int h = 0; h < Hq; ++h) {
            for (int d = 0; d < d_qk; ++d)
                qh[d] = bf16_decode(q_rows[((size_t)r * Hq + h) * d_qk + d]);
            double m = -INFINITY;
            for (int i = 0; i < n; ++i) {
                const uint16_t* c_s = kv + (size_t)(k_base + sel[i]) * d_qk;
                double dot = 0.0;
                for (int d = 0; d < d_qk; ++d)
                    dot += qh[d] * bf16_decode(c_s[d]);
                z[i] = scale * dot;
                if (z[i] > m)
                    m = z[i];
            }
            double l = 0.0;
            for (int i = 0; i < n; ++i)
                l += exp(z[i] - m);
            for (int i = 0; i < n; ++i)
                p[i] += exp(z[i] - m) / l;
        }
        double psum = 0.0;
        for (int i = 0; i < n; ++i)
            psum += p[i];
        for (int i = 0; i < n; ++i)
            p[i] /= psum;
        /* index scores over S_t and their log-softmax */
        double mI = -INFINITY;
        for (int i = 0; i < n; ++i) {
            const uint8_t* ks = k_idx + (size_t)(k_base + sel[i]) * d_I;
            double acc = 0.0;
            for (int j = 0; j < H_I; ++j) {
                double dot = 0.0;
                for (int d = 0; d < d_I; ++d)
                    dot += E4M3[qi[(size_t)j * d_I + d]] * E4M3[ks[d]];
                u[(size_t)i * H_I + j] = dot;
                acc += (double)w[j] * (dot > 0.0 ? dot : 0.0);
            }
            I[i] = acc;
            if (acc > mI)
                mI = acc;
        }
        double lI = 0.0;
        for (int i = 0; i < n; ++i)
            lI += exp(I[i] - mI);
        const double lseI = mI + log(lI);
        double L = 0.0;
        for (int i = 0; i < n; ++i)
            if (p[i] > 0.0)
                L += p[i] * (log(p[i]) - (I[i] - lseI));
        loss[r] = L;
        /* gradients through the index score */
        for (int i = 0; i < n; ++i) {
            const double dI = exp(I[i] - lseI) - p[i];
            const uint8_t* ks = k_idx + (size_t)(k_base + sel[i]) * d_I;
            double* dk_s = dki + (size_t)(k_base + sel[i]) * d_I;
            for (int j = 0; j < H_I; ++j) {
                const double uj = u[(size_t)i * H_I + j];
                dw_r[j] += dI * (uj > 0.0 ? uj : 0.0);
                if (uj > 0.0) {
                    const double c = dI * (double)w[j];
                    for (int d = 0; d < d_I; ++d) {
                        dq_r[(size_t)j * d_I + d] += c * E4M3[ks[d]];
                        dk_s[d] += c * E4M3[qi[(size_t)j * d_I + d]];
                    }
                }
            }
        }
    }
    free(qh);
    free(u);
    free(I);
    free(p);
    free(z);
    free(sel);
}

/* MLA in MHA mode over a causal sequence (the bilingual paper summary's list of
 * sections, "Appendix A MHA and MQA Modes of MLA", title only; "Paper
 * Breakdown: DeepSeek-V3.2", section 2, "DSA under MLA (MQA Mode)"). Reading:
 * in MHA mode every head has its own key and value rows (the latent row
 * expanded per head), where MQA mode shares one latent row across heads. For a
 * short prefill (L <= k) the selector keeps every causal key, so the mode is
 * dense causal attention, per row t and head h over s = 0..pos:
 *   z_s = scale q_{t,h}.k_{s,h},  o_{t,h} = sum_s softmax(z)_s v_{s,h},
 *   lse = log sum_s exp(z_s)
 * q [R, Hq, d_h] (row r at position pos_rows[r]), k [S, Hq, d_h], v [S, Hq, d_hv]
 * (bf16); keys of row r at base_rows[r] + s. */
void oracle_mha_attn_rows(const uint16_t* q_rows, const uint16_t* k, const uint16_t* v,
                          const int32_t* pos_rows, const int32_t* base_rows, int R, int Hq, int d_h,
                          int d_hv, double scale, double* out, double* lse)
{
    for (int r = 0; r < R; ++r) {
        const int64_t n = (int64_t)pos_rows[r] + 1, base = base_rows[r];
        double* z = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        for (int h = 0; h < Hq; ++h) {
            double* o = out + ((size_t)r * Hq + h) * d_hv;
            for (int c = 0; c < d_hv; ++c)
                o[c] = 0.0;
            if (n <= 0) {
                lse[(size_t)r * Hq + h] = -INFINITY;
                continue;
            }
            const uint16_t* qh = q_rows + ((size_t)r * Hq + h) * d_h;
            double m = -INFINITY;
            for (int64_t s = 0; s < n; ++s) {
                const uint16_t* ks = k + ((size_t)(base + s) * Hq + h) * d_h;
                double dot = 0.0;
                for (int d = 0; d < d_h; ++d)
                    dot += bf16_decode(qh[d]) * bf16_decode(ks[d]);
                z[s] = scale * dot;
                if (z[s] > m)
                    m = z[s];
            }
            double l = 0.0;
            for (int64_t s = 0; s < n; ++s)
                l += exp(z[s] - m);
            for (int64_t s = 0; s < n; ++s) {
                const double p = exp(z[s] - m) / l;
                const uint16_t* vs = v + ((size_t)(base + s) * Hq + h) * d_hv;
                for (int c = 0; c < d_hv; ++c)
                    o[c] += p * bf16_decode(vs[c]);
            }
            lse[(size_t)r * Hq + h] = m + log(l);
        }
        free(z);
    }
}

/* ------------------------------------------- index scores of many rows */

/* I_{t,s} of a list of query rows, one oracle_indexer_row per row (rows run
 * in parallel; the arithmetic is that function's):
 *   q_rows [R, H_I, d_I] e4m3, w_rows [R, H_I], pos_rows [R], base_rows [R];
 *   out [R, ld] fp32: row r holds s = 0..pos_rows[r]; entries past that are
 *   left untouched (ld >= max pos + 1). */
void oracle_indexer_scores_rows(const uint8_t* q_rows, const float* w_rows, const uint8_t* keys,
                                const int32_t* pos_rows, const int32_t* base_rows, int R, int H_I,
                                int d_I, int64_t ld, float* out)
{
    e4m3_init();
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < R; ++r)
        oracle_indexer_row(q_rows + (size_t)r * H_I * d_I, w_rows + (size_t)r * H_I, keys,
                           base_rows[r], (int64_t)pos_rows[r] + 1, H_I, d_I, out + (size_t)r * ld);
}
