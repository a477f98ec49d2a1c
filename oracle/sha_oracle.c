/*
 * sha_oracle.c -- float64 CPU oracle for Selective Head Attention (SHA) decode.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * reference that the CUDA path is checked against.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline / reference arm may load it.
 * It shares no code, header, table or helper with the CUDA library, and the
 * CUDA library never calls it.
 *
 * What it computes (sources: the pages about "Polar Sparsity: High Throughput
 * Batched LLM Inferencing with Scalable Contextual Sparsity"):
 *
 *  - attention of one query row against one head's cache, as the equation
 *    under "Attention Head 稀疏性" (papernotes.org summary) defines it:
 *        O = softmax(scale * q K^T) V,   scale = 1/sqrt(d_h) by default;
 *  - the same quantity by the tiled online-softmax recurrence of Algorithm 1,
 *    "Selective Head Flash Attention (Decode)" (ri.k117.org reproducibility
 *    record, "Pseudocode" row), which renormalises the accumulator after
 *    every tile of Bc keys;
 *  - the routing of Algorithm 1 and of the "Selective Head Attention (SHA)
 *    Kernel" section (papernotes.org): for every batch row b and slot k the
 *    head id h = batch_head_index[b,k] is looked up, only that head's K/V are
 *    read and only its output rows are written; all other output rows keep
 *    whatever the caller put there.  For GQA the unit of selection is a KV
 *    group (same section: "group sparsity"); query head h*G + j, j < G, reads
 *    KV head h.
 *
 * Inputs are the raw 16-bit patterns of IEEE binary16 (fp16) or bfloat16
 * values.  Each is widened to double exactly; every sum, product and exp is
 * then done in double, in the plain order of the definition.
 *
 * Function pins (tests/test_oracle_pins.py): all 65536 patterns of each
 * format against numpy's widening; hand-derived exact results
 * (tests/golden/); torch's scaled_dot_product_attention in float64 when every
 * head is active; closed forms (one key, equal keys, zero scale); the
 * online recurrence against the two-pass definition; permutation and shift
 * invariance; convexity; untouched inactive rows.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_FP16 = 0, ORACLE_BF16 = 1 };

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double fp16_to_double(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int exponent = (bits >> 10) & 0x1f;
    int fraction = bits & 0x3ff;
    double magnitude;
    if (exponent == 0)          /* zero or subnormal: fraction * 2^-24 */
        magnitude = ldexp((double)fraction, -24);
    else if (exponent == 31)    /* infinity or NaN */
        magnitude = fraction ? NAN : INFINITY;
    else                        /* normal: (1 + fraction/1024) * 2^(exponent-15) */
        magnitude = ldexp((double)(1024 + fraction), exponent - 25);
    return sign ? -magnitude : magnitude;
}

/* bfloat16 is the upper half of an IEEE binary32 pattern. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t word = (uint32_t)bits << 16;
    float value;
    memcpy(&value, &word, sizeof value);
    return (double)value;
}

static double widen(uint16_t bits, int dtype)
{
    return dtype == ORACLE_BF16 ? bf16_to_double(bits) : fp16_to_double(bits);
}

double sha_oracle_widen(uint16_t bits, int dtype) { return widen(bits, dtype); }

/* scale * <q, K[n]> for one key row n. */
static double score(const uint16_t *q, const uint16_t *key_row, int d,
                    double scale, int dtype)
{
    double dot = 0.0;
    for (int c = 0; c < d; ++c)
        dot += widen(q[c], dtype) * widen(key_row[c], dtype);
    return scale * dot;
}

/*
 * Definition: O = softmax(scale * q K^T) V over all n_kv keys.
 * Pass 1 forms the scores and their maximum M; pass 2 forms
 * p[n] = exp(s[n] - M), L = sum p[n] and O[c] = sum_n p[n] V[n,c] / L.
 * Subtracting M leaves the quotient unchanged; it only keeps exp finite.
 * s is caller scratch of n_kv doubles.
 */
static void attention_definition(const uint16_t *q, const uint16_t *K,
                                 const uint16_t *V, int n_kv, int d,
                                 double scale, int dtype, double *s, double *o)
{
    double M = -INFINITY;
    for (int n = 0; n < n_kv; ++n) {
        s[n] = score(q, K + (size_t)n * d, d, scale, dtype);
        if (s[n] > M) M = s[n];
    }
    double L = 0.0;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int n = 0; n < n_kv; ++n) {
        double p = exp(s[n] - M);
        L += p;
        const uint16_t *v_row = V + (size_t)n * d;
        for (int c = 0; c < d; ++c) o[c] += p * widen(v_row[c], dtype);
    }
    for (int c = 0; c < d; ++c) o[c] /= L;
}

/*
 * Algorithm 1's recurrence, taken as the pages give it: state
 * (O_acc, l_acc, m_acc) starts at (0, 0, -inf); the keys are visited in
 * Tc = ceil(n_kv / Bc) tiles [kstart, kend), kend = min(j*Bc, n_kv).  Per tile:
 *   S_j = scale * q K_j^T,  m_j = max S_j,  P_j = exp(S_j - m_j),  l_j = sum P_j
 *   m_new = max(m_acc, m_j),  alpha = exp(m_acc - m_new),  beta = exp(m_j - m_new)
 *   l_new = alpha*l_acc + beta*l_j
 *   O_acc = (alpha*l_acc*O_acc + beta*(P_j V_j)) / l_new
 * so O_acc is a normalised average after every tile.
 * s and pv are caller scratch of Bc and d doubles.
 */
static void attention_online(const uint16_t *q, const uint16_t *K,
                             const uint16_t *V, int n_kv, int d, double scale,
                             int dtype, int Bc, double *s, double *pv,
                             double *o)
{
    double m_acc = -INFINITY, l_acc = 0.0;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    int Tc = (n_kv + Bc - 1) / Bc;
    for (int j = 1; j <= Tc; ++j) {
        int kstart = (j - 1) * Bc;
        int kend = j * Bc < n_kv ? j * Bc : n_kv;
        double m_j = -INFINITY;
        for (int n = kstart; n < kend; ++n) {
            s[n - kstart] = score(q, K + (size_t)n * d, d, scale, dtype);
            if (s[n - kstart] > m_j) m_j = s[n - kstart];
        }
        double l_j = 0.0;
        for (int c = 0; c < d; ++c) pv[c] = 0.0;
        for (int n = kstart; n < kend; ++n) {
            double p = exp(s[n - kstart] - m_j);
            l_j += p;
            const uint16_t *v_row = V + (size_t)n * d;
            for (int c = 0; c < d; ++c) pv[c] += p * widen(v_row[c], dtype);
        }
        double m_new = m_acc > m_j ? m_acc : m_j;
        double alpha = exp(m_acc - m_new);
        double beta = exp(m_j - m_new);
        double l_new = alpha * l_acc + beta * l_j;
        for (int c = 0; c < d; ++c)
            o[c] = (alpha * l_acc * o[c] + beta * pv[c]) / l_new;
        l_acc = l_new;
        m_acc = m_new;
    }
}

/* One (query row, head) pair by either method; Bc <= 0 selects the definition. */
static void attention(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                      int n_kv, int d, double scale, int dtype, int Bc,
                      double *o)
{
    if (Bc <= 0) {
        double *s = (double *)malloc(sizeof(double) * (size_t)n_kv);
        attention_definition(q, K, V, n_kv, d, scale, dtype, s, o);
        free(s);
    } else {
        double *s = (double *)malloc(sizeof(double) * (size_t)Bc);
        double *pv = (double *)malloc(sizeof(double) * (size_t)d);
        attention_online(q, K, V, n_kv, d, scale, dtype, Bc, s, pv, o);
        free(pv);
        free(s);
    }
}

/*
 * Selective head decode over the full layout
 *   Q, out : [B, H_q, d]        K, V : [B, H_kv, N_kv, d]
 *   batch_head_index : [B, top_k], values are KV-head ids in [0, H_kv)
 * G = H_q / H_kv query heads share one KV head (G = 1 is plain multi-head
 * attention).  For every (b, k) with h = batch_head_index[b,k] in range, rows
 * out[b, h*G + j, :], j < G, are overwritten; an id out of range writes
 * nothing and is counted.  No other element of out is touched.
 * Bc <= 0 uses the definition, Bc > 0 Algorithm 1's tiled recurrence.
 * Returns the number of out-of-range ids, or -1 for inconsistent sizes.
 */
long long sha_oracle_decode(const uint16_t *Q, const uint16_t *K,
                            const uint16_t *V, const int32_t *batch_head_index,
                            int B, int H_q, int H_kv, int N_kv, int d,
                            int top_k, double scale, int dtype, int Bc,
                            double *out)
{
    if (B < 0 || H_kv <= 0 || H_q <= 0 || H_q % H_kv != 0 || N_kv <= 0 ||
        d <= 0 || top_k < 0)
        return -1;
    int G = H_q / H_kv;
    long long bad = 0;
    long long units = (long long)B * top_k;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (long long u = 0; u < units; ++u) {
        long long b = u / top_k;
        int h = batch_head_index[u];
        if (h < 0 || h >= H_kv) {
            bad += 1;
            continue;
        }
        const uint16_t *K_bh = K + ((size_t)b * H_kv + h) * (size_t)N_kv * d;
        const uint16_t *V_bh = V + ((size_t)b * H_kv + h) * (size_t)N_kv * d;
        for (int j = 0; j < G; ++j) {
            size_t row = ((size_t)b * H_q + (size_t)h * G + j) * (size_t)d;
            attention(Q + row, K_bh, V_bh, N_kv, d, scale, dtype, Bc, out + row);
        }
    }
    return bad;
}

/*
 * The same per-unit computation on units already gathered by the caller:
 *   Qu, out : [n_units, G, d]     Ku, Vu : [n_units, N_kv, d]
 * (unit i is one selected (batch row, KV head) pair with its G query rows).
 * Used to check sampled units of workloads too large to widen whole.
 */
int sha_oracle_units(const uint16_t *Qu, const uint16_t *Ku, const uint16_t *Vu,
                     int n_units, int G, int N_kv, int d, double scale,
                     int dtype, int Bc, double *out)
{
    if (n_units < 0 || G <= 0 || N_kv <= 0 || d <= 0) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_units; ++i) {
        const uint16_t *K_i = Ku + (size_t)i * N_kv * d;
        const uint16_t *V_i = Vu + (size_t)i * N_kv * d;
        for (int j = 0; j < G; ++j) {
            size_t row = ((size_t)i * G + j) * (size_t)d;
            attention(Qu + row, K_i, V_i, N_kv, d, scale, dtype, Bc, out + row);
        }
    }
    return 0;
}

/* Number of host threads the parallel loops above use. */
int sha_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Head selection: the step that turns the attention router's per-head scores
 * into batch_head_index (papernotes.org summary, "Router 训练": the attention
 * router is one fully connected layer whose top-k heads are kept; atlas.scime.ai
 * summary: a router picks the top-k attention heads or GQA groups per token).
 * For every row b the top_k heads with the largest scores[b, :] are written in
 * order of decreasing score; equal scores are ordered by increasing head id.
 * Done here by top_k rounds of "take the best head not yet taken".
 * Returns -1 for inconsistent sizes.
 */
int sha_oracle_select_heads(const float *scores, int B, int H, int top_k,
                            int32_t *batch_head_index)
{
    if (B < 0 || H <= 0 || top_k < 0 || top_k > H) return -1;
    unsigned char *taken = (unsigned char *)malloc((size_t)H);
    for (int b = 0; b < B; ++b) {
        const float *row = scores + (size_t)b * H;
        memset(taken, 0, (size_t)H);
        for (int k = 0; k < top_k; ++k) {
            int best = -1;
            for (int h = 0; h < H; ++h) {
                if (taken[h]) continue;
                if (best < 0 || row[h] > row[best]) best = h;   /* ties keep the lower id */
            }
            taken[best] = 1;
            batch_head_index[(size_t)b * top_k + k] = best;
        }
    }
    free(taken);
    return 0;
}

/*
 * Selective head decode when every batch row has its own cache length: row b
 * attends to keys [0, seqlens[b]) of its [N_max]-long cache (a decode batch
 * whose sequences have different lengths).  Each selected unit is exactly the
 * operation of sha_oracle_decode on that row's first seqlens[b] keys.  Rows
 * whose length is outside [1, N_max] are skipped and counted like out-of-range
 * ids.  Returns the count, or -1 for inconsistent sizes.
 */
long long sha_oracle_decode_varlen(const uint16_t *Q, const uint16_t *K,
                                   const uint16_t *V, const int32_t *batch_head_index,
                                   const int32_t *seqlens, int B, int H_q, int H_kv,
                                   int N_max, int d, int top_k, double scale, int dtype,
                                   double *out)
{
    if (B < 0 || H_kv <= 0 || H_q <= 0 || H_q % H_kv != 0 || N_max <= 0 ||
        d <= 0 || top_k < 0)
        return -1;
    int G = H_q / H_kv;
    long long bad = 0;
    long long units = (long long)B * top_k;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (long long u = 0; u < units; ++u) {
        long long b = u / top_k;
        int h = batch_head_index[u];
        int n = seqlens[b];
        if (h < 0 || h >= H_kv || n < 1 || n > N_max) {
            bad += 1;
            continue;
        }
        const uint16_t *K_bh = K + ((size_t)b * H_kv + h) * (size_t)N_max * d;
        const uint16_t *V_bh = V + ((size_t)b * H_kv + h) * (size_t)N_max * d;
        for (int j = 0; j < G; ++j) {
            size_t row = ((size_t)b * H_q + (size_t)h * G + j) * (size_t)d;
            attention(Q + row, K_bh, V_bh, n, d, scale, dtype, 0, out + row);
        }
    }
    return bad;
}

/*
 * Head x token sparsity.  The pages name it only as future work: combining
 * head sparsity with token sparsity "may give multiplicative speedups"
 * (papernotes.org summary, "局限与展望"); they give no method.  The plainest
 * reading: each selected (batch row, head) unit attends to a given subset of
 * its own head's keys,
 *     tokens : [B, top_k, n_sel], key positions in [0, N_kv) of the head
 *              selected by slot k of row b,
 * and the unit's output is the attention equation restricted to those keys:
 *     s_i = scale * <q, K[t_i]>,  O = sum_i exp(s_i - M) V[t_i] / sum_i exp(s_i - M),
 * M = max_i s_i, i < n_sel.  A position listed twice counts twice (the subset
 * is a list).  A unit with a position outside [0, N_kv) is skipped (nothing
 * written) and counted with the out-of-range head ids.  Returns the count,
 * or -1 for inconsistent sizes.
 */
long long sha_oracle_decode_tokens(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                                   const int32_t *batch_head_index, const int32_t *tokens,
                                   int B, int H_q, int H_kv, int N_kv, int d, int top_k,
                                   int n_sel, double scale, int dtype, double *out)
{
    if (B < 0 || H_kv <= 0 || H_q <= 0 || H_q % H_kv != 0 || N_kv <= 0 || d <= 0 ||
        top_k < 0 || n_sel <= 0)
        return -1;
    int G = H_q / H_kv;
    long long bad = 0;
    long long units = (long long)B * top_k;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (long long u = 0; u < units; ++u) {
        long long b = u / top_k;
        int h = batch_head_index[u];
        const int32_t *t = tokens + (size_t)u * n_sel;
        int ok = h >= 0 && h < H_kv;
        for (int i = 0; ok && i < n_sel; ++i) ok = t[i] >= 0 && t[i] < N_kv;
        if (!ok) {
            bad += 1;
            continue;
        }
        const uint16_t *K_bh = K + ((size_t)b * H_kv + h) * (size_t)N_kv * d;
        const uint16_t *V_bh = V + ((size_t)b * H_kv + h) * (size_t)N_kv * d;
        double *sc = (double *)malloc(sizeof(double) * (size_t)n_sel);
        for (int j = 0; j < G; ++j) {
            size_t row = ((size_t)b * H_q + (size_t)h * G + j) * (size_t)d;
            double M = -INFINITY;
            for (int i = 0; i < n_sel; ++i) {
                sc[i] = score(Q + row, K_bh + (size_t)t[i] * d, d, scale, dtype);
                if (sc[i] > M) M = sc[i];
            }
            double L = 0.0;
            double *o = out + row;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int i = 0; i < n_sel; ++i) {
                double p = exp(sc[i] - M);
                L += p;
                const uint16_t *v_row = V_bh + (size_t)t[i] * d;
                for (int c = 0; c < d; ++c) o[c] += p * widen(v_row[c], dtype);
            }
            for (int c = 0; c < d; ++c) o[c] /= L;
        }
        free(sc);
    }
    return bad;
}

/*
 * Selective head decode over a paged KV cache (the serving layout in which a
 * sequence's keys live in fixed-size pages of a shared pool):
 *   K, V        : [num_pages, H_kv, page_size, d]
 *   block_table : [B, max_pages]; key n of row b is at page
 *                 block_table[b, n / page_size], position n % page_size
 *   seqlens     : [B]; row b attends to keys [0, seqlens[b])
 * Each unit gathers its row's keys and values through the block table and is
 * then exactly the per-row-length decode.  A row whose length is outside
 * [1, max_pages * page_size], or that needs a page id outside [0, num_pages),
 * is skipped and counted with the out-of-range head ids.
 */
long long sha_oracle_decode_paged(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                                  const int32_t *batch_head_index, const int32_t *seqlens,
                                  const int32_t *block_table, int B, int H_q, int H_kv,
                                  int num_pages, int page_size, int max_pages, int d,
                                  int top_k, double scale, int dtype, double *out)
{
    if (B < 0 || H_kv <= 0 || H_q <= 0 || H_q % H_kv != 0 || num_pages <= 0 ||
        page_size <= 0 || max_pages <= 0 || d <= 0 || top_k < 0)
        return -1;
    int G = H_q / H_kv;
    long long bad = 0;
    long long units = (long long)B * top_k;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (long long u = 0; u < units; ++u) {
        long long b = u / top_k;
        int h = batch_head_index[u];
        int n = seqlens[b];
        int ok = h >= 0 && h < H_kv && n >= 1 && n <= max_pages * page_size;
        for (int p = 0; ok && p < (n + page_size - 1) / page_size; ++p) {
            int page = block_table[b * (long long)max_pages + p];
            if (page < 0 || page >= num_pages) ok = 0;
        }
        if (!ok) {
            bad += 1;
            continue;
        }
        uint16_t *Kg = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)n * d);
        uint16_t *Vg = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)n * d);
        for (int key = 0; key < n; ++key) {
            int page = block_table[b * (long long)max_pages + key / page_size];
            size_t src = (((size_t)page * H_kv + h) * page_size + key % page_size) * (size_t)d;
            memcpy(Kg + (size_t)key * d, K + src, sizeof(uint16_t) * (size_t)d);
            memcpy(Vg + (size_t)key * d, V + src, sizeof(uint16_t) * (size_t)d);
        }
        for (int j = 0; j < G; ++j) {
            size_t row = ((size_t)b * H_q + (size_t)h * G + j) * (size_t)d;
            attention(Q + row, Kg, Vg, n, d, scale, dtype, 0, out + row);
        }
        free(Vg);
        free(Kg);
    }
    return bad;
}

/*
 * Selective GEMM -- the MLP half of Polar Sparsity (papernotes.org summary,
 * "MLP 层动态稀疏"): for a decode batch x [B, d] and the union S_B of the
 * neurons active for any row of the batch,
 *     MLP_{S_B}(x) = sigma(x W1[:, S_B]) W2[:, S_B]^T,
 * with W1, W2 of shape [d, D].  Both are passed transposed, neuron-major:
 * W1t = W1^T and W2t = W2^T, [D, d], so neuron j's weights are row j.
 * sigma is ReLU (act = 1) or the identity (act = 0).
 */
int sha_oracle_mlp_union(const uint8_t *active, int B, int D, int32_t *S)
{
    if (B < 0 || D <= 0) return -1;
    int n = 0;
    for (int j = 0; j < D; ++j) {
        int any = 0;
        for (int b = 0; b < B; ++b) any |= active[(size_t)b * D + j] != 0;
        if (any) S[n++] = j;
    }
    return n;
}

/* W2t may hold a subset of the output columns: [D, d_out], y [B, d_out]
 * (output columns are independent, so this is the same sum restricted). */
int sha_oracle_selective_mlp(const uint16_t *x, const uint16_t *W1t, const uint16_t *W2t,
                             const int32_t *S, int n_S, int B, int d, int d_out, int D,
                             int act, int dtype, double *y)
{
    if (B < 0 || d <= 0 || d_out <= 0 || D <= 0 || n_S < 0 || n_S > D) return -1;
    for (int t = 0; t < n_S; ++t)
        if (S[t] < 0 || S[t] >= D) return -1;
#pragma omp parallel for schedule(static)
    for (int b = 0; b < B; ++b) {
        double *yb = y + (size_t)b * d_out;
        for (int c = 0; c < d_out; ++c) yb[c] = 0.0;
        for (int t = 0; t < n_S; ++t) {
            const int j = S[t];
            const uint16_t *w1 = W1t + (size_t)j * d, *w2 = W2t + (size_t)j * d_out;
            double pre = 0.0;
            for (int i = 0; i < d; ++i) pre += widen(x[(size_t)b * d + i], dtype) * widen(w1[i], dtype);
            const double h = (act == 1 && pre < 0.0) ? 0.0 : pre;
            for (int c = 0; c < d_out; ++c) yb[c] += h * widen(w2[c], dtype);
        }
    }
    return 0;
}
