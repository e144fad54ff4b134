/*
 * TEST INFRASTRUCTURE — fp64 CPU oracle for MLA decode attention.
 *
 * Only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg call this file.  It shares no code with the CUDA library.
 *
 * What it computes (FlashMLA-ETAP technical summary, "Methodology": the
 * standard attention S = Q K^T, P = softmax(S), O = P V, and the transposed
 * ETAP form S^T = K Q^T, P^T = softmax(S^T), O^T = V^T P^T, O = (O^T)^T):
 *
 *   for every sequence b, query token t and head hd (column n = t*h + hd):
 *     s_j  = scale * sum_{k<576} Q[b,t,hd,k] * KV[b,j,k]     for visible j
 *     m    = max_j s_j
 *     O    = sum_j exp(s_j - m) * KV[b,j,0:512] / sum_j exp(s_j - m)
 *     LSE  = m + ln sum_j exp(s_j - m)                        (natural log)
 *
 * V is the first 512 of the 576 columns of the shared latent KV row (the
 * pages' "low-rank joint compression": one latent row serves as key and value).
 * Visible rows: j < L_b, and for causal multi-token decode j <= L_b - q_len + t
 * (the q_len new tokens are the last q_len cache rows).  A column with no
 * visible row gives O = 0 and LSE = -inf.
 *
 * Ragged multi-token decode (a different number of new tokens per sequence,
 * q_lens[b] <= q_len; the pages decode one token per forward and name more
 * as a limitation: FlashMLA-ETAP Chinese abstract page, "Limitations"): token t of sequence b is a real query iff
 * t < q_lens[b], and then it sees j <= L_b - q_lens[b] + t when causal (its
 * q_lens[b] new tokens are the last q_lens[b] cache rows) or j < L_b; padding
 * tokens t >= q_lens[b] see no row (O = 0, LSE = -inf).
 *
 * Inputs are bf16 bit patterns (uint16), widened exactly to fp64.  All
 * arithmetic is fp64.  Paged caches ([num_blocks, page, 576]) are resolved
 * through the block table; contiguous caches are [B, kv_rows, 576].
 *
 * FP8 latent cache (an adjacent storage format; the pages keep the cache in
 * bf16): every cache row is 576 OCP FP8 E4M3 codes plus one fp32 scale for the
 * row, and element k of row r stands for scale[r] * e4m3(code[r][k]).  The
 * oracle widens every element to that fp64 value and then computes exactly the
 * definition above; the scale array is indexed like the rows ([B, kv_rows], or
 * [num_blocks, page] when paged).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Row j of sequence b's latent KV cache (576 bf16 values). */
static const uint16_t *kv_row(const uint16_t *kv, const int32_t *block_table, int b, int j,
                              int kv_rows, int max_blocks, int page, int d_qk)
{
    if (block_table) {
        int blk = block_table[(int64_t)b * max_blocks + j / page];
        return kv + ((int64_t)blk * page + (j % page)) * d_qk;
    }
    return kv + ((int64_t)b * kv_rows + j) * d_qk;
}

/*
 * OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits (bias 7),
 * 3 mantissa bits, no infinities; exponent 0 is subnormal (m/8 * 2^-6) and the
 * all-ones exponent and mantissa (0x7F, 0xFF) is NaN.  Largest finite value 448.
 */
static double e4m3_to_double(uint8_t code)
{
    int e = (code >> 3) & 0xF, m = code & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);          /* (m / 8) * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m / 8) * 2^(e - 7) */
    return (code & 0x80) ? -v : v;
}

/* A latent cache in either storage format. */
typedef struct {
    const uint16_t *bf16;     /* bf16 bit patterns, or NULL */
    const uint8_t *e4m3;      /* E4M3 codes (with row_scale), or NULL */
    const float *row_scale;   /* one scale per cache row */
    const double *e4m3_value; /* [256] decoded codes */
    const int32_t *block_table;
    int kv_rows, max_blocks, page, d_qk;
} kv_cache;

/* Widen the first n values of row j of sequence b to fp64. */
static void widen_row(const kv_cache *c, int b, int j, int n, double *dst)
{
    int64_t r = c->block_table
                    ? (int64_t)c->block_table[(int64_t)b * c->max_blocks + j / c->page] * c->page + j % c->page
                    : (int64_t)b * c->kv_rows + j;
    if (c->e4m3) {
        const uint8_t *src = c->e4m3 + r * c->d_qk;
        double s = (double)c->row_scale[r];
        for (int k = 0; k < n; ++k) dst[k] = s * c->e4m3_value[src[k]];
    } else {
        const uint16_t *src = c->bf16 + r * c->d_qk;
        for (int k = 0; k < n; ++k) dst[k] = bf16_to_double(src[k]);
    }
}

static int visible_rows(int L, int q_len, int t, int causal)
{
    int vis = causal ? (L - q_len + t + 1) : L;
    return vis < 0 ? 0 : vis;
}

/* Visible rows of token t of sequence b: uniform q_len, or ragged when q_lens != NULL. */
static int token_visible_rows(int L, int q_len, const int32_t *q_lens, int b, int t, int causal)
{
    if (!q_lens) return visible_rows(L, q_len, t, causal);
    int qb = q_lens[b];
    if (t >= qb) return 0;
    return visible_rows(L, qb, t, causal);
}

static int decode_standard(const uint16_t *q, const kv_cache *c, const int32_t *seqlens,
                           const int32_t *q_lens, int B, int q_len, int h, int d_v, double scale,
                           int causal, double *o, double *lse);

static kv_cache bf16_cache(const uint16_t *kv, const int32_t *block_table, int kv_rows, int max_blocks,
                           int page, int d_qk)
{
    kv_cache c = {kv, NULL, NULL, NULL, block_table, kv_rows, max_blocks, page, d_qk};
    return c;
}

/*
 * Standard form: S = Q K^T, P = softmax(S) over the KV axis, O = P V.
 * q: [B, q_len, h, d_qk]; o: [B, q_len, h, d_v]; lse: [B, q_len, h].
 * Returns 0, or -1 on an allocation failure.
 */
int oracle_mla_decode(const uint16_t *q, const uint16_t *kv, const int32_t *seqlens,
                      const int32_t *block_table, int B, int q_len, int h, int d_qk, int d_v,
                      int kv_rows, int max_blocks, int page, double scale, int causal,
                      double *o, double *lse)
{
    kv_cache c = bf16_cache(kv, block_table, kv_rows, max_blocks, page, d_qk);
    return decode_standard(q, &c, seqlens, NULL, B, q_len, h, d_v, scale, causal, o, lse);
}

/* The same with q_lens[b] real query tokens in sequence b (0 <= q_lens[b] <= q_len). */
int oracle_mla_decode_ragged(const uint16_t *q, const uint16_t *kv, const int32_t *seqlens,
                             const int32_t *q_lens, const int32_t *block_table, int B, int q_len,
                             int h, int d_qk, int d_v, int kv_rows, int max_blocks, int page,
                             double scale, int causal, double *o, double *lse)
{
    kv_cache c = bf16_cache(kv, block_table, kv_rows, max_blocks, page, d_qk);
    return decode_standard(q, &c, seqlens, q_lens, B, q_len, h, d_v, scale, causal, o, lse);
}

/*
 * FP8 cache: kv8 holds E4M3 codes laid out like the bf16 cache, kv_scale one
 * fp32 scale per cache row.  q_lens may be NULL (every sequence has q_len
 * query tokens).
 */
int oracle_mla_decode_fp8(const uint16_t *q, const uint8_t *kv8, const float *kv_scale,
                          const int32_t *seqlens, const int32_t *q_lens, const int32_t *block_table,
                          int B, int q_len, int h, int d_qk, int d_v, int kv_rows, int max_blocks,
                          int page, double scale, int causal, double *o, double *lse)
{
    double table[256];
    for (int i = 0; i < 256; ++i) table[i] = e4m3_to_double((uint8_t)i);
    kv_cache c = {NULL, kv8, kv_scale, table, block_table, kv_rows, max_blocks, page, d_qk};
    return decode_standard(q, &c, seqlens, q_lens, B, q_len, h, d_v, scale, causal, o, lse);
}

static int decode_standard(const uint16_t *q, const kv_cache *c, const int32_t *seqlens,
                           const int32_t *q_lens, int B, int q_len, int h, int d_v, double scale,
                           int causal, double *o, double *lse)
{
    int d_qk = c->d_qk;
    int rows = B * q_len * h;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int r = 0; r < rows; ++r) {
        int b = r / (q_len * h);
        int t = (r / h) % q_len;
        int L = seqlens[b];
        int vis = token_visible_rows(L, q_len, q_lens, b, t, causal);
        const uint16_t *qr = q + (int64_t)r * d_qk;
        double *orow = o + (int64_t)r * d_v;
        double qd[1024], kd[1024];
        for (int k = 0; k < d_qk; ++k) qd[k] = bf16_to_double(qr[k]);
        for (int d = 0; d < d_v; ++d) orow[d] = 0.0;
        if (vis == 0) {
            lse[r] = -INFINITY;
            continue;
        }
        double *s = (double *)malloc(sizeof(double) * (size_t)vis);
        if (!s) {
            failed = 1;
            continue;
        }
        /* S row: s_j = scale * q . k_j */
        for (int j = 0; j < vis; ++j) {
            widen_row(c, b, j, d_qk, kd);
            double acc = 0.0;
            for (int k = 0; k < d_qk; ++k) acc += qd[k] * kd[k];
            s[j] = scale * acc;
        }
        /* softmax over the KV axis, two passes */
        double m = s[0];
        for (int j = 1; j < vis; ++j)
            if (s[j] > m) m = s[j];
        double den = 0.0;
        for (int j = 0; j < vis; ++j) {
            s[j] = exp(s[j] - m);
            den += s[j];
        }
        /* O = P V with V = the first d_v columns of the latent row */
        for (int j = 0; j < vis; ++j) {
            widen_row(c, b, j, d_v, kd);
            double p = s[j] / den;
            for (int d = 0; d < d_v; ++d) orow[d] += p * kd[d];
        }
        lse[r] = m + log(den);
        free(s);
    }
    return failed ? -1 : 0;
}

/*
 * Transposed (ETAP) form, step by step for one sequence at a time:
 *   1. S^T = K Q^T          [L x N]   (N = q_len*h query columns)
 *   2. P^T = softmax(S^T) down each column (over the KV rows)
 *   3. O^T = V^T P^T        [d_v x N]
 *   4. O = (O^T)^T          [N x d_v]
 * Same outputs and layouts as oracle_mla_decode.
 */
int oracle_mla_decode_etap(const uint16_t *q, const uint16_t *kv, const int32_t *seqlens,
                           const int32_t *block_table, int B, int q_len, int h, int d_qk, int d_v,
                           int kv_rows, int max_blocks, int page, double scale, int causal,
                           double *o, double *lse)
{
    int N = q_len * h;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int b = 0; b < B; ++b) {
        int L = seqlens[b];
        int Lc = L > 0 ? L : 1;
        double *ST = (double *)malloc(sizeof(double) * (size_t)Lc * N);
        double *OT = (double *)malloc(sizeof(double) * (size_t)d_v * N);
        double *QT = (double *)malloc(sizeof(double) * (size_t)d_qk * N);
        if (!ST || !OT || !QT) {
            free(ST); free(OT); free(QT);
            failed = 1;
            continue;
        }
        /* Q^T [d_qk x N] */
        for (int n = 0; n < N; ++n)
            for (int k = 0; k < d_qk; ++k)
                QT[(int64_t)k * N + n] = bf16_to_double(q[((int64_t)b * N + n) * d_qk + k]);
        /* 1. S^T = K Q^T (scaled); invisible entries are -inf */
        for (int j = 0; j < L; ++j) {
            const uint16_t *kr = kv_row(kv, block_table, b, j, kv_rows, max_blocks, page, d_qk);
            for (int n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int k = 0; k < d_qk; ++k) acc += bf16_to_double(kr[k]) * QT[(int64_t)k * N + n];
                int t = n / h;
                ST[(int64_t)j * N + n] = (j < visible_rows(L, q_len, t, causal)) ? scale * acc : -INFINITY;
            }
        }
        /* 2. P^T = column softmax of S^T (over j); keeps m and the sum for the LSE */
        for (int n = 0; n < N; ++n) {
            int r = b * N + n;
            int vis = visible_rows(L, q_len, n / h, causal);
            if (vis == 0) {
                for (int j = 0; j < L; ++j) ST[(int64_t)j * N + n] = 0.0;
                lse[r] = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (int j = 0; j < L; ++j)
                if (ST[(int64_t)j * N + n] > m) m = ST[(int64_t)j * N + n];
            double den = 0.0;
            for (int j = 0; j < L; ++j) {
                double e = exp(ST[(int64_t)j * N + n] - m);
                ST[(int64_t)j * N + n] = e;
                den += e;
            }
            for (int j = 0; j < L; ++j) ST[(int64_t)j * N + n] /= den;
            lse[r] = m + log(den);
        }
        /* 3. O^T = V^T P^T */
        for (int64_t i = 0; i < (int64_t)d_v * N; ++i) OT[i] = 0.0;
        for (int j = 0; j < L; ++j) {
            const uint16_t *vr = kv_row(kv, block_table, b, j, kv_rows, max_blocks, page, d_qk);
            for (int d = 0; d < d_v; ++d) {
                double v = bf16_to_double(vr[d]);
                for (int n = 0; n < N; ++n) OT[(int64_t)d * N + n] += v * ST[(int64_t)j * N + n];
            }
        }
        /* 4. O = (O^T)^T */
        for (int n = 0; n < N; ++n)
            for (int d = 0; d < d_v; ++d)
                o[((int64_t)b * N + n) * d_v + d] = OT[(int64_t)d * N + n];
        free(ST); free(OT); free(QT);
    }
    return failed ? -1 : 0;
}

/*
 * Merge of attention results over disjoint KV ranges (the log-sum-exp
 * identity): given S partial results (o_s [S x d_v], lse_s [S]) over disjoint
 * row sets, lse = ln sum_s exp(lse_s) and O = sum_s exp(lse_s - lse) o_s.
 * A partial with lse_s = -inf contributes nothing; all -inf gives O = 0.
 */
void oracle_lse_merge(int S, int d_v, const double *o_s, const double *lse_s, double *o, double *lse)
{
    double m = -INFINITY;
    for (int s = 0; s < S; ++s)
        if (lse_s[s] > m) m = lse_s[s];
    for (int d = 0; d < d_v; ++d) o[d] = 0.0;
    if (m == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double sum = 0.0;
    for (int s = 0; s < S; ++s) sum += exp(lse_s[s] - m);
    double l = m + log(sum);
    for (int s = 0; s < S; ++s) {
        double w = exp(lse_s[s] - l);
        for (int d = 0; d < d_v; ++d) o[d] += w * o_s[(int64_t)s * d_v + d];
    }
    *lse = l;
}
