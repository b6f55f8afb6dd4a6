/*
 * Fathom key-scan ORACLE -- test infrastructure only.
 *
 * A plain, slow, obviously-correct CPU statement of what the Fathom scan
 * computes, in double precision, written from the paper's prose
 * ("Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded KV
 * Caches", arXiv 2609.17652, as retold on the yeyulingfeng.com article
 * sections "方法一" (bit planes) and "方法二" (reverse water-filling)).
 * Only the test suite, the package's smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header,
 * table or constant with the CUDA path.
 *
 * Precision: fp64 everywhere, except the channel importance w_j, which is
 * evaluated with IEEE single-precision operations in a fixed order (see
 * orc_plan) so that the integer plan it feeds is defined bit for bit.
 * Build with -ffp-contract=off so no multiply-add is fused.
 *
 * Every function is a direct transcription of a definition:
 *   orc_fp16_bits      IEEE 754 binary16 round-to-nearest-even
 *   orc_code4          4-bit uniform symmetric code (bit planes section)
 *   orc_dequant        t-plane prefix dequantisation (bit planes section)
 *   orc_pack           block scales + channel-major bit planes
 *   orc_plan           reverse water-filling plan (water-filling section)
 *   orc_plan_fixed     fixed-depth r-channel plan (byte-accounting section)
 *   orc_scan           variable-depth scores (water-filling section, last
 *                      paragraph: one plan shared by the G heads)
 *   orc_topk           full sort per query head + union per KV head
 *                      (byte-accounting section, top-k bullet)
 *   orc_dequant_rows   whole key rows rebuilt from the planes (limits
 *                      section, storage-overhead paragraph)
 *   orc_calibrate      per-KV-head key statistics from the session's own
 *                      keys: mean, population variance (the sigma^2 of the
 *                      water-filling section) and covariance (experiments
 *                      section, calibration-domain paragraph; rotated
 *                      basis of the multi-model paragraph)
 *   orc_union_attention  softmax attention of each query head over its KV
 *                      head's union of winner rows (byte-accounting
 *                      section: the winner rows a step fetches)
 *   orc_layer_budgets  greedy split of a total plane-bit budget across
 *                      layers (water-filling section, per-layer plan
 *                      paragraph)
 *   orc_pack_nibbles   the same 4-bit codes stored whole, 4 bits per token
 *                      (the fixed-depth scans' 4-bit coordinates of the
 *                      byte-accounting section), 16 tokens per 64-bit word
 *   orc_rotate_keys    the keys' coordinates in a rotated orthonormal basis
 *                      (base-choice section: models without QK-norm store
 *                      keys in the KLT basis), in a fixed single-precision
 *                      order of fused multiply-adds; orc_pack of them is
 *                      the rotated index
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_ENOMEM (-2)

/* ------------------------------------------------------------------ */
/* IEEE 754 binary16, round to nearest, ties to even.                  */
/* Written from the standard: binary16 has 1 sign bit, 5 exponent bits  */
/* (bias 15) and 10 fraction bits; normal numbers are (1+f/1024)*2^(e-15)*/
/* for e in 1..30, subnormals f/1024 * 2^-14, and anything that rounds  */
/* to 2^16 or more becomes infinity.                                    */
/* ------------------------------------------------------------------ */
uint16_t orc_fp16_bits(double x)
{
    uint16_t sign = 0;
    if (x != x) return 0x7E00; /* NaN */
    if (signbit(x)) { sign = 0x8000; x = -x; }
    if (x == 0.0) return sign;
    if (isinf(x)) return sign | 0x7C00;

    /* Quantum (spacing of representable values) at x's binade. */
    int e2;
    frexp(x, &e2);               /* x = m * 2^e2, m in [0.5, 1) */
    int unbiased = e2 - 1;       /* x in [2^unbiased, 2^(unbiased+1)) */
    if (unbiased < -14) unbiased = -14; /* subnormal range shares the 2^-24 quantum */
    double quantum = ldexp(1.0, unbiased - 10);

    double r = x / quantum;      /* exact: dividing by a power of two */
    double fl = floor(r);
    double frac = r - fl;
    double m;
    if (frac > 0.5) m = fl + 1.0;
    else if (frac < 0.5) m = fl;
    else m = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0; /* tie: to even */

    double y = m * quantum;      /* rounded magnitude */
    if (y >= 65536.0) return sign | 0x7C00; /* overflow to infinity */

    /* Encode y. */
    if (y < ldexp(1.0, -14)) {   /* subnormal (or smallest normal reached by rounding) */
        int f = (int)(y / ldexp(1.0, -24));
        if (f >= 1024) return sign | (uint16_t)(1 << 10); /* rounded up to min normal */
        return sign | (uint16_t)f;
    }
    int ey;
    double my = frexp(y, &ey);   /* y = my * 2^ey, my in [0.5,1) */
    int e = ey - 1 + 15;         /* biased exponent */
    int f = (int)((my * 2.0 - 1.0) * 1024.0);
    return sign | (uint16_t)(e << 10) | (uint16_t)f;
}

double orc_fp16_value(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)f, -24);
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp(1.0 + f / 1024.0, e - 15);
    return s ? -v : v;
}

/* bf16 -> value: bf16 is the top half of an IEEE binary32 word. */
static double orc_bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* ------------------------------------------------------------------ */
/* Quantiser (bit planes section).  A block of 64 tokens of one        */
/* channel has scale s = fp16(max |k|); 16 uniform cells of width      */
/* s/8 cover [-s, s]; the code is the cell index, clamped to 0..15, so  */
/* code 8 is the cell [0, s/8) and the top bit is the sign.            */
/* ------------------------------------------------------------------ */
int orc_code4(double k, double s)
{
    if (!(s > 0.0) || isinf(s)) return 8;
    double cell = floor(8.0 * k / s); /* exact for fp32/bf16 k and fp16 s */
    double c = cell + 8.0;
    if (c < 0.0) c = 0.0;
    if (c > 15.0) c = 15.0;
    return (int)c;
}

/* Prefix dequantisation: the first t planes give c_t = c >> (4 - t), and  */
/* the value is the centre of cell c_t of the t-bit mid-rise quantiser on  */
/* [-s, s], i.e. -s + (c_t + 1/2) * 2s / 2^t.  t = 0 reads nothing: 0.      */
double orc_dequant(int c4, int t, double s)
{
    if (t <= 0) return 0.0;
    int ct = c4 >> (4 - t);
    double cells = ldexp(1.0, t);
    return -s + (ct + 0.5) * (2.0 * s / cells);
}

/* keys: [H][n][D] token-major with the given strides (elements);
 * key_dtype 0 = fp32, 1 = bf16 (raw uint16 bits).
 * planes: [H][D][4][nb_stride] uint64, scales: [H][D][nb_stride] fp16 bits. */
int orc_pack(const void* keys, int key_dtype, int64_t H, int64_t n, int D,
             int64_t stride_h, int64_t stride_tok,
             uint64_t* planes, uint16_t* scales, int64_t nb_stride)
{
    if (!keys || !planes || !scales || H < 0 || n < 0 || D <= 0) return ORC_EINVAL;
    int64_t nb = (n + 63) / 64;
    if (nb_stride < nb) return ORC_EINVAL;
    for (int64_t h = 0; h < H; ++h) {
        for (int j = 0; j < D; ++j) {
            for (int64_t b = 0; b < nb; ++b) {
                double kv[64];
                int cnt = 0;
                double m = 0.0;
                for (int i = 0; i < 64; ++i) {
                    int64_t tok = b * 64 + i;
                    if (tok >= n) break;
                    int64_t off = h * stride_h + tok * stride_tok + j;
                    double v = key_dtype == 1 ? orc_bf16_value(((const uint16_t*)keys)[off])
                                              : (double)((const float*)keys)[off];
                    kv[i] = v;
                    if (fabs(v) > m) m = fabs(v);
                    cnt++;
                }
                uint16_t sb = orc_fp16_bits(m);
                double s = orc_fp16_value(sb);
                uint64_t w[4] = {0, 0, 0, 0};
                for (int i = 0; i < cnt; ++i) {
                    int c = orc_code4(kv[i], s);
                    for (int p = 0; p < 4; ++p)
                        if ((c >> (3 - p)) & 1) w[p] |= (uint64_t)1 << i;
                }
                for (int p = 0; p < 4; ++p)
                    planes[(((h * D) + j) * 4 + p) * nb_stride + b] = w[p];
                scales[((h * D) + j) * nb_stride + b] = sb;
            }
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Reverse water-filling plan (water-filling section).                 */
/* w_j = sigma2_j * sum_g q_{g,j}^2 (single precision, fixed order).    */
/* Reading t planes leaves error variance proportional to 4^-t, so the  */
/* (t+1)-th plane of channel j is worth w_j * 4^-t.  Depth t_j counts   */
/* the items w_j*4^-t (t = 0..3) above the water level theta; theta* is */
/* the smallest theta >= 0 with sum_j t_j(theta) <= B, i.e. the         */
/* (B+1)-th largest item (0 when fewer than B+1 items are positive).    */
/* ------------------------------------------------------------------ */
static int cmp_desc_double(const void* a, const void* b)
{
    double x = *(const double*)a, y = *(const double*)b;
    return (x < y) - (x > y);
}

/* fp32 importance, exactly as the plan defines it. */
float orc_importance(const float* sigma2_j, const float* q_col, int G, int64_t q_stride)
{
    float acc = q_col[0] * q_col[0];
    for (int g = 1; g < G; ++g) {
        float sq = q_col[g * q_stride] * q_col[g * q_stride];
        acc = acc + sq;
    }
    return sigma2_j[0] * acc;
}

int orc_plan(const float* sigma2, const float* q, int64_t H, int G, int D,
             const int32_t* budget, uint8_t* depth, uint16_t* active,
             int32_t* n_active, double* theta, float* w_out)
{
    if (!sigma2 || !q || !budget || !depth || H < 0 || G <= 0 || D <= 0) return ORC_EINVAL;
    double* items = (double*)malloc(sizeof(double) * 4 * (size_t)D);
    float* w = (float*)malloc(sizeof(float) * (size_t)D);
    if (!items || !w) { free(items); free(w); return ORC_ENOMEM; }
    for (int64_t h = 0; h < H; ++h) {
        int B = budget[h];
        if (B < 0) B = 0;
        if (B > 4 * D) B = 4 * D;
        int npos = 0;
        for (int j = 0; j < D; ++j) {
            w[j] = orc_importance(&sigma2[h * D + j], &q[(h * G) * D + j], G, D);
            if (w_out) w_out[h * D + j] = w[j];
            if (w[j] > 0.0f)
                for (int t = 0; t < 4; ++t) items[npos++] = ldexp((double)w[j], -2 * t);
        }
        qsort(items, (size_t)npos, sizeof(double), cmp_desc_double);
        double th = (npos > B) ? items[B] : 0.0;
        int na = 0;
        for (int j = 0; j < D; ++j) {
            int t = 0;
            if (w[j] > 0.0f)
                for (int u = 0; u < 4; ++u)
                    if (ldexp((double)w[j], -2 * u) > th) t++;
            depth[h * D + j] = (uint8_t)t;
            if (t > 0 && active) active[h * D + na] = (uint16_t)(j | (t << 8));
            if (t > 0) na++;
        }
        if (active)
            for (int j = na; j < D; ++j) active[h * D + j] = 0;
        if (n_active) n_active[h] = na;
        if (theta) theta[h] = th;
    }
    free(items);
    free(w);
    return ORC_OK;
}

/* Fixed-depth comparator plan: the r channels with the largest         */
/* sum_g |q_{g,j}| (single precision, fixed order; ties to the lower j) */
/* are read at `bits` planes -- with r = 32 and 4 planes, the 32-channel */
/* 4-bit scan the byte-accounting section puts at 136 bits per token.   */
typedef struct { float a; int j; } orc_rank_t;

static int cmp_rank(const void* x, const void* y)
{
    const orc_rank_t* u = (const orc_rank_t*)x;
    const orc_rank_t* v = (const orc_rank_t*)y;
    if (u->a > v->a) return -1;
    if (u->a < v->a) return 1;
    return (u->j > v->j) - (u->j < v->j);
}

int orc_plan_fixed(const float* q, int64_t H, int G, int D, int r, int bits,
                   uint8_t* depth, uint16_t* active, int32_t* n_active)
{
    if (!q || !depth || H < 0 || G <= 0 || D <= 0 || r < 0 || r > D || bits < 1 || bits > 4) return ORC_EINVAL;
    orc_rank_t* rk = (orc_rank_t*)malloc(sizeof(orc_rank_t) * (size_t)D);
    if (!rk) return ORC_ENOMEM;
    for (int64_t h = 0; h < H; ++h) {
        for (int j = 0; j < D; ++j) {
            float acc = fabsf(q[(h * G) * D + j]);
            for (int g = 1; g < G; ++g) acc = acc + fabsf(q[(h * G + g) * D + j]);
            rk[j].a = acc;
            rk[j].j = j;
        }
        qsort(rk, (size_t)D, sizeof(orc_rank_t), cmp_rank);
        for (int j = 0; j < D; ++j) depth[h * D + j] = 0;
        for (int i = 0; i < r; ++i) depth[h * D + rk[i].j] = (uint8_t)bits;
        int na = 0;
        for (int j = 0; j < D; ++j)
            if (depth[h * D + j] && active) active[h * D + na++] = (uint16_t)(j | (bits << 8));
            else if (depth[h * D + j]) na++;
        if (active)
            for (int j = na; j < D; ++j) active[h * D + j] = 0;
        if (n_active) n_active[h] = na;
    }
    free(rk);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Variable-depth scores.  For token i < n and query head g of group h: */
/*   s_{g,i} = sum_{j : t_j > 0} q_{g,j} * khat^{t_j}_{i,j}             */
/* with khat the t-plane prefix dequantisation of the stored code.      */
/* l1 (optional) receives sum_j |q_{g,j} * khat|, the scale of rounding. */
/* ------------------------------------------------------------------ */
int orc_scan(const uint64_t* planes, const uint16_t* scales, int64_t H, int D, int64_t n,
             int64_t nb_stride, const uint8_t* depth, const float* q, int G,
             double* scores, double* l1)
{
    if (!planes || !scales || !depth || !q || !scores || H < 0 || D <= 0 || n < 0 || G <= 0)
        return ORC_EINVAL;
    for (int64_t h = 0; h < H; ++h) {
        for (int64_t i = 0; i < n; ++i) {
            int64_t b = i / 64;
            int bit = (int)(i % 64);
            double acc[64], sum_abs[64];
            for (int g = 0; g < G; ++g) { acc[g] = 0.0; sum_abs[g] = 0.0; }
            for (int j = 0; j < D; ++j) {
                int t = depth[h * D + j];
                if (t == 0) continue;
                int c4 = 0; /* the planes not read stay zero; only the top t bits matter */
                for (int p = 0; p < t; ++p) {
                    uint64_t w = planes[(((h * D) + j) * 4 + p) * nb_stride + b];
                    if ((w >> bit) & 1) c4 |= 1 << (3 - p);
                }
                double s = orc_fp16_value(scales[(h * D + j) * nb_stride + b]);
                double kh = orc_dequant(c4, t, s);
                for (int g = 0; g < G; ++g) {
                    double term = (double)q[(h * G + g) * D + j] * kh;
                    acc[g] += term;
                    sum_abs[g] += fabs(term);
                }
            }
            for (int g = 0; g < G; ++g) {
                scores[(h * G + g) * n + i] = acc[g];
                if (l1) l1[(h * G + g) * n + i] = sum_abs[g];
            }
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Top-k per query head by a full sort on (score descending, index     */
/* ascending), then the sorted, de-duplicated union of the G winner     */
/* lists of each KV head.                                               */
/* ------------------------------------------------------------------ */
typedef struct { double s; int32_t i; } orc_cand_t;

static int cmp_cand(const void* x, const void* y)
{
    const orc_cand_t* u = (const orc_cand_t*)x;
    const orc_cand_t* v = (const orc_cand_t*)y;
    if (u->s > v->s) return -1;
    if (u->s < v->s) return 1;
    return (u->i > v->i) - (u->i < v->i);
}

static int cmp_i32(const void* x, const void* y)
{
    int32_t a = *(const int32_t*)x, b = *(const int32_t*)y;
    return (a > b) - (a < b);
}

int orc_topk(const double* scores, int64_t H, int G, int64_t n, int k,
             int32_t* idx, int32_t* union_idx, int32_t* union_count)
{
    if (!scores || !idx || H < 0 || G <= 0 || n <= 0 || k <= 0 || k > n) return ORC_EINVAL;
    orc_cand_t* c = (orc_cand_t*)malloc(sizeof(orc_cand_t) * (size_t)n);
    int32_t* u = (int32_t*)malloc(sizeof(int32_t) * (size_t)G * (size_t)k);
    if (!c || !u) { free(c); free(u); return ORC_ENOMEM; }
    for (int64_t h = 0; h < H; ++h) {
        for (int g = 0; g < G; ++g) {
            const double* s = scores + (h * G + g) * n;
            for (int64_t i = 0; i < n; ++i) { c[i].s = s[i]; c[i].i = (int32_t)i; }
            qsort(c, (size_t)n, sizeof(orc_cand_t), cmp_cand);
            for (int r = 0; r < k; ++r) {
                idx[(h * G + g) * k + r] = c[r].i;
                u[g * k + r] = c[r].i;
            }
        }
        if (union_idx) {
            qsort(u, (size_t)G * (size_t)k, sizeof(int32_t), cmp_i32);
            int cnt = 0;
            for (int r = 0; r < G * k; ++r)
                if (r == 0 || u[r] != u[r - 1]) union_idx[h * G * k + cnt++] = u[r];
            for (int r = cnt; r < G * k; ++r) union_idx[h * G * k + r] = -1;
            if (union_count) union_count[h] = cnt;
        }
    }
    free(c);
    free(u);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Key rows rebuilt from the stored planes: for list entry r of group h */
/* (token i = rows[h*M + r]) and channel j, the `bits`-plane prefix     */
/* value of the stored code.  Entries outside [0, n), and entries past  */
/* row_count[h] (a negative count reads as 0), give 0.                  */
/* ------------------------------------------------------------------ */
int orc_dequant_rows(const uint64_t* planes, const uint16_t* scales, int64_t H, int D, int64_t n,
                     int64_t nb_stride, const int32_t* rows, int64_t M, const int32_t* row_count,
                     int bits, double* out)
{
    if (!planes || !scales || !rows || !out || H < 0 || D <= 0 || M < 0 || bits < 1 || bits > 4)
        return ORC_EINVAL;
    for (int64_t h = 0; h < H; ++h) {
        int64_t count = M;
        if (row_count) count = row_count[h] < 0 ? 0 : (row_count[h] > M ? M : row_count[h]);
        for (int64_t r = 0; r < M; ++r) {
            int64_t i = rows[h * M + r];
            for (int j = 0; j < D; ++j) {
                double v = 0.0;
                if (r < count && i >= 0 && i < n) {
                    int64_t b = i / 64;
                    int c4 = 0;
                    for (int p = 0; p < 4; ++p)
                        if ((planes[(((h * D) + j) * 4 + p) * nb_stride + b] >> (i % 64)) & 1) c4 |= 1 << (3 - p);
                    v = orc_dequant(c4, bits, orc_fp16_value(scales[(h * D + j) * nb_stride + b]));
                }
                out[(h * M + r) * D + j] = v;
            }
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Key statistics of each group over its first n keys (experiments     */
/* section: sigma^2 "measured once on calibration keys"; the session's */
/* own prefill keys may serve, one covariance per KV head).  Two passes */
/* in double: mean_j = (1/n) sum_i k_ij, then the centred population    */
/* moments cov_ab = (1/n) sum_i (k_ia - mean_a)(k_ib - mean_b), whose   */
/* diagonal is var_j.  mean and cov may be NULL; n = 0 gives zeros.     */
/* ------------------------------------------------------------------ */
int orc_calibrate(const void* keys, int key_dtype, int64_t H, int64_t n, int D,
                  int64_t stride_h, int64_t stride_tok, double* mean, double* var, double* cov)
{
    if (!keys || !var || H < 0 || n < 0 || D <= 0) return ORC_EINVAL;
    double* mu = (double*)calloc((size_t)D, sizeof(double));
    double* row = (double*)calloc((size_t)D, sizeof(double));
    if (!mu || !row) { free(mu); free(row); return ORC_ENOMEM; }
    for (int64_t h = 0; h < H; ++h) {
        for (int j = 0; j < D; ++j) mu[j] = 0.0;
        for (int64_t i = 0; i < n; ++i)
            for (int j = 0; j < D; ++j) {
                int64_t off = h * stride_h + i * stride_tok + j;
                mu[j] += key_dtype == 1 ? orc_bf16_value(((const uint16_t*)keys)[off]) : (double)((const float*)keys)[off];
            }
        for (int j = 0; j < D; ++j) mu[j] = n > 0 ? mu[j] / (double)n : 0.0;
        double* c = cov ? cov + h * (int64_t)D * D : NULL;
        if (c) for (int64_t e = 0; e < (int64_t)D * D; ++e) c[e] = 0.0;
        for (int j = 0; j < D; ++j) var[h * D + j] = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            for (int j = 0; j < D; ++j) {
                int64_t off = h * stride_h + i * stride_tok + j;
                double v = key_dtype == 1 ? orc_bf16_value(((const uint16_t*)keys)[off]) : (double)((const float*)keys)[off];
                row[j] = v - mu[j];
                var[h * D + j] += row[j] * row[j];
            }
            if (c)
                for (int a = 0; a < D; ++a)
                    for (int b = 0; b < D; ++b) c[(int64_t)a * D + b] += row[a] * row[b];
        }
        for (int j = 0; j < D; ++j) {
            var[h * D + j] = n > 0 ? var[h * D + j] / (double)n : 0.0;
            if (mean) mean[h * D + j] = mu[j];
        }
        if (c && n > 0)
            for (int64_t e = 0; e < (int64_t)D * D; ++e) c[e] /= (double)n;
    }
    free(mu);
    free(row);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Attention over the union of winners (byte-accounting section: each    */
/* step fetches the KV rows of the union of the G heads' top-k, at most  */
/* G*k rows per KV head).  For group h, head g and the rows i in         */
/* union[h][0 .. count_h):                                               */
/*   s_i = scale * q_g . K_i,  p_i = exp(s_i - max s) / sum exp(s - max), */
/*   out_g = sum_i p_i V_i.                                              */
/* A count <= 0 (no rows, or an error status) gives a zero output.       */
/* K and V: [H][n][D] with the given strides, fp32 or bf16 bits.         */
/* ------------------------------------------------------------------ */
int orc_union_attention(const void* kc, const void* vc, int kv_dtype, int64_t H, int64_t n, int D,
                        int64_t stride_h, int64_t stride_tok, const float* q, int G, const int32_t* uni,
                        const int32_t* count, int64_t M, double scale, double* out)
{
    if (!kc || !vc || !q || !uni || !count || !out || H < 0 || n < 0 || D <= 0 || G <= 0 || M < 0) return ORC_EINVAL;
    double* sc = (double*)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1));
    if (!sc) return ORC_ENOMEM;
    for (int64_t h = 0; h < H; ++h) {
        int64_t c = count[h] < 0 ? 0 : (count[h] > M ? M : count[h]);
        for (int g = 0; g < G; ++g) {
            const float* qg = q + (h * G + g) * (int64_t)D;
            double* o = out + (h * G + g) * (int64_t)D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (c == 0) continue;
            double mx = -INFINITY;
            for (int64_t r = 0; r < c; ++r) {
                int64_t i = uni[h * M + r];
                if (i < 0 || i >= n) { free(sc); return ORC_EINVAL; }
                double dot = 0.0;
                for (int d = 0; d < D; ++d) {
                    int64_t off = h * stride_h + i * stride_tok + d;
                    double kv = kv_dtype == 1 ? orc_bf16_value(((const uint16_t*)kc)[off]) : (double)((const float*)kc)[off];
                    dot += (double)qg[d] * kv;
                }
                sc[r] = scale * dot;
                if (sc[r] > mx) mx = sc[r];
            }
            double den = 0.0;
            for (int64_t r = 0; r < c; ++r) {
                sc[r] = exp(sc[r] - mx);
                den += sc[r];
            }
            for (int64_t r = 0; r < c; ++r) {
                int64_t i = uni[h * M + r];
                for (int d = 0; d < D; ++d) {
                    int64_t off = h * stride_h + i * stride_tok + d;
                    double vv = kv_dtype == 1 ? orc_bf16_value(((const uint16_t*)vc)[off]) : (double)((const float*)vc)[off];
                    o[d] += sc[r] / den * vv;
                }
            }
        }
    }
    free(sc);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Nibble store of the same codes (byte-accounting section: a fixed-depth */
/* scan reads each chosen coordinate's whole 4-bit code).  Word w of     */
/* block b of channel j holds tokens 64b + 16w .. 64b + 16w + 15, token  */
/* 64b + 16w + e in bits 4e .. 4e + 3.  Layout [H][D][4][nb_stride] like  */
/* the planes: row (h, j, w) is contiguous along the blocks.  Padding    */
/* tokens (past n) hold code 0.  Scales are those of orc_pack.           */
/* ------------------------------------------------------------------ */
int orc_pack_nibbles(const void* keys, int key_dtype, int64_t H, int64_t n, int D,
                     int64_t stride_h, int64_t stride_tok, uint64_t* nib, int64_t nb_stride)
{
    if (!keys || !nib || H < 0 || n < 0 || D <= 0) return ORC_EINVAL;
    int64_t nb = (n + 63) / 64;
    if (nb_stride < nb) return ORC_EINVAL;
    for (int64_t h = 0; h < H; ++h) {
        for (int j = 0; j < D; ++j) {
            for (int64_t b = 0; b < nb; ++b) {
                double kv[64];
                int cnt = 0;
                double m = 0.0;
                for (int i = 0; i < 64; ++i) {
                    int64_t tok = b * 64 + i;
                    if (tok >= n) break;
                    int64_t off = h * stride_h + tok * stride_tok + j;
                    double v = key_dtype == 1 ? orc_bf16_value(((const uint16_t*)keys)[off])
                                              : (double)((const float*)keys)[off];
                    kv[i] = v;
                    if (fabs(v) > m) m = fabs(v);
                    cnt++;
                }
                double s = orc_fp16_value(orc_fp16_bits(m));
                uint64_t w[4] = {0, 0, 0, 0};
                for (int i = 0; i < cnt; ++i)
                    w[i / 16] |= (uint64_t)orc_code4(kv[i], s) << (4 * (i % 16));
                for (int p = 0; p < 4; ++p) nib[(((h * D) + j) * 4 + p) * nb_stride + b] = w[p];
            }
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Per-layer budgets (water-filling section: layers differ in how sharp  */
/* their scores are, so a greedy pass on calibration data may give each  */
/* layer its own budget; the default is the flat budget).                */
/* The groups of layer l are h = l*P .. l*P + P - 1 (P = H / layers),    */
/* and all get the layer's budget B_l.  A group's expected squared score */
/* error under its plan is E_h(B) = sum_j w_j 4^-t_j, and reading the    */
/* b-th largest item v (an item w_j 4^-t) lowers it by 3v/4.  The cost   */
/* of layer l is its groups' error relative to their unread error,      */
/*   C_l(B) = sum_h E_h(B) / N_l,   N_l = sum_h sum_j w_hj,              */
/* so one more bit for every group of the layer gains                    */
/*   g_l(b) = 0.75 * (sum_h v_h,(b)) / N_l,   b = B_l + 1,               */
/* which does not grow with b.  The greedy gives the total budget one    */
/* bit per step to the layer with the largest next gain (ties to the     */
/* lower layer), at most 4D bits per layer.  Sums run in double, in the  */
/* order written (h ascending, then j ascending).                        */
/* ------------------------------------------------------------------ */
int orc_layer_budgets(const float* sigma2, const float* q, int64_t H, int G, int D, int layers,
                      int64_t total_bits, int32_t* budget_out)
{
    if (!sigma2 || !q || !budget_out || H <= 0 || G <= 0 || D <= 0 || layers <= 0 || H % layers) return ORC_EINVAL;
    int64_t P = H / layers, NI = 4 * (int64_t)D;
    double* items = (double*)calloc((size_t)(H * NI), sizeof(double));
    double* N = (double*)calloc((size_t)layers, sizeof(double));
    int64_t* ptr = (int64_t*)calloc((size_t)layers, sizeof(int64_t));
    if (!items || !N || !ptr) { free(items); free(N); free(ptr); return ORC_ENOMEM; }
    for (int64_t h = 0; h < H; ++h) {
        double* it = items + h * NI;
        int npos = 0;
        for (int j = 0; j < D; ++j) {
            float w = orc_importance(&sigma2[h * D + j], &q[(h * G) * D + j], G, D);
            if (w > 0.0f) {
                N[h / P] += (double)w;
                for (int t = 0; t < 4; ++t) it[npos++] = ldexp((double)w, -2 * t);
            }
        }
        qsort(it, (size_t)npos, sizeof(double), cmp_desc_double);   /* the rest stays 0 */
    }
    int64_t T = total_bits < 0 ? 0 : total_bits;
    if (T > layers * NI) T = layers * NI;
    for (int64_t step = 0; step < T; ++step) {
        int best = -1;
        double bg = 0.0;
        for (int l = 0; l < layers; ++l) {
            if (ptr[l] >= NI) continue;
            double S = 0.0;
            for (int64_t h = l * P; h < (l + 1) * P; ++h) S += items[h * NI + ptr[l]];
            double g = N[l] > 0.0 ? 0.75 * S / N[l] : 0.0;
            if (best < 0 || g > bg) { best = l; bg = g; }
        }
        ptr[best]++;
    }
    for (int64_t h = 0; h < H; ++h) budget_out[h] = (int32_t)ptr[h / P];
    free(items);
    free(N);
    free(ptr);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Keys in a rotated basis (base-choice section: for a model without    */
/* QK-norm the planes hold the keys' coordinates in an orthonormal      */
/* basis of directions u_i, the columns of U, and the queries are       */
/* rotated to match, so q'.y = q.k).  Coordinate i of key k is           */
/* y_i = sum_d k_d U[d][i].  So that the codes packed from y are        */
/* defined bit for bit, the sum has one stated single-precision order:  */
/* y_i starts at +0 and takes k_d * U[d][i] for d = 0, 1, ..., D-1,     */
/* each step one IEEE fused multiply-add (C99 fmaf: the exact           */
/* k_d * U[d][i] + y_i, rounded once to nearest-even binary32).  bf16   */
/* keys are widened to binary32 exactly.  U is [H][D][D] fp32,          */
/* U[h][d][i]; out is [H][n][D] fp32, contiguous.                        */
/* ------------------------------------------------------------------ */
int orc_rotate_keys(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t stride_h,
                    int64_t stride_tok, const float* U, float* out)
{
    if (!keys || !U || !out || H < 0 || n < 0 || D <= 0) return ORC_EINVAL;
    float* x = (float*)malloc(sizeof(float) * (size_t)D);
    if (!x) return ORC_ENOMEM;
    for (int64_t h = 0; h < H; ++h) {
        const float* Uh = U + h * (int64_t)D * D;
        for (int64_t tok = 0; tok < n; ++tok) {
            for (int d = 0; d < D; ++d) {
                int64_t off = h * stride_h + tok * stride_tok + d;
                x[d] = key_dtype == 1 ? (float)orc_bf16_value(((const uint16_t*)keys)[off])
                                      : ((const float*)keys)[off];
            }
            for (int i = 0; i < D; ++i) {
                float y = 0.0f;
                for (int d = 0; d < D; ++d) y = fmaf(x[d], Uh[(int64_t)d * D + i], y);
                out[(h * n + tok) * D + i] = y;
            }
        }
    }
    free(x);
    return ORC_OK;
}
