/*
 * CPU oracle for the lightning-indexer decode path and its selection
 * evaluation.  TEST INFRASTRUCTURE ONLY: the product never links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant with the
 * CUDA library.
 *
 * Every routine is the plain definition written out, in double precision,
 * with no blocking, fusion or reordering beyond what the definition states:
 *
 *  - orc_index_score  head-weighted ReLU index score
 *        s[b,t,j] = sum_h w[b,t,h] * max(q[b,t,h,:] . k[b,j,:], 0)
 *        (lightning indexer: DeepSeek-V4-Flash architecture post, section
 *        (B); "native ReLU-MQA" and the head-fused gate form in the
 *        FlashMemory-DeepSeek-V4 write-up, reply #2; the pages name the rule
 *        but print no formula, and this is its plainest reading)
 *  - orc_topk          the k largest scores, ties to the lower index
 *        (n_indexer_top_k = 512 / 1024: architecture post, section (B))
 *  - orc_attn          softmax attention of one decode query over the
 *        selected compressed rows plus the sliding-window rows, K = V = the
 *        full 512-wide row (architecture post, sections (A) and (B))
 *  - orc_golden        head-mean of per-head dense softmax over all entries
 *        (FlashMemory vs native indexer post, Act 3: unmasked dense attention
 *        as ground truth; write-up section 3.2 step 1)
 *  - orc_golden_index  the other reading of the golden probabilities: the
 *        softmax over all entries of the indexer's own logits (write-up
 *        section 3.2 step 1 softmaxes the indexer logits)
 *  - orc_topp          the minimal prefix of entries (descending probability)
 *        whose mass reaches the fraction p of the total (write-up 3.2 step 2)
 *  - orc_vote          entries chosen by at least m of the layers (write-up
 *        3.2 step 3); orc_union: union over the queries of a tau window
 *  - orc_lsa_gate      sigmoid(logit) >= 0.5 <=> logit >= 0, OR over the
 *        gate layers (write-up sections 2.2 and 4.1)
 *  - orc_overlap       |A & B|, |A|, |B| (FlashMemory vs native post, Act 1/3)
 *  - orc_encode_rows   the cache write side: rows stored as E4M3 + per-64
 *        power-of-two scales + bf16 RoPE dims, or bf16 / fp32 (architecture
 *        post, "why quantising the KV does not save memory")
 *
 * Storage decoding (architecture post, "why you cannot quantise the KV"):
 * non-RoPE dims are OCP E4M3FN bytes, one E8M0 power-of-two scale per 64
 * consecutive elements, RoPE dims bf16.  A row of width D holds D-64 FP8 dims
 * followed by 64 bf16 RoPE dims.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENAN 2
#define ORC_ERANGE 3
#define ORC_ENOMEM 4

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2

/* One set of stored rows.  Row r of plane P starts at P + r * ld_P. */
typedef struct {
    int32_t dtype;
    int32_t dim;
    const void *data;     /* F32: float, BF16: uint16 bits, E4M3: uint8 codes */
    const uint8_t *scale; /* E4M3: E8M0 codes, (dim-64)/64 per row */
    const uint16_t *rope; /* E4M3: bf16 bits, 64 per row */
    int64_t ld, ld_scale, ld_rope;
} orc_rows;

/* ---------------------------------------------------------------- decoding */

/* bf16: sign, 8 exponent bits (bias 127), 7 mantissa bits. */
static double bf16_value(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xFF;
    int m = b & 0x7F;
    double v;
    if (e == 0xFF)
        v = m ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)m, -126 - 7);
    else
        v = ldexp(1.0 + m / 128.0, e - 127);
    return sign ? -v : v;
}

/* OCP E4M3FN: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
 * subnormal (m * 2^-9); S.1111.111 is NaN; no infinities. */
static double e4m3_value(uint8_t b)
{
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* E8M0: unsigned power of two 2^(c-127); 0xFF is NaN. */
static double e8m0_value(uint8_t c)
{
    return c == 0xFF ? NAN : ldexp(1.0, (int)c - 127);
}

static void decode_row(const orc_rows *r, int64_t row, double *out)
{
    int D = r->dim;
    if (r->dtype == ORC_F32) {
        const float *p = (const float *)r->data + row * r->ld;
        for (int d = 0; d < D; d++) out[d] = (double)p[d];
    } else if (r->dtype == ORC_BF16) {
        const uint16_t *p = (const uint16_t *)r->data + row * r->ld;
        for (int d = 0; d < D; d++) out[d] = bf16_value(p[d]);
    } else {
        const uint8_t *p = (const uint8_t *)r->data + row * r->ld;
        const uint8_t *sc = r->scale + row * r->ld_scale;
        const uint16_t *rp = r->rope + row * r->ld_rope;
        int nope = D - 64;
        for (int d = 0; d < nope; d++) out[d] = e4m3_value(p[d]) * e8m0_value(sc[d / 64]);
        for (int d = 0; d < 64; d++) out[nope + d] = bf16_value(rp[d]);
    }
}

/* exported so the tests can pin the decoders against published code points */
double orc_decode_bf16(uint16_t b) { return bf16_value(b); }
double orc_decode_e4m3(uint8_t b) { return e4m3_value(b); }
double orc_decode_e8m0(uint8_t b) { return e8m0_value(b); }

int orc_decode_rows(const orc_rows *r, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; i++) decode_row(r, i, out + i * r->dim);
    return ORC_OK;
}

/* ---------------------------------------------------------------- encoding
 *
 * The cache write side (architecture post, "why quantising the KV does not
 * save memory", point 1): the non-RoPE dims of a row are stored as OCP
 * E4M3FN codes with one power-of-two (E8M0) scale per 64 elements, the 64
 * RoPE dims as bf16.  The page fixes the format, not how the scale is chosen;
 * the reading taken here is the finest scale that still fits the block: the
 * smallest integer e with amax <= 448 * 2^e (448 is the largest E4M3FN
 * value), clamped to [-127, 127], stored as the byte e + 127; a block whose
 * finite values are all zero takes e = 0.  Values are divided by 2^e and
 * rounded to the nearest E4M3 value, ties to the even code; magnitudes
 * above 448 saturate to 448 (infinities included); NaN is stored as the
 * code 0x7F.  RoPE dims and bf16 rows round to nearest even from the fp32
 * input.
 */

/* nearest E4M3FN code of v (ties to even); |v| > 448 saturates */
static uint8_t e4m3_encode(double v)
{
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;
    int ex;
    (void)frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1): floor(log2 a) = ex - 1 */
    int e = ex - 1;
    double q; /* the value on the integer grid of its binade */
    int E;
    if (a == 0.0 || e < -6) { /* subnormal: m * 2^-9, m = 0..7 (8 rounds up to the smallest normal) */
        q = ldexp(a, 9);
        E = 0;
    } else {                  /* normal: 2^e * (1 + m/8): q = 8 + m in [8, 16) */
        q = ldexp(a, 3 - e);
        E = e + 7;
    }
    double fl = floor(q);
    double rem = q - fl;
    long n = (long)fl;
    if (rem > 0.5 || (rem == 0.5 && (n & 1))) n++;
    int code;
    if (E == 0) {
        code = (int)n;                  /* n = 8 is exponent field 1, mantissa 0 */
    } else {
        if (n == 16) { n = 8; E++; }    /* carry into the next binade */
        code = (E << 3) | (int)(n - 8);
    }
    if (code > 0x7E) code = 0x7E;       /* 0x7F is NaN: the rounding saturates */
    return (uint8_t)(sign | code);
}

/* nearest bf16 of a float (ties to even); NaN stays a quiet NaN */
static uint16_t bf16_encode(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lower = u & 0xFFFFu, upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper++;
    return (uint16_t)upper;
}

/* E8M0 code of the block scale for largest finite magnitude amax */
static uint8_t e8m0_for(double amax)
{
    if (amax == 0.0) return 127;
    int e = -127;
    while (e < 127 && amax > ldexp(448.0, e)) e++;
    return (uint8_t)(e + 127);
}

uint8_t orc_encode_e4m3(double v) { return e4m3_encode(v); }
uint16_t orc_encode_bf16(float x) { return bf16_encode(x); }
uint8_t orc_e8m0_for(double amax) { return e8m0_for(amax); }

/*
 * Encode `rows` rows of `dim` fp32 values x[rows][dim] in format `dtype`
 * into packed planes:
 *   F32:  f32[rows][dim] (copied)
 *   BF16: bits[rows][dim]
 *   E4M3: codes[rows][dim-64], scales[rows][(dim-64)/64], bits[rows][64] (RoPE)
 * Returns ORC_ENAN (after encoding every row) when an input was not finite.
 */
int orc_encode_rows(const float *x, int64_t rows, int dim, int dtype, float *f32, uint16_t *bits,
                    uint8_t *codes, uint8_t *scales)
{
    if (rows < 0 || dim < 64 || dim % 64) return ORC_EINVAL;
    int nonfinite = 0;
    for (int64_t r = 0; r < rows; r++) {
        const float *xr = x + r * dim;
        for (int d = 0; d < dim; d++) nonfinite |= !isfinite(xr[d]);
        if (dtype == ORC_F32) {
            memcpy(f32 + r * dim, xr, sizeof(float) * (size_t)dim);
        } else if (dtype == ORC_BF16) {
            for (int d = 0; d < dim; d++) bits[r * dim + d] = bf16_encode(xr[d]);
        } else if (dtype == ORC_E4M3) {
            int nope = dim - 64, nb = nope / 64;
            for (int blk = 0; blk < nb; blk++) {
                double amax = 0.0;
                for (int d = 64 * blk; d < 64 * blk + 64; d++) {
                    double a = fabs((double)xr[d]);
                    if (isfinite(a) && a > amax) amax = a;
                }
                uint8_t sc = e8m0_for(amax);
                scales[r * nb + blk] = sc;
                for (int d = 64 * blk; d < 64 * blk + 64; d++)
                    codes[r * nope + d] = e4m3_encode(ldexp((double)xr[d], 127 - (int)sc));
            }
            for (int d = 0; d < 64; d++) bits[r * 64 + d] = bf16_encode(xr[nope + d]);
        } else {
            return ORC_EINVAL;
        }
    }
    return nonfinite ? ORC_ENAN : ORC_OK;
}

/* ------------------------------------------------------------- index score */

/*
 * q: rows B*Q*H of width D (query (b,t,h) is row (b*Q+t)*H+h)
 * w: float [B][Q][H]
 * keys: rows B*key_batch_rows, entry (b,j) is row b*key_batch_rows + j
 * scores: float [B][Q][N] (row stride ld_s)
 * cond (optional): double [B][Q][N], sum_h |w_h| * sum_d |q_hd k_jd| -- the
 *   magnitude a rounding-error bound of the score scales with.
 * cond_dot (optional): double [B][Q][N], sum_h |w_h| * |q_h . k_j| -- the
 *   absolute floor of the score tolerance (the scores must agree to 1e-5
 *   relative; this term only keeps that bar finite where the head terms
 *   cancel to near zero).
 */
int orc_index_score(int B, int Q, int H, int N, const orc_rows *q, const float *w,
                    const orc_rows *keys, int64_t key_batch_rows, float *scores,
                    int64_t ld_s, double *cond, double *cond_dot)
{
    int D = keys->dim;
    if (q->dim != D || B < 0 || Q < 0 || H < 1 || N < 0) return ORC_EINVAL;
    double *qv = (double *)malloc(sizeof(double) * (size_t)H * D);
    double *kv = (double *)malloc(sizeof(double) * (size_t)D);
    if (!qv || !kv) { free(qv); free(kv); return ORC_ENOMEM; }
    for (int b = 0; b < B; b++)
        for (int t = 0; t < Q; t++) {
            for (int h = 0; h < H; h++) decode_row(q, ((int64_t)b * Q + t) * H + h, qv + (size_t)h * D);
            const float *wt = w + ((int64_t)b * Q + t) * H;
            for (int j = 0; j < N; j++) {
                decode_row(keys, (int64_t)b * key_batch_rows + j, kv);
                double s = 0.0, c = 0.0, cd = 0.0;
                for (int h = 0; h < H; h++) {
                    double dot = 0.0, mag = 0.0;
                    for (int d = 0; d < D; d++) {
                        dot += qv[(size_t)h * D + d] * kv[d];
                        mag += fabs(qv[(size_t)h * D + d] * kv[d]);
                    }
                    double relu = dot > 0.0 ? dot : 0.0;
                    s += (double)wt[h] * relu;
                    c += fabs((double)wt[h]) * mag;
                    cd += fabs((double)wt[h]) * fabs(dot);
                }
                scores[((int64_t)b * Q + t) * ld_s + j] = (float)s;
                if (cond) cond[((int64_t)b * Q + t) * N + j] = c;
                if (cond_dot) cond_dot[((int64_t)b * Q + t) * N + j] = cd;
            }
        }
    free(qv);
    free(kv);
    return ORC_OK;
}

/* ------------------------------------------------------------------- top-k */

typedef struct { float v; int32_t i; } orc_vi;

/* descending value, then ascending index */
static int cmp_desc_then_index(const void *a, const void *b)
{
    const orc_vi *x = (const orc_vi *)a, *y = (const orc_vi *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->i > y->i) - (x->i < y->i);
}

static int cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Select the k largest of s[0..N) among entries with allowed[j] != 0 (all
 * when allowed is NULL).  Equal values (including +0 and -0) are ordered by
 * index, lower first.  NaN entries are never selected; their count is
 * returned through *n_nan.  ids[0..k) receives the selected indices in
 * ascending order followed by -1 padding; *n_sel = min(k, #eligible).
 */
int orc_topk(int N, int k, const float *s, const uint8_t *allowed, int32_t *ids,
             int32_t *n_sel, int32_t *n_nan)
{
    if (N < 0 || k < 1) return ORC_EINVAL;
    orc_vi *v = (orc_vi *)malloc(sizeof(orc_vi) * (size_t)(N > 0 ? N : 1));
    if (!v) return ORC_ENOMEM;
    int n = 0, nan = 0;
    for (int j = 0; j < N; j++) {
        if (allowed && !allowed[j]) continue;
        if (isnan(s[j])) { nan++; continue; }
        v[n].v = s[j];
        v[n].i = j;
        n++;
    }
    qsort(v, (size_t)n, sizeof(orc_vi), cmp_desc_then_index);
    int m = n < k ? n : k;
    for (int i = 0; i < m; i++) ids[i] = v[i].i;
    qsort(ids, (size_t)m, sizeof(int32_t), cmp_i32);
    for (int i = m; i < k; i++) ids[i] = -1;
    *n_sel = m;
    if (n_nan) *n_nan = nan;
    free(v);
    return ORC_OK;
}

/* --------------------------------------------------------------- attention */

/*
 * One decode query (H heads) attending over the multiset
 *   R = { kv row ids[i] : 0 <= i < n_ids, ids[i] >= 0 }  U  { swa rows 0..swa_len-1 }
 * with logits scale * q_h . x_r, K = V = the full row:
 *   o_h = sum_r softmax_r(logit_hr) x_r,  lse_h = log sum_r exp(logit_hr).
 * An id >= N returns ORC_ERANGE.  Empty R gives o = 0 and lse = -inf.
 * q: rows H of width D; kv: rows [0, N); swa: rows [0, swa_len).
 */
int orc_attn(int H, const orc_rows *q, const orc_rows *kv, int N, const int32_t *ids,
             int n_ids, const orc_rows *swa, int swa_len, double scale, float *out, float *lse)
{
    int D = kv->dim;
    if (q->dim != D || (swa && swa_len > 0 && swa->dim != D)) return ORC_EINVAL;
    int nr = 0;
    for (int i = 0; i < n_ids; i++) {
        if (ids[i] < 0) continue;
        if (ids[i] >= N) return ORC_ERANGE;
        nr++;
    }
    int R = nr + (swa ? swa_len : 0);
    double *X = (double *)malloc(sizeof(double) * (size_t)(R > 0 ? R : 1) * D);
    double *qv = (double *)malloc(sizeof(double) * (size_t)D);
    double *lg = (double *)malloc(sizeof(double) * (size_t)(R > 0 ? R : 1));
    if (!X || !qv || !lg) { free(X); free(qv); free(lg); return ORC_ENOMEM; }
    int r = 0;
    for (int i = 0; i < n_ids; i++)
        if (ids[i] >= 0) decode_row(kv, ids[i], X + (size_t)(r++) * D);
    for (int i = 0; swa && i < swa_len; i++) decode_row(swa, i, X + (size_t)(r++) * D);
    for (int h = 0; h < H; h++) {
        decode_row(q, h, qv);
        float *o = out + (size_t)h * D;
        if (R == 0) {
            for (int d = 0; d < D; d++) o[d] = 0.0f;
            if (lse) lse[h] = -INFINITY;
            continue;
        }
        double mx = -INFINITY;
        for (int i = 0; i < R; i++) {
            double dot = 0.0;
            for (int d = 0; d < D; d++) dot += qv[d] * X[(size_t)i * D + d];
            lg[i] = scale * dot;
            if (lg[i] > mx) mx = lg[i];
        }
        double l = 0.0;
        for (int i = 0; i < R; i++) { lg[i] = exp(lg[i] - mx); l += lg[i]; }
        for (int d = 0; d < D; d++) {
            double acc = 0.0;
            for (int i = 0; i < R; i++) acc += lg[i] * X[(size_t)i * D + d];
            o[d] = (float)(acc / l);
        }
        if (lse) lse[h] = (float)(mx + log(l));
    }
    free(X);
    free(qv);
    free(lg);
    return ORC_OK;
}

/* ------------------------------------------------------- golden probability */

/*
 * One layer of the dense ground truth: for each query t,
 *   p[t,j] = (1/H) sum_h softmax_j(scale * qa[t,h] . x_j)   over all N entries.
 * qa: rows T*H of width D ((t,h) is row t*H+h); kv: rows [0, N).
 */
int orc_golden(int T, int H, int N, const orc_rows *qa, const orc_rows *kv, double scale,
               float *p)
{
    int D = kv->dim;
    if (qa->dim != D || N < 1) return ORC_EINVAL;
    double *X = (double *)malloc(sizeof(double) * (size_t)N * D);
    double *qv = (double *)malloc(sizeof(double) * (size_t)D);
    double *lg = (double *)malloc(sizeof(double) * (size_t)N);
    double *acc = (double *)malloc(sizeof(double) * (size_t)N);
    if (!X || !qv || !lg || !acc) { free(X); free(qv); free(lg); free(acc); return ORC_ENOMEM; }
    for (int j = 0; j < N; j++) decode_row(kv, j, X + (size_t)j * D);
    for (int t = 0; t < T; t++) {
        for (int j = 0; j < N; j++) acc[j] = 0.0;
        for (int h = 0; h < H; h++) {
            decode_row(qa, (int64_t)t * H + h, qv);
            double mx = -INFINITY;
            for (int j = 0; j < N; j++) {
                double dot = 0.0;
                for (int d = 0; d < D; d++) dot += qv[d] * X[(size_t)j * D + d];
                lg[j] = scale * dot;
                if (lg[j] > mx) mx = lg[j];
            }
            double l = 0.0;
            for (int j = 0; j < N; j++) { lg[j] = exp(lg[j] - mx); l += lg[j]; }
            for (int j = 0; j < N; j++) acc[j] += lg[j] / l;
        }
        for (int j = 0; j < N; j++) p[(size_t)t * N + j] = (float)(acc[j] / H);
    }
    free(X);
    free(qv);
    free(lg);
    free(acc);
    return ORC_OK;
}

/*
 * Softmax over the N entries of each of R rows of scores (row r at
 * s + r * ld): p_j = exp(s_j - m) / sum_i exp(s_i - m), m the row's largest
 * score.  NaN and -inf scores take no mass (p = 0); a row without any finite
 * score is all zeros.  Rounded to fp32 at the end.
 */
int orc_golden_index(int R, int N, const float *s, int64_t ld, float *p)
{
    if (R < 1 || N < 1 || ld < N) return ORC_EINVAL;
    for (int r = 0; r < R; r++) {
        const float *x = s + (size_t)r * ld;
        float *out = p + (size_t)r * N;
        double m = -INFINITY;
        for (int j = 0; j < N; j++)
            if (x[j] == x[j] && (double)x[j] > m) m = x[j];
        double l = 0.0;
        if (m > -INFINITY)
            for (int j = 0; j < N; j++)
                if (x[j] == x[j]) l += exp((double)x[j] - m);
        for (int j = 0; j < N; j++)
            out[j] = (m > -INFINITY && x[j] == x[j]) ? (float)(exp((double)x[j] - m) / l) : 0.0f;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------- top-p */

/*
 * Nucleus set of one probability row.  Masses are taken in fixed point,
 * m_j = floor(p_j * 2^shift) (exact for fp32 p_j in [0,1]), total M = sum m_j,
 * threshold T = ceil(M * num / den).  Entries are ranked by p descending,
 * ties to the lower index; the set is the shortest prefix of that ranking
 * whose mass reaches T (empty when T == 0).  Output: bitset [ceil(N/32)].
 * Negative or NaN p returns ORC_EINVAL; a total that does not fit 64 bits
 * returns ORC_ERANGE.
 */
int orc_topp(int N, const float *p, uint32_t num, uint32_t den, int shift, uint32_t *bits,
             int32_t *count)
{
    if (N < 1 || den == 0 || num > den || shift < 0 || shift > 62) return ORC_EINVAL;
    orc_vi *v = (orc_vi *)malloc(sizeof(orc_vi) * (size_t)N);
    if (!v) return ORC_ENOMEM;
    unsigned __int128 M = 0;
    for (int j = 0; j < N; j++) {
        if (!(p[j] >= 0.0f) || p[j] > 1.0f) { free(v); return ORC_EINVAL; }
        v[j].v = p[j];
        v[j].i = j;
        M += (uint64_t)floor(ldexp((double)p[j], shift));
    }
    if (M >> 64) { free(v); return ORC_ERANGE; }
    unsigned __int128 prod = M * num;
    uint64_t T = (uint64_t)(prod / den + (prod % den != 0));
    qsort(v, (size_t)N, sizeof(orc_vi), cmp_desc_then_index);
    int W = (N + 31) / 32;
    memset(bits, 0, sizeof(uint32_t) * (size_t)W);
    uint64_t cum = 0;
    int n = 0;
    for (int i = 0; i < N && cum < T; i++) {
        cum += (uint64_t)floor(ldexp((double)v[i].v, shift));
        bits[v[i].i / 32] |= 1u << (v[i].i % 32);
        n++;
    }
    if (count) *count = n;
    free(v);
    return ORC_OK;
}

/* -------------------------------------------------------------------- vote */

static int bit_at(const uint32_t *b, int j) { return (b[j / 32] >> (j % 32)) & 1u; }

/* out[j] = [ #{l < L : j in layer l's set} >= min_votes ];  sets [L][W]. */
int orc_vote(int L, int N, const uint32_t *sets, int min_votes, uint32_t *out)
{
    int W = (N + 31) / 32;
    memset(out, 0, sizeof(uint32_t) * (size_t)W);
    for (int j = 0; j < N; j++) {
        int c = 0;
        for (int l = 0; l < L; l++) c += bit_at(sets + (size_t)l * W, j);
        if (c >= min_votes) out[j / 32] |= 1u << (j % 32);
    }
    return ORC_OK;
}

/* out = union of the T sets [T][W]. */
int orc_union(int T, int N, const uint32_t *sets, uint32_t *out)
{
    int W = (N + 31) / 32;
    memset(out, 0, sizeof(uint32_t) * (size_t)W);
    for (int j = 0; j < N; j++)
        for (int t = 0; t < T; t++)
            if (bit_at(sets + (size_t)t * W, j)) { out[j / 32] |= 1u << (j % 32); break; }
    return ORC_OK;
}

/* ---------------------------------------------------------------- LSA gate */

/*
 * Fetched set: entry j is fetched when, for any gate layer g,
 * sigmoid(logit[g][j] + beta) >= 0.5, i.e. logit + beta >= 0 with the sum
 * rounded to fp32 (sigmoid(0) = 0.5 exactly, so no exp is needed).
 */
int orc_lsa_gate(int G, int N, const float *logits, float beta, uint32_t *out)
{
    int W = (N + 31) / 32;
    memset(out, 0, sizeof(uint32_t) * (size_t)W);
    for (int j = 0; j < N; j++)
        for (int g = 0; g < G; g++) {
            float z = logits[(size_t)g * N + j] + beta;
            if (z >= 0.0f) { out[j / 32] |= 1u << (j % 32); break; }
        }
    return ORC_OK;
}

/* ----------------------------------------------------------------- overlap */

/* counts = { |A & B|, |A|, |B| } over entries [0, N). */
int orc_overlap(int N, const uint32_t *a, const uint32_t *b, int64_t *counts)
{
    int64_t both = 0, na = 0, nb = 0;
    for (int j = 0; j < N; j++) {
        int x = bit_at(a, j), y = bit_at(b, j);
        both += x & y;
        na += x;
        nb += y;
    }
    counts[0] = both;
    counts[1] = na;
    counts[2] = nb;
    return ORC_OK;
}
