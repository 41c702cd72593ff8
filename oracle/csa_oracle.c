/*
 * csa_oracle.c -- plain, slow CPU oracle for the CSA2 FP4 compressed sparse-KV decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls this file; only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg do.  It shares no code, header,
 * table or constant generator with the CUDA library.
 *
 * Sources (the three pages on DeepSeek-V4.1-Flash's KV cache):
 *   [yomxxx]    yomxxx.com long-form post on KV-cache compression limits
 *   [rebasdaily] rebasdaily.com article on DeepSeek-V4.1-Flash KV compression
 *   [ailily]    ailily.cc article "每个 token 只占 890 字节：DeepSeek 削掉的是 Agent 最贵的隐形账"
 *
 * Every floating-point step is written out in the order stated next to it; the file must be
 * compiled with -ffp-contract=off and without -ffast-math so that no step is fused or reordered.
 * Single-threaded.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ---------------------------------------------------------------------------------------------
 * Element formats.  The pages name them only ([ailily] §二 "每 16 个通道配一个 E4M3 缩放因子";
 * §三 "FP4 的 E2M1 格式 ... 448 × 6 = 2688"); the bit layouts below are the public OCP FP8 / MX
 * definitions.
 * ------------------------------------------------------------------------------------------- */

/* E4M3 ("fn" variant): sign | 4 exponent bits (bias 7) | 3 mantissa bits.  No infinities;
 * S.1111.111 is NaN; the largest finite magnitude is 1.75 * 2^8 = 448; exponent field 0 holds the
 * subnormals m * 2^-9. */
double ora_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* E2M1: sign | 2 exponent bits (bias 1) | 1 mantissa bit.  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
 * no infinities or NaN. */
double ora_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v;
    if (e == 0)
        v = 0.5 * m;
    else
        v = ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* Round to the nearest representable magnitude; an exact tie goes to the code with an even
 * mantissa (round-to-nearest-even); magnitudes beyond the largest finite value saturate to it.
 * The search is written as a plain scan over all non-negative finite codes, which are ordered by
 * value. */
static int nearest_even_code(double a, int ncodes, double (*decode)(uint8_t))
{
    int best = 0;
    double bestd = fabs(a - decode(0));
    for (int c = 1; c < ncodes; ++c) {
        double d = fabs(a - decode((uint8_t)c));
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* Float -> E4M3, round-to-nearest-even, saturating to +-448.  The sign is kept, so a negative
 * value that rounds to zero gives negative zero (0x80).  NaN -> 0x7F. */
uint8_t ora_e4m3_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (isnan(x))
        return 0x7F;
    if (a >= 448.0)
        return sign | 0x7E;
    return sign | (uint8_t)nearest_even_code(a, 0x7F, ora_e4m3_decode);
}

/* Float -> E2M1, round-to-nearest-even, saturating to +-6, sign kept (so -0.1 -> 0x8). */
uint8_t ora_e2m1_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs((double)x);
    if (a >= 6.0)
        return sign | 0x7;
    return sign | (uint8_t)nearest_even_code(a, 8, ora_e2m1_decode);
}

/* ---------------------------------------------------------------------------------------------
 * Step 1: pack one token.  [rebasdaily] §"同一份笔记，多层一起用": main KV in FP4, SWA KV stays FP8;
 * [ailily] §二: one E4M3 scale per 16 channels.
 *
 * Main entry, per 16-channel group g of the 512-channel latent x (bf16 -> f32 is exact):
 *   a      = max_i |x_i|
 *   s32    = a / 6                      (binary32 division, correctly rounded)
 *   s      = E4M3(s32), s_d = decode(s)
 *   code_i = 0 if s_d == 0, else E2M1(x_i / s_d)   (binary32 division, correctly rounded)
 * Codes are stored two per byte, channel 2i in the low nibble and 2i+1 in the high nibble.
 * ------------------------------------------------------------------------------------------- */
void ora_pack_main(const uint16_t *latent, uint8_t *codes, uint8_t *scales)
{
    for (int g = 0; g < 32; ++g) {
        float x[16];
        float a = 0.0f;
        for (int i = 0; i < 16; ++i) {
            x[i] = bf16_to_f32(latent[16 * g + i]);
            float ax = fabsf(x[i]);
            if (ax > a)
                a = ax;
        }
        float s32 = a / 6.0f;
        uint8_t s = ora_e4m3_encode(s32);
        float sd = (float)ora_e4m3_decode(s);
        scales[g] = s;
        for (int i = 0; i < 16; i += 2) {
            uint8_t c0 = 0, c1 = 0;
            if (sd != 0.0f) {
                c0 = ora_e2m1_encode(x[i] / sd);
                c1 = ora_e2m1_encode(x[i + 1] / sd);
            }
            codes[8 * g + i / 2] = (uint8_t)(c0 | (c1 << 4));
        }
    }
}

/* Indexer key: each of the 128 bf16 channels cast to E4M3 with no scale. */
void ora_pack_key(const uint16_t *key, uint8_t *key8)
{
    for (int d = 0; d < 128; ++d)
        key8[d] = ora_e4m3_encode(bf16_to_f32(key[d]));
}

/* SWA entry: the same latent in FP8 E4M3 with one binary32 scale per token:
 *   scale = (max_c |x_c|) / 448 (correctly rounded); value_c = E4M3(x_c / scale); scale 0 -> 0. */
void ora_pack_swa(const uint16_t *latent, uint8_t *swa, float *swa_scale)
{
    float a = 0.0f;
    for (int c = 0; c < 512; ++c) {
        float ax = fabsf(bf16_to_f32(latent[c]));
        if (ax > a)
            a = ax;
    }
    float scale = a / 448.0f;
    *swa_scale = scale;
    for (int c = 0; c < 512; ++c)
        swa[c] = (scale == 0.0f) ? 0 : ora_e4m3_encode(bf16_to_f32(latent[c]) / scale);
}

/* binary32 -> bf16, round to nearest even (NaN stays a quiet NaN). */
static uint16_t f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u)
        return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------------------------------------
 * Step 0, before the pack: RMSNorm of the 512-channel pre-norm latent with a caller-given weight,
 * then the rotary embedding of channels 448..511 with caller-given (cos, sin) per pair, rounded to
 * bf16.  The pages fix only that the latent is RMS-normalised (weights of magnitude about 1) and
 * rotated by RoPE, which keeps its norm ([ailily] §三); the arithmetic is this build's reading, in
 * binary32, in exactly this order:
 *   s_g = FMA chain of v_c * v_c over c = 16g .. 16g+15, from 0 (g = 0..31);
 *   for d = 16, 8, 4, 2, 1: s_g <- s_g + s_(g xor d) for every g at once; ss = s_0;
 *   r = 1 / sqrt(ss / 512 + 1e-6), every operation correctly rounded;
 *   y_c = (v_c * r) * w_c;
 *   pair i = 0..31, (a, b) = (y_(448+2i), y_(449+2i)):
 *     y_(448+2i) = (a * cos_i) - (b * sin_i),  y_(449+2i) = (a * sin_i) + (b * cos_i);
 *   out_c = bf16(y_c).
 * n tokens: x bf16 [n][512], w [512], cs [n][32][2] = (cos_i, sin_i), out bf16 [n][512].
 * ------------------------------------------------------------------------------------------- */
void ora_norm_rope(int64_t n, const uint16_t *x, const float *w, const float *cs, uint16_t *out)
{
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t *xt = x + 512 * t;
        float v[512], y[512], s[32], s2[32];
        for (int c = 0; c < 512; ++c)
            v[c] = bf16_to_f32(xt[c]);
        for (int g = 0; g < 32; ++g) {
            float acc = 0.0f;
            for (int c = 16 * g; c < 16 * g + 16; ++c)
                acc = fmaf(v[c], v[c], acc);
            s[g] = acc;
        }
        for (int d = 16; d >= 1; d >>= 1) {
            for (int g = 0; g < 32; ++g)
                s2[g] = s[g] + s[g ^ d];
            memcpy(s, s2, sizeof s);
        }
        const float mean = s[0] / 512.0f;
        const float q = sqrtf(mean + 1e-6f);
        const float r = 1.0f / q;
        for (int c = 0; c < 512; ++c) {
            const float vr = v[c] * r;
            y[c] = vr * w[c];
        }
        const float *cst = cs + 64 * t;
        for (int i = 0; i < 32; ++i) {
            const float a = y[448 + 2 * i], b = y[449 + 2 * i];
            const float co = cst[2 * i], si = cst[2 * i + 1];
            const float ac = a * co, bs = b * si, as = a * si, bc = b * co;
            y[448 + 2 * i] = ac - bs;
            y[449 + 2 * i] = as + bc;
        }
        for (int c = 0; c < 512; ++c)
            out[512 * t + c] = f32_to_bf16(y[c]);
    }
}

/* n tokens, outputs packed densely per token.  swa/swa_scale may be NULL. */
void ora_pack_tokens(int64_t n, const uint16_t *latent, const uint16_t *key, uint8_t *codes,
                     uint8_t *scales, uint8_t *key8, uint8_t *swa, float *swa_scale)
{
    for (int64_t t = 0; t < n; ++t) {
        ora_pack_main(latent + 512 * t, codes + 256 * t, scales + 32 * t);
        ora_pack_key(key + 128 * t, key8 + 128 * t);
        if (swa)
            ora_pack_swa(latent + 512 * t, swa + 512 * t, swa_scale + t);
    }
}

/* ---------------------------------------------------------------------------------------------
 * Step 2: indexer score of one position.  The pages fix only that a Top-K of 8-position blocks is
 * chosen by an indexer ([rebasdaily] §"同一份笔记，多层一起用"); the score itself is
 *   t = sum_h w_h * ReLU(q_h . k)      over 8 heads, 128-dim keys in E4M3,
 * evaluated in binary32 in exactly this order:
 *   per head h: eight 16-dim chains part_j = fma(q[16j+t], k[16j+t], part_j), t = 0..15, from 0;
 *               d_h = ((part0+part4)+(part2+part6)) + ((part1+part5)+(part3+part7));
 *               r_h = d_h > 0 ? d_h : 0;
 *   score = fma(w_h, r_h, score) for h = 0..7, from 0.
 * ------------------------------------------------------------------------------------------- */
float ora_index_score(const uint16_t *iq, const float *iw, const uint8_t *key8)
{
    float k[128];
    for (int d = 0; d < 128; ++d)
        k[d] = (float)ora_e4m3_decode(key8[d]);
    float score = 0.0f;
    for (int h = 0; h < 8; ++h) {
        float part[8];
        for (int j = 0; j < 8; ++j) {
            float p = 0.0f;
            for (int t = 0; t < 16; ++t)
                p = fmaf(bf16_to_f32(iq[128 * h + 16 * j + t]), k[16 * j + t], p);
            part[j] = p;
        }
        float d = ((part[0] + part[4]) + (part[2] + part[6])) + ((part[1] + part[5]) + (part[3] + part[7]));
        float r = d > 0.0f ? d : 0.0f;
        score = fmaf(iw[h], r, score);
    }
    return score;
}

/* Block score of block b = max of the position scores over positions 8b .. 8b+7 that are < L.
 * keys8 is [L][128]; scores gets ceil(L/8) values. */
void ora_block_scores(int64_t L, const uint16_t *iq, const float *iw, const uint8_t *keys8,
                      float *scores)
{
    int64_t nb = (L + 7) / 8;
    for (int64_t b = 0; b < nb; ++b) {
        float m = -INFINITY;
        for (int64_t p = 8 * b; p < 8 * b + 8 && p < L; ++p) {
            float t = ora_index_score(iq, iw, keys8 + 128 * p);
            if (t > m)
                m = t;
        }
        scores[b] = m;
    }
}

/* ---------------------------------------------------------------------------------------------
 * Step 3: Top-K over blocks.  Order: larger score first; equal scores -> lower block id first.
 * The first min(k, n) of that order are returned sorted by ascending block id.
 * ------------------------------------------------------------------------------------------- */
typedef struct {
    float s;
    int32_t b;
} ora_cand;

static int cmp_score_desc_block_asc(const void *pa, const void *pb)
{
    const ora_cand *a = pa, *b = pb;
    if (a->s > b->s)
        return -1;
    if (a->s < b->s)
        return 1;
    return (a->b > b->b) - (a->b < b->b);
}

static int cmp_i32(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Candidates are (blocks[i], scores[i]), i < n.  Returns the count written to out. */
int32_t ora_topk(int64_t n, const int32_t *blocks, const float *scores, int32_t k, int32_t *out)
{
    ora_cand *c = (ora_cand *)malloc(sizeof(ora_cand) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) {
        c[i].s = scores[i];
        c[i].b = blocks[i];
    }
    qsort(c, (size_t)n, sizeof(ora_cand), cmp_score_desc_block_asc);
    int32_t cnt = (int32_t)(n < k ? n : k);
    for (int32_t i = 0; i < cnt; ++i)
        out[i] = c[i].b;
    qsort(out, (size_t)cnt, sizeof(int32_t), cmp_i32);
    free(c);
    return cnt;
}

/* ---------------------------------------------------------------------------------------------
 * Step 4: sparse decode attention for one sequence, in binary64.
 * [rebasdaily] §"同一份笔记，多层一起用" (sparse attention over the chosen positions) and
 * §"先让长输入少走一半路" (the sliding-window branch), merged through one softmax:
 *   segment E: nE FP4 entries, value v_c = e2m1(code_c) * e4m3(scale_{c/16})   (exact)
 *   segment F: nF SWA entries, value u_c = e4m3(swa_c) * swa_scale             (binary64)
 *   z_i   = tau * sum_c q_c * val_i,c     (the 512-channel latent is both key and value)
 *   o_h   = sum_i exp(z_i - M) val_i / sum_i exp(z_i - M),  M = max_i z_i
 *   lse_h = M + ln sum_i exp(z_i - M)
 * q is [H][512] bf16; out is [H][512]; lse is [H].
 * ------------------------------------------------------------------------------------------- */
void ora_dequant_main(const uint8_t *codes, const uint8_t *scales, double *v)
{
    for (int c = 0; c < 512; ++c) {
        uint8_t byte = codes[c / 2];
        uint8_t code = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
        v[c] = ora_e2m1_decode(code) * ora_e4m3_decode(scales[c / 16]);
    }
}

void ora_dequant_swa(const uint8_t *swa, float swa_scale, double *u)
{
    for (int c = 0; c < 512; ++c)
        u[c] = ora_e4m3_decode(swa[c]) * (double)swa_scale;
}

int ora_attention(int32_t H, const uint16_t *q, double tau, int64_t nE, const uint8_t *codes,
                  const uint8_t *scales, int64_t nF, const uint8_t *swa, const float *swa_scale,
                  double *out, double *lse)
{
    int64_t n = nE + nF;
    double *val = (double *)malloc(sizeof(double) * 512 * (size_t)(n > 0 ? n : 1));
    double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!val || !z) {
        free(val);
        free(z);
        return -1;
    }
    for (int64_t i = 0; i < nE; ++i)
        ora_dequant_main(codes + 256 * i, scales + 32 * i, val + 512 * i);
    for (int64_t i = 0; i < nF; ++i)
        ora_dequant_swa(swa + 512 * i, swa_scale[i], val + 512 * (nE + i));

    for (int32_t h = 0; h < H; ++h) {
        double qh[512];
        for (int c = 0; c < 512; ++c)
            qh[c] = (double)bf16_to_f32(q[512 * h + c]);
        double M = -INFINITY;
        for (int64_t i = 0; i < n; ++i) {
            double dot = 0.0;
            for (int c = 0; c < 512; ++c)
                dot += qh[c] * val[512 * i + c];
            z[i] = tau * dot;
            if (z[i] > M)
                M = z[i];
        }
        double den = 0.0;
        double num[512];
        for (int c = 0; c < 512; ++c)
            num[c] = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            double e = exp(z[i] - M);
            den += e;
            for (int c = 0; c < 512; ++c)
                num[c] += e * val[512 * i + c];
        }
        for (int c = 0; c < 512; ++c)
            out[512 * h + c] = num[c] / den;
        lse[h] = M + log(den);
    }
    free(val);
    free(z);
    return 0;
}

/* ---------------------------------------------------------------------------------------------
 * Array forms of the codecs, so that tests can sweep many values in one call.
 * ------------------------------------------------------------------------------------------- */
void ora_e4m3_encode_n(int64_t n, const float *x, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = ora_e4m3_encode(x[i]);
}

void ora_e2m1_encode_n(int64_t n, const float *x, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = ora_e2m1_encode(x[i]);
}

void ora_e4m3_decode_n(int64_t n, const uint8_t *c, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = ora_e4m3_decode(c[i]);
}

void ora_e2m1_decode_n(int64_t n, const uint8_t *c, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = ora_e2m1_decode(c[i]);
}

/* Position scores for n keys (no block max). */
void ora_index_scores(int64_t n, const uint16_t *iq, const float *iw, const uint8_t *keys8, float *out)
{
    for (int64_t p = 0; p < n; ++p)
        out[p] = ora_index_score(iq, iw, keys8 + 128 * p);
}
