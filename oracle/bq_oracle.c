/*
 * bq_oracle.c -- plain, slow CPU oracle for linear layers on packed binary-g128 and
 * ternary-g128 weights.
 *
 * TEST INFRASTRUCTURE ONLY. It is called by the test suite, by the smoke check and by
 * the CPU-baseline leg of the benchmark. The product library (libbq) never links,
 * loads or calls it, and the two share no code: not a header, not a helper, not a table.
 *
 * Every floating-point result is computed in IEEE binary64 ("fp64"), summing k in
 * ascending order; there is no blocking, fusion or reordering.
 *
 * What it follows
 *   [card]    "prism-ml/Bonsai-27B-mlx-1bit - Hugging Face" model card.
 *             Section "Weight representation: Binary g128": each weight is one sign
 *             bit, 0 maps to -scale and 1 maps to +scale, and every 128 weights share
 *             one FP16 scale (1 + 16/128 = 1.125 bits per weight).
 *             Section "MLX packaging": scale-only groups are stored in MLX's
 *             scale+bias form with s_mlx = 2*s_g and bias = -s_g, which reproduces
 *             +-s_g exactly at 1.25 bits per weight.
 *             Section "CUDA (NVIDIA GPUs)": the fused kernel unpacks the sign codes
 *             inside the matrix product and applies the group scale; the model is
 *             never expanded to a dense FP16 tensor.
 *   [tern]    "Ternary Bonsai 27B vs ..." article (wmrh.cn), section
 *             "三元量化技术突破" and "局限性与未来发展": ternary weights in {-1, 0, +1}
 *             with the same FP16 scale per 128 weights, currently kept in 2-bit storage.
 *   [agent]   "Bonsai 27B 将 270 亿参数 AI 带到手机" (agentlenshq), section
 *             "两种硬件对应的运行点": ternary (-1, 0, +1) and binary (-1, +1) share the
 *             same group scaling.
 *
 * Readings taken where the pages are silent (each is a choice, not a page fact):
 *   - The group of 128 runs along K, the reduction axis of y = x W^T; weights are
 *     row-major over the N output rows with K inner.
 *   - Binary bits are LSB-first: bit (k % 32) of word (k / 32) of a row holds weight k,
 *     so one group is 4 consecutive uint32 words.
 *   - Ternary codes are 2-bit fields, LSB-first: bits 2*(k % 16)..2*(k % 16)+1 of word
 *     (k / 16) hold code c with value c - 1 (0 -> -1, 1 -> 0, 2 -> +1); c = 3 is invalid.
 *   - Scales are IEEE binary16 [N, K/128]; x is binary16 or bfloat16 [M, K].
 *   - Base-3 ternary storage (BQO_TERNARY_B3): see the section "Ternary g128 in base-3
 *     storage" below for the byte layout, which the pages leave open.
 *   - The tolerance bound of an output is 2e-3 * sum_k |x[m,k] * s[n, k/128]|; for
 *     ternary weights the scale counts even where the code is 0.
 */
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>

#include "bq_oracle.h"

/* ---------------------------------------------------------------------------------------
 * Number formats.  Written from the IEEE 754-2008 binary16 definition and from bfloat16
 * being the upper 16 bits of a binary32.
 * ------------------------------------------------------------------------------------- */

double bqo_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);     /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

double bqo_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to a binary format with `p` significant bits, minimum normal exponent
 * `emin` (value 2^emin) and largest finite value `maxv`; ties to even. Returns the
 * rounded value as a double (inf on overflow). */
static double round_to_format(double v, int p, int emin, double maxv)
{
    if (isnan(v) || isinf(v) || v == 0.0)
        return v;
    int e;
    frexp(v, &e);                 /* v = m * 2^e, 0.5 <= |m| < 1 */
    int exp_unbiased = e - 1;     /* v = 1.xxx * 2^(e-1) */
    if (exp_unbiased < emin)
        exp_unbiased = emin;      /* subnormal range: fixed quantum */
    int quantum_exp = exp_unbiased - (p - 1);
    double q = nearbyint(ldexp(v, -quantum_exp));   /* default rounding mode: ties-to-even */
    double r = ldexp(q, quantum_exp);
    if (fabs(r) > maxv)
        return v > 0 ? INFINITY : -INFINITY;
    return r;
}

uint16_t bqo_f64_to_bf16(double v)
{
    if (isnan(v))
        return 0x7fc0;
    double r = round_to_format(v, 8, -126, 3.38953138925153547590470800371487866880e+38);
    float f = (float)r;           /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

void bqo_f64_to_bf16_array(const double *v, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = bqo_f64_to_bf16(v[i]);
}

uint16_t bqo_f64_to_f16(double v)
{
    if (isnan(v))
        return 0x7e00;
    double r = round_to_format(v, 11, -14, 65504.0);
    uint16_t sign = signbit(r) ? 0x8000 : 0;
    double a = fabs(r);
    if (isinf(a))
        return sign | 0x7c00;
    if (a == 0.0)
        return sign;
    if (a < ldexp(1.0, -14))                           /* subnormal */
        return sign | (uint16_t)ldexp(a, 24);
    int e;
    double m = frexp(a, &e);                           /* a = m * 2^e */
    int biased = (e - 1) + 15;
    uint16_t frac = (uint16_t)(ldexp(m, 11) - 1024.0);
    return sign | (uint16_t)(biased << 10) | frac;
}

/* ---------------------------------------------------------------------------------------
 * Sizes.
 * ------------------------------------------------------------------------------------- */

int64_t bqo_words_per_row(int fmt, int64_t K)
{
    if (K <= 0 || K % 128)
        return -1;
    if (fmt == BQO_BINARY)
        return K / 32;            /* one bit per weight */
    if (fmt == BQO_TERNARY)
        return K / 16;            /* two bits per weight */
    return -1;
}

int64_t bqo_row_bytes(int fmt, int64_t K)
{
    if (K <= 0 || K % 128)
        return -1;
    if (fmt == BQO_BINARY)
        return K / 8;
    if (fmt == BQO_TERNARY)
        return K / 4;
    if (fmt == BQO_TERNARY_B3)
        return 26 * (K / 128);    /* 26 bytes per group of 128 */
    return -1;
}

/* ---------------------------------------------------------------------------------------
 * Pack / unpack: loop over every k and set or read its bit (binary) or 2-bit field
 * (ternary). [card] "Weight representation: Binary g128"; [tern] 2-bit storage.
 * ------------------------------------------------------------------------------------- */

int bqo_pack_binary_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                         uint32_t *words, uint16_t *s_out)
{
    int64_t W = bqo_words_per_row(BQO_BINARY, K);
    if (W < 0 || N < 0)
        return BQO_ERR_SHAPE;
    for (int64_t i = 0; i < N * W; i++)
        words[i] = 0;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) {
            int8_t v = q[n * K + k];
            if (v == 1)
                words[n * W + k / 32] |= (uint32_t)1 << (k % 32);   /* 1 -> +scale */
            else if (v != -1)
                return BQO_ERR_CODE;                                 /* 0 -> -scale */
        }
    }
    for (int64_t i = 0; i < N * (K / 128); i++)
        s_out[i] = s_in[i];
    return BQO_OK;
}

int bqo_pack_ternary_g128(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                          uint32_t *words, uint16_t *s_out)
{
    int64_t W = bqo_words_per_row(BQO_TERNARY, K);
    if (W < 0 || N < 0)
        return BQO_ERR_SHAPE;
    for (int64_t i = 0; i < N * W; i++)
        words[i] = 0;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) {
            int8_t v = q[n * K + k];
            if (v < -1 || v > 1)
                return BQO_ERR_CODE;
            uint32_t code = (uint32_t)(v + 1);                       /* -1->0, 0->1, +1->2 */
            words[n * W + k / 16] |= code << (2 * (k % 16));
        }
    }
    for (int64_t i = 0; i < N * (K / 128); i++)
        s_out[i] = s_in[i];
    return BQO_OK;
}

int64_t bqo_unpack_binary_g128(const uint32_t *words, int64_t N, int64_t K, int8_t *q)
{
    int64_t W = bqo_words_per_row(BQO_BINARY, K);
    if (W < 0 || N < 0)
        return -1;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            uint32_t bit = (words[n * W + k / 32] >> (k % 32)) & 1u;
            q[n * K + k] = bit ? 1 : -1;
        }
    return 0;
}

/* Returns the number of invalid (code 3) fields; their q is set to 0. */
int64_t bqo_unpack_ternary_g128(const uint32_t *words, int64_t N, int64_t K, int8_t *q)
{
    int64_t W = bqo_words_per_row(BQO_TERNARY, K);
    if (W < 0 || N < 0)
        return -1;
    int64_t bad = 0;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            uint32_t code = (words[n * W + k / 16] >> (2 * (k % 16))) & 3u;
            if (code == 3) {
                bad++;
                q[n * K + k] = 0;
            } else {
                q[n * K + k] = (int8_t)((int)code - 1);
            }
        }
    return bad;
}

/* ---------------------------------------------------------------------------------------
 * Ternary g128 in base-3 storage (BQO_TERNARY_B3).
 * [tern] "局限性与未来发展": the deployed ternary model keeps 2-bit codes (7.2 GB) while the
 * information is 1.71 bits per weight (5.9 GB), and native ternary kernels are still to
 * come; [agent] "两种硬件对应的运行点" gives the same 1.71 bits per weight and 5.9 GB. The
 * pages give no base-3 layout; this is the library's reading:
 *   - The codes c = value + 1 in {0, 1, 2} of a group of 128 are stored in 26 bytes:
 *     bytes 0..23 hold five codes each (positions 5j .. 5j+4 of the group), bytes 24 and
 *     25 four codes each (positions 120..123 and 124..127).
 *   - A byte holding n codes c_0 .. c_{n-1} (c_0 at the lowest position) stores
 *     ceil(256 v / 3^n), v = sum_p c_p 3^(n-1-p): the codes read as a base-3 number,
 *     first code most significant, kept as the fraction v / 3^n in 8-bit fixed point
 *     rounded up. v is floor(byte * 3^n / 256).
 *   - A row is a run of blocks of 8 groups (the last block may hold fewer, nb). A block
 *     stores the 24 five-code bytes of each of its groups first (group i of the block at
 *     byte 24 i) and then the two four-code bytes of each (group i at 24 nb + 2 i). A row
 *     is 26 K / 128 bytes; with the fp16 scale, (26 * 8 + 16) / 128 = 1.75 bits per weight.
 *   - 243 of the 256 byte values are written for five codes and 81 for four; any other
 *     value is invalid (the pack never writes it; the unpack counts it).
 * ------------------------------------------------------------------------------------- */

static const int64_t kPow3[6] = {1, 3, 9, 27, 81, 243};

/* Byte j (0..25) of a group holds b3_count(j) codes starting at position b3_first(j). */
static int b3_count(int j) { return j < 24 ? 5 : 4; }
static int b3_first(int j) { return j < 24 ? 5 * j : 120 + 4 * (j - 24); }

/* The byte of a group that holds position kk (0..127). */
static int b3_byte_of(int kk) { return kk < 120 ? kk / 5 : 24 + (kk - 120) / 4; }

/* Offset, within a row of G groups, of byte j of group g. */
static int64_t b3_byte_offset(int64_t G, int64_t g, int j)
{
    int64_t first = 8 * (g / 8);                      /* first group of g's block */
    int64_t nb = G - first < 8 ? G - first : 8;       /* groups in that block */
    if (j < 24)
        return 26 * first + 24 * (g - first) + j;
    return 26 * first + 24 * nb + 2 * (g - first) + (j - 24);
}

static uint8_t b3_encode(int64_t v, int n)
{
    return (uint8_t)((256 * v + kPow3[n] - 1) / kPow3[n]);   /* ceil(256 v / 3^n) */
}

/* v of a stored byte holding n codes; *valid says whether the encoding writes that byte. */
static int64_t b3_decode(uint8_t byte, int n, int *valid)
{
    int64_t v = ((int64_t)byte * kPow3[n]) / 256;
    *valid = b3_encode(v, n) == byte;
    return v;
}

/* Code p (0 = first, the most significant digit) of the n codes with value v. */
static int b3_code(int64_t v, int n, int p)
{
    return (int)((v / kPow3[n - 1 - p]) % 3);
}

int bqo_pack_ternary_b3(const int8_t *q, const uint16_t *s_in, int64_t N, int64_t K,
                        uint8_t *bytes, uint16_t *s_out)
{
    int64_t RB = bqo_row_bytes(BQO_TERNARY_B3, K);
    if (RB < 0 || N < 0)
        return BQO_ERR_SHAPE;
    int64_t G = K / 128;
    for (int64_t n = 0; n < N; n++)
        for (int64_t g = 0; g < G; g++)
            for (int j = 0; j < 26; j++) {
                int cnt = b3_count(j);
                int64_t v = 0;
                for (int p = 0; p < cnt; p++) {
                    int8_t w = q[n * K + 128 * g + b3_first(j) + p];
                    if (w < -1 || w > 1)
                        return BQO_ERR_CODE;
                    v = 3 * v + (w + 1);                 /* first code most significant */
                }
                bytes[n * RB + b3_byte_offset(G, g, j)] = b3_encode(v, cnt);
            }
    for (int64_t i = 0; i < N * G; i++)
        s_out[i] = s_in[i];
    return BQO_OK;
}

/* Returns the number of invalid bytes; the q of their codes is set to 0. */
int64_t bqo_unpack_ternary_b3(const uint8_t *bytes, int64_t N, int64_t K, int8_t *q)
{
    int64_t RB = bqo_row_bytes(BQO_TERNARY_B3, K);
    if (RB < 0 || N < 0)
        return -1;
    int64_t G = K / 128, bad = 0;
    for (int64_t n = 0; n < N; n++)
        for (int64_t g = 0; g < G; g++)
            for (int j = 0; j < 26; j++) {
                int cnt = b3_count(j), valid;
                int64_t v = b3_decode(bytes[n * RB + b3_byte_offset(G, g, j)], cnt, &valid);
                if (!valid)
                    bad++;
                for (int p = 0; p < cnt; p++)
                    q[n * K + 128 * g + b3_first(j) + p] = valid ? (int8_t)(b3_code(v, cnt, p) - 1) : 0;
            }
    return bad;
}

/* Code of weight (n, k) of a base-3 matrix, or -1 if its byte is invalid. */
static int b3_code_at(const uint8_t *bytes, int64_t K, int64_t n, int64_t k)
{
    int64_t G = K / 128;
    int kk = (int)(k % 128);
    int j = b3_byte_of(kk), cnt = b3_count(j), valid;
    int64_t v = b3_decode(bytes[n * 26 * G + b3_byte_offset(G, k / 128, j)], cnt, &valid);
    return valid ? b3_code(v, cnt, kk - b3_first(j)) : -1;
}

/* ---------------------------------------------------------------------------------------
 * Dequantised weight W[n, k] = s[n, k/128] * (2b - 1)   (binary, [card])
 *                            = s[n, k/128] * (c - 1)    (ternary, either storage, [tern])
 * The weight buffer is uint32 words for the binary and 2-bit formats and bytes for base-3.
 * ------------------------------------------------------------------------------------- */

double bqo_weight(int fmt, const uint32_t *words, const uint16_t *scales, int64_t K,
                  int64_t n, int64_t k)
{
    double s = bqo_f16_to_f64(scales[n * (K / 128) + k / 128]);
    if (fmt == BQO_BINARY) {
        uint32_t bit = (words[n * (K / 32) + k / 32] >> (k % 32)) & 1u;
        return bit ? s : -s;
    }
    if (fmt == BQO_TERNARY_B3) {
        int c = b3_code_at((const uint8_t *)words, K, n, k);
        return c < 0 ? NAN : s * (double)(c - 1);
    }
    uint32_t code = (words[n * (K / 16) + k / 16] >> (2 * (k % 16))) & 3u;
    if (code == 3)
        return NAN;
    return s * (double)((int)code - 1);
}

int bqo_dequant(int fmt, const uint32_t *words, const uint16_t *scales, int64_t N, int64_t K,
                double *Wd)
{
    if (bqo_row_bytes(fmt, K) < 0 || N < 0)
        return BQO_ERR_SHAPE;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++)
            Wd[n * K + k] = bqo_weight(fmt, words, scales, K, n, k);
    return BQO_OK;
}

static double x_value(const uint16_t *x, int xt, int64_t i)
{
    return xt == BQO_X_F16 ? bqo_f16_to_f64(x[i]) : bqo_bf16_to_f64(x[i]);
}

/* ---------------------------------------------------------------------------------------
 * y[m, r] = sum_k x[m, k] * W[rows[r], k]   in fp64, k ascending, and the tolerance bound
 * bound[m, r] = 2e-3 * sum_k |x[m, k] * s[rows[r], k/128]|.
 * The same function serves the decode GEMV (M <= 8) and the prefill GEMM (any M): a GEMM
 * is the GEMV for every row of x. Outputs are [M, R] row-major.
 * ------------------------------------------------------------------------------------- */

int bqo_gemv_rows(int fmt, const uint16_t *x, int xt, int64_t M, int64_t K,
                  const uint32_t *words, const uint16_t *scales, int64_t N,
                  const int64_t *rows, int64_t R, double *y, double *bound)
{
    if (bqo_row_bytes(fmt, K) < 0 || M < 0 || N < 0 || R < 0)
        return BQO_ERR_SHAPE;
    for (int64_t r = 0; r < R; r++) {
        int64_t n = rows[r];
        if (n < 0 || n >= N)
            return BQO_ERR_SHAPE;
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double xv = x_value(x, xt, m * K + k);
                acc += xv * bqo_weight(fmt, words, scales, K, n, k);
                mag += fabs(xv * bqo_f16_to_f64(scales[n * (K / 128) + k / 128]));
            }
            y[m * R + r] = acc;
            if (bound)
                bound[m * R + r] = 2e-3 * mag;
        }
    }
    return BQO_OK;
}

/* ---------------------------------------------------------------------------------------
 * Embedding lookup: out[t, k] = W[ids[t], k]. [card] "Highlights": the embedding is one
 * of the binary layers. Ids outside [0, N) give a row of zeros and are counted.
 * ------------------------------------------------------------------------------------- */

int64_t bqo_embed(int fmt, const int32_t *ids, int64_t T, const uint32_t *words,
                  const uint16_t *scales, int64_t N, int64_t K, double *out)
{
    if (bqo_row_bytes(fmt, K) < 0 || T < 0 || N < 0)
        return -1;
    int64_t bad = 0;
    for (int64_t t = 0; t < T; t++) {
        int64_t id = ids[t];
        for (int64_t k = 0; k < K; k++) {
            if (id < 0 || id >= N)
                out[t * K + k] = 0.0;
            else
                out[t * K + k] = bqo_weight(fmt, words, scales, K, id, k);
        }
        if (id < 0 || id >= N)
            bad++;
    }
    return bad;
}

/* ---------------------------------------------------------------------------------------
 * Top-k of the logits and sampling from it. [card] "Generation parameters": temperature 0.7,
 * top-p 0.95, top-k 20 for every reported benchmark run. The pages do not state the order of
 * the three filters; the reading taken here: the k largest logits (equal values in ascending
 * index order) are the candidates; their probabilities are softmax(logit / T) over the k; top-p
 * keeps the shortest leading run of candidates whose probabilities sum to at least top_p (at
 * least one); the token is the first kept candidate whose cumulative probability, renormalised
 * over the kept ones, exceeds u, a uniform number in [0, 1) drawn by the caller.
 * ------------------------------------------------------------------------------------- */

/* a ranks before b: larger value, or the same value and a smaller index */
static int ranks_before(double va, int64_t ia, double vb, int64_t ib)
{
    return va > vb || (va == vb && ia < ib);
}

int bqo_topk(const double *y, int64_t M, int64_t N, int k, int64_t *idx, double *vals)
{
    if (M < 0 || N < 1 || k < 1 || k > N)
        return BQO_ERR_SHAPE;
    for (int64_t m = 0; m < M; m++) {
        const double *row = y + m * N;
        for (int j = 0; j < k; j++) {
            /* the best entry that ranks after the (j-1)-th pick */
            int64_t best = -1;
            for (int64_t n = 0; n < N; n++) {
                if (j > 0 && !ranks_before(vals[m * k + j - 1], idx[m * k + j - 1], row[n], n))
                    continue;
                if (best < 0 || ranks_before(row[n], n, row[best], best))
                    best = n;
            }
            idx[m * k + j] = best;
            vals[m * k + j] = row[best];
        }
    }
    return BQO_OK;
}

int64_t bqo_sample_topk(const double *vals, const int64_t *idx, int k, double T, double top_p, double u)
{
    if (k < 1 || !(T > 0.0))
        return -1;
    double p[64];
    if (k > 64)
        return -1;
    double z = 0.0;
    for (int i = 0; i < k; i++) {
        p[i] = exp((vals[i] - vals[0]) / T);      /* vals[0] is the largest: no overflow */
        z += p[i];
    }
    int keep = 0;
    double c = 0.0;
    while (keep < k) {
        c += p[keep] / z;
        keep++;
        if (c >= top_p)
            break;
    }
    double kept = 0.0;
    for (int i = 0; i < keep; i++)
        kept += p[i];
    double cum = 0.0;
    for (int i = 0; i < keep; i++) {
        cum += p[i] / kept;
        if (cum > u)
            return idx[i];
    }
    return idx[keep - 1];                           /* u just below 1 and rounding */
}

/* ---------------------------------------------------------------------------------------
 * SwiGLU MLP of a decode step. [card] "Model overview": the blocks use a SwiGLU MLP. For each
 * token row m: g = x W_gate^T and u = x W_up^T (the product above, fp64, k ascending),
 * a = silu(g) * u with silu(z) = z / (1 + e^(-z)), y = a W_down^T (fp64, j ascending). The bound
 * of y[m, n] is 2e-3 * sum_j |a[m, j] * s_down[n, j / 128]|. a is returned too ([M, F]).
 * ------------------------------------------------------------------------------------- */

int bqo_mlp_swiglu(int fmt_gu, const uint16_t *x, int xt, int64_t M, int64_t K, const uint32_t *wg,
                   const uint16_t *sg, const uint32_t *wu, const uint16_t *su, int64_t F, int fmt_d,
                   const uint32_t *wd, const uint16_t *sd, int64_t N, double *a, double *y, double *bound)
{
    if (bqo_row_bytes(fmt_gu, K) < 0 || bqo_row_bytes(fmt_d, F) < 0 || M < 0 || N < 0)
        return BQO_ERR_SHAPE;
    for (int64_t m = 0; m < M; m++) {
        for (int64_t f = 0; f < F; f++) {
            double g = 0.0, u = 0.0;
            for (int64_t k = 0; k < K; k++) {
                const double xk = x_value(x, xt, m * K + k);
                g += xk * bqo_weight(fmt_gu, wg, sg, K, f, k);
                u += xk * bqo_weight(fmt_gu, wu, su, K, f, k);
            }
            a[m * F + f] = g / (1.0 + exp(-g)) * u;
        }
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0, mag = 0.0;
            for (int64_t j = 0; j < F; j++) {
                double av = a[m * F + j];
                acc += av * bqo_weight(fmt_d, wd, sd, F, n, j);
                mag += fabs(av * bqo_f16_to_f64(sd[n * (F / 128) + j / 128]));
            }
            y[m * N + n] = acc;
            bound[m * N + n] = 2e-3 * mag;
        }
    }
    return BQO_OK;
}

/* ---------------------------------------------------------------------------------------
 * Dense -> g128 quantiser. The pages name the format but not how q and s are obtained ([card]
 * "Weight representation: Binary g128" points to a whitepaper that is not among them). The
 * reading taken: the least-squares fit of each group of 128 weights w,
 *   binary:  q = +1 where w >= 0, else -1; s = mean |w| (for fixed signs, sum (w - s q)^2 is
 *            smallest at s = sum |w| / 128);
 *   ternary: q and s >= 0 minimising sum (w - s q)^2 over q in {-1, 0, +1}^128: on a support of
 *            j weights the best q is their sign and the best s their mean |w|, leaving
 *            sum w^2 - (sum_support |w|)^2 / j; so the support is the j largest |w| (equal |w|:
 *            lower position first) with j maximising (sum of those |w|)^2 / j, the smallest such
 *            j on a tie, and none for a group of zeros.
 * s is then rounded to binary16 (ties to even). Inputs are binary32.
 * ------------------------------------------------------------------------------------- */

struct absw {
    double a;
    int k;
};

static int absw_desc(const void *pa, const void *pb)
{
    const struct absw *a = pa, *b = pb;
    if (a->a != b->a)
        return a->a > b->a ? -1 : 1;
    return a->k - b->k;
}

int bqo_quantize_g128(int fmt, const float *w, int64_t N, int64_t K, int8_t *q, uint16_t *s)
{
    if (N < 0 || K <= 0 || K % 128 || (fmt != BQO_BINARY && fmt != BQO_TERNARY && fmt != BQO_TERNARY_B3))
        return BQO_ERR_SHAPE;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t g = 0; g < K / 128; g++) {
            const float *wg = w + n * K + 128 * g;
            int8_t *qg = q + n * K + 128 * g;
            if (fmt == BQO_BINARY) {
                double sum = 0.0;
                for (int k = 0; k < 128; k++) {
                    qg[k] = wg[k] >= 0.0f ? 1 : -1;
                    sum += fabs((double)wg[k]);
                }
                s[n * (K / 128) + g] = bqo_f64_to_f16(sum / 128.0);
                continue;
            }
            struct absw order[128];
            for (int k = 0; k < 128; k++) {
                order[k].a = fabs((double)wg[k]);
                order[k].k = k;
                qg[k] = 0;
            }
            qsort(order, 128, sizeof order[0], absw_desc);
            double best = 0.0, prefix = 0.0, best_sum = 0.0;
            int best_j = 0;
            for (int j = 1; j <= 128; j++) {
                prefix += order[j - 1].a;
                double score = prefix * prefix / j;
                if (score > best) {
                    best = score;
                    best_j = j;
                    best_sum = prefix;
                }
            }
            for (int j = 0; j < best_j; j++) {
                int k = order[j].k;
                qg[k] = wg[k] >= 0.0f ? 1 : -1;
            }
            s[n * (K / 128) + g] = bqo_f64_to_f16(best_j ? best_sum / best_j : 0.0);
        }
    }
    return BQO_OK;
}

/* ---------------------------------------------------------------------------------------
 * MLX affine form ([card] "MLX packaging"): w = s_mlx * q + bias with q in {0, 1},
 * s_mlx = 2 * s and bias = -s, each stored and each operation rounded in binary16.
 * Returns the binary16 bits of w.
 * ------------------------------------------------------------------------------------- */

uint16_t bqo_mlx_affine_dequant(uint16_t s_f16, int q01)
{
    double s = bqo_f16_to_f64(s_f16);
    uint16_t s_mlx = bqo_f64_to_f16(2.0 * s);
    uint16_t bias = bqo_f64_to_f16(-s);
    double prod = bqo_f16_to_f64(bqo_f64_to_f16(bqo_f16_to_f64(s_mlx) * (double)q01));
    return bqo_f64_to_f16(prod + bqo_f16_to_f64(bias));
}
