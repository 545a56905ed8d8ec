/*
 * CPU oracle for the CSA2 decode hot path (DeepSeek V4.1 Flash KV cache pages).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. The CUDA library never links it and it
 * shares no code, header, table or helper with the CUDA sources.
 *
 * Everything here is the plain definition of each step, written for a reader to
 * check by eye: exact format definitions, int64 dot products, a full sort for
 * top-k, fp64 softmax attention. Nothing is blocked, fused or reordered.
 *
 * Sources (page title + section):
 *  [G]  "DeepSeek V4.1 Flash KV Cache: 890 Bytes per Token Explained"
 *       (deepseekv4guide.org), sections on the hierarchical sparse indexer and
 *       on FP4 storage of the main KV.
 *  [N]  "DeepSeek-V4.1-Flash: 890 Bytes Per Token, 437x Smaller KV Cache"
 *       (aimastery.page), sections "CSA2: Sharing Main KV, Indexer K, and
 *       Top-K Indices Across Layers" and "FP4 KV Quantization and Cache
 *       Lifetime Management".
 *  [T]  "890 bytes per token: how DeepSeek V4.1-Flash's KV cache works"
 *       (runaii.cloud), "Mechanism 4: the hierarchical sparse indexer".
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - FP4 scale: amax/6 of the 16-channel group, fp32 IEEE division, rounded to
 *    the nearest E4M3 value (ties to even mantissa), saturating at 448.
 *  - FP4 element: x / scale in fp32 IEEE division, then nearest E2M1 value,
 *    ties to the even code, saturating at 6, sign taken from x. A zero scale
 *    encodes every element as +0.
 *  - MXFP4 variant: E8M0 scale per 32 channels = 2^(floor(log2(amax)) - 2),
 *    clamped to 2^-127..2^127 (2^-127 for an all-zero block); element = nearest
 *    E2M1 value of x / scale, ties to even, saturating at 6, sign from x.
 *  - Indexer score: (sum over heads and dims of int8*int8, exact) converted to
 *    fp32 with round-to-nearest-even, then one fp32 multiply by the key's scale.
 *  - Block score: max of the visible token scores in the 8-token block.
 *  - Selection order: score descending, then position ascending; outputs are
 *    listed in ascending position order.
 *  - Attention: K = V = the dequantized main-KV row (one shared head), logits
 *    scaled by 1/sqrt(C), fp64 throughout.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* The library is built twice: plain (what every test loads) and with
 * -fopenmp, a timing build for the CPU baseline in which the independent
 * outer loops (rows, tokens, heads) are shared among threads. The pragmas
 * change no arithmetic: every output element is computed by one thread in
 * the same order as in the plain build. */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* bf16: the upper 16 bits of an IEEE binary32.                        */
/* ------------------------------------------------------------------ */
static float bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------ */
/* E4M3 ("fn" flavour of the OCP 8-bit float): 1 sign bit, 4 exponent  */
/* bits with bias 7, 3 mantissa bits. Exponent field 0 is subnormal    */
/* (m * 2^-9). S.1111.111 is NaN; there is no infinity; the largest     */
/* finite magnitude is 1.75 * 2^8 = 448. [G] FP4 section, [N] FP4 section */
/* name E4M3 as the per-16-channel scale type.                         */
/* ------------------------------------------------------------------ */
double orc_e4m3_value(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        mag = m * ldexp(1.0, -9);
    else
        mag = (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return sign ? -mag : mag;
}

/* Nearest finite E4M3 value to x. Ties go to the even code (even
 * mantissa). Magnitudes above 448 become 448 (saturating conversion); the
 * clamp comes first so that every distance below is exact in fp64. The
 * sign bit copies x's.                                                  */
uint8_t orc_e4m3_encode(float x)
{
    double ax = fabs((double)x);
    if (ax > 448.0)
        ax = 448.0;
    int best = 0;            /* code 0 is +0 */
    double best_d = ax;
    for (int c = 1; c <= 0x7E; c++) {
        double d = fabs(ax - orc_e4m3_value((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(best | (signbit(x) ? 0x80 : 0));
}

/* ------------------------------------------------------------------ */
/* E2M1 (4-bit float): 1 sign bit, 2 exponent bits with bias 1, 1      */
/* mantissa bit. Exponent field 0 is subnormal (m * 0.5). Magnitudes:   */
/* 0, 0.5, 1, 1.5, 2, 3, 4, 6. No NaN, no infinity. [G] and [N] FP4     */
/* sections.                                                            */
/* ------------------------------------------------------------------ */
double orc_e2m1_value(uint8_t code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 0x3;
    int m = code & 0x1;
    double mag = (e == 0) ? m * 0.5 : (1.0 + m / 2.0) * ldexp(1.0, e - 1);
    return sign ? -mag : mag;
}

/* Nearest E2M1 magnitude to |v| (ties to the even code), saturating at 6
 * (clamped first, as above); the sign bit copies v's, so a negative value
 * that rounds to zero gives -0.                                          */
uint8_t orc_e2m1_encode(float v)
{
    double av = fabs((double)v);
    if (av > 6.0)
        av = 6.0;
    int best = 0;
    double best_d = av;
    for (int c = 1; c <= 7; c++) {
        double d = fabs(av - orc_e2m1_value((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(best | (signbit(v) ? 0x8 : 0));
}

/* Element-wise forms of the two encoders (used by the format tests). */
void orc_e4m3_encode_n(const float *x, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = orc_e4m3_encode(x[i]);
}

void orc_e2m1_encode_n(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = orc_e2m1_encode(v[i]);
}

/* ------------------------------------------------------------------ */
/* FP4 main-KV quantize-and-pack ([G] FP4 section: E2M1 values, one    */
/* E4M3 scale per 16 channels; [N] FP4 section: the NVFP4 scheme        */
/* without its global scale).                                           */
/*   x      : rows x C bf16 bit patterns                                */
/*   packed : rows x C/2 bytes; byte i = code[2i] | code[2i+1] << 4      */
/*   sf     : rows x C/16 E4M3 scale codes                              */
/* ------------------------------------------------------------------ */
void orc_fp4_quantize(const uint16_t *x, int64_t rows, int C, uint8_t *packed, uint8_t *sf)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        const uint16_t *xr = x + r * C;
        for (int g = 0; g < C / 16; g++) {
            float amax = 0.0f;
            for (int c = 0; c < 16; c++) {
                float v = fabsf(bf16_to_float(xr[g * 16 + c]));
                if (v > amax)
                    amax = v;
            }
            float s_f = amax / 6.0f; /* fp32 IEEE division */
            uint8_t s_code = orc_e4m3_encode(s_f);
            float s = (float)orc_e4m3_value(s_code);
            sf[r * (C / 16) + g] = s_code;
            for (int c = 0; c < 16; c += 2) {
                uint8_t code[2];
                for (int u = 0; u < 2; u++) {
                    float xv = bf16_to_float(xr[g * 16 + c + u]);
                    if (s == 0.0f) {
                        code[u] = 0;
                    } else {
                        float v = xv / s; /* fp32 IEEE division */
                        code[u] = orc_e2m1_encode(v);
                    }
                }
                packed[r * (C / 2) + (g * 16 + c) / 2] = (uint8_t)(code[0] | (code[1] << 4));
            }
        }
    }
}

/* Dequantize: value = e2m1(code) * e4m3(scale). */
void orc_fp4_dequantize(const uint8_t *packed, const uint8_t *sf, int64_t rows, int C, double *out)
{
    for (int64_t r = 0; r < rows; r++) {
        for (int c = 0; c < C; c++) {
            uint8_t byte = packed[r * (C / 2) + c / 2];
            uint8_t code = (c & 1) ? (byte >> 4) : (byte & 0xF);
            double s = orc_e4m3_value(sf[r * (C / 16) + c / 16]);
            out[r * C + c] = orc_e2m1_value(code) * s;
        }
    }
}

/* ------------------------------------------------------------------ */
/* MXFP4 variant. [T] mechanism 3 names the cache format MXFP4 and     */
/* gives no detail; read as the OCP Microscaling format: E2M1 elements  */
/* sharing one E8M0 scale per block of 32 channels.                     */
/* E8M0: 8 exponent bits, bias 127, no sign, no mantissa; code e is     */
/* 2^(e - 127) for e = 0..254, and code 255 is NaN.                     */
/* ------------------------------------------------------------------ */
double orc_e8m0_value(uint8_t code)
{
    if (code == 255)
        return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* Shared exponent of a block whose largest magnitude is amax: the
 * exponent of amax (floor(log2(amax))) minus 2, the largest E2M1
 * exponent, clamped to the E8M0 range [-127, 127]; an all-zero block
 * takes -127. frexp gives amax = m * 2^ex with m in [0.5, 1), so
 * floor(log2(amax)) = ex - 1 exactly.                                    */
int orc_mx_shared_exp(double amax)
{
    if (amax == 0.0)
        return -127;
    int ex;
    frexp(amax, &ex);
    int e = (ex - 1) - 2;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return e;
}

/* MXFP4 quantize-and-pack: per block of 32 channels, the shared scale
 * 2^e (e from orc_mx_shared_exp of the block's amax); each element is the
 * nearest E2M1 value of x / 2^e (an exact division by a power of two),
 * ties to the even code, saturating at 6, sign taken from x.
 *   packed : rows x C/2 bytes; byte i = code[2i] | code[2i+1] << 4
 *   sf     : rows x C/32 E8M0 codes (e + 127)                           */
void orc_mxfp4_quantize(const uint16_t *x, int64_t rows, int C, uint8_t *packed, uint8_t *sf)
{
    for (int64_t r = 0; r < rows; r++) {
        const uint16_t *xr = x + r * C;
        for (int g = 0; g < C / 32; g++) {
            double amax = 0.0;
            for (int c = 0; c < 32; c++) {
                double v = fabs((double)bf16_to_float(xr[g * 32 + c]));
                if (v > amax)
                    amax = v;
            }
            int e = orc_mx_shared_exp(amax);
            sf[r * (C / 32) + g] = (uint8_t)(e + 127);
            for (int c = 0; c < 32; c += 2) {
                uint8_t code[2];
                for (int u = 0; u < 2; u++) {
                    double v = ldexp((double)bf16_to_float(xr[g * 32 + c + u]), -e);
                    code[u] = orc_e2m1_encode((float)v);
                }
                packed[r * (C / 2) + (g * 32 + c) / 2] = (uint8_t)(code[0] | (code[1] << 4));
            }
        }
    }
}

/* Dequantize: value = e2m1(code) * e8m0(scale of the 32-channel block). */
void orc_mxfp4_dequantize(const uint8_t *packed, const uint8_t *sf, int64_t rows, int C,
                          double *out)
{
    for (int64_t r = 0; r < rows; r++) {
        for (int c = 0; c < C; c++) {
            uint8_t byte = packed[r * (C / 2) + c / 2];
            uint8_t code = (c & 1) ? (byte >> 4) : (byte & 0xF);
            double s = orc_e8m0_value(sf[r * (C / 32) + c / 32]);
            out[r * C + c] = orc_e2m1_value(code) * s;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Indexer ([N] CSA2 section: Full layers project indexer K and select  */
/* fresh top-512; Reindex layers rescore the pool with their own        */
/* indexer Q; [T] mechanism 4: indexer keys are a structure separate    */
/* from the FP4 main cache). Score of token t:                          */
/*   S[t] = sum_h sum_d q[h,d] * k[t,h,d]   (exact integer)             */
/*   score[t] = fp32(S[t]) * scale[t]       (one fp32 multiply)         */
/* HD = heads * dims per head.                                          */
/* ------------------------------------------------------------------ */
void orc_index_dots(const int8_t *q, const int8_t *k, int64_t n, int HD, int64_t *S)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; t++) {
        int64_t acc = 0;
        for (int i = 0; i < HD; i++)
            acc += (int64_t)q[i] * (int64_t)k[t * HD + i];
        S[t] = acc;
    }
}

/* Returns 0, or -1 if some dot product leaves the int32 range. */
int orc_index_scores(const int8_t *q, const int8_t *k, const float *kscale, int64_t n, int HD,
                     float *score)
{
    int out_of_range = 0;
#pragma omp parallel for schedule(static) reduction(|| : out_of_range)
    for (int64_t t = 0; t < n; t++) {
        int64_t acc = 0;
        for (int i = 0; i < HD; i++)
            acc += (int64_t)q[i] * (int64_t)k[t * HD + i];
        if (acc > INT32_MAX || acc < INT32_MIN) {
            out_of_range = 1;
            continue;
        }
        float s = (float)acc; /* round to nearest even */
        score[t] = s * kscale[t];
    }
    return out_of_range ? -1 : 0;
}

/* Block score: max over the visible tokens of each 8-token block.
 * nblk = ceil(n_visible / 8); a last partial block only sees its visible
 * tokens. [G] indexer section: the pool is made of 8-token blocks.      */
void orc_block_max(const float *score, int64_t n_visible, float *blk)
{
    int64_t nblk = (n_visible + 7) / 8;
    for (int64_t j = 0; j < nblk; j++) {
        float m = score[8 * j];
        for (int64_t t = 8 * j + 1; t < 8 * j + 8 && t < n_visible; t++)
            if (score[t] > m)
                m = score[t];
        blk[j] = m;
    }
}

/* ------------------------------------------------------------------ */
/* Top-k by full sort. Candidates (score[i], pos[i]) are ordered by     */
/* score descending, then position ascending; the first min(k, n) are   */
/* taken and written in ascending position order, then -1 padding up to */
/* k entries. Returns the number of real entries.                       */
/* ------------------------------------------------------------------ */
typedef struct {
    float s;
    int64_t p;
} orc_cand;

static int orc_cmp_rank(const void *a, const void *b)
{
    const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    if (x->p < y->p) return -1;
    if (x->p > y->p) return 1;
    return 0;
}

static int orc_cmp_i64(const void *a, const void *b)
{
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x > y) - (x < y);
}

int64_t orc_topk(const float *score, const int64_t *pos, int64_t n, int64_t k, int64_t *out)
{
    orc_cand *c = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; i++) {
        c[i].s = score[i];
        c[i].p = pos[i];
    }
    qsort(c, (size_t)n, sizeof(orc_cand), orc_cmp_rank);
    int64_t m = n < k ? n : k;
    for (int64_t i = 0; i < m; i++)
        out[i] = c[i].p;
    qsort(out, (size_t)m, sizeof(int64_t), orc_cmp_i64);
    for (int64_t i = m; i < k; i++)
        out[i] = -1;
    free(c);
    return m;
}

/* ------------------------------------------------------------------ */
/* Softmax attention of one query's heads over n key rows ([T]          */
/* mechanism 4: attention runs only over the selected candidates; [N]   */
/* CED and CSA2 sections: every layer has its own main Q and SWA KV,     */
/* the window being the last 128 tokens). K and V are the same row.     */
/*   q   : Hq x C bf16 bit patterns                                     */
/*   kv  : n x C values (fp64)                                          */
/*   out : Hq x C, out[h] = sum_j softmax_j(scale * q[h].kv[j]) kv[j]     */
/* ------------------------------------------------------------------ */
void orc_attention(const uint16_t *q, int Hq, int C, const double *kv, int64_t n, double scale,
                   double *out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < Hq; h++) {
        if (n == 0) {
            /* no key: no softmax; the output is defined as zero */
            for (int c = 0; c < C; c++)
                out[h * C + c] = 0.0;
            continue;
        }
        double *logit = (double *)malloc(sizeof(double) * (size_t)n);
        double mx = -INFINITY;
        for (int64_t j = 0; j < n; j++) {
            double dot = 0.0;
            for (int c = 0; c < C; c++)
                dot += (double)bf16_to_float(q[h * C + c]) * kv[j * C + c];
            logit[j] = scale * dot;
            if (logit[j] > mx)
                mx = logit[j];
        }
        double z = 0.0;
        for (int64_t j = 0; j < n; j++) {
            logit[j] = exp(logit[j] - mx);
            z += logit[j];
        }
        for (int c = 0; c < C; c++) {
            double acc = 0.0;
            for (int64_t j = 0; j < n; j++)
                acc += logit[j] * kv[j * C + c];
            out[h * C + c] = acc / z;
        }
        free(logit);
    }
}
