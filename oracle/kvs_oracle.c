/*
 * kvs_oracle.c -- plain, slow, single-threaded CPU oracle for host-streamed
 * paged quantized KV attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library,
 * its Python binding) may include, link or call this file.  Only the tests,
 * the smoke check and the CPU-baseline leg of the benchmark use it.  It shares
 * no code, header, table or constant with the CUDA path.
 *
 * What it computes (sources are the three web pages on the subject):
 *  - the K cache is Q8_0 and the V cache is Q4_0, blocks of 32 values with an
 *    fp16 scale ("RaymondHuang210129/llama.cpp-adaptive-kv-streaming",
 *    Summary; "llama.cpp adaptive KV streaming - spec fork notes", Results);
 *    V may also be Q8_0 (the q8_0/q8_0 runs of PR #326) or another of the
 *    legal cache types of the flash-attention build ("llama.cpp adaptive KV
 *    streaming - spec fork notes", TLDR: -DGGML_CUDA_FA_QUANTS), each with its
 *    own block rule below;
 *  - the KV history is quantized once, when a token is appended, and attention
 *    is exact over every token of the history; streaming only changes where
 *    the bytes live ("Feature/adaptive kv stream integration", PR #326,
 *    section 1 "Correctness -- PPL parity, streaming on vs off");
 *  - residency: 256-token pages, the newest pages resident, the rest streamed
 *    in order; auto sizing = 10 % of the context per layer, 2048-token floor,
 *    8192 MiB ceiling (PR #326, commit list and "Diagnostic log").
 *
 * Floating point: quantization decisions are taken in IEEE binary32 (the
 * precision in which the block formats define their scale), the attention is
 * computed in binary64.  Compile with -ffp-contract=off and without
 * -ffast-math.
 *
 * Every function here is pinned by the CPU tests under tests/ against closed
 * forms, hand-worked examples and library routines (see test_oracle_*.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "kvs_oracle.h"

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 <-> binary32/binary64, written from the format's        */
/* definition: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.       */
/* ------------------------------------------------------------------------ */

double oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);              /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(f | 0x400), e - 25); /* (1024+f) * 2^(e-15-10) */
    }
    return sign ? -v : v;
}

float oracle_half_to_float(uint16_t h) {
    /* every binary16 value is exactly representable in binary32 */
    return (float)oracle_half_to_double(h);
}

static uint32_t float_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

uint16_t oracle_float_to_half(float f) {
    /* round to nearest, ties to even */
    uint32_t x = float_bits(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    int exp = (int)((x >> 23) & 0xff);
    uint32_t mant = x & 0x7fffffu;
    if (exp == 255) return (uint16_t)(sign | 0x7c00u | (mant ? 0x200u : 0u));
    if (exp == 0) return sign; /* binary32 zero/subnormal (< 2^-126) -> +-0 */
    int e = exp - 127 + 15;    /* binary16 biased exponent */
    if (e >= 31) return (uint16_t)(sign | 0x7c00u);
    if (e >= 1) {
        uint32_t hm = mant >> 13;
        uint32_t rem = mant & 0x1fffu;
        if (rem > 0x1000u || (rem == 0x1000u && (hm & 1u))) {
            hm += 1;
            if (hm == 0x400u) {
                hm = 0;
                e += 1;
                if (e == 31) return (uint16_t)(sign | 0x7c00u);
            }
        }
        return (uint16_t)(sign | ((uint32_t)e << 10) | hm);
    }
    /* binary16 subnormal range: value = m * 2^(exp-150), unit 2^-24, so the
     * count of units is m * 2^(exp-126) = m >> (126-exp). */
    uint32_t m = mant | 0x800000u;
    int s = 126 - exp; /* >= 14 */
    if (s > 25) return sign;
    uint32_t hm = m >> s;
    uint32_t rem = m & ((1u << s) - 1u);
    uint32_t halfway = 1u << (s - 1);
    if (rem > halfway || (rem == halfway && (hm & 1u))) hm += 1;
    return (uint16_t)(sign | hm); /* hm == 0x400 encodes the smallest normal */
}

/* ------------------------------------------------------------------------ */
/* Block quantization.  Canonical block byte layout (little endian):          */
/*   Q8_0: 2-byte fp16 scale d, then 32 signed bytes q      (34 bytes)        */
/*   Q4_0: 2-byte fp16 scale d, then 16 bytes, byte j holding q_j in its low  */
/*         nibble and q_{j+16} in its high nibble             (18 bytes)      */
/*   Q5_0: 2-byte fp16 scale d, a 4-byte word whose bit j is bit 4 of q_j,    */
/*         then 16 bytes holding the low 4 bits of q_j / q_{j+16} as Q4_0    */
/*         does                                               (22 bytes)      */
/*   Q4_1: fp16 d, fp16 m (the block minimum), then the 16 code bytes of      */
/*         Q4_0                                               (20 bytes)      */
/*   Q5_1: fp16 d, fp16 m, the fifth-bit word, then the 16 bytes of Q5_0      */
/*                                                            (24 bytes)      */
/* ------------------------------------------------------------------------ */

void oracle_q8_0_block(const uint16_t x_h[32], uint8_t out[34]) {
    float x[32];
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
        x[i] = oracle_half_to_float(x_h[i]);
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float d = amax / 127.0f; /* d = amax/127 in binary32 */
    uint16_t dh = oracle_float_to_half(d);
    out[0] = (uint8_t)(dh & 0xff);
    out[1] = (uint8_t)(dh >> 8);
    for (int i = 0; i < 32; ++i) {
        int q = 0;
        if (d != 0.0f) q = (int)roundf(x[i] / d); /* half away from zero */
        out[2 + i] = (uint8_t)(int8_t)q;
    }
}

void oracle_q4_0_block(const uint16_t x_h[32], uint8_t out[18]) {
    float x[32];
    float amax = 0.0f, m = 0.0f;
    for (int i = 0; i < 32; ++i) {
        x[i] = oracle_half_to_float(x_h[i]);
        float a = fabsf(x[i]);
        if (a > amax) { /* strict: the first index of the largest |x| wins */
            amax = a;
            m = x[i];
        }
    }
    float d = m / -8.0f; /* signed max over -8 */
    uint16_t dh = oracle_float_to_half(d);
    out[0] = (uint8_t)(dh & 0xff);
    out[1] = (uint8_t)(dh >> 8);
    int q[32];
    for (int i = 0; i < 32; ++i) {
        if (d == 0.0f) {
            q[i] = 8;
        } else {
            int t = (int)(x[i] / d + 8.5f); /* argument >= 0.5: truncation */
            q[i] = t < 15 ? t : 15;
        }
    }
    for (int j = 0; j < 16; ++j) out[2 + j] = (uint8_t)(q[j] | (q[j + 16] << 4));
}

/* Q5_0: the 5-bit member of the same family, one of the cache types the
 * flash-attention build lists as legal ("llama.cpp adaptive KV streaming -
 * spec fork notes", TLDR: -DGGML_CUDA_FA_QUANTS).  The pages
 * give no rule; it is read as Q4_0's with 32 levels: d = (signed max)/-16,
 * q = min(31, trunc(x/d + 16.5)), so x ~ d (q - 16). */
void oracle_q5_0_block(const uint16_t x_h[32], uint8_t out[22]) {
    float x[32];
    float amax = 0.0f, m = 0.0f;
    for (int i = 0; i < 32; ++i) {
        x[i] = oracle_half_to_float(x_h[i]);
        float a = fabsf(x[i]);
        if (a > amax) { /* the first index of the largest |x| wins (strict) */
            amax = a;
            m = x[i];
        }
    }
    float d = m / -16.0f; /* signed max over -16 */
    uint16_t dh = oracle_float_to_half(d);
    out[0] = (uint8_t)(dh & 0xff);
    out[1] = (uint8_t)(dh >> 8);
    int q[32];
    for (int i = 0; i < 32; ++i) {
        if (d == 0.0f) {
            q[i] = 16;
        } else {
            int t = (int)(x[i] / d + 16.5f); /* argument >= 0.5: truncation */
            q[i] = t < 31 ? t : 31;
        }
    }
    uint32_t high = 0;
    for (int i = 0; i < 32; ++i) high |= (uint32_t)(q[i] >> 4) << i;
    for (int b = 0; b < 4; ++b) out[2 + b] = (uint8_t)(high >> (8 * b));
    for (int j = 0; j < 16; ++j) out[6 + j] = (uint8_t)((q[j] & 15) | ((q[j + 16] & 15) << 4));
}

/* Q4_1 / Q5_1: the asymmetric members of the family, also among the legal
 * cache types of the flash-attention build (same page and section as Q5_0).
 * The pages give no rule; it is read as the block's range split into 15 (31)
 * steps from its minimum: d = (max - min)/levels, q = min(levels,
 * trunc((x - min)/d + 0.5)), q = 0 when d = 0, so x ~ d q + min. */
static void min_block(const uint16_t x_h[32], int levels, uint16_t* dh, uint16_t* mh, int q[32]) {
    float x[32];
    float lo = 0.0f, hi = 0.0f;
    for (int i = 0; i < 32; ++i) {
        x[i] = oracle_half_to_float(x_h[i]);
        if (i == 0 || x[i] < lo) lo = x[i];
        if (i == 0 || x[i] > hi) hi = x[i];
    }
    float d = (hi - lo) / (float)levels; /* binary32 difference, then division */
    *dh = oracle_float_to_half(d);
    *mh = oracle_float_to_half(lo);
    for (int i = 0; i < 32; ++i) {
        if (d == 0.0f) {
            q[i] = 0;
        } else {
            int t = (int)((x[i] - lo) / d + 0.5f); /* argument >= 0.5: truncation */
            q[i] = t < levels ? t : levels;
        }
    }
}

void oracle_q4_1_block(const uint16_t x_h[32], uint8_t out[20]) {
    uint16_t dh, mh;
    int q[32];
    min_block(x_h, 15, &dh, &mh, q);
    out[0] = (uint8_t)(dh & 0xff);
    out[1] = (uint8_t)(dh >> 8);
    out[2] = (uint8_t)(mh & 0xff);
    out[3] = (uint8_t)(mh >> 8);
    for (int j = 0; j < 16; ++j) out[4 + j] = (uint8_t)(q[j] | (q[j + 16] << 4));
}

void oracle_q5_1_block(const uint16_t x_h[32], uint8_t out[24]) {
    uint16_t dh, mh;
    int q[32];
    min_block(x_h, 31, &dh, &mh, q);
    out[0] = (uint8_t)(dh & 0xff);
    out[1] = (uint8_t)(dh >> 8);
    out[2] = (uint8_t)(mh & 0xff);
    out[3] = (uint8_t)(mh >> 8);
    uint32_t top = 0;
    for (int i = 0; i < 32; ++i) top |= (uint32_t)(q[i] >> 4) << i;
    for (int b = 0; b < 4; ++b) out[4 + b] = (uint8_t)(top >> (8 * b));
    for (int j = 0; j < 16; ++j) out[8 + j] = (uint8_t)((q[j] & 15) | ((q[j + 16] & 15) << 4));
}

void oracle_dequant_q8_0(const uint8_t blk[34], double out[32]) {
    double d = oracle_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    for (int i = 0; i < 32; ++i) out[i] = d * (double)(int8_t)blk[2 + i];
}

void oracle_dequant_q4_0(const uint8_t blk[18], double out[32]) {
    double d = oracle_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    for (int j = 0; j < 16; ++j) {
        out[j] = d * (double)((int)(blk[2 + j] & 0x0f) - 8);
        out[j + 16] = d * (double)((int)(blk[2 + j] >> 4) - 8);
    }
}

void oracle_dequant_q5_0(const uint8_t blk[22], double out[32]) {
    double d = oracle_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    uint32_t high = (uint32_t)blk[2] | ((uint32_t)blk[3] << 8) | ((uint32_t)blk[4] << 16) | ((uint32_t)blk[5] << 24);
    for (int j = 0; j < 16; ++j) {
        int lo = (int)(blk[6 + j] & 0x0f) | (int)(((high >> j) & 1u) << 4);
        int hi = (int)(blk[6 + j] >> 4) | (int)(((high >> (j + 16)) & 1u) << 4);
        out[j] = d * (double)(lo - 16);
        out[j + 16] = d * (double)(hi - 16);
    }
}

void oracle_dequant_q4_1(const uint8_t blk[20], double out[32]) {
    double d = oracle_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    double m = oracle_half_to_double((uint16_t)(blk[2] | (blk[3] << 8)));
    for (int j = 0; j < 16; ++j) {
        out[j] = d * (double)(blk[4 + j] & 0x0f) + m;
        out[j + 16] = d * (double)(blk[4 + j] >> 4) + m;
    }
}

void oracle_dequant_q5_1(const uint8_t blk[24], double out[32]) {
    double d = oracle_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    double m = oracle_half_to_double((uint16_t)(blk[2] | (blk[3] << 8)));
    uint32_t top = (uint32_t)blk[4] | ((uint32_t)blk[5] << 8) | ((uint32_t)blk[6] << 16) | ((uint32_t)blk[7] << 24);
    for (int j = 0; j < 16; ++j) {
        int a = (int)(blk[8 + j] & 0x0f) | (int)(((top >> j) & 1u) << 4);
        int b = (int)(blk[8 + j] >> 4) | (int)(((top >> (j + 16)) & 1u) << 4);
        out[j] = d * (double)a + m;
        out[j + 16] = d * (double)b + m;
    }
}

/* F16 V: the values themselves, 32 fp16 per block (64 bytes, little endian);
 * f16 is a legal cache type of the same build list.  Nothing is rounded. */
static void f16_block(const uint16_t x_h[32], uint8_t out[64]) {
    for (int i = 0; i < 32; ++i) {
        out[2 * i] = (uint8_t)(x_h[i] & 0xff);
        out[2 * i + 1] = (uint8_t)(x_h[i] >> 8);
    }
}

static void f16_dequant(const uint8_t blk[64], double out[32]) {
    for (int i = 0; i < 32; ++i) out[i] = oracle_half_to_double((uint16_t)(blk[2 * i] | (blk[2 * i + 1] << 8)));
}

/* bytes of one 32-value block of a V type (1 = F16, 2 = Q4_0, 3 = Q4_1,
 * 6 = Q5_0, 7 = Q5_1, 8 = Q8_0), 0 if unknown */
static int v_block_bytes(int v_type) {
    switch (v_type) {
        case 1: return 64;
        case 2: return 18;
        case 3: return 20;
        case 6: return 22;
        case 7: return 24;
        case 8: return 34;
        default: return 0;
    }
}

static void v_block(int v_type, const uint16_t* x, uint8_t* out) {
    if (v_type == 1) f16_block(x, out);
    else if (v_type == 2) oracle_q4_0_block(x, out);
    else if (v_type == 3) oracle_q4_1_block(x, out);
    else if (v_type == 6) oracle_q5_0_block(x, out);
    else if (v_type == 7) oracle_q5_1_block(x, out);
    else oracle_q8_0_block(x, out);
}

static void v_dequant(int v_type, const uint8_t* blk, double* out) {
    if (v_type == 1) f16_dequant(blk, out);
    else if (v_type == 2) oracle_dequant_q4_0(blk, out);
    else if (v_type == 3) oracle_dequant_q4_1(blk, out);
    else if (v_type == 6) oracle_dequant_q5_0(blk, out);
    else if (v_type == 7) oracle_dequant_q5_1(blk, out);
    else oracle_dequant_q8_0(blk, out);
}

/* K types: Q8_0 (8, 34-byte blocks) or F16 (1, the 64-byte blocks of the
 * values; "f16-f16 is always compiled" in the flash-attention build of "llama.cpp
 * adaptive KV streaming - spec fork notes", TLDR) */
static int k_block_bytes(int k_type) {
    return k_type == 8 ? 34 : (k_type == 1 ? 64 : 0);
}

/* K rows -> blocks of the K type; V rows -> blocks of the V type (1 F16,
 * 2 Q4_0, 3 Q4_1, 6 Q5_0, 7 Q5_1, 8 Q8_0) */
int oracle_quantize_rows_kv(int n_rows, int dim, const uint16_t* k, const uint16_t* v,
                            uint8_t* k_blocks, uint8_t* v_blocks, int k_type, int v_type) {
    int nb = dim / 32;
    int kbb = k_block_bytes(k_type);
    int vbb = v_block_bytes(v_type);
    if (!vbb || !kbb) return -1;
    for (int r = 0; r < n_rows; ++r) {
        for (int b = 0; b < nb; ++b) {
            const uint16_t* kx = k + (size_t)r * dim + (size_t)b * 32;
            const uint16_t* vx = v + (size_t)r * dim + (size_t)b * 32;
            if (k_type == 8) oracle_q8_0_block(kx, k_blocks + ((size_t)r * nb + b) * kbb);
            else f16_block(kx, k_blocks + ((size_t)r * nb + b) * kbb);
            v_block(v_type, vx, v_blocks + ((size_t)r * nb + b) * vbb);
        }
    }
    return 0;
}

int oracle_quantize_rows_t(int n_rows, int dim, const uint16_t* k, const uint16_t* v,
                           uint8_t* k_blocks, uint8_t* v_blocks, int v_type) {
    return oracle_quantize_rows_kv(n_rows, dim, k, v, k_blocks, v_blocks, 8, v_type);
}

void oracle_quantize_rows(int n_rows, int dim, const uint16_t* k, const uint16_t* v,
                          uint8_t* k_blocks, uint8_t* v_blocks) {
    oracle_quantize_rows_t(n_rows, dim, k, v, k_blocks, v_blocks, 2);
}

/* ------------------------------------------------------------------------ */
/* Attention over the quantized history, binary64.                            */
/*                                                                            */
/* k_blocks: [n_keys][n_kv][dim/32] Q8_0 blocks (token-major history)         */
/* v_blocks: [n_keys][n_kv][dim/32] blocks of the V type (v_block_bytes)     */
/* q:        [n_q][n_qh][dim] fp16; query j sits at absolute position pos0+j  */
/*           and sees keys 0..pos0+j (causal).                                */
/* q head h reads kv head h / (n_qh/n_kv) (contiguous grouping).              */
/* out:      [n_q][n_qh][dim] ; lse: [n_q][n_qh] natural log of the sum of    */
/*           exp(scaled logits).                                              */
/* ------------------------------------------------------------------------ */

int oracle_attention_kv(int n_kv, int n_qh, int dim, const uint8_t* k_blocks,
                        const uint8_t* v_blocks, int n_q, int pos0, const uint16_t* q,
                        double* out, double* lse, int k_type, int v_type) {
    int vbb = v_block_bytes(v_type);
    int kbb = k_block_bytes(k_type);
    if (n_kv <= 0 || n_qh % n_kv != 0 || dim % 32 != 0 || n_q <= 0 || pos0 < 0 || !vbb || !kbb) return -1;
    int group = n_qh / n_kv;
    int nb = dim / 32;
    int max_keys = pos0 + n_q;
    double scale = 1.0 / sqrt((double)dim);
    double* s = (double*)malloc(sizeof(double) * (size_t)max_keys);
    double* qd = (double*)malloc(sizeof(double) * (size_t)dim);
    double* kd = (double*)malloc(sizeof(double) * 32);
    double* vd = (double*)malloc(sizeof(double) * 32);
    if (!s || !qd || !kd || !vd) {
        free(s); free(qd); free(kd); free(vd);
        return -2;
    }
    for (int j = 0; j < n_q; ++j) {
        int n_keys = pos0 + j + 1;
        for (int h = 0; h < n_qh; ++h) {
            int g = h / group;
            const uint16_t* qh = q + ((size_t)j * n_qh + h) * dim;
            for (int d = 0; d < dim; ++d) qd[d] = oracle_half_to_double(qh[d]);
            /* scores */
            double m = -INFINITY;
            for (int i = 0; i < n_keys; ++i) {
                double acc = 0.0;
                for (int b = 0; b < nb; ++b) {
                    const uint8_t* kblk = k_blocks + (((size_t)i * n_kv + g) * nb + b) * kbb;
                    if (k_type == 8) oracle_dequant_q8_0(kblk, kd);
                    else f16_dequant(kblk, kd);
                    for (int t = 0; t < 32; ++t) acc += qd[b * 32 + t] * kd[t];
                }
                s[i] = acc * scale;
                if (s[i] > m) m = s[i];
            }
            /* softmax-weighted sum of values */
            double* o = out + ((size_t)j * n_qh + h) * dim;
            for (int d = 0; d < dim; ++d) o[d] = 0.0;
            double sum = 0.0;
            for (int i = 0; i < n_keys; ++i) {
                double p = exp(s[i] - m);
                sum += p;
                for (int b = 0; b < nb; ++b) {
                    const uint8_t* vblk = v_blocks + (((size_t)i * n_kv + g) * nb + b) * vbb;
                    v_dequant(v_type, vblk, vd);
                    for (int t = 0; t < 32; ++t) o[b * 32 + t] += p * vd[t];
                }
            }
            for (int d = 0; d < dim; ++d) o[d] /= sum;
            lse[(size_t)j * n_qh + h] = m + log(sum);
        }
    }
    free(s); free(qd); free(kd); free(vd);
    return 0;
}

int oracle_attention_t(int n_kv, int n_qh, int dim, const uint8_t* k_blocks,
                       const uint8_t* v_blocks, int n_q, int pos0, const uint16_t* q,
                       double* out, double* lse, int v_type) {
    return oracle_attention_kv(n_kv, n_qh, dim, k_blocks, v_blocks, n_q, pos0, q, out, lse, 8, v_type);
}

int oracle_attention(int n_kv, int n_qh, int dim, const uint8_t* k_blocks,
                     const uint8_t* v_blocks, int n_q, int pos0, const uint16_t* q,
                     double* out, double* lse) {
    return oracle_attention_t(n_kv, n_qh, dim, k_blocks, v_blocks, n_q, pos0, q, out, lse, 2);
}

/* ------------------------------------------------------------------------ */
/* Page policy.                                                               */
/* ------------------------------------------------------------------------ */

long oracle_pages_for(long n_tokens, int page_tokens) {
    return (n_tokens + page_tokens - 1) / page_tokens;
}

/* "--kv-stream auto": 10 % of the context resident per layer rounded up to a
 * whole page, a 2048-token floor, then an 8192 MiB ceiling on the resident
 * bytes of all layers (PR #326 commit list; "Diagnostic log" shows 65536 ->
 * 6656 tokens and the 262144-token run shows 26368 tokens). */
long oracle_auto_resident_pages(long max_ctx, int page_tokens, long page_bytes, int n_layers) {
    long tenth_tokens_x10 = max_ctx; /* 10 % of max_ctx, kept as max_ctx/10 */
    long pages = (tenth_tokens_x10 + 10L * page_tokens - 1) / (10L * page_tokens);
    long floor_pages = (2048 + page_tokens - 1) / page_tokens;
    if (pages < floor_pages) pages = floor_pages;
    long ceiling_bytes = 8192L * 1024L * 1024L;
    long cap = ceiling_bytes / (page_bytes * (long)n_layers);
    if (pages > cap) pages = cap;
    if (pages < 1) pages = 1;
    return pages;
}

/* Location of page `page` of a layer holding n_tokens tokens with R resident
 * page slots: the R most recent pages are resident (slot = page mod R), the
 * older ones stream in ascending page order (ordinal = page). */
int oracle_page_location(long n_tokens, int page_tokens, long n_resident, long page,
                         int* kind, long* index) {
    long P = oracle_pages_for(n_tokens, page_tokens);
    if (page < 0 || page >= P) {
        *kind = ORACLE_PAGE_ABSENT;
        *index = -1;
        return -1;
    }
    if (page >= P - n_resident) {
        *kind = ORACLE_PAGE_RESIDENT;
        *index = page % n_resident;
    } else {
        *kind = ORACLE_PAGE_STREAMED;
        *index = page;
    }
    return 0;
}
