/*
 * q4_oracle.c -- CPU oracle for group-wise INT4 weight quantization and the
 * W4A16 matrix-vector product.  TEST INFRASTRUCTURE ONLY: nothing on the
 * product path may link, load or call this file.  Only tests/, the smoke
 * check in __graft_entry__.py and the cpu_baseline / reference legs of
 * bench.py use it.
 *
 * Plain, single-threaded C11.  No CUDA headers, no code shared with the GPU
 * library.  Compiled without -ffast-math and with -ffp-contract=off so that
 * every fp32 operation below is one IEEE-754 binary32 operation rounded to
 * nearest-even, exactly as written.
 *
 * What it computes, and where the pages define it:
 *
 *  - the affine quantizer  q = clamp(round(w/s) + z, qmin, qmax),
 *    dequant  w_hat = s * (q - z)
 *      "LLM 后训练量化深度实战" (ybb.press), section 二, first equation;
 *      arganzheng.life post-training-quantization-gptq-awq-and-rotation,
 *      section 二.2 (基本形式与粒度), first equation;
 *      "量化：PTQ、GPTQ、AWQ 与 SmoothQuant" (charles2530.github.io),
 *      section 1 (量化的统一形式).
 *  - symmetric scale s = max|w| / (2^(b-1) - 1) = amax / 7 with z = 0, and
 *    asymmetric scale s = (max - min) / (2^b - 1) = (max - min) / 15 with an
 *    integer zero-point z: arganzheng.life, section 二.2.
 *  - group-wise granularity along in_features, symmetric INT4 range [-8, 7]:
 *    ybb.press, section 二, function quantize_per_group;
 *    charles2530.github.io, section 1 (q in {-8..7}).
 *  - zero-point as the integer code of real 0, z = round(-min / s):
 *    arganzheng.life section 二.2 (z is added on the integer side);
 *    "压缩算法" (cs-knowledge-wiki), section 7.4.1.1 (INT8 asymmetric form).
 *  - two 4-bit codes per byte: "压缩算法" section 7.4.1.2 (pack_int4).
 *  - the decode product y = x W^T of the dequantised weights:
 *    arganzheng.life section 二.1 ([B,k] x [k,n] decode GEMM) and 二.3.
 *  - per-output-channel INT8 weights, s = max(amax, 1e-6) / 127, codes in
 *    [-127, 127]: charles2530.github.io, section 13 (快速代码示例).
 *  - INT8 KV cache, one scale per token row of head_dim values, codes in
 *    [-128, 127], and its dequantization: "压缩算法" section 7.4.1.1.
 *  - E2M1, E4M3, MXFP4 (E8M0 scale per 32, the OCP rule) and NVFP4 (E4M3
 *    scale per 16 and an fp32 tensor scale): arganzheng.life sections 九.1
 *    and 九.2 (the scale choices and E2M1 rounding are readings, stated with
 *    the functions below).
 *
 * Readings taken where the pages leave a step open:
 *  - the scale is computed in fp32 (IEEE division), stored as fp16, and the
 *    STORED fp16 scale is the one that quantizes and dequantizes;
 *  - round() is round-half-to-even (torch.round in the ybb.press code);
 *  - a group whose stored scale is 0 gets all codes 0 (sym) / z = 0 (asym);
 *  - asymmetric: z = clamp(rne(-min / s), 0, 15), stored as an fp16 integer;
 *    codes are clamp(rne(w / s) + z, 0, 15);
 *  - packing: element 2j in the low nibble of byte j, element 2j+1 in the
 *    high nibble; symmetric codes stored as two's complement (q & 0xF).
 *
 * fp16 and bf16 codecs are written from the IEEE-754 binary16 definition and
 * from bfloat16 = the upper 16 bits of binary32 (round to nearest even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------ codecs */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
ORACLE_API float oracle_f16_to_f32(uint16_t h) {
    uint32_t sign = (uint32_t)(h >> 15) & 1u;
    uint32_t exp = (uint32_t)(h >> 10) & 0x1Fu;
    uint32_t frac = (uint32_t)h & 0x3FFu;
    float mag;
    if (exp == 0x1F) {
        mag = frac ? NAN : INFINITY;
    } else if (exp == 0) {
        mag = ldexpf((float)frac, -24);            /* subnormal: frac * 2^-24 */
    } else {
        mag = ldexpf((float)(frac | 0x400u), (int)exp - 25); /* 1.f * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

/* Round a binary32 value to the nearest binary16 value, ties to even.
 * Works on the exact value: v = m * 2^e with a 24-bit integer m. */
ORACLE_API uint16_t oracle_f32_to_f16(float f) {
    uint32_t u = f32_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t exp = (u >> 23) & 0xFFu;
    uint32_t frac = u & 0x7FFFFFu;
    if (exp == 0xFF) return (uint16_t)(sign | 0x7C00u | (frac ? 0x200u : 0u));
    if (exp == 0 && frac == 0) return sign;
    /* exact value = mant * 2^(e2) with mant < 2^24 */
    uint32_t mant = exp ? (frac | 0x800000u) : frac;
    int e2 = exp ? (int)exp - 150 : -149;
    /* binary16 quantum for this magnitude: representable values are
     * k * 2^q with q = max(unbiased_exp - 10, -24), unbiased exponent of the
     * result computed from the leading bit of mant. */
    int lead = 31 - __builtin_clz(mant);          /* position of leading 1 */
    int unb = lead + e2;                          /* floor(log2 |v|) */
    int q = unb - 10;
    if (q < -24) q = -24;
    int shift = q - e2;                           /* bits to drop from mant */
    uint64_t k;
    if (shift <= 0) {
        k = (uint64_t)mant << (-shift);
    } else if (shift > 40) {
        k = 0;
    } else {
        uint64_t m = mant;
        uint64_t kq = m >> shift;
        uint64_t rem = m - (kq << shift);
        uint64_t half = 1ull << (shift - 1);
        if (rem > half || (rem == half && (kq & 1ull))) kq += 1;
        k = kq;
    }
    /* value = k * 2^q; encode */
    if (k == 0) return sign;
    /* k may have overflowed into 2^11 after rounding: renormalise */
    while (k >= 2048) { k >>= 1; q += 1; }    /* k even here, exact */
    if (q == -24 && k < 1024) return (uint16_t)(sign | (uint16_t)k); /* subnormal */
    /* normal: k in [1024, 2047], value = k * 2^q = 1.f * 2^(q+10) */
    int be = q + 10 + 15;
    if (be >= 31) return (uint16_t)(sign | 0x7C00u);  /* overflow -> inf */
    return (uint16_t)(sign | (uint16_t)(be << 10) | (uint16_t)(k - 1024));
}

ORACLE_API float oracle_bf16_to_f32(uint16_t b) { return bits_f32((uint32_t)b << 16); }

ORACLE_API uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u = f32_bits(f);
    if (((u >> 23) & 0xFFu) == 0xFFu && (u & 0x7FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lower = u & 0xFFFFu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1; /* may carry into inf: correct */
    return (uint16_t)upper;
}

/* array forms of the codecs (n elements) */
ORACLE_API void oracle_f16_to_f32_n(const uint16_t* h, float* f, int64_t n) {
    for (int64_t i = 0; i < n; ++i) f[i] = oracle_f16_to_f32(h[i]);
}
ORACLE_API void oracle_f32_to_f16_n(const float* f, uint16_t* h, int64_t n) {
    for (int64_t i = 0; i < n; ++i) h[i] = oracle_f32_to_f16(f[i]);
}
ORACLE_API void oracle_bf16_to_f32_n(const uint16_t* b, float* f, int64_t n) {
    for (int64_t i = 0; i < n; ++i) f[i] = oracle_bf16_to_f32(b[i]);
}
ORACLE_API void oracle_f32_to_bf16_n(const float* f, uint16_t* b, int64_t n) {
    for (int64_t i = 0; i < n; ++i) b[i] = oracle_f32_to_bf16(f[i]);
}

/* ---------------------------------------------------------------- rounding */

/* round half to even of a binary32 value (default IEEE rounding mode). */
static float rne(float v) { return nearbyintf(v); }

/* q = clamp(rne(w / s) + z, qmin, qmax): the affine quantizer of one value
 * with an externally supplied fp32 scale (the worked rounding and clipping
 * examples of "模型量化技术工程实践" (iopencloud.com), section 1.2, use it). */
ORACLE_API int32_t oracle_quantize_value(float w, float s, int32_t z, int32_t qmin, int32_t qmax) {
    float t = rne(w / s);                       /* IEEE fp32 division, RN */
    /* add z and clamp in float, where t is an exact integer-valued float */
    float v = t + (float)z;
    if (!(v >= (float)qmin)) v = (float)qmin;   /* also maps NaN to qmin */
    if (v > (float)qmax) v = (float)qmax;
    return (int32_t)v;
}

/* -------------------------------------------------------------- quantizer */

/*
 * Group-wise INT4 round-to-nearest quantization and packing.
 *   W        [out, in] fp32 values (the exact values of the fp16/bf16 input)
 *   qweight  [out, in/2] bytes, element 2j low nibble, 2j+1 high nibble
 *   scales   [out, in/g] fp16 bit patterns
 *   zeros    [out, in/g] fp16 bit patterns (integer-valued), NULL iff symmetric
 * Returns 0, or -1 on bad arguments (g not dividing in, g or in odd).
 */
ORACLE_API int oracle_quantize_pack(const float* W, int64_t out, int64_t in, int32_t g,
                                    int32_t symmetric, uint8_t* qweight, uint16_t* scales,
                                    uint16_t* zeros) {
    if (g <= 0 || in <= 0 || out < 0 || (in % g) != 0 || (g % 2) != 0) return -1;
    if (!symmetric && zeros == NULL) return -1;
    const int64_t G = in / g;
    int32_t* codes = (int32_t*)malloc(sizeof(int32_t) * (size_t)g);
    if (!codes) return -1;
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t j = 0; j < G; ++j) {
            const float* w = W + r * in + j * g;
            uint16_t s16;
            float sf;
            int32_t z = 0;
            if (symmetric) {
                /* a = max |w| over the group; s = a / 7 (2^(b-1) - 1 = 7) */
                float a = 0.0f;
                for (int32_t k = 0; k < g; ++k) {
                    float m = fabsf(w[k]);
                    if (m > a) a = m;
                }
                float s32 = a / 7.0f;
                s16 = oracle_f32_to_f16(s32);
                sf = oracle_f16_to_f32(s16);
                for (int32_t k = 0; k < g; ++k)
                    codes[k] = (sf == 0.0f) ? 0 : oracle_quantize_value(w[k], sf, 0, -8, 7);
            } else {
                /* s = (max - min) / 15, z = clamp(rne(-min / s), 0, 15) */
                float mn = w[0], mx = w[0];
                for (int32_t k = 1; k < g; ++k) {
                    if (w[k] < mn) mn = w[k];
                    if (w[k] > mx) mx = w[k];
                }
                float s32 = (mx - mn) / 15.0f;
                s16 = oracle_f32_to_f16(s32);
                sf = oracle_f16_to_f32(s16);
                if (sf == 0.0f) {
                    z = 0;
                    for (int32_t k = 0; k < g; ++k) codes[k] = 0;
                } else {
                    z = oracle_quantize_value(-mn, sf, 0, 0, 15);
                    for (int32_t k = 0; k < g; ++k)
                        codes[k] = oracle_quantize_value(w[k], sf, z, 0, 15);
                }
                zeros[r * G + j] = oracle_f32_to_f16((float)z);
            }
            scales[r * G + j] = s16;
            /* pack: two codes per byte, even element in the low nibble */
            uint8_t* dst = qweight + r * (in / 2) + j * (g / 2);
            for (int32_t k = 0; k < g; k += 2) {
                uint8_t lo = (uint8_t)(codes[k] & 0xF);
                uint8_t hi = (uint8_t)(codes[k + 1] & 0xF);
                dst[k / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    free(codes);
    return 0;
}

/*
 * Act-order quantization ("post-training-quantization-gptq-awq-and-rotation"
 * (arganzheng.life) section 五.3: desc_act quantizes the columns in the
 * order of decreasing input-channel variance, and the kernels then need a
 * reorder index g_idx; section 九.2: that reorder is a gather).  The columns
 * are taken in the order perm[0], perm[1], ...: groups are g consecutive
 * positions of that order and the codes and scales are stored in it, so
 *   packed column j  <->  original column perm[j],   g_idx[perm[j]] = j / g.
 * This is oracle_quantize_pack applied to the column-permuted matrix.
 */
ORACLE_API int oracle_quantize_pack_perm(const float* W, int64_t out, int64_t in, int32_t g,
                                         int32_t symmetric, const int32_t* perm, uint8_t* qweight,
                                         uint16_t* scales, uint16_t* zeros) {
    if (in <= 0 || out < 0) return -1;
    for (int64_t j = 0; j < in; ++j)
        if (perm[j] < 0 || perm[j] >= in) return -1;
    float* Wp = (float*)malloc(sizeof(float) * (size_t)(out > 0 ? out : 1) * (size_t)in);
    if (!Wp) return -1;
    for (int64_t r = 0; r < out; ++r)
        for (int64_t j = 0; j < in; ++j) Wp[r * in + j] = W[r * in + perm[j]];
    const int rc = oracle_quantize_pack(Wp, out, in, g, symmetric, qweight, scales, zeros);
    free(Wp);
    return rc;
}

/*
 * Range (clipping) search of symmetric INT4 group quantization
 * ("post-training-quantization-gptq-awq-and-rotation" (arganzheng.life),
 * section 三.2, 裁剪与舍入的权衡: scan a set of ranges alpha between 0.8 and
 * 1.0 of max|w| and keep the one with the smallest error).  Readings:
 *  - candidates alpha_j = amax (K - j) / K, j = 0 .. n-1, K = 5 (n - 1)
 *    (alpha_0 = amax, alpha_{n-1} = 0.8 amax; n = 1: amax only);
 *  - s_j = fp16(fp32(amax (K - j)) / fp32(7 K)) with IEEE division; the
 *    product and 7 K are exact in fp32, so s_0 is bit-for-bit the RTN scale;
 *  - codes q = clamp(rne(w / s_j), -7, 7): the section's symmetric grid of
 *    2^b - 1 points (RTN's -8 is unreachable at alpha = amax, so j = 0
 *    reproduces RTN's codes);
 *  - error E_j = sum over the group of (w - s_j q)^2 in fp64; a candidate
 *    whose fp16 scale is 0 is skipped unless it is the first;
 *  - j replaces the best so far only if E_j < E_best (1 - 1e-12), so ties
 *    keep the wider range.
 * Fills the group's E_j (and fp16 scale bits) for j < n; returns the index.
 */
ORACLE_API int32_t oracle_clip_search_group(const float* w, int32_t g, int32_t n,
                                            double* err, uint16_t* s16_out) {
    float a = 0.0f;
    for (int32_t k = 0; k < g; ++k) {
        float m = fabsf(w[k]);
        if (m > a) a = m;
    }
    const int32_t K = 5 * (n - 1);
    int32_t best = 0;
    double best_e = 0.0;
    for (int32_t j = 0; j < n; ++j) {
        const float num = (n == 1) ? a : a * (float)(K - j);
        const float den = (n == 1) ? 7.0f : 7.0f * (float)K;
        const uint16_t s16 = oracle_f32_to_f16(num / den);
        const float sf = oracle_f16_to_f32(s16);
        double e = 0.0;
        for (int32_t k = 0; k < g; ++k) {
            const int32_t q = (sf == 0.0f) ? 0 : oracle_quantize_value(w[k], sf, 0, -7, 7);
            const double d = (double)w[k] - (double)sf * (double)q;
            e += d * d;
        }
        if (err) err[j] = e;
        if (s16_out) s16_out[j] = s16;
        if (j == 0) {
            best_e = e;
        } else if (sf != 0.0f && e < best_e * (1.0 - 1e-12)) {
            best = j;
            best_e = e;
        }
    }
    return best;
}

/* Symmetric INT4 quantization with the range search above, packed like
 * oracle_quantize_pack; alpha_idx (may be NULL) receives each group's j. */
ORACLE_API int oracle_quantize_pack_clip(const float* W, int64_t out, int64_t in, int32_t g,
                                         int32_t n, uint8_t* qweight, uint16_t* scales,
                                         int32_t* alpha_idx) {
    if (g <= 0 || in <= 0 || out < 0 || (in % g) != 0 || (g % 2) != 0 || n < 1 || n > 64)
        return -1;
    const int64_t G = in / g;
    uint16_t* s16 = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)n);
    if (!s16) return -1;
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t j = 0; j < G; ++j) {
            const float* w = W + r * in + j * g;
            const int32_t best = oracle_clip_search_group(w, g, n, NULL, s16);
            const float sf = oracle_f16_to_f32(s16[best]);
            scales[r * G + j] = s16[best];
            if (alpha_idx) alpha_idx[r * G + j] = best;
            uint8_t* dst = qweight + r * (in / 2) + j * (g / 2);
            for (int32_t k = 0; k < g; k += 2) {
                const int32_t q0 = (sf == 0.0f) ? 0 : oracle_quantize_value(w[k], sf, 0, -7, 7);
                const int32_t q1 = (sf == 0.0f) ? 0 : oracle_quantize_value(w[k + 1], sf, 0, -7, 7);
                dst[k / 2] = (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
            }
        }
    }
    free(s16);
    return 0;
}

/* Unpack one code: low nibble for even k, high for odd k; symmetric codes are
 * two's complement 4-bit integers, asymmetric codes are unsigned. */
ORACLE_API int32_t oracle_code_at(const uint8_t* qweight, int64_t in, int64_t r, int64_t k,
                                  int32_t symmetric) {
    uint8_t b = qweight[r * (in / 2) + k / 2];
    int32_t n = (k & 1) ? (b >> 4) : (b & 0xF);
    if (symmetric && n >= 8) n -= 16;
    return n;
}

/*
 * Dequantisation w_hat = s * (q - z), in fp32.  The product of an fp16 scale
 * (11 significant bits) and an integer of magnitude <= 15 is exact in fp32.
 * W_hat [out, in] fp32.
 */
ORACLE_API int oracle_dequant_f32(const uint8_t* qweight, const uint16_t* scales,
                                  const uint16_t* zeros, int64_t out, int64_t in, int32_t g,
                                  int32_t symmetric, float* W_hat) {
    if (g <= 0 || (in % g) != 0 || (g % 2) != 0) return -1;
    if (!symmetric && zeros == NULL) return -1;
    const int64_t G = in / g;
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t k = 0; k < in; ++k) {
            int64_t j = k / g;
            float sf = oracle_f16_to_f32(scales[r * G + j]);
            int32_t z = symmetric ? 0 : (int32_t)oracle_f16_to_f32(zeros[r * G + j]);
            int32_t q = oracle_code_at(qweight, in, r, k, symmetric);
            W_hat[r * in + k] = sf * (float)(q - z);
        }
    }
    return 0;
}

/*
 * y[b, i] = sum_k w_hat[rows[i], k] * x[b, k] in fp64, for a list of rows.
 *   x [B, in] fp64 (exact values of the bf16/fp16 activations)
 *   y [B, nrows] fp64
 * The dequantised weights are exact in fp64; only the summation rounds.
 */
ORACLE_API int oracle_gemv_rows_f64(const uint8_t* qweight, const uint16_t* scales,
                                    const uint16_t* zeros, int64_t out, int64_t in, int32_t g,
                                    int32_t symmetric, const double* x, int64_t B,
                                    const int64_t* rows, int64_t nrows, double* y) {
    if (g <= 0 || (in % g) != 0 || (g % 2) != 0) return -1;
    if (!symmetric && zeros == NULL) return -1;
    const int64_t G = in / g;
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t r = rows[i];
        if (r < 0 || r >= out) return -1;
        for (int64_t b = 0; b < B; ++b) {
            double acc = 0.0;
            for (int64_t k = 0; k < in; ++k) {
                int64_t j = k / g;
                double sf = (double)oracle_f16_to_f32(scales[r * G + j]);
                double z = symmetric ? 0.0 : (double)oracle_f16_to_f32(zeros[r * G + j]);
                double q = (double)oracle_code_at(qweight, in, r, k, symmetric);
                acc += sf * (q - z) * x[b * in + k];
            }
            y[b * nrows + i] = acc;
        }
    }
    return 0;
}

/* All rows: y [B, out]. */
ORACLE_API int oracle_gemv_f64(const uint8_t* qweight, const uint16_t* scales,
                               const uint16_t* zeros, int64_t out, int64_t in, int32_t g,
                               int32_t symmetric, const double* x, int64_t B, double* y) {
    int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)(out > 0 ? out : 1));
    if (!rows) return -1;
    for (int64_t r = 0; r < out; ++r) rows[r] = r;
    int rc = oracle_gemv_rows_f64(qweight, scales, zeros, out, in, g, symmetric, x, B, rows, out, y);
    free(rows);
    return rc;
}

/*
 * The unquantised reference product y[b, i] = sum_k W[rows[i], k] * x[b, k]
 * in fp64, for W given as exact fp32 values (of bf16 weights).  This is the
 * bf16 decode matmul the INT4 path is compared with (ybb.press section 一,
 * roofline_bound example; arganzheng.life section 二.4 batch table).
 */
ORACLE_API int oracle_dense_rows_f64(const float* W, int64_t out, int64_t in, const double* x,
                                     int64_t B, const int64_t* rows, int64_t nrows, double* y) {
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t r = rows[i];
        if (r < 0 || r >= out) return -1;
        for (int64_t b = 0; b < B; ++b) {
            double acc = 0.0;
            for (int64_t k = 0; k < in; ++k) acc += (double)W[r * in + k] * x[b * in + k];
            y[b * nrows + i] = acc;
        }
    }
    return 0;
}

/* ------------------------------------------------- per-channel INT8 weights */

/*
 * Per-output-channel INT8 weight quantization ("量化：PTQ、GPTQ、AWQ 与
 * SmoothQuant" (charles2530.github.io), section 13, 快速代码示例
 * per_channel_int8_quant): one scale per row,
 *   s[r] = max(max_k |W[r, k]|, eps) / 127,   eps = 1e-6,
 *   q[r, k] = clamp(rne(W[r, k] / s[r]), -127, 127)   (int8),
 *   w_hat = q * s.
 * All in fp32 (the page's w is a float tensor), IEEE division, RNE.
 */
ORACLE_API int oracle_q8_quantize_per_channel(const float* W, int64_t out, int64_t in,
                                              int8_t* q, float* scales) {
    if (out < 0 || in <= 0) return -1;
    const float eps = 1e-6f;
    for (int64_t r = 0; r < out; ++r) {
        const float* w = W + r * in;
        float a = 0.0f;
        for (int64_t k = 0; k < in; ++k) {
            float m = fabsf(w[k]);
            if (m > a) a = m;
        }
        if (a < eps) a = eps;                    /* clamp_min(eps) */
        const float s = a / 127.0f;
        scales[r] = s;
        for (int64_t k = 0; k < in; ++k)
            q[r * in + k] = (int8_t)oracle_quantize_value(w[k], s, 0, -127, 127);
    }
    return 0;
}

/* w_hat[r, k] = q[r, k] * s[r], one fp32 multiplication. */
ORACLE_API int oracle_q8_dequant_f32(const int8_t* q, const float* scales, int64_t out,
                                     int64_t in, float* W_hat) {
    if (out < 0 || in <= 0) return -1;
    for (int64_t r = 0; r < out; ++r)
        for (int64_t k = 0; k < in; ++k) W_hat[r * in + k] = (float)q[r * in + k] * scales[r];
    return 0;
}

/*
 * y[b, i] = s[rows[i]] * sum_k q[rows[i], k] * x[b, k] in fp64 (the W8A16
 * decode product of the dequantised per-channel weights).
 */
ORACLE_API int oracle_q8_gemv_rows_f64(const int8_t* q, const float* scales, int64_t out,
                                       int64_t in, const double* x, int64_t B,
                                       const int64_t* rows, int64_t nrows, double* y) {
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t r = rows[i];
        if (r < 0 || r >= out) return -1;
        for (int64_t b = 0; b < B; ++b) {
            double acc = 0.0;
            for (int64_t k = 0; k < in; ++k) acc += (double)q[r * in + k] * x[b * in + k];
            y[b * nrows + i] = (double)scales[r] * acc;
        }
    }
    return 0;
}

/* ------------------------------------------------------- INT8 KV cache */

static uint16_t to_cache_dtype(float f, int is_bf16) {
    return is_bf16 ? oracle_f32_to_bf16(f) : oracle_f32_to_f16(f);
}
static float from_cache_dtype(uint16_t h, int is_bf16) {
    return is_bf16 ? oracle_bf16_to_f32(h) : oracle_f16_to_f32(h);
}

/*
 * Symmetric INT8 quantization of a KV cache [batch, heads, seq, head_dim]
 * along head_dim ("压缩算法" (cs-knowledge-wiki), section 7.4.1.1,
 * quantize_kv_cache_int8 with its default axis = -1): one scale per
 * (batch, head, token) row of head_dim values,
 *   s = max |x| / 127  (stored in the cache's 16-bit type),
 *   q = clamp(rne(x / s), -128, 127),
 * and the dequantization q * s rounded to the cache type
 * (dequantize_kv_cache_int8).  rows = batch * heads * seq, row-major.
 * Readings: fp32 arithmetic with the stored scale (as for the weights); a
 * row whose stored scale is 0 gets codes 0.
 */
ORACLE_API int oracle_kv_quantize_int8(const float* kv, int64_t rows, int64_t d, int32_t is_bf16,
                                       int8_t* codes, uint16_t* scales) {
    if (rows < 0 || d <= 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const float* v = kv + r * d;
        float a = 0.0f;
        for (int64_t k = 0; k < d; ++k) {
            float m = fabsf(v[k]);
            if (m > a) a = m;
        }
        const uint16_t sb = to_cache_dtype(a / 127.0f, is_bf16);
        const float s = from_cache_dtype(sb, is_bf16);
        scales[r] = sb;
        for (int64_t k = 0; k < d; ++k)
            codes[r * d + k] = (int8_t)(s == 0.0f ? 0 : oracle_quantize_value(v[k], s, 0, -128, 127));
    }
    return 0;
}

ORACLE_API int oracle_kv_dequant_int8(const int8_t* codes, const uint16_t* scales, int64_t rows,
                                      int64_t d, int32_t is_bf16, uint16_t* out) {
    if (rows < 0 || d <= 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const float s = from_cache_dtype(scales[r], is_bf16);
        for (int64_t k = 0; k < d; ++k)
            out[r * d + k] = to_cache_dtype((float)codes[r * d + k] * s, is_bf16);
    }
    return 0;
}

/* ------------------------------------------- FP4 microscaling formats */

/*
 * E2M1 ("post-training-quantization-gptq-awq-and-rotation" (arganzheng.life)
 * section 九.1, format table): 1 sign, 2 exponent, 1 mantissa bit; the
 * magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.  A code is sign << 3 | m with
 * magnitude index m in 0..7 in that order.
 */
static const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

ORACLE_API float oracle_e2m1_to_f32(uint8_t c) {
    float m = kE2M1[c & 7u];
    return (c & 8u) ? -m : m;
}

/* Nearest E2M1 value of a finite fp32 value, ties to the even magnitude
 * index (mantissa bit 0), magnitudes above 6 saturating to 6; the sign is
 * kept, so small negative values give -0 (code 8).  NaN gives +0. */
ORACLE_API uint8_t oracle_f32_to_e2m1(float v) {
    if (v != v) return 0;
    uint8_t sign = (v < 0.0f || (v == 0.0f && signbit(v))) ? 8u : 0u;
    double a = fabs((double)v);
    if (a >= 6.0) return (uint8_t)(sign | 7u);
    uint8_t best = 0;
    for (uint8_t m = 1; m < 8; ++m) {
        double dm = fabs(a - (double)kE2M1[m]);
        double db = fabs(a - (double)kE2M1[best]);
        if (dm < db || (dm == db && (m & 1u) == 0u)) best = m;
    }
    return (uint8_t)(sign | best);
}

/* E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities, 0x7F / 0xFF NaN, largest finite 448, subnormals m * 2^-9). */
ORACLE_API float oracle_e4m3_to_f32(uint8_t c) {
    uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
    float mag;
    if (e == 0xFu && m == 7u) mag = NAN;
    else if (e == 0) mag = ldexpf((float)m, -9);
    else mag = ldexpf((float)(8u | m), (int)e - 10);
    return (c & 0x80u) ? -mag : mag;
}

/* Nearest E4M3 value of a non-negative finite fp32 value, ties to even,
 * saturating at 448 (the block scales are never negative). */
ORACLE_API uint8_t oracle_f32_to_e4m3_sat(float v) {
    if (!(v > 0.0f)) return 0;
    if (v >= 448.0f) return 0x7E;
    uint8_t best = 0;
    double bd = fabs((double)v);
    for (uint32_t c = 1; c <= 0x7E; ++c) {
        double d = fabs((double)v - (double)oracle_e4m3_to_f32((uint8_t)c));
        if (d < bd || (d == bd && (c & 1u) == 0u)) { best = (uint8_t)c; bd = d; }
    }
    return best;
}

/* floor(log2(a)) of a positive finite fp32 value, exactly. */
static int floor_log2_f32(float a) {
    int e;
    (void)frexpf(a, &e);          /* a = f * 2^e, f in [0.5, 1) */
    return e - 1;
}

/*
 * MXFP4 ("post-training-quantization-gptq-awq-and-rotation" section 九.1 and
 * 九.2: E2M1 elements with one E8M0 power-of-two scale per 32, the OCP
 * standard; the scale rule is the OCP one): per block of 32 consecutive
 * elements of a row,
 *   e = clamp(floor(log2(max |v|)) - 2, -127, 127)   (2 = E2M1's largest exponent)
 *   X = 2^e,  scale byte = e + 127,  q = e2m1(v / X) (saturating at 6),
 * and an all-zero block gets scale byte 0 and codes +0.  Codes packed two
 * per byte, even element in the low nibble.
 *   W [out, in] fp32;  packed [out, in/2];  scales [out, in/32] E8M0 bytes.
 */
ORACLE_API int oracle_mxfp4_quantize(const float* W, int64_t out, int64_t in, uint8_t* packed,
                                     uint8_t* scales) {
    if (out < 0 || in <= 0 || (in % 32) != 0) return -1;
    uint8_t codes[32];
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t b = 0; b < in / 32; ++b) {
            const float* v = W + r * in + b * 32;
            float a = 0.0f;
            for (int k = 0; k < 32; ++k) if (fabsf(v[k]) > a) a = fabsf(v[k]);
            int e = -127;
            if (a > 0.0f) {
                e = floor_log2_f32(a) - 2;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            for (int k = 0; k < 32; ++k)
                codes[k] = (a > 0.0f) ? oracle_f32_to_e2m1(ldexpf(v[k], -e)) : 0u;
            scales[r * (in / 32) + b] = (uint8_t)(e + 127);
            for (int k = 0; k < 32; k += 2)
                packed[r * (in / 2) + b * 16 + k / 2] = (uint8_t)(codes[k] | (codes[k + 1] << 4));
        }
    }
    return 0;
}

/* w_hat = e2m1(q) * 2^(scale - 127) in fp32 (exact). */
ORACLE_API int oracle_mxfp4_dequant(const uint8_t* packed, const uint8_t* scales, int64_t out,
                                    int64_t in, float* W_hat) {
    if (out < 0 || in <= 0 || (in % 32) != 0) return -1;
    for (int64_t r = 0; r < out; ++r)
        for (int64_t k = 0; k < in; ++k) {
            uint8_t byte = packed[r * (in / 2) + k / 2];
            uint8_t c = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
            int e = (int)scales[r * (in / 32) + k / 32] - 127;
            W_hat[r * in + k] = ldexpf(oracle_e2m1_to_f32(c), e);
        }
    return 0;
}

/*
 * NVFP4 (the same section: E2M1 elements, one E4M3 scale per 16 and one fp32
 * scale per tensor).  Readings: the tensor scale maps the largest block scale
 * amax/6 onto E4M3's largest value 448, and each block scale is amax_b / 6
 * expressed in units of the tensor scale, all in fp32 IEEE arithmetic:
 *   s_t = A / 2688  (A = max |W| over the tensor; 2688 = 6 * 448; s_t = 1 if A = 0)
 *   c_b = e4m3_sat(fp32(amax_b / 6) / s_t),   S_b = fp32(e4m3(c_b) * s_t)
 *   q = e2m1(v / S_b) (saturating at 6), codes 0 where S_b = 0,
 * and w_hat = fp32(e2m1(q) * S_b).
 *   packed [out, in/2];  scales [out, in/16] E4M3 bytes;  *tensor_scale fp32.
 */
ORACLE_API int oracle_nvfp4_quantize(const float* W, int64_t out, int64_t in, uint8_t* packed,
                                     uint8_t* scales, float* tensor_scale) {
    if (out < 0 || in <= 0 || (in % 16) != 0) return -1;
    float A = 0.0f;
    for (int64_t i = 0; i < out * in; ++i) if (fabsf(W[i]) > A) A = fabsf(W[i]);
    const float st = (A > 0.0f) ? A / 2688.0f : 1.0f;
    *tensor_scale = st;
    uint8_t codes[16];
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t b = 0; b < in / 16; ++b) {
            const float* v = W + r * in + b * 16;
            float a = 0.0f;
            for (int k = 0; k < 16; ++k) if (fabsf(v[k]) > a) a = fabsf(v[k]);
            const uint8_t cb = oracle_f32_to_e4m3_sat((a / 6.0f) / st);
            const float S = oracle_e4m3_to_f32(cb) * st;
            for (int k = 0; k < 16; ++k) codes[k] = (S > 0.0f) ? oracle_f32_to_e2m1(v[k] / S) : 0u;
            scales[r * (in / 16) + b] = cb;
            for (int k = 0; k < 16; k += 2)
                packed[r * (in / 2) + b * 8 + k / 2] = (uint8_t)(codes[k] | (codes[k + 1] << 4));
        }
    }
    return 0;
}

ORACLE_API int oracle_nvfp4_dequant(const uint8_t* packed, const uint8_t* scales,
                                    float tensor_scale, int64_t out, int64_t in, float* W_hat) {
    if (out < 0 || in <= 0 || (in % 16) != 0) return -1;
    for (int64_t r = 0; r < out; ++r)
        for (int64_t k = 0; k < in; ++k) {
            uint8_t byte = packed[r * (in / 2) + k / 2];
            uint8_t c = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
            const float S = oracle_e4m3_to_f32(scales[r * (in / 16) + k / 16]) * tensor_scale;
            W_hat[r * in + k] = oracle_e2m1_to_f32(c) * S;
        }
    return 0;
}

/*
 * The W4A4 product of two FP4 operands (the use of the microscaling formats
 * on Blackwell's block-scaled tensor cores, arganzheng.life sections 九.1,
 * 九.2: FP4 puts the non-uniform grid into activation quantization too):
 *   y[b, r] = sum_k w_hat[r, k] * x_hat[b, k]   in fp64,
 * with w_hat, x_hat the values of the packed codes and block scales taken
 * exactly in fp64 (e2m1 * 2^e for MXFP4; e2m1 * e4m3 * s_t for NVFP4, the
 * product of three short significands, exact), i.e. the product a
 * block-scaled MMA computes before its fp32 rounding.
 *   fmt 0 = MXFP4 (scales [rows, in/32] E8M0), 1 = NVFP4 (scales [rows, in/16]
 *   E4M3, tensor scales w_st, x_st); packed [rows, in/2].
 */
static double fp4_value_f64(const uint8_t* packed, const uint8_t* scales, double st, int fmt,
                            int64_t in, int64_t r, int64_t k) {
    uint8_t byte = packed[r * (in / 2) + k / 2];
    uint8_t c = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
    double e = (double)oracle_e2m1_to_f32(c);
    if (fmt == 0) return ldexp(e, (int)scales[r * (in / 32) + k / 32] - 127);
    return e * (double)oracle_e4m3_to_f32(scales[r * (in / 16) + k / 16]) * st;
}

ORACLE_API int oracle_fp4_gemm_f64(const uint8_t* wq, const uint8_t* ws, float w_st,
                                   const uint8_t* xq, const uint8_t* xs, float x_st, int32_t fmt,
                                   int64_t out, int64_t in, int64_t B, double* y) {
    const int64_t blk = fmt == 0 ? 32 : 16;
    if (out < 0 || B < 0 || in <= 0 || (in % blk) != 0 || (fmt != 0 && fmt != 1)) return -1;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t r = 0; r < out; ++r) {
            double acc = 0.0;
            for (int64_t k = 0; k < in; ++k)
                acc += fp4_value_f64(wq, ws, (double)w_st, fmt, in, r, k) *
                       fp4_value_f64(xq, xs, (double)x_st, fmt, in, b, k);
            y[b * out + r] = acc;
        }
    return 0;
}
