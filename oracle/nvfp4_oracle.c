/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for the NVFP4 W4A4 linear
 *
 *     y = dequant(Q(x.H)) . dequant(Q(W.H))^T + b
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file: it is used by tests/, by the smoke check and by the CPU-baseline leg
 * of bench.py.  It shares no code, header, table or constant generator with the
 * CUDA library; it is written from the definitions on the pages cited below.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -fPIC -shared
 * (contraction off so that every float expression is one IEEE-754 binary32
 * operation rounded to nearest-even, exactly as written; x86-64 evaluates float
 * in SSE single precision).  OpenMP only splits independent rows; it never
 * changes the order of any sum or comparison.
 *
 * Sources (page title -- section):
 *  [P1] minimax_h3_nvfp4_decoder (FastVideo API docs) -- nvfp4_linear_inference,
 *       NVFP4DecoderLinear (__init__, from_linear, _activation_global_sf, forward),
 *       module docstring (block Hadamard rotation folded into the weight).
 *  [P2] convert_minimax_h3_text_encoder_nvfp4.py -- module docstring,
 *       probe_relative_error, quantize_language_linear.
 *  [P5] FastH3-QAD-v2 and NVFP4 VAE Decoders -- "The whole stack in NVFP4"
 *       (4-bit values plus one FP8 scale for every 16).
 *
 * Readings taken where the pages are silent:
 *  R1 FP4_E4M3_RANGE = 448 * 6 = 2688 (largest E4M3 scale times largest E2M1 value).
 *  R2 dynamic global scale = 2688 / max(amax, 1e-12), amax over the whole call.
 *  R3 per-block order: bmax -> s_raw = rn(rn(gsf*bmax)/6) -> s8 = E4M3(s_raw) ->
 *     s = dec(s8) -> inv = rn(gsf/s) -> code = E2M1(rn(x*inv)); s == 0 -> all codes 0.
 *  R4 E2M1 and E4M3 encodes are round-to-nearest-even with saturation to the
 *     largest finite value; E2M1 keeps the sign of its input (so -0.1 -> code 8).
 *  R5 packing: element 2i in the low nibble, element 2i+1 in the high nibble.
 *  R6 layout_128x4: offset(r,c) = ((r/128)*(Cp/4) + c/4)*512 + (r%32)*16
 *     + ((r%128)/32)*4 + c%4, rows padded to 128, scale columns to 4, padding 0.
 *  R7 Hadamard: Sylvester H_g (H[i][j] = (-1)^popcount(i&j)) times rn(1/sqrt(g)),
 *     computed by an fp32 butterfly with stages h = 1,2,..,g/2, pair (j, j+h) ->
 *     (a+b, a-b), then one multiply by the scale, then RNE to bf16.
 *  R8 alpha = rn(1 / rn(gsf_x * gsf_w)) in fp32.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                              */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the upper half of an fp32 bit pattern; widening is exact. */
EXPORT float ora_bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* Round an fp32 value to the nearest bf16, ties to the even bf16 (IEEE RNE):
 * add half an ulp of the target, plus one more unit when the kept LSB is odd,
 * then truncate.  NaN stays a quiet NaN. */
EXPORT uint16_t ora_f32_to_bf16(float f) {
    uint32_t u = f32_to_bits(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

/* ------------------------------------------------------------------------ */
/* E2M1 (FP4) -- [P5] "4-bit values"; magnitudes of codes 0..7                */
/* ------------------------------------------------------------------------ */

static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* code bit 3 is the sign, bits 0..2 index E2M1_MAG. */
EXPORT double ora_e2m1_decode(uint8_t code) {
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* R4: nearest of the eight magnitudes; an exact tie goes to the even code (the
 * code whose mantissa bit, bit 0, is clear); anything beyond 6 becomes 6. */
EXPORT uint8_t ora_e2m1_encode(float v) {
    double a = fabs((double)v);
    if (a >= 6.0) return (uint8_t)(7 | (signbit(v) ? 8 : 0));   /* saturate (also inf) */
    int best = 0;
    double best_d = fabs(a - E2M1_MAG[0]);
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - E2M1_MAG[c]);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(best | (signbit(v) ? 8 : 0));
}

/* ------------------------------------------------------------------------ */
/* E4M3 (OCP E4M3FN) -- [P1] "inv_scale" / [P5] "a shared FP8 scale"           */
/* ------------------------------------------------------------------------ */

/* bias 7, 3 mantissa bits, no infinities; S.1111.111 is NaN; exponent field 0
 * is subnormal with step 2^-9. */
EXPORT double ora_e4m3_decode(uint8_t b) {
    int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* R4 for a non-negative input: the finite codes 0x00..0x7E are increasing in
 * value, so find the bracketing pair by bisection, then take the nearer one, the
 * even code on an exact tie; inputs above 448 saturate to 0x7E (448). */
EXPORT uint8_t ora_e4m3_encode(float v) {
    double a = (double)v;
    if (!(a > 0.0)) return 0;            /* zero (and negative, unused) -> +0 */
    if (a >= 448.0) return 0x7e;
    int lo = 0, hi = 0x7e;               /* dec(lo) <= a < dec(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (ora_e4m3_decode((uint8_t)mid) <= a) lo = mid; else hi = mid;
    }
    double dl = a - ora_e4m3_decode((uint8_t)lo);
    double dh = ora_e4m3_decode((uint8_t)hi) - a;
    if (dl < dh) return (uint8_t)lo;
    if (dh < dl) return (uint8_t)hi;
    return (uint8_t)((lo & 1) ? hi : lo);
}

/* Element-wise forms of the two encoders and of the bf16 rounding, for sweeps. */
EXPORT void ora_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = ora_e2m1_encode(v[i]);
}

EXPORT void ora_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = ora_e4m3_encode(v[i]);
}

EXPORT void ora_f32_to_bf16_array(const float* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = ora_f32_to_bf16(v[i]);
}

/* ------------------------------------------------------------------------ */
/* Global scale -- [P1] _activation_global_sf ("FP4_E4M3_RANGE / amax"),      */
/* nvfp4_linear_inference (global_sf_x = None -> computed per call), R1, R2   */
/* ------------------------------------------------------------------------ */

/* max |x| over n bf16 values (exact: max needs no rounding). */
EXPORT float ora_amax_bf16(const uint16_t* x, int64_t n) {
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(ora_bf16_to_f32(x[i]));
        if (a > m) m = a;
    }
    return m;
}

EXPORT float ora_global_scale(float amax) {
    float clamped = amax > 1e-12f ? amax : 1e-12f;
    return 2688.0f / clamped;
}

/* R8, [P1] nvfp4_linear_inference: 1.0 / (global_sf_x * global_sf_w). */
EXPORT float ora_alpha(float gsf_x, float gsf_w) {
    float p = gsf_x * gsf_w;
    return 1.0f / p;
}

/* ------------------------------------------------------------------------ */
/* Block quantizer -- [P1] NVFP4_BLOCK_SIZE = 16 along in_features,           */
/* [P2] quantize_language_linear (packed [out, in/2] uint8), R3, R5           */
/* ------------------------------------------------------------------------ */

/* One block of 16 values (already in fp32, exactly the bf16 inputs).  Writes
 * 8 packed bytes and returns the E4M3 scale byte. */
static uint8_t quantize_block16(const float* v, float gsf, uint8_t* packed8) {
    float bmax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(v[i]);
        if (a > bmax) bmax = a;
    }
    float t = gsf * bmax;
    float s_raw = t / 6.0f;
    uint8_t s8 = ora_e4m3_encode(s_raw);
    float s = (float)ora_e4m3_decode(s8);
    uint8_t codes[16];
    if (s == 0.0f) {
        for (int i = 0; i < 16; ++i) codes[i] = 0;
    } else {
        float inv = gsf / s;
        for (int i = 0; i < 16; ++i) {
            float q = v[i] * inv;
            codes[i] = ora_e2m1_encode(q);
        }
    }
    for (int i = 0; i < 8; ++i)
        packed8[i] = (uint8_t)(codes[2 * i] | (codes[2 * i + 1] << 4));
    return s8;
}

/* x: bf16 [R, K] row-major, K % 16 == 0.  packed: [R, K/2].  sf_lin: the
 * scale bytes in plain row-major order [R, K/16] (the un-swizzled form). */
EXPORT void ora_quantize_rows(const uint16_t* x, int64_t R, int64_t K, float gsf,
                              uint8_t* packed, uint8_t* sf_lin) {
    int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        float v[16];
        for (int64_t j = 0; j < nb; ++j) {
            for (int i = 0; i < 16; ++i) v[i] = ora_bf16_to_f32(x[r * K + j * 16 + i]);
            sf_lin[r * nb + j] = quantize_block16(v, gsf, packed + r * (K / 2) + j * 8);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* layout_128x4 -- [P1] SfLayout.layout_128x4; [P2] nvfp4_scale_shape, R6     */
/* ------------------------------------------------------------------------ */

EXPORT int64_t ora_scale_rows_padded(int64_t R) { return (R + 127) / 128 * 128; }
EXPORT int64_t ora_scale_cols_padded(int64_t K) { return (K / 16 + 3) / 4 * 4; }
EXPORT int64_t ora_scale_bytes(int64_t R, int64_t K) {
    return ora_scale_rows_padded(R) * ora_scale_cols_padded(K);
}

EXPORT int64_t ora_scale_offset(int64_t r, int64_t c, int64_t K) {
    int64_t cp = ora_scale_cols_padded(K);
    return ((r / 128) * (cp / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* Places sf_lin [R, K/16] at its 128x4 offsets; every padding byte becomes 0. */
EXPORT void ora_scale_swizzle(const uint8_t* sf_lin, int64_t R, int64_t K, uint8_t* out) {
    int64_t nb = K / 16;
    memset(out, 0, (size_t)ora_scale_bytes(R, K));
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < nb; ++c)
            out[ora_scale_offset(r, c, K)] = sf_lin[r * nb + c];
}

EXPORT void ora_scale_unswizzle(const uint8_t* sf, int64_t R, int64_t K, uint8_t* sf_lin) {
    int64_t nb = K / 16;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < nb; ++c)
            sf_lin[r * nb + c] = sf[ora_scale_offset(r, c, K)];
}

/* ------------------------------------------------------------------------ */
/* Block Hadamard -- [P1] module docstring and from_linear (orthonormal,      */
/* symmetric H; "y = x W^T = (x H)(W H)^T"), forward (rotate before quant), R7 */
/* ------------------------------------------------------------------------ */

EXPORT float ora_hadamard_scale(int g) { return (float)(1.0 / sqrt((double)g)); }

/* In-place fp32 butterfly on g values; result = H_g v without normalisation. */
static void fwht_f32(float* v, int g) {
    for (int h = 1; h < g; h *= 2) {
        for (int j = 0; j < g; ++j) {
            if (j & h) continue;
            float a = v[j], b = v[j + h];
            v[j] = a + b;
            v[j + h] = a - b;
        }
    }
}

/* x, y: bf16 [R, K]; every g-group of every row is rotated; K % g == 0. */
EXPORT void ora_hadamard_rotate(const uint16_t* x, int64_t R, int64_t K, int g, uint16_t* y) {
    float c = ora_hadamard_scale(g);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        float v[256];
        for (int64_t j0 = 0; j0 < K; j0 += g) {
            for (int i = 0; i < g; ++i) v[i] = ora_bf16_to_f32(x[r * K + j0 + i]);
            fwht_f32(v, g);
            for (int i = 0; i < g; ++i) {
                float s = v[i] * c;
                y[r * K + j0 + i] = ora_f32_to_bf16(s);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Dequantization and the fp64 GEMM -- [P1] nvfp4_linear_inference            */
/* (mm_fp4(x_fp4, packed.T, x_sf, w_sf.T, alpha) then out.add_(bias))          */
/* ------------------------------------------------------------------------ */

/* Element (r, k) of a packed NVFP4 matrix, before the global scale:
 * E2M1(code) * E4M3(block scale), exact in fp64. */
static double dequant_elem(const uint8_t* packed, const uint8_t* sf, int64_t r, int64_t k,
                           int64_t K) {
    uint8_t byte = packed[r * (K / 2) + k / 2];
    uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);
    return ora_e2m1_decode(code) * ora_e4m3_decode(sf[ora_scale_offset(r, k / 16, K)]);
}

/* Expands rows [0, R) of a packed matrix to fp64 [R, K] (no global scale). */
EXPORT void ora_dequantize(const uint8_t* packed, const uint8_t* sf, int64_t R, int64_t K,
                           double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k) out[r * K + k] = dequant_elem(packed, sf, r, k, K);
}

/* NVFP4 -> bf16 expansion of a packed tensor (the W4A16 path: "decode dynamic-scale
 * NVFP4 H3 VAE tiles one at a time" -- FASTVIDEO_H3_ENCODER_FUSED_DEQUANT, which expands
 * the serialized NVFP4 text encoder to bf16 on GPUs without an FP4 GEMM).  Reading: the
 * value is E2M1(code) * E4M3(scale) (exact in fp32), divided by the global scale in fp32
 * (IEEE, round to nearest even) and rounded to nearest even to bf16. */
EXPORT void ora_dequantize_bf16(const uint8_t* packed, const uint8_t* sf, int64_t R, int64_t K,
                                float gsf, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k) {
            const float v = (float)dequant_elem(packed, sf, r, k, K);
            const float q = v / gsf;
            out[r * K + k] = ora_f32_to_bf16(q);
        }
}

/* y[i, n] = alpha * sum_k deq_a(rows[i], k) * deq_b(n, k) + bias[n], in fp64,
 * k ascending; every product is exact in fp64.  rows == NULL means rows 0..M-1
 * (then n_rows = M).  bias_bf16 may be NULL.  Each operand row is dequantized once
 * (dequant_elem, exact) and the sum runs over the two dequantized rows; on an
 * allocation failure every output is NaN. */
EXPORT void ora_gemm_f64(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                         const uint8_t* sfb, int64_t N, int64_t K, float alpha,
                         const uint16_t* bias_bf16, const int64_t* rows, int64_t n_rows,
                         double* y) {
    double* da = (double*)malloc((size_t)(n_rows > 0 ? n_rows : 1) * (size_t)K * sizeof(double));
    if (!da) {
        for (int64_t i = 0; i < n_rows * N; ++i) y[i] = NAN;
        return;
    }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t m = rows ? rows[i] : i;
        for (int64_t k = 0; k < K; ++k) da[i * K + k] = dequant_elem(a, sfa, m, k, K);
    }
    int failed = 0;
#pragma omp parallel
    {
        double* db = (double*)malloc((size_t)K * sizeof(double));
        if (!db) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t n = 0; n < N; ++n) {
            if (!db) continue;
            for (int64_t k = 0; k < K; ++k) db[k] = dequant_elem(b, sfb, n, k, K);
            double bias = bias_bf16 ? (double)ora_bf16_to_f32(bias_bf16[n]) : 0.0;
            for (int64_t i = 0; i < n_rows; ++i) {
                const double* ra = da + i * K;
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += ra[k] * db[k];
                y[i * N + n] = (double)alpha * acc + bias;
            }
        }
        free(db);
    }
    free(da);
    if (failed)
        for (int64_t i = 0; i < n_rows * N; ++i) y[i] = NAN;
}

/* ------------------------------------------------------------------------ */
/* Whole-path helpers                                                         */
/* ------------------------------------------------------------------------ */

/* Quantize a bf16 [R, K] tensor to the packed + 128x4 form.  gsf_in < 0 means
 * dynamic (R2: amax over all R*K values); otherwise gsf_in is used as is.
 * sf_lin_scratch must hold R*K/16 bytes.  Returns the global scale used. */
EXPORT float ora_quantize(const uint16_t* x, int64_t R, int64_t K, float gsf_in,
                          uint8_t* packed, uint8_t* sf, uint8_t* sf_lin_scratch) {
    float gsf = gsf_in < 0.0f ? ora_global_scale(ora_amax_bf16(x, R * K)) : gsf_in;
    ora_quantize_rows(x, R, K, gsf, packed, sf_lin_scratch);
    ora_scale_swizzle(sf_lin_scratch, R, K, sf);
    return gsf;
}

/* ------------------------------------------------------------------------- */
/* int8 per-row W8A8 linear ("FastH3-4-step-Preview-v1-r16-int8", "What is    */
/* inside": weight = round(W / scale) clamped to -127..127 with scale =       */
/* amax(|W[row]|) / 127 per output row; activations quantized per row at call */
/* time and multiplied with an int8 GEMM).                                     */
/* Readings: the division and the scale are fp32 (IEEE, round to nearest      */
/* even); round() is half to even; an all-zero row has scale 0 and codes 0;   */
/* activations use the same per-row rule; the product is                      */
/* y = bf16(fp32(fp32(acc) * s_x[m]) * s_w[n] + bias[n]) with an exact integer */
/* accumulator.                                                                */
/* ------------------------------------------------------------------------- */

/* Row r of x (bf16 [R, K]) -> int8 codes and the fp32 row scale. */
EXPORT void ora_int8_quantize_rows(const uint16_t* x, int64_t R, int64_t K, int8_t* q,
                                   float* scale) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(ora_bf16_to_f32(x[r * K + k]));
            if (a > amax) amax = a;
        }
        const float s = amax / 127.0f;
        scale[r] = s;
        for (int64_t k = 0; k < K; ++k) {
            int8_t c = 0;
            if (s != 0.0f) {
                const float v = ora_bf16_to_f32(x[r * K + k]) / s;
                double t = nearbyint((double)v);          /* half to even (default mode) */
                if (t > 127.0) t = 127.0;
                if (t < -127.0) t = -127.0;
                c = (int8_t)t;
            }
            q[r * K + k] = c;
        }
    }
}

/* y[i, n] = s_x[m] * s_w[n] * sum_k qx[m, k] qw[n, k] + bias[n] in fp64 (the integer sum
 * exact), rows as in ora_gemm_f64. */
EXPORT void ora_int8_gemm_f64(const int8_t* qx, const float* sx, const int8_t* qw,
                              const float* sw, int64_t N, int64_t K, const uint16_t* bias_bf16,
                              const int64_t* rows, int64_t n_rows, double* y) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t m = rows ? rows[i] : i;
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k) acc += (int64_t)qx[m * K + k] * (int64_t)qw[n * K + k];
            double v = (double)acc * (double)sx[m] * (double)sw[n];
            if (bias_bf16) v += (double)ora_bf16_to_f32(bias_bf16[n]);
            y[i * N + n] = v;
        }
    }
}
