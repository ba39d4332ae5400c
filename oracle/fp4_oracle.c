/*
 * fp4_oracle.c -- plain, slow CPU oracle for the block-scaled FP4 quantized linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA path shares no
 * code, header, table or constant with it.
 *
 * What it computes (sources are the model-card pages this project implements):
 *   - E2M1 (FP4) elements, two per byte, with one E8M0 scale per 32 values along K
 *     ("MXFP4", Wan2.2-I2V-A14B-Lightning-Diffusers-MXFP4-AutoRound, Quantization
 *     Details, coverage list; Wan2.2-Animate-14B-Diffusers-MXFP4-AutoRound, Coverage).
 *   - E2M1 elements with one FP8 E4M3 scale per 16 values and an FP32 per-tensor
 *     global scale ("NVFP4", Wan2.2-T2V-A14B-Diffusers-NVFP4-AutoRound, Model
 *     Details: format and activation-scaling bullets).
 *   - dynamic MXFP8 activations for the W4A8 SVDQuant linear (wan2.2-ti2v-w4a8-svd
 *     README, opening paragraph).
 *   - the quantized linear itself, y = deq(A) deq(W)^T + bias, evaluated in fp64 on
 *     the dequantized operands (the quantize-dequantize view named on the NVFP4
 *     page's "How to Use" section), plus the rank-32 low-rank term X L1 L2 for W4A8.
 *
 * Where the pages are silent the plain readings below are taken (each is also
 * listed with its reason in the design notes):
 *   R1 E2M1 rounding: nearest grid value, ties to the even code, saturate at 6.
 *   R2 signed zero: -0 and negatives that round to zero keep the sign bit (0x8).
 *   R3 MXFP4 scale: 2^(floor(log2 amax) - 2), clamped to the E8M0 range; amax = 0
 *      gives byte 0x00.  MXFP8 uses the same rule with E4M3's emax 8.
 *   R4 NVFP4 arithmetic order, each step one IEEE fp32 operation:
 *        g  = T / 2688                      (T = tensor amax, 2688 = 6 * 448; T = 0 -> g = 1)
 *        s  = amax_block / (6 * g)          -> E4M3 (round to nearest even, saturate 448)
 *        d  = dec(sf) * g ;  r = 1 / d ;  code_i = e2m1(x_i * r)
 *      a block whose scale rounds to zero stores all-zero codes.
 *   R5 nibble order: element 2i in bits 3:0, element 2i+1 in bits 7:4.
 *   R6 scale-factor layout: 128-row x 4-group atoms of 512 bytes,
 *        off(r, j) = ((r/128)*(Kg/4) + j/4)*512 + (r%32)*16 + ((r%128)/32)*4 + j%4,
 *      rows padded to a multiple of 128 with zero bytes.
 *   R7 W4A8 low-rank term uses the unquantized bf16 input: u = x L1 (fp64).
 *   R10 the activation between the FFN's two quantized linears (ffn.net.0.proj ->
 *      ffn.net.2 in the MXFP4 pages' coverage lists) is the tanh-approximated GELU,
 *        gelu(z) = 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))),
 *      applied to the bf16 up-projection output z and rounded to bf16 before the down
 *      projection quantizes it.  The oracle takes the plain definition: gelu in fp64
 *      (orc_gelu_f64), then round to nearest even bf16 (orc_f64_to_bf16_rn).  A GPU that
 *      evaluates gelu in fp32 can land one bf16 step away where the exact value sits
 *      next to a rounding midpoint; the tests judge such results against the interval
 *      its stated error bound allows, not bit for bit.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math), so every
 * float operation is one IEEE round-to-nearest operation.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_MX 0
#define ORC_NV 1

/* ------------------------------------------------------------------------------------
 * Element and scale codecs
 * ---------------------------------------------------------------------------------- */

/* The eight E2M1 magnitudes: 1 sign, 2 exponent, 1 mantissa bit (MXFP4 page: weights
 * stored as packed 4-bit E2M1 codes). Index = the 3 low bits of the code. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_decode(uint8_t code) {
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* Nearest E2M1 value to v (R1, R2): scan the 8 magnitudes, keep the closest, and on an
 * exact tie prefer the even index (round-to-nearest-even on the mantissa bit).
 * Magnitudes of 6 and above saturate to 6 (code 7). */
uint8_t orc_e2m1_encode(float v) {
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    if (a >= 6.0) return sign | 7;
    int best = 0;
    double bestd = a;                       /* distance to magnitude 0 */
    for (int i = 1; i < 8; ++i) {
        double d = fabs(a - E2M1_MAG[i]);
        if (d < bestd || (d == bestd && (i % 2) == 0)) {
            best = i;
            bestd = d;
        }
    }
    return sign | (uint8_t)best;
}

/* OCP FP8 E4M3 ("fn"): bias 7, no infinities, 0x7F/0xFF are NaN, max 448 = 0x7E. */
double orc_e4m3_decode(uint8_t b) {
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Nearest finite E4M3 value to v, ties to the even code, saturating at 448 (R4's
 * "round to nearest even, saturate"); the sign bit is kept for zero results (R2). */
uint8_t orc_e4m3_encode(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;
    int best = 0;
    double bestd = a;
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs(a - orc_e4m3_decode((uint8_t)c));
        if (d < bestd || (d == bestd && (c % 2) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return sign | (uint8_t)best;
}

/* E8M0: one unsigned exponent byte, value 2^(b - 127); 0xFF is NaN (never produced). */
double orc_e8m0_decode(uint8_t b) {
    if (b == 0xFF) return NAN;
    return ldexp(1.0, (int)b - 127);
}

float orc_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static double f16_to_double(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp(1.0 + (double)m / 1024.0, e - 15);
    return s ? -v : v;
}

double orc_f16_to_double(uint16_t h) { return f16_to_double(h); }

/* floor(log2(a)) for finite a > 0, exact (frexp returns a = f * 2^ex, f in [0.5, 1)). */
static int floor_log2(double a) {
    int ex;
    frexp(a, &ex);
    return ex - 1;
}

/* ------------------------------------------------------------------------------------
 * Scale-factor layout (R6) and sizes
 * ---------------------------------------------------------------------------------- */
int64_t orc_sf_offset(int64_t r, int64_t j, int64_t Kg) {
    int64_t rb = r / 128, kb = j / 4;
    return (rb * (Kg / 4) + kb) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (j % 4);
}

int64_t orc_sf_bytes(int64_t rows, int64_t Kg) { return ((rows + 127) / 128) * 128 * Kg; }

/* ------------------------------------------------------------------------------------
 * Tensor amax and the NVFP4 global scale (R4)
 * ---------------------------------------------------------------------------------- */
float orc_tensor_amax(const uint16_t* x, int64_t n) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(orc_bf16_to_f32(x[i]));
        if (a > amax) amax = a;
    }
    return amax;
}

float orc_nv_global(float T) {
    if (T == 0.0f) return 1.0f;
    return T / 2688.0f;
}

/* ------------------------------------------------------------------------------------
 * GELU-tanh (R10): the plain definition, in fp64, then rounded to bf16.
 * ---------------------------------------------------------------------------------- */

/* gelu(z) = 0.5 z (1 + tanh(v)),  v = sqrt(2/pi) (z + 0.044715 z^3).
 * For v < 0, 1 + tanh(v) cancels (it is about 2 e^{2v}); there the exact identity
 * 0.5 (1 + tanh(v)) = 1 / (1 + e^{-2v}) is used instead, which loses nothing.  Once
 * e^{-2v} overflows the result is a zero of z's sign (the true value is below 2^-1000 |z|). */
double orc_gelu_f64(double z) {
    const double k = sqrt(2.0 / 3.14159265358979323846);
    const double v = k * (z + 0.044715 * z * z * z);
    if (v >= 0.0) return 0.5 * z * (1.0 + tanh(v));
    return z / (1.0 + exp(-2.0 * v));
}

/* Round a finite double to the nearest bf16 (8 significant bits, fp32's exponent range,
 * subnormals down to 2^-133), ties to even, and return its bits.  Values at or beyond the
 * largest finite bf16 plus half an ulp become infinities (gelu(z) never gets there: it
 * is at most z). */
uint16_t orc_f64_to_bf16_rn(double x) {
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);                      /* a = f 2^ex, f in [0.5, 1): ulp is 2^(ex - 8) */
    int q = ex - 8;
    if (q < -133) q = -133;             /* the subnormal quantum */
    double r = ldexp(rint(ldexp(a, -q)), q);   /* rint: nearest, ties to even */
    if (r >= 0x1p128) return sign | 0x7F80;  /* rounded past the largest finite bf16, 0x1.fep127 */
    float f = (float)r;                 /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)((u >> 16) & 0x7FFF);
}

/* h = bf16_rn(gelu(z)) element-wise: the down projection's input (R10). */
void orc_gelu_bf16(const uint16_t* z, int64_t n, uint16_t* h) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) h[i] = orc_f64_to_bf16_rn(orc_gelu_f64((double)orc_bf16_to_f32(z[i])));
}

/* ------------------------------------------------------------------------------------
 * Quantizers.  x is bf16 [rows, K] row-major; codes [rows, K/2]; sf in layout R6.
 * ---------------------------------------------------------------------------------- */

/* MXFP4: per 32 consecutive values along K (MXFP4 pages; R1-R3, R5, R6). */
void orc_quant_mxfp4(const uint16_t* x, int64_t rows, int64_t K, uint8_t* codes, uint8_t* sf) {
    const int64_t G = 32, Kg = K / G;
    memset(sf, 0, (size_t)orc_sf_bytes(rows, Kg));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < Kg; ++j) {
            const uint16_t* xb = x + r * K + j * G;
            float amax = 0.0f;
            for (int i = 0; i < G; ++i) {
                float a = fabsf(orc_bf16_to_f32(xb[i]));
                if (a > amax) amax = a;
            }
            int e = (amax == 0.0f) ? -127 : floor_log2((double)amax) - 2;
            if (e < -127) e = -127;
            if (e > 127) e = 127;
            sf[orc_sf_offset(r, j, Kg)] = (uint8_t)(e + 127);
            for (int i = 0; i < G; ++i) {
                /* x * 2^-e is exact in fp32 for every bf16 x and e in [-127, 125] */
                float q = (float)ldexp((double)orc_bf16_to_f32(xb[i]), -e);
                uint8_t c = orc_e2m1_encode(q);
                int64_t k = j * G + i;
                uint8_t* byte = codes + r * (K / 2) + k / 2;
                if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | c);
                else *byte = (uint8_t)((*byte & 0x0F) | (c << 4));
            }
        }
    }
}

/* NVFP4: per 16 consecutive values along K under the fp32 global g (NVFP4 page; R4). */
void orc_quant_nvfp4(const uint16_t* x, int64_t rows, int64_t K, float g, uint8_t* codes,
                     uint8_t* sf) {
    const int64_t G = 16, Kg = K / G;
    memset(sf, 0, (size_t)orc_sf_bytes(rows, Kg));
    const float six_g = 6.0f * g;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < Kg; ++j) {
            const uint16_t* xb = x + r * K + j * G;
            float amax = 0.0f;
            for (int i = 0; i < G; ++i) {
                float a = fabsf(orc_bf16_to_f32(xb[i]));
                if (a > amax) amax = a;
            }
            float s = amax / six_g;
            uint8_t sfb = orc_e4m3_encode(s);
            sf[orc_sf_offset(r, j, Kg)] = sfb;
            float d = (float)orc_e4m3_decode(sfb) * g;
            for (int i = 0; i < G; ++i) {
                uint8_t c;
                if (d == 0.0f) {
                    c = 0;
                } else {
                    float rcp = 1.0f / d;
                    c = orc_e2m1_encode(orc_bf16_to_f32(xb[i]) * rcp);
                }
                int64_t k = j * G + i;
                uint8_t* byte = codes + r * (K / 2) + k / 2;
                if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | c);
                else *byte = (uint8_t)((*byte & 0x0F) | (c << 4));
            }
        }
    }
}

/* MXFP8 (E4M3 elements, per-32 E8M0 scale) for the W4A8 linear's activations (R3). */
void orc_quant_mxfp8(const uint16_t* x, int64_t rows, int64_t K, uint8_t* elems, uint8_t* sf) {
    const int64_t G = 32, Kg = K / G;
    memset(sf, 0, (size_t)orc_sf_bytes(rows, Kg));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < Kg; ++j) {
            const uint16_t* xb = x + r * K + j * G;
            float amax = 0.0f;
            for (int i = 0; i < G; ++i) {
                float a = fabsf(orc_bf16_to_f32(xb[i]));
                if (a > amax) amax = a;
            }
            int e = (amax == 0.0f) ? -127 : floor_log2((double)amax) - 8;
            if (e < -127) e = -127;
            if (e > 127) e = 127;
            sf[orc_sf_offset(r, j, Kg)] = (uint8_t)(e + 127);
            for (int i = 0; i < G; ++i) {
                float q = (float)ldexp((double)orc_bf16_to_f32(xb[i]), -e);
                elems[r * K + j * G + i] = orc_e4m3_encode(q);
            }
        }
    }
}

/* ------------------------------------------------------------------------------------
 * Dequantization to fp64 (exact: every product of a code value, a scale and g fits
 * in 53 bits).  row_ids selects which rows to expand; out is [nrows, K].
 * ---------------------------------------------------------------------------------- */
void orc_dequant_fp4(int fmt, const uint8_t* codes, const uint8_t* sf, int64_t K, double g,
                     const int64_t* row_ids, int64_t nrows, double* out) {
    const int64_t G = (fmt == ORC_MX) ? 32 : 16, Kg = K / G;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nrows; ++t) {
        int64_t r = row_ids[t];
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            uint8_t sb = sf[orc_sf_offset(r, k / G, Kg)];
            double scale = (fmt == ORC_MX) ? orc_e8m0_decode(sb) : orc_e4m3_decode(sb) * g;
            out[t * K + k] = orc_e2m1_decode(c) * scale;
        }
    }
}

void orc_dequant_mxfp8(const uint8_t* elems, const uint8_t* sf, int64_t K, const int64_t* row_ids,
                       int64_t nrows, double* out) {
    const int64_t G = 32, Kg = K / G;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nrows; ++t) {
        int64_t r = row_ids[t];
        for (int64_t k = 0; k < K; ++k) {
            uint8_t sb = sf[orc_sf_offset(r, k / G, Kg)];
            out[t * K + k] = orc_e4m3_decode(elems[r * K + k]) * orc_e8m0_decode(sb);
        }
    }
}

/* ------------------------------------------------------------------------------------
 * The linear in fp64 (quantize-dequantize view): for the selected rows of A,
 *   Y[t, n] = sum_k A[t, k] * W[n, k] + bias[n]
 *   S[t, n] = sum_k |A[t, k] * W[n, k]|        (magnitude sum for the tolerance)
 * A is [nrows, K] fp64, W is [N, K] fp64, bias fp16 bits [N] or NULL.
 * Each sum runs over k in order; four output columns are processed side by side.
 * ---------------------------------------------------------------------------------- */
void orc_linear_fp64(const double* A, int64_t nrows, const double* W, int64_t N, int64_t K,
                     const uint16_t* bias, double* Y, double* S) {
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int64_t t = 0; t < nrows; ++t) {
        for (int64_t n0 = 0; n0 < N; n0 += 4) {
            const double* a = A + t * K;
            int64_t nn = (N - n0 < 4) ? (N - n0) : 4;
            for (int64_t q = 0; q < nn; ++q) {
                const double* w = W + (n0 + q) * K;
                double y = 0.0, s = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double p = a[k] * w[k];
                    y += p;
                    s += fabs(p);
                }
                if (bias) y += f16_to_double(bias[n0 + q]);
                Y[t * N + n0 + q] = y;
                S[t * N + n0 + q] = s;
            }
        }
    }
}

/* Low-rank term of the W4A8 SVDQuant linear (R7), for the selected rows:
 *   u[t, r]   = sum_k x[t, k] * L1[k, r]            (x: unquantized bf16 input)
 *   LR[t, n]  = sum_r u[t, r] * L2[r, n]
 *   LS[t, n]  = sum_r |u[t, r] * L2[r, n]|
 * x bf16 [*, K], L1 bf16 [K, rank], L2 bf16 [rank, N]. */
void orc_lowrank_fp64(const uint16_t* x, int64_t K, const int64_t* row_ids, int64_t nrows,
                      const uint16_t* l1, const uint16_t* l2, int64_t rank, int64_t N,
                      double* LR, double* LS) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nrows; ++t) {
        double u[256];
        int64_t r0 = row_ids[t];
        for (int64_t r = 0; r < rank; ++r) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)orc_bf16_to_f32(x[r0 * K + k]) * (double)orc_bf16_to_f32(l1[k * rank + r]);
            u[r] = acc;
        }
        for (int64_t n = 0; n < N; ++n) {
            double y = 0.0, s = 0.0;
            for (int64_t r = 0; r < rank; ++r) {
                double p = u[r] * (double)orc_bf16_to_f32(l2[r * N + n]);
                y += p;
                s += fabs(p);
            }
            LR[t * N + n] = y;
            LS[t * N + n] = s;
        }
    }
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
