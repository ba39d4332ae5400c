// gelu.cuh -- GELU-tanh in fp32 for the fused FFN activation.
//
// The FFN of the Wan2.2 blocks applies GELU-tanh between its two quantized linears
// (ffn.net.0.proj -> ffn.net.2, the MXFP4 model cards' coverage lists):
//   gelu(z) = 0.5 z (1 + tanh(v)),  v = sqrt(2/pi) (z + 0.044715 z^3).
// The down projection quantizes h = bf16_rn(gelu(z)).  This file evaluates gelu in fp32
// with no library transcendental and no division, in a fixed order of IEEE fp32
// operations (fused multiply-adds included), on pairs of values with the packed f32x2
// operations of sm_100:
//   q = z z;  p = q 0.044715;  w = fma(p, z, z)                  [w = z + 0.044715 z^3]
//   t = w (-2 sqrt(2/pi) / ln 2)                                 [exp(-2v) = 2^t]
//   t > 125:  gelu = z * 0   (the true value is below 2^-118 |z|)
//   else:     t = max(t, -126)
//             2^t: n = (t + 1.5 2^23) - 1.5 2^23 (t rounded to the nearest integer, ties
//             to even, by two additions), f = t - n (exact, |f| <= 1/2), 2^f by the
//             degree-6 Taylor polynomial in ln2 f (Horner with fma; truncation error
//             below 2^-22 on |f| <= 1/2), times 2^n exactly
//             d = 1 + 2^t;  y = 1/d by Newton-Raphson from a guess read off the bits
//             of d, three steps r = fma(-d, y, 1), y = fma(y, r, y)
//             gelu = z y           using 0.5 (1 + tanh v) = 1 / (1 + exp(-2v))
// The reciprocal guess: the bits of a positive float read as an integer are, to first
// order, 2^23 (log2 x + 127 - c) for a small bias c, so bits(1/d) ~ K - bits(d) with
// K = 2^24 (127 - c).  The relative error |d y0 - 1| of y0 = K - bits(d) depends only on
// d's mantissa; K = 0x7EF311C2 minimizes its maximum over a binade (0.0505, found by
// exhaustive search over the 2^23 mantissas), and three Newton steps, each squaring the
// error, leave 0.0505^8 < 2^-34 before rounding.
// Error bound (checked on the GPU for every finite bf16 z against the fp64 definition):
// |gelu_f32(z) - gelu(z)| <= (2 |a| + 16) 2^-23 |gelu(z)| + 2^-126, a = -2v, and for
// t > 125 the result is a zero of z's sign.  h is the nearest bf16 to gelu_f32(z), so it
// equals the correctly rounded bf16 of gelu(z) except where gelu(z) lies within that bound
// of a rounding midpoint, where it may be the other neighbour.
#pragma once
#include "ptx.cuh"

namespace fp4 {

// bf16_rn of a finite fp32 value, returned as fp32 (round to nearest even on the bits)
FP4_DEV float bf16_rn_f32(float g) {
    uint32_t u = __float_as_uint(g);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return __uint_as_float(u & 0xFFFF0000u);
}

// gelu_tanh(z) in fp32 for the pair (z0, z1), before the bf16 rounding
FP4_DEV void gelu_f32_x2(float z0, float z1, float& g0, float& g1) {
    const uint64_t z = f2_pack(z0, z1);
    const uint64_t p = f2_mul(f2_mul(z, z), f2_splat(0x1.6e4e26p-5f));  // 0.044715 z^2
    const uint64_t w = f2_fma(p, z, z);                                  // z + 0.044715 z^3
    float t0, t1;
    f2_unpack(f2_mul(w, f2_splat(-0x1.26aec2p+1f)), t0, t1);            // -2 sqrt(2/pi) / ln2
    const bool cut0 = t0 > 125.0f, cut1 = t1 > 125.0f;
    const uint64_t t = f2_pack(fminf(fmaxf(t0, -126.0f), 125.0f), fminf(fmaxf(t1, -126.0f), 125.0f));
    // 2^t
    const uint64_t big = f2_add(t, f2_splat(0x1.8p23f));
    const uint64_t f = f2_sub(t, f2_sub(big, f2_splat(0x1.8p23f)));
    uint64_t e = f2_splat(0x1.430912p-13f);                // (ln2)^6 / 6!
    e = f2_fma(e, f, f2_splat(0x1.5d87fep-10f));           // (ln2)^5 / 5!
    e = f2_fma(e, f, f2_splat(0x1.3b2ab6p-7f));            // (ln2)^4 / 4!
    e = f2_fma(e, f, f2_splat(0x1.c6b08ep-5f));            // (ln2)^3 / 3!
    e = f2_fma(e, f, f2_splat(0x1.ebfbe0p-3f));            // (ln2)^2 / 2!
    e = f2_fma(e, f, f2_splat(0x1.62e430p-1f));            // ln2
    e = f2_fma(e, f, f2_splat(1.0f));
    float b0, b1;
    f2_unpack(big, b0, b1);  // n in the low mantissa bits of big
    const uint64_t s2 = f2_pack(__uint_as_float((__float_as_uint(b0) - 0x4B400000u + 127u) << 23),
                                __uint_as_float((__float_as_uint(b1) - 0x4B400000u + 127u) << 23));
    const uint64_t d = f2_add(f2_splat(1.0f), f2_mul(e, s2));
    // y = 1/d by Newton-Raphson from the exponent-bit guess
    float d0, d1;
    f2_unpack(d, d0, d1);
    uint64_t y = f2_pack(__uint_as_float(0x7EF311C2u - __float_as_uint(d0)),
                         __uint_as_float(0x7EF311C2u - __float_as_uint(d1)));
    const uint64_t nd = d ^ 0x8000000080000000ull;  // -d, exactly
#pragma unroll
    for (int i = 0; i < 3; ++i) y = f2_fma(y, f2_fma(nd, y, f2_splat(1.0f)), y);
    f2_unpack(f2_mul(z, y), g0, g1);
    if (cut0) g0 = __fmul_rn(z0, 0.0f);
    if (cut1) g1 = __fmul_rn(z1, 0.0f);
}

// h = bf16_rn(gelu_tanh(z)) for the pair (z0, z1)
FP4_DEV void gelu_bf16_x2(float z0, float z1, float& h0, float& h1) {
    float g0, g1;
    gelu_f32_x2(z0, z1, g0, g1);
    h0 = bf16_rn_f32(g0);
    h1 = bf16_rn_f32(g1);
}

}  // namespace fp4
