// gelu.cuh -- GELU-tanh in fp32, evaluated in a fixed order of IEEE operations.
//
// The FFN of the Wan2.2 blocks applies GELU-tanh between its two quantized linears
// (ffn.net.0.proj -> ffn.net.2, the MXFP4 model cards' coverage lists):
//   gelu(z) = 0.5 z (1 + tanh(v)),  v = sqrt(2/pi) (z + 0.044715 z^3).
// The down projection quantizes bf16_rn(gelu(z)), so the integer codes depend on every
// rounding of this evaluation; it is therefore written out step by step (no library
// transcendental, no contracted multiply-add) as
//   q = 0.044715 (z z);  w = (q + 1) z;  a = w (-2 sqrt(2/pi))          [a = -2v]
//   a > 88:  gelu = z * 0     (exp(a) leaves fp32; the true value is below 2^-120)
//   else:    gelu = z / (1 + exp(max(a, -87)))    using 0.5 (1 + tanh v) = 1 / (1 + exp(-2v))
// with exp by Cody-Waite argument reduction (W. J. Cody and W. Waite, "Software Manual
// for the Elementary Functions", 1980): n = floor(a / ln2 + 1/2), r = (a - n ln2_hi) -
// n ln2_lo with a 16-bit ln2_hi (so n ln2_hi is exact), exp(r) for |r| <= ln2/2 by the
// degree-7 Taylor polynomial in Horner form, then the exact scaling by 2^n (a normal
// float for a in [-87, 88]).  Every constant is written exactly as an fp32 hex literal.
#pragma once
#include "ptx.cuh"

namespace fp4 {

FP4_DEV float exp_cw_f32(float a) {
    const float t = __fmul_rn(a, 0x1.715476p+0f);  // 1/ln2
    const float fn = floorf(__fadd_rn(t, 0.5f));
    const float r = __fsub_rn(__fsub_rn(a, __fmul_rn(fn, 0x1.62e4p-1f)), __fmul_rn(fn, 0x1.7f7d1cp-20f));
    float p = 0x1.a01a02p-13f;                          // 1/7!
    p = __fadd_rn(__fmul_rn(p, r), 0x1.6c16c2p-10f);    // 1/6!
    p = __fadd_rn(__fmul_rn(p, r), 0x1.111112p-7f);     // 1/5!
    p = __fadd_rn(__fmul_rn(p, r), 0x1.555556p-5f);     // 1/4!
    p = __fadd_rn(__fmul_rn(p, r), 0x1.555556p-3f);     // 1/3!
    p = __fadd_rn(__fmul_rn(p, r), 0.5f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    const int n = (int)fn;  // in [-126, 127] for a in [-87, 88]
    return __fmul_rn(p, __int_as_float((n + 127) << 23));
}

FP4_DEV float gelu_tanh_f32(float z) {
    const float q = __fmul_rn(0x1.6e4e26p-5f, __fmul_rn(z, z));  // 0.044715 z^2
    const float w = __fmul_rn(__fadd_rn(q, 1.0f), z);
    float a = __fmul_rn(w, -0x1.988454p+0f);  // -2 sqrt(2/pi)
    if (a > 88.0f) return __fmul_rn(z, 0.0f);
    a = fmaxf(a, -87.0f);
    return __fdiv_rn(z, __fadd_rn(1.0f, exp_cw_f32(a)));
}

// bf16_rn(gelu(z)) as an fp32 value
FP4_DEV float gelu_bf16_f32(float z) { return __bfloat162float(__float2bfloat16_rn(gelu_tanh_f32(z))); }

}  // namespace fp4
