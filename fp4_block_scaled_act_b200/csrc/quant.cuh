// quant.cuh -- activation / weight quantization kernels (HBM-bound).
//
// Work unit: 128 consecutive elements of one row (K is a multiple of 128), handled by
// 16 consecutive lanes with one 128-bit load each (8 bf16).  A warp holds two units.
// Units are numbered linearly over the [Mpad, K] buffer, so loads and code stores are
// fully contiguous.  Group amax is reduced with shuffles (4 lanes per 32-group, 2 lanes
// per 16-group); the group scale bytes of a unit are gathered by shuffle into 32-bit
// words and written straight into the 128x4 scale-factor atoms the tensor core reads.
// Rows in [M, Mpad) only write zero scale bytes (the layout's padding).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace fp4 {

enum QuantKind { Q_MXFP4 = 0, Q_NVFP4 = 1, Q_MXFP8 = 2 };

constexpr int QUANT_THREADS = 256;
constexpr int QUANT_UNROLL = 4;

FP4_DEV void bf16x8_to_f32(const uint4& u, float (&v)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Offset of the 32-bit word holding groups 4*atom_k .. 4*atom_k+3 of row r.
FP4_DEV int64_t sf_word_offset(int64_t r, int64_t atom_k, int64_t atoms_per_rowblock) {
    return ((r >> 7) * atoms_per_rowblock + atom_k) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4;
}

// MX scale byte from the group amax: 2^(floor(log2 amax) - emax) as E8M0, clamped at 0.
// amax >= 0 so its biased exponent field is floor(log2) + 127 for normals and 0 for
// zero / subnormals (which all clamp to byte 0).
template <int EMAX>
FP4_DEV uint32_t mx_scale_byte(float amax) {
    const int eb = (int)(__float_as_uint(amax) >> 23);
    return (uint32_t)max(eb - EMAX, 0);
}
// 2^-e for e = byte - 127, exact (byte <= 252 keeps the result a normal float).
FP4_DEV float mx_inv_scale(uint32_t byte) { return __uint_as_float((254u - byte) << 23); }

template <int KIND>
__global__ void __launch_bounds__(QUANT_THREADS) quant_kernel(const uint4* __restrict__ x, int64_t M, int64_t K,
                                                              const float* __restrict__ g_ptr,
                                                              uint8_t* __restrict__ out, uint8_t* __restrict__ sf) {
    // Each CTA owns a contiguous range of units; per pass its 16 half-warps take 16
    // consecutive units, QUANT_UNROLL passes are loaded before any is processed.  Row and
    // chunk of a unit are advanced incrementally (no per-unit division).
    constexpr uint32_t UPB = QUANT_THREADS / 16;  // units per pass
    const uint32_t upr = (uint32_t)(K >> 7);
    const uint32_t Mpad = (uint32_t)((M + 127) & ~int64_t(127));
    const uint32_t total = Mpad * upr;  // even: Mpad is a multiple of 128
    const uint32_t span = UPB * QUANT_UNROLL;
    const uint32_t per_cta = ((total + gridDim.x - 1) / gridDim.x + span - 1) / span * span;
    const uint32_t u_begin = blockIdx.x * per_cta;
    const uint32_t u_end = min(total, u_begin + per_cta);
    const int lane = threadIdx.x & 31;
    const int part = lane & 15;
    const uint32_t my = threadIdx.x >> 4;
    const uint32_t adv_rows = UPB / upr, adv_chunk = UPB % upr;

    float g = 1.0f, six_g = 6.0f;
    if (KIND == Q_NVFP4) {
        g = *g_ptr;
        six_g = __fmul_rn(6.0f, g);
    }
    // atoms (4 groups) per 128-row block along K
    const uint32_t apr = (KIND == Q_NVFP4) ? (uint32_t)(K >> 6) : upr;

    uint32_t row = (u_begin + my) / upr;
    uint32_t chunk = (u_begin + my) - row * upr;
    for (uint32_t ub = u_begin; ub < u_end; ub += span) {
        uint4 raw[QUANT_UNROLL];
        uint32_t rows[QUANT_UNROLL], chunks[QUANT_UNROLL];
#pragma unroll
        for (int it = 0; it < QUANT_UNROLL; ++it) {
            rows[it] = row;
            chunks[it] = chunk;
            const uint32_t u = ub + it * UPB + my;
            raw[it] = (u < u_end && row < (uint32_t)M) ? __ldcs(x + (size_t)u * 16 + part) : make_uint4(0, 0, 0, 0);
            chunk += adv_chunk;
            row += adv_rows;
            if (chunk >= upr) {
                chunk -= upr;
                ++row;
            }
        }
#pragma unroll
        for (int it = 0; it < QUANT_UNROLL; ++it) {
            const uint32_t u = ub + it * UPB + my;
            if (u >= u_end) break;  // uniform across the warp (ranges are even)
            float v[8];
            bf16x8_to_f32(raw[it], v);
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            if (KIND != Q_NVFP4) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));

            uint32_t sfb;
            if (KIND == Q_NVFP4) {
                const float s = __fdiv_rn(amax, six_g);
                sfb = cvt_e4m3x2(s, 0.0f) & 0xFFu;
                const float d = __fmul_rn(e4m3_to_f32(sfb), g);
                if (d == 0.0f) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = 0.0f;
                } else {
                    const float r = __frcp_rn(d);
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], r);
                }
            } else {
                sfb = mx_scale_byte<(KIND == Q_MXFP4) ? 2 : 8>(amax);
                const float inv = mx_inv_scale(sfb);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], inv);
            }

            if (rows[it] < (uint32_t)M) {
                if (KIND == Q_MXFP8) {
                    uint2 w;
                    w.x = cvt_e4m3x2(v[0], v[1]) | (cvt_e4m3x2(v[2], v[3]) << 16);
                    w.y = cvt_e4m3x2(v[4], v[5]) | (cvt_e4m3x2(v[6], v[7]) << 16);
                    reinterpret_cast<uint2*>(out)[(size_t)u * 16 + part] = w;
                } else {
                    reinterpret_cast<uint32_t*>(out)[(size_t)u * 16 + part] = cvt_e2m1x8(v);
                }
            }

            // gather the unit's scale bytes into 32-bit words (padding rows give zeros):
            // every lane of a group holds its group's byte; shift it to the group's slot and
            // OR across the 4 groups of a word
            uint32_t word;
            if (KIND == Q_NVFP4) {
                word = sfb << (8 * ((part >> 1) & 3));  // groups of 2 lanes, words of 8 lanes
                word |= __shfl_xor_sync(0xffffffffu, word, 2);
                word |= __shfl_xor_sync(0xffffffffu, word, 4);
                if ((part & 7) == 0)
                    *reinterpret_cast<uint32_t*>(sf + sf_word_offset(rows[it], chunks[it] * 2 + (part >> 3), apr)) =
                        word;
            } else {
                word = sfb << (8 * (part >> 2));        // groups of 4 lanes, one word per unit
                word |= __shfl_xor_sync(0xffffffffu, word, 4);
                word |= __shfl_xor_sync(0xffffffffu, word, 8);
                if (part == 0)
                    *reinterpret_cast<uint32_t*>(sf + sf_word_offset(rows[it], chunks[it], apr)) = word;
            }
        }
    }
}

// ---------------------------------------------------------------- tensor amax
// max |x| over n bf16 values; result accumulated as fp32 bits with atomicMax (values
// are non-negative, so their bit patterns order like the values).  *out must be zero
// before the launch.
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ x, int64_t n,
                                                   unsigned int* __restrict__ out) {
    float m = 0.0f;
    const int64_t nvec = n >> 3;
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = tid; i < nvec; i += stride) {
        float v[8];
        bf16x8_to_f32(__ldcs(xv + i), v);
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    }
    for (int64_t i = (nvec << 3) + tid; i < n; i += stride) m = fmaxf(m, fabsf(__uint_as_float((uint32_t)x[i] << 16)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float wm[8];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wm[w]);
        atomicMax(out, __float_as_uint(m));
    }
}

// In place: amax bits -> NVFP4 global g = T / 2688 (T = 0 gives 1).
__global__ void nv_global_kernel(float* g) {
    const float T = *g;
    *g = (T == 0.0f) ? 1.0f : __fdiv_rn(T, 2688.0f);
}

// ---------------------------------------------------------------- low-rank down-projection
// u[m, r] = sum_k x[m, k] * L1[k, r] in fp32, fixed summation order (k ascending), for the
// W4A8 SVDQuant linear.  Block: 256 threads, 32 rows x RANK outputs; K staged in chunks.
template <int RANK>
__global__ void __launch_bounds__(256) lowrank_down_kernel(const __nv_bfloat16* __restrict__ x,
                                                           const __nv_bfloat16* __restrict__ l1, int64_t M,
                                                           int64_t K, float* __restrict__ u) {
    constexpr int ROWS = 32, KC = 64;
    constexpr int RPT = ROWS * RANK / 256;  // rows per thread
    __shared__ float xs[ROWS][KC + 1];
    __shared__ float ls[KC][RANK];
    const int r = threadIdx.x % RANK;
    const int rg = threadIdx.x / RANK;  // 0 .. 256/RANK-1
    const int64_t m0 = (int64_t)blockIdx.x * ROWS;
    float acc[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) acc[i] = 0.0f;
    for (int64_t k0 = 0; k0 < K; k0 += KC) {
        for (int i = threadIdx.x; i < ROWS * KC; i += 256) {
            const int rr = i / KC, kk = i % KC;
            const int64_t m = m0 + rr;
            xs[rr][kk] = (m < M) ? __bfloat162float(x[m * K + k0 + kk]) : 0.0f;
        }
        for (int i = threadIdx.x; i < KC * RANK; i += 256) {
            const int kk = i / RANK, rr = i % RANK;
            ls[kk][rr] = __bfloat162float(l1[(k0 + kk) * RANK + rr]);
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < KC; ++kk) {
            const float l = ls[kk][r];
#pragma unroll
            for (int i = 0; i < RPT; ++i) acc[i] = __fmaf_rn(xs[rg * RPT + i][kk], l, acc[i]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int64_t m = m0 + rg * RPT + i;
        if (m < M) u[m * RANK + r] = acc[i];
    }
}

}  // namespace fp4
