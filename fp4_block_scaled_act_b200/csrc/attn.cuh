// attn.cuh -- FP4 attention beyond the score GEMM: the V operand quantized along tokens,
// the row softmax of the scores and its MXFP4 quantization (the P operand), all HBM-bound.
//
// Reading followed (the Wan2.2-Animate-14B MXFP4 card, "Results", names SageAttention v3 as
// Blackwell microscaling FP4 attention without giving its algorithm): per query row, the
// unnormalized softmax weights P~ = 2^(s c - max) (c = scale log2 e; the largest is exactly
// 1) over the T_kv keys, quantized in blocks of G consecutive keys, and their fp32 sum l; V of
// a head quantized per head-dim channel in blocks of G consecutive tokens; O = deq(P~) deq(V)
// by the block-scaled GEMM (its K is the key axis, so both operands carry their scales along
// the keys), then each row divided by its l.  MXFP4: G = 32, E8M0 scales.  NVFP4: G = 16,
// E4M3 scales under one fp32 global per tensor (V's from its amax; P~'s is a caller's
// constant, 1 / 2688 for p <= 1), by the same steps as the activation quantizer.
//
// Layouts (head-major, as the score operands):
//   V^T  codes [H][128 dims][Tpad/2] bytes (tokens along K; padding tokens hold zero codes),
//        scales per head: the atom layout of a [128, Tpad] matrix, heads one after another.
//   P    codes [T_q][T_kv_pad/2], scales: the atom layout of a [T_q, T_kv_pad] matrix
//        (padding keys and padding query rows get zero codes / zero scale bytes).
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace fp4 {

constexpr int VT_TOKENS = 128;  // tokens per V^T quantizer block (one scale atom along K)
constexpr int VT_PITCH = 136;   // bf16 elements per staged token row (16 bytes of padding)
constexpr int SOFTMAX_THREADS = 256;

// V^T quantizer: block (token block tb, head h) stages V[tb*128 .. +127][h*128 .. +127] in
// shared memory; thread d (a head-dim channel) quantizes the 128 / G groups of its column
// and writes their 64 code bytes and its scale word(s) (one MXFP4 atom, two NVFP4 atoms).
template <int KIND>
__global__ void __launch_bounds__(128) quant_vt_kernel(const __nv_bfloat16* __restrict__ v, int64_t T, int H,
                                                       int64_t tpad, const float* __restrict__ g_ptr,
                                                       uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
    constexpr int G = (KIND == Q_NVFP4) ? 16 : 32;
    __shared__ __align__(16) __nv_bfloat16 tile[VT_TOKENS * VT_PITCH];
    __shared__ float nv_rcp[128];
    const int tb = blockIdx.x, h = blockIdx.y;
    const int64_t t0 = (int64_t)tb * VT_TOKENS;
    const int64_t row_elems = (int64_t)H * 128;
    float six_g = 6.0f;
    if (KIND == Q_NVFP4) {
        // 1 / (e4m3(sf) * g) for every scale byte, by the activation quantizer's operations
        const float g = *g_ptr;
        six_g = __fmul_rn(6.0f, g);
        const float d = __fmul_rn(e4m3_to_f32(threadIdx.x), g);
        nv_rcp[threadIdx.x] = d == 0.0f ? 0.0f : __frcp_rn(d);
    }
    // 128 token rows x 256 bytes as 16-byte chunks: 2048 chunks over 128 threads
    for (int c = threadIdx.x; c < VT_TOKENS * 16; c += 128) {
        const int r = c >> 4, q = c & 15;
        uint4 w = make_uint4(0, 0, 0, 0);
        if (t0 + r < T) w = *reinterpret_cast<const uint4*>(v + (t0 + r) * row_elems + (int64_t)h * 128 + q * 8);
        *reinterpret_cast<uint4*>(tile + r * VT_PITCH + q * 8) = w;
    }
    __syncthreads();
    const int d = threadIdx.x;
    uint32_t words[2] = {0u, 0u};
    uint8_t* crow = codes + ((int64_t)h * 128 + d) * (tpad / 2) + t0 / 2;
#pragma unroll
    for (int g = 0; g < 128 / G; ++g) {
        float x[G];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < G; ++i) {
            x[i] = __bfloat162float(tile[(g * G + i) * VT_PITCH + d]);
            amax = fmaxf(amax, fabsf(x[i]));
        }
        uint32_t sfb;
        if (KIND == Q_NVFP4) {
            sfb = cvt_e4m3x2(__fdiv_rn(amax, six_g), 0.0f) & 0xFFu;
            const float r = nv_rcp[sfb & 0x7Fu];
#pragma unroll
            for (int i = 0; i < G; ++i) x[i] = (r == 0.0f) ? 0.0f : __fmul_rn(x[i], r);
        } else {
            sfb = mx_scale_byte<2>(amax);
            const float inv = mx_inv_scale(sfb);
#pragma unroll
            for (int i = 0; i < G; ++i) x[i] = __fmul_rn(x[i], inv);
        }
        uint32_t cw[G / 8];
#pragma unroll
        for (int q = 0; q < G / 8; ++q) cw[q] = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(x + 8 * q));
        if constexpr (G == 32)
            *reinterpret_cast<uint4*>(crow + g * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        else
            *reinterpret_cast<uint2*>(crow + g * 8) = make_uint2(cw[0], cw[1]);
        words[g >> 2] |= sfb << (8 * (g & 3));
    }
    // head h's scales: rows = the 128 channels (one row block), atoms along the Tpad tokens
    constexpr int ATOMS = 128 / (G * 4);  // atoms per 128 tokens: MXFP4 1, NVFP4 2
    const int64_t apr = tpad / (G * 4);
#pragma unroll
    for (int a = 0; a < ATOMS; ++a)
        *reinterpret_cast<uint32_t*>(sf + (int64_t)h * apr * 512 + sf_word_offset(d, (int64_t)tb * ATOMS + a, apr)) =
            words[a];
}

// The softmax argument of a score in fp32: t = fl(fl(s * c) - m), c = scale * log2(e), m =
// the row maximum of fl(s * c) (softmax_max_kernel), so the largest score gives t = 0.
FP4_DEV float softmax_t(float s, float c, float m) { return __fsub_rn(__fmul_rn(s, c), m); }

// Block reduction in a fixed order (warp shuffles, then the warp results in index order).
template <bool MAX, int NT = SOFTMAX_THREADS>
FP4_DEV float block_reduce(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float w = __shfl_xor_sync(0xffffffffu, v, o);
        v = MAX ? fmaxf(v, w) : __fadd_rn(v, w);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();  // red[] is free again
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = red[0];
    for (int i = 1; i < NT / 32; ++i) r = MAX ? fmaxf(r, red[i]) : __fadd_rn(r, red[i]);
    return r;
}

// Row maximum of the softmax argument: m = max_j fl(s_j c) over the T_kv valid keys (one
// block per query row; a maximum is exact, so the order does not matter).
__global__ void __launch_bounds__(SOFTMAX_THREADS) softmax_max_kernel(const __nv_bfloat16* __restrict__ s,
                                                                     int64_t kpad, int64_t T_kv, float c,
                                                                     float2* __restrict__ stats) {
    __shared__ float red[SOFTMAX_THREADS / 32];
    const __nv_bfloat16* row = s + (int64_t)blockIdx.x * kpad;
    const int64_t nvec = kpad / 8;
    float m = -INFINITY;
    for (int64_t i = threadIdx.x; i < nvec; i += SOFTMAX_THREADS) {
        float v[8];
        bf16x8_to_f32(__ldcs(reinterpret_cast<const uint4*>(row + i * 8)), v);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i * 8 + k < T_kv) m = fmaxf(m, __fmul_rn(v[k], c));
    }
    m = block_reduce<true>(m, red);
    if (threadIdx.x == 0) stats[blockIdx.x] = make_float2(m, 0.0f);
}

// P~ = exp2(t_j), quantized in groups of G keys (MXFP4 32, NVFP4 16 under the global
// *g_ptr), and the row sum l = sum_j P~_j in fp32 (each thread adds its keys in order, then
// the fixed block tree) into stats[r].y.  One block per query row of the padded
// [T_q_pad, T_kv_pad] layout; its 8 warps take 256-key chunks in turn, a lane 8 keys
// (16-byte load, 4-byte code store), G / 8 lanes a group.  Keys j >= T_kv give p = 0; rows
// >= T_q write only zero scale bytes (the layout's padding).
template <int KIND>
__global__ void __launch_bounds__(SOFTMAX_THREADS) softmax_quant_kernel(const __nv_bfloat16* __restrict__ s,
                                                                       int64_t T_q, int64_t kpad, int64_t T_kv,
                                                                       float c, float2* __restrict__ stats,
                                                                       const float* __restrict__ g_ptr,
                                                                       uint8_t* __restrict__ p_codes,
                                                                       uint8_t* __restrict__ p_sf) {
    constexpr int G = (KIND == Q_NVFP4) ? 16 : 32;
    __shared__ float nv_rcp[128];
    __shared__ float red[SOFTMAX_THREADS / 32];
    const int64_t r = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t apr = kpad / (G * 4);
    const bool real = r < T_q;
    float six_g = 6.0f;
    if (KIND == Q_NVFP4) {
        const float g = *g_ptr;
        six_g = __fmul_rn(6.0f, g);
        if (threadIdx.x < 128) {
            const float d = __fmul_rn(e4m3_to_f32(threadIdx.x), g);
            nv_rcp[threadIdx.x] = d == 0.0f ? 0.0f : __frcp_rn(d);
        }
        __syncthreads();
    }
    const float m = real ? stats[r].x : 0.0f;
    float l = 0.0f;
    for (int64_t chunk = warp; chunk * 256 < kpad; chunk += SOFTMAX_THREADS / 32) {
        const int64_t col = chunk * 256 + lane * 8;
        const bool in = col < kpad;  // T_kv_pad = 128 (mod 256): the last chunk's upper half is absent
        float p[8];
        float amax = 0.0f;
        if (real && in) {
            float v[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(s + r * kpad + col), v);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                p[k] = (col + k < T_kv) ? exp2f(softmax_t(v[k], c, m)) : 0.0f;
                l = __fadd_rn(l, p[k]);
                amax = fmaxf(amax, p[k]);
            }
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) p[k] = 0.0f;
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        if (G == 32) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        uint32_t sfb;
        if (KIND == Q_NVFP4) {
            sfb = cvt_e4m3x2(__fdiv_rn(amax, six_g), 0.0f) & 0xFFu;
            const float rr = nv_rcp[sfb & 0x7Fu];
#pragma unroll
            for (int k = 0; k < 8; ++k) p[k] = (rr == 0.0f) ? 0.0f : __fmul_rn(p[k], rr);
        } else {
            sfb = mx_scale_byte<2>(amax);
            const float inv = mx_inv_scale(sfb);
#pragma unroll
            for (int k = 0; k < 8; ++k) p[k] = __fmul_rn(p[k], inv);
        }
        if (real && in) *reinterpret_cast<uint32_t*>(p_codes + r * (kpad / 2) + col / 2) = cvt_e2m1x8(p);
        // the 4 group bytes of each atom word: MXFP4 16 lanes (128 keys) per word, NVFP4 8 (64)
        constexpr int LW = G / 2;  // lanes per word
        uint32_t word = sfb << (8 * ((lane % LW) / (G / 8)));
        word |= __shfl_xor_sync(0xffffffffu, word, G / 8);
        word |= __shfl_xor_sync(0xffffffffu, word, G / 4);
        if (lane % LW == 0 && in)
            *reinterpret_cast<uint32_t*>(p_sf + sf_word_offset(r, (chunk * 256 + lane * 8) / (G * 4), apr)) = word;
    }
    l = block_reduce<false>(l, red);  // uniform per block: real is the same for every thread
    if (real && threadIdx.x == 0) stats[r].y = l;
}

// O's rows divided by their softmax sums, in place: o = bf16_rn(o * fl(1 / l)).
__global__ void __launch_bounds__(256) attn_row_scale_kernel(__nv_bfloat16* __restrict__ o, int64_t rows, int D,
                                                             const float2* __restrict__ stats) {
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;  // one 8-element vector
    const int64_t per_row = D / 8;
    if (i >= rows * per_row) return;
    const float inv = __frcp_rn(stats[i / per_row].y);
    uint4 w = *reinterpret_cast<uint4*>(o + i * 8);
    float v[8];
    bf16x8_to_f32(w, v);
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(v[2 * k], inv), __fmul_rn(v[2 * k + 1], inv));
        out[k] = *reinterpret_cast<uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(o + i * 8) = make_uint4(out[0], out[1], out[2], out[3]);
}

}  // namespace fp4
