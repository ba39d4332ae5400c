// attn.cuh -- FP4 attention beyond the score GEMM: the V operand quantized along tokens,
// the row softmax of the scores and its MXFP4 quantization (the P operand), all HBM-bound.
//
// Reading followed (the Wan2.2-Animate-14B MXFP4 card, "Results", names SageAttention v3 as
// Blackwell microscaling FP4 attention without giving its algorithm): P = softmax(S * scale)
// per query row over the T_kv keys, quantized in MXFP4 blocks of 32 consecutive keys; V of a
// head quantized per head-dim channel in MXFP4 blocks of 32 consecutive tokens; O = deq(P)
// deq(V) by the block-scaled GEMM (its K is the key axis, so both operands carry their
// scales along the keys).
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
// shared memory; thread d (a head-dim channel) quantizes the four 32-token groups of its
// column and writes their 64 code bytes and one scale word.
__global__ void __launch_bounds__(128) quant_vt_kernel(const __nv_bfloat16* __restrict__ v, int64_t T, int H,
                                                       int64_t tpad, uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ sf) {
    __shared__ __align__(16) __nv_bfloat16 tile[VT_TOKENS * VT_PITCH];
    const int tb = blockIdx.x, h = blockIdx.y;
    const int64_t t0 = (int64_t)tb * VT_TOKENS;
    const int64_t row_elems = (int64_t)H * 128;
    // 128 token rows x 256 bytes as 16-byte chunks: 2048 chunks over 128 threads
    for (int c = threadIdx.x; c < VT_TOKENS * 16; c += 128) {
        const int r = c >> 4, q = c & 15;
        uint4 w = make_uint4(0, 0, 0, 0);
        if (t0 + r < T) w = *reinterpret_cast<const uint4*>(v + (t0 + r) * row_elems + (int64_t)h * 128 + q * 8);
        *reinterpret_cast<uint4*>(tile + r * VT_PITCH + q * 8) = w;
    }
    __syncthreads();
    const int d = threadIdx.x;
    uint32_t word = 0;
    uint8_t* crow = codes + ((int64_t)h * 128 + d) * (tpad / 2) + t0 / 2;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        float x[32];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            x[i] = __bfloat162float(tile[(g * 32 + i) * VT_PITCH + d]);
            amax = fmaxf(amax, fabsf(x[i]));
        }
        const uint32_t sfb = mx_scale_byte<2>(amax);
        const float inv = mx_inv_scale(sfb);
        uint32_t cw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float e[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) e[i] = __fmul_rn(x[q * 8 + i], inv);
            cw[q] = cvt_e2m1x8(e);
        }
        *reinterpret_cast<uint4*>(crow + g * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        word |= sfb << (8 * g);
    }
    // head h's scales: rows = the 128 channels (one row block), atoms along the Tpad tokens
    const int64_t apr = tpad / 128;
    *reinterpret_cast<uint32_t*>(sf + (int64_t)h * apr * 512 + sf_word_offset(d, tb, apr)) = word;
}

// The softmax argument of a score in fp32, the same two roundings in both softmax kernels:
// t = fl(fl(s * c) - m), c = scale * log2(e), m = the row maximum of fl(s * c).
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

// Row statistics of the softmax: m = max_j fl(s_j c) over the T_kv valid keys and
// l = sum_j exp2(t_j), each thread summing its columns in order, then the fixed block tree.
// One block per query row; the row (T_kv_pad bf16) is read twice, the second time from L2.
__global__ void __launch_bounds__(SOFTMAX_THREADS) softmax_stats_kernel(const __nv_bfloat16* __restrict__ s,
                                                                       int64_t kpad, int64_t T_kv, float c,
                                                                       float2* __restrict__ stats) {
    __shared__ float red[SOFTMAX_THREADS / 32];
    const __nv_bfloat16* row = s + (int64_t)blockIdx.x * kpad;
    const int64_t nvec = kpad / 8;
    float m = -INFINITY;
    for (int64_t i = threadIdx.x; i < nvec; i += SOFTMAX_THREADS) {
        float v[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + i * 8), v);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i * 8 + k < T_kv) m = fmaxf(m, __fmul_rn(v[k], c));
    }
    m = block_reduce<true>(m, red);
    float l = 0.0f;
    for (int64_t i = threadIdx.x; i < nvec; i += SOFTMAX_THREADS) {
        float v[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + i * 8), v);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i * 8 + k < T_kv) l = __fadd_rn(l, exp2f(softmax_t(v[k], c, m)));
    }
    l = block_reduce<false>(l, red);
    if (threadIdx.x == 0) stats[blockIdx.x] = make_float2(m, l);
}

// P = exp2(t_j) * (1 / l), quantized in MXFP4 groups of 32 keys.  One block per query row
// of the padded [T_q_pad, T_kv_pad] layout; its 8 warps take 256-key chunks in turn, a lane
// 8 keys (16-byte load, 4-byte code store), 4 lanes a group.  Keys j >= T_kv give p = 0;
// rows >= T_q write only zero scale bytes (the layout's padding).
__global__ void __launch_bounds__(SOFTMAX_THREADS) softmax_quant_kernel(const __nv_bfloat16* __restrict__ s,
                                                                       int64_t T_q, int64_t kpad, int64_t T_kv,
                                                                       float c, const float2* __restrict__ stats,
                                                                       uint8_t* __restrict__ p_codes,
                                                                       uint8_t* __restrict__ p_sf) {
    const int64_t r = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t apr = kpad / 128;
    const bool real = r < T_q;
    float m = 0.0f, inv_l = 0.0f;
    if (real) {
        const float2 st = stats[r];
        m = st.x;
        inv_l = __frcp_rn(st.y);
    }
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
                p[k] = (col + k < T_kv) ? __fmul_rn(exp2f(softmax_t(v[k], c, m)), inv_l) : 0.0f;
                amax = fmaxf(amax, p[k]);
            }
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) p[k] = 0.0f;
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const uint32_t sfb = mx_scale_byte<2>(amax);
        if (real && in) {
            const float inv = mx_inv_scale(sfb);
#pragma unroll
            for (int k = 0; k < 8; ++k) p[k] = __fmul_rn(p[k], inv);
            *reinterpret_cast<uint32_t*>(p_codes + r * (kpad / 2) + col / 2) = cvt_e2m1x8(p);
        }
        // the 4 group bytes of each 128-key unit into one word (lanes 0-15: unit 2 chunk,
        // lanes 16-31: unit 2 chunk + 1)
        uint32_t word = sfb << (8 * ((lane & 15) >> 2));
        word |= __shfl_xor_sync(0xffffffffu, word, 4);
        word |= __shfl_xor_sync(0xffffffffu, word, 8);
        if ((lane & 15) == 0 && in)
            *reinterpret_cast<uint32_t*>(p_sf + sf_word_offset(r, chunk * 2 + (lane >> 4), apr)) = word;
    }
}

}  // namespace fp4
