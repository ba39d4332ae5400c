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

#include "gelu.cuh"
#include "ptx.cuh"

namespace fp4 {

enum QuantKind { Q_MXFP4 = 0, Q_NVFP4 = 1, Q_MXFP8 = 2 };

constexpr int QUANT_THREADS = 256;
constexpr int QUANT_UNROLL = 6;  // units in flight per half-warp (measured best of 4, 6, 8 at 75600 x 5120)

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

// GELU = true: the input is the bf16 up-projection output z and the quantized value is
// bf16_rn(gelu_tanh(z)) (gelu.cuh), the down projection's activation.
// HEADS = true: x is [M tokens, H heads x 128] (attention Q or K, head_dim 128), so a unit
// is one token's head (chunk = head), and the output is head-major: codes
// [H][Mpad][64 bytes] (padding tokens get zero codes) and per head the scale atoms of a
// [Mpad, 128] matrix, heads one after another.  Each head's codes and scales are then the
// A or B operand layout of a GEMM with K = head_dim.
template <int KIND, bool GELU = false, bool HEADS = false>
__global__ void __launch_bounds__(QUANT_THREADS, 4) quant_kernel(const uint4* __restrict__ x, int64_t M, int64_t K,
                                                              const float* __restrict__ g_ptr,
                                                              uint8_t* __restrict__ out, uint8_t* __restrict__ sf) {
    // Each CTA owns a contiguous range of units; per pass its 16 half-warps take 16
    // consecutive units, QUANT_UNROLL passes are loaded before any is processed.  Row and
    // chunk of a unit are advanced incrementally (no per-unit division).
    // a GEMM launched after us with programmatic serialization may be scheduled now (its
    // prologue overlaps our work; it still waits for our completion before reading)
    griddep_launch_dependents();
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
    // NVFP4: the group's decoded scale d = e4m3(sf) * g takes one of at most 127 values per
    // tensor (sf = 0 .. 0x7E, amax >= 0), so the reciprocal 1 / d is tabulated once per CTA
    // by the same operations; 0 marks d = 0 (no finite d > 0 has a zero reciprocal)
    __shared__ float nv_rcp[128];
    if (KIND == Q_NVFP4) {
        g = *g_ptr;
        six_g = __fmul_rn(6.0f, g);
        if (threadIdx.x < 128) {
            const float d = __fmul_rn(e4m3_to_f32(threadIdx.x), g);
            nv_rcp[threadIdx.x] = d == 0.0f ? 0.0f : __frcp_rn(d);
        }
        __syncthreads();
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
            if (GELU) {
#pragma unroll
                for (int i = 0; i < 8; i += 2) gelu_bf16_x2(v[i], v[i + 1], v[i], v[i + 1]);
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            if (KIND != Q_NVFP4) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));

            uint32_t sfb;
            if (KIND == Q_NVFP4) {
                const float s = __fdiv_rn(amax, six_g);
                sfb = cvt_e4m3x2(s, 0.0f) & 0xFFu;
                const float r = nv_rcp[sfb & 0x7Fu];  // sfb <= 0x7E: s >= 0, satfinite
                if (r == 0.0f) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = 0.0f;
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], r);
                }
            } else {
                sfb = mx_scale_byte<(KIND == Q_MXFP4) ? 2 : 8>(amax);
                const float inv = mx_inv_scale(sfb);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], inv);
            }

            if (HEADS) {
                static_assert(!HEADS || KIND != Q_MXFP8, "head-major output is FP4 only");
                reinterpret_cast<uint32_t*>(out)[((size_t)chunks[it] * Mpad + rows[it]) * 16 + part] = cvt_e2m1x8(v);
            } else if (rows[it] < (uint32_t)M) {
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
                if ((part & 7) == 0) {
                    if (HEADS)  // head chunks[it]: two atoms per row block
                        *reinterpret_cast<uint32_t*>(sf + (size_t)chunks[it] * (Mpad >> 7) * 1024 +
                                                     sf_word_offset(rows[it], part >> 3, 2)) = word;
                    else
                        *reinterpret_cast<uint32_t*>(sf + sf_word_offset(rows[it], chunks[it] * 2 + (part >> 3), apr)) =
                            word;
                }
            } else {
                word = sfb << (8 * (part >> 2));        // groups of 4 lanes, one word per unit
                word |= __shfl_xor_sync(0xffffffffu, word, 4);
                word |= __shfl_xor_sync(0xffffffffu, word, 8);
                if (part == 0) {
                    if (HEADS)  // head chunks[it]: one atom per row block
                        *reinterpret_cast<uint32_t*>(sf + (size_t)chunks[it] * (Mpad >> 7) * 512 +
                                                     sf_word_offset(rows[it], 0, 1)) = word;
                    else
                        *reinterpret_cast<uint32_t*>(sf + sf_word_offset(rows[it], chunks[it], apr)) = word;
                }
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

// NVFP4 global g = T / 2688 (T = 0 gives 1), one IEEE fp32 division.
FP4_DEV float nv_global_of(float T) { return (T == 0.0f) ? 1.0f : __fdiv_rn(T, 2688.0f); }

// In place: amax bits -> NVFP4 global.
__global__ void nv_global_kernel(float* g) { *g = nv_global_of(*g); }

// g_out = NVFP4 global of the amax in *amax (kept).
__global__ void nv_global_from_kernel(const float* amax, float* g_out) { *g_out = nv_global_of(*amax); }

// ---------------------------------------------------------------- low-rank down-projection
// W4A8 SVDQuant: u[m, r] = sum_k x[m, k] * L1[k, r] (rank 32) with bf16 inputs and fp32
// accumulation, on the warp-level tensor-core MMA (mma.sync m16n8k16): a skinny,
// HBM-bound contraction (the kernel is bound by reading X), for which the warp-level MMA
// is ample.  The result is stored as a bf16 pair per value, hi = bf16(u), lo = bf16(u - hi)
// (u_pair[m][r] = hi, u_pair[m][32 + r] = lo), so the GEMM can add u L2 on the tensor core
// as u_hi L2 + u_lo L2 with |u - hi - lo| <= 2^-18 |u|.
// Block: 256 threads = 8 warps x 16 rows = 128 rows, all 32 ranks; K in 64-element chunks
// through a ring of LR_STAGES cp.async stages.  At the W4A8 shape (4290 rows) only 34 blocks
// exist, each streaming 786 KB of X, so bytes in flight per SM set the speed: with two
// stages the kernel took 33 us (about 32 GB/s per SM), hence a deep ring.
constexpr int LR_ROWS = 128, LR_THREADS = 256, LR_KC = 64, LR_STAGES = 6;
constexpr int LR_XP = LR_KC + 8;  // padded X row (elements): conflict-free ldmatrix
constexpr int LR_LP = 32 + 8;     // padded L1 row
constexpr int LR_SMEM_BYTES = LR_STAGES * (LR_ROWS * LR_XP + LR_KC * LR_LP) * 2;  // dynamic shared memory
constexpr int LR_NO_QUANT = -1;

FP4_DEV void cp_async16(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
FP4_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
FP4_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Split K (partial != nullptr): block (i, j) covers chunks [j * kc_per_split, (j + 1) *
// kc_per_split) of row block i and writes its fp32 sums to partial[j][m][r] (rows padded to
// whole blocks); lowrank_reduce_kernel adds the splits in index order.  Otherwise the block
// covers all of K and writes the pair itself.
// The same pass can quantize X (QK = Q_MXFP8 for W4A8, Q_MXFP4 for W4A4 SVDQuant; LR_NO_QUANT
// for the projection alone): every chunk,
// once it has fed the MMAs, is read back from its stage by groups of 32 (thread t: group t & 1
// of row t >> 1) and turned into codes and E8M0 scale bytes by the steps quant_kernel takes,
// so X crosses HBM once for both results.  Rows in [M, Mpad) get zero scale bytes.
template <int QK>
__global__ void __launch_bounds__(LR_THREADS) lowrank_down_kernel(const __nv_bfloat16* __restrict__ x,
                                                                  const __nv_bfloat16* __restrict__ l1, int M,
                                                                  int K, __nv_bfloat16* __restrict__ u_pair,
                                                                  float* __restrict__ partial, int kc_per_split,
                                                                  uint8_t* __restrict__ codes,
                                                                  uint8_t* __restrict__ sf) {
    static_assert(QK == Q_MXFP8 || QK == Q_MXFP4 || QK == LR_NO_QUANT, "MX activations or none");
    extern __shared__ __align__(16) uint8_t lr_smem[];
    auto xs = reinterpret_cast<__nv_bfloat16(*)[LR_ROWS][LR_XP]>(lr_smem);
    auto ls = reinterpret_cast<__nv_bfloat16(*)[LR_KC][LR_LP]>(lr_smem + LR_STAGES * LR_ROWS * LR_XP * 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * LR_ROWS;
    const int nkc = partial ? kc_per_split : K / LR_KC;
    const int kc0 = partial ? (int)blockIdx.y * kc_per_split : 0;

    auto load = [&](int kc, int st) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // X: 128 rows x 8 pieces of 16 bytes
            const int idx = tid + i * LR_THREADS;
            const int row = idx >> 3, c = idx & 7;
            const bool ok = m0 + row < M;
            const __nv_bfloat16* src = ok ? x + (size_t)(m0 + row) * K + (kc0 + kc) * LR_KC + c * 8 : x;
            cp_async16(&xs[st][row][c * 8], src, ok);
        }
        {  // L1: 64 rows x 4 pieces of 16 bytes
            const int row = tid >> 2, c = tid & 3;
            cp_async16(&ls[st][row][c * 8], l1 + (size_t)((kc0 + kc) * LR_KC + row) * 32 + c * 8, true);
        }
        cp_async_commit();
    };

    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.0f;

    // prologue: chunks 0 .. LR_STAGES - 2 in flight (one commit group per chunk; empty groups
    // past the end keep the count uniform, so "chunk kc landed" is "at most LR_STAGES - 2
    // groups pending")
#pragma unroll
    for (int c = 0; c < LR_STAGES - 1; ++c) {
        if (c < nkc)
            load(c, c);
        else
            cp_async_commit();
    }
    for (int kc = 0; kc < nkc; ++kc) {
        const int st = kc % LR_STAGES;
        cp_async_wait<LR_STAGES - 2>();
        __syncthreads();
        // refill the stage chunk kc - 1 used: every thread is past it (the barrier above)
        const int nk = kc + LR_STAGES - 1;
        if (nk < nkc)
            load(nk, nk % LR_STAGES);
        else
            cp_async_commit();
#pragma unroll
        for (int ks = 0; ks < LR_KC / 16; ++ks) {
            uint32_t a[4];
            const uint32_t aaddr = smem_u32(&xs[st][warp * 16 + (lane & 15)][ks * 16 + (lane >> 4) * 8]);
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                         : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                         : "r"(aaddr));
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b[4];
                const uint32_t baddr = smem_u32(&ls[st][ks * 16 + (lane & 15)][np * 16 + (lane >> 4) * 8]);
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
                             : "r"(baddr));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float* d = acc[np * 2 + h];
                    asm volatile(
                        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                        "{%8, %9}, {%0, %1, %2, %3};"
                        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[2 * h]), "r"(b[2 * h + 1]));
                }
            }
        }
        // quantize the chunk from the stage (it is refilled only after the next barrier)
        if constexpr (QK != LR_NO_QUANT) {
            const int qr = tid >> 1, qg = tid & 1;
            const int m = m0 + qr;
            const int col = (kc0 + kc) * LR_KC + qg * 32;  // the group's first column
            const uint4* src = reinterpret_cast<const uint4*>(&xs[st][qr][qg * 32]);
            float v[32];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float w[8];
                bf16x8_to_f32(src[i], w);
#pragma unroll
                for (int e = 0; e < 8; ++e) v[8 * i + e] = w[e];
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
            const uint32_t sfb = mx_scale_byte<(QK == Q_MXFP4) ? 2 : 8>(amax);
            const float inv = mx_inv_scale(sfb);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], inv);
            if (m < M) {
                if (QK == Q_MXFP8) {
                    uint32_t c[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        c[i] = cvt_e4m3x2(v[4 * i], v[4 * i + 1]) | (cvt_e4m3x2(v[4 * i + 2], v[4 * i + 3]) << 16);
                    uint4* dst = reinterpret_cast<uint4*>(codes + (size_t)m * K + col);
                    dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
                    dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
                } else {
                    uint32_t c[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float e8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) e8[e] = v[8 * i + e];
                        c[i] = cvt_e2m1x8(e8);
                    }
                    *reinterpret_cast<uint4*>(codes + (size_t)m * (K / 2) + col / 2) = make_uint4(c[0], c[1], c[2], c[3]);
                }
            }
            const int j = col >> 5;  // group index in the row: byte j & 3 of atom word j >> 2
            sf[sf_word_offset(m, j >> 2, K >> 7) + (j & 3)] = (uint8_t)sfb;
        }
    }
    // accumulator fragment: acc[j][0..1] -> row lane/4, acc[j][2..3] -> row lane/4 + 8,
    // columns 8j + 2(lane%4) + {0, 1}
    if (partial) {
        const size_t mpad = (size_t)gridDim.x * LR_ROWS;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int m = m0 + warp * 16 + (lane >> 2) + half * 8;
            float* row = partial + ((size_t)blockIdx.y * mpad + m) * 32;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<float2*>(row + j * 8 + 2 * (lane & 3)) =
                    make_float2(acc[j][2 * half], acc[j][2 * half + 1]);
        }
        return;
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int m = m0 + warp * 16 + (lane >> 2) + half * 8;
        if (m >= M) continue;
        __nv_bfloat16* row = u_pair + (size_t)m * 64;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = j * 8 + 2 * (lane & 3);
            const float u0 = acc[j][2 * half], u1 = acc[j][2 * half + 1];
            const __nv_bfloat16 h0 = __float2bfloat16_rn(u0), h1 = __float2bfloat16_rn(u1);
            const __nv_bfloat16 l0 = __float2bfloat16_rn(u0 - __bfloat162float(h0));
            const __nv_bfloat16 l1v = __float2bfloat16_rn(u1 - __bfloat162float(h1));
            *reinterpret_cast<__nv_bfloat162*>(row + c) = __halves2bfloat162(h0, h1);
            *reinterpret_cast<__nv_bfloat162*>(row + 32 + c) = __halves2bfloat162(l0, l1v);
        }
    }
}

// u[m][r] = the splits' partial sums added in split order (a fixed order: the result does not
// depend on scheduling), stored as the bf16 pair hi, lo like lowrank_down_kernel.
__global__ void __launch_bounds__(256) lowrank_reduce_kernel(const float* __restrict__ partial, int M, int mpad,
                                                             int splits, __nv_bfloat16* __restrict__ u_pair) {
    const int i = blockIdx.x * 256 + threadIdx.x;  // (row, rank)
    if (i >= M * 32) return;
    float u = partial[i];
    for (int j = 1; j < splits; ++j) u = __fadd_rn(u, partial[(size_t)j * mpad * 32 + i]);
    const __nv_bfloat16 hi = __float2bfloat16_rn(u);
    const __nv_bfloat16 lo = __float2bfloat16_rn(u - __bfloat162float(hi));
    const int m = i >> 5, r = i & 31;
    u_pair[(size_t)m * 64 + r] = hi;
    u_pair[(size_t)m * 64 + 32 + r] = lo;
}

}  // namespace fp4
