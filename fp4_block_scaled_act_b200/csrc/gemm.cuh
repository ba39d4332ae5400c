// gemm.cuh -- persistent block-scaled GEMM for sm_100a (tcgen05 + TMA), fused epilogue.
//
//   y[m, n] = bf16_rn( gs * sum_k deq(a[m, k]) * deq(w[n, k]) (+ u[m,:] L2[:, n]) + bias[n] )
//
// Tile 128 x 256 (M x N), one CTA per SM, tiles assigned round-robin (tile t -> CTA
// t mod grid), N fastest so concurrently running CTAs share the activation rows in L2.
// Per K-stage the operands take one 128-byte swizzle atom per row:
//   W4A4 (kind::mxf4nvf4): 256 packed E2M1 values, 4 MMAs of K = 64
//   W4A8 (kind::mxf8f6f4): 128 E4M3 / unpacked E2M1 values, 4 MMAs of K = 32
// Warp roles (320 threads):
//   warp 0      TMA producer: A/B tiles (tensor maps) + scale-factor atoms (bulk copies)
//   warp 1      TMEM owner and MMA issuer: tcgen05.cp scale atoms into TMEM, then
//               tcgen05.mma block_scale into a 128 x 256 fp32 accumulator in TMEM
//   warps 2..9  epilogue: drain the accumulator to registers (freeing TMEM for the next
//               tile's MMAs at once), then scale, add bias (and the low-rank term), round
//               to bf16 and store
// Every mbarrier wait is bounded; a wait that runs out sets the device status word and
// the shared abort flag, and all roles leave their loops, drain in-flight copies/MMAs and
// free TMEM before the CTA exits.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace fp4 {

enum GemmKind { G_MXFP4 = 0, G_NVFP4 = 1, G_W4A8 = 2 };

constexpr int GEMM_THREADS = 320;
constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_STAGES = 4;
constexpr int GEMM_ACC_COLS = 256;
constexpr int GEMM_TMEM_COLS = 512;
constexpr int STATUS_TIMEOUT = 7;

template <int KIND>
struct GemmCfg {
    static constexpr int BK = (KIND == G_W4A8) ? 128 : 256;     // K elements per stage
    static constexpr int G = (KIND == G_NVFP4) ? 16 : 32;       // scale group size
    static constexpr int MMA_K = (KIND == G_W4A8) ? 32 : 64;
    static constexpr int ATOMS = BK / (G * 4);                  // SF atoms per 128 rows per stage
    static constexpr int A_BYTES = GEMM_BM * 128;
    static constexpr int B_BYTES = GEMM_BN * 128;
    static constexpr int SFA_BYTES = ATOMS * 512;
    static constexpr int SFB_BYTES = 2 * ATOMS * 512;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int SF_COLS = ATOMS * 4 * 3;               // SFA + SFB TMEM columns
    static constexpr int SMEM_BYTES = 1024 + GEMM_STAGES * STAGE_BYTES + 256;
    // instruction descriptor (block-scaled): formats, N>>3, scale format, M>>4
    static constexpr uint32_t A_FMT = (KIND == G_W4A8) ? 0u : 1u;  // E4M3 : E2M1
    static constexpr uint32_t B_FMT = (KIND == G_W4A8) ? 5u : 1u;  // E2M1 (f8f6f4) : E2M1 (mxf4)
    static constexpr uint32_t SCALE_FMT = (KIND == G_NVFP4) ? 0u : 1u;  // UE4M3 : UE8M0
    static constexpr uint32_t IDESC = (A_FMT << 7) | (B_FMT << 10) | ((uint32_t)(GEMM_BN >> 3) << 17) |
                                      (SCALE_FMT << 23) | ((uint32_t)(GEMM_BM >> 4) << 24);
    static_assert(GEMM_ACC_COLS + 2 * SF_COLS <= GEMM_TMEM_COLS, "TMEM budget");
};

struct GemmParams {
    int M, N, K;
    const uint8_t* sfa;       // activation scale factors (128x4 atoms)
    const uint8_t* sfb;       // weight scale factors
    const float* g_a;         // NVFP4 globals (device scalars) or null
    const float* g_w;
    const __half* bias;       // [N] or null
    __nv_bfloat16* y;         // [M, N]
    const float* u;           // W4A8: [M, 32] fp32
    const __nv_bfloat16* l2;  // W4A8: [32, N] bf16
    uint64_t timeout_ns;
    int skip_iter;            // test hook: producer skips this k-iteration (-1: none)
    int* status;              // device status word
};

FP4_DEV void gemm_fail(const GemmParams& p, volatile int* abort) {
    *abort = 1;
    atomicCAS(p.status, 0, STATUS_TIMEOUT);
}

template <int KIND>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p) {
    using C = GemmCfg<KIND>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + GEMM_STAGES * C::A_BYTES;
    uint8_t* sSFA = sB + GEMM_STAGES * C::B_BYTES;
    uint8_t* sSFB = sSFA + GEMM_STAGES * C::SFA_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + GEMM_STAGES * C::SFB_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = bars + GEMM_STAGES;
    uint64_t* tmem_full = bars + 2 * GEMM_STAGES;
    uint64_t* tmem_empty = tmem_full + 1;
    uint64_t* mma_done = tmem_full + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < GEMM_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tmem_full, 1);
        mbar_init(tmem_empty, 8);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, GEMM_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int M = p.M, N = p.N, K = p.K;
    const int num_m = (M + GEMM_BM - 1) / GEMM_BM;
    const int num_n = (N + GEMM_BN - 1) / GEMM_BN;
    const int num_tiles = num_m * num_n;
    const int num_kb = (K + C::BK - 1) / C::BK;
    const int atoms_per_rowblock = K / (C::G * 4);      // SF atoms per 128-row block along K
    const int n_rowblocks = (N + 127) / 128;

    if (warp == 0) {
        // ============================================================ producer
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_normal();
            const uint64_t pol_b = policy_evict_last();
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int mb = tile / num_n, nb = tile % num_n;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % GEMM_STAGES;
                    const uint32_t ph = (uint32_t)(it / GEMM_STAGES) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, p.timeout_ns, abort)) {
                        gemm_fail(p, abort);
                        ok = false;
                        break;
                    }
                    if (it == p.skip_iter) continue;  // test hook: never arrive on this stage
                    const int k_elems = min(C::BK, K - kb * C::BK);
                    const int n_atoms = k_elems / (C::G * 4);
                    const int rb1_ok = (nb * 2 + 1) < n_rowblocks;
                    // the unpacking map for W4A8's E2M1 operand counts the packed (global) bytes
                    const uint32_t b_tx = (KIND == G_W4A8) ? C::B_BYTES / 2 : C::B_BYTES;
                    const uint32_t bytes = C::A_BYTES + b_tx + n_atoms * 512 * (2 + rb1_ok);
                    mbar_arrive_expect_tx(&full[s], bytes);
                    // A: x in bytes of the row (packed FP4: BK/2 bytes per stage; E4M3: BK bytes)
                    const int ax = (KIND == G_W4A8) ? kb * C::BK : kb * (C::BK / 2);
                    tma_load_2d(sA + s * C::A_BYTES, &tmA, &full[s], ax, mb * GEMM_BM, pol_a);
                    // B: packed FP4 addressed in bytes; W4A8's unpacking map is addressed in elements
                    const int bx = (KIND == G_W4A8) ? kb * C::BK : kb * (C::BK / 2);
                    tma_load_2d(sB + s * C::B_BYTES, &tmB, &full[s], bx, nb * GEMM_BN, pol_b);
                    const size_t a_off = ((size_t)mb * atoms_per_rowblock + (size_t)kb * C::ATOMS) * 512;
                    bulk_load(sSFA + s * C::SFA_BYTES, p.sfa + a_off, n_atoms * 512, &full[s], pol_a);
                    for (int rb = 0; rb < 1 + rb1_ok; ++rb) {
                        const size_t b_off =
                            ((size_t)(nb * 2 + rb) * atoms_per_rowblock + (size_t)kb * C::ATOMS) * 512;
                        bulk_load(sSFB + s * C::SFB_BYTES + rb * C::ATOMS * 512, p.sfb + b_off, n_atoms * 512,
                                  &full[s], pol_b);
                    }
                }
            }
            // drain: every copy issued into the ring must have landed before the CTA exits
            for (int j = max(0, it - GEMM_STAGES); j < it; ++j) {
                if (j == p.skip_iter) continue;
                if (!mbar_wait_drain(&full[j % GEMM_STAGES], (uint32_t)(j / GEMM_STAGES) & 1u, p.timeout_ns)) {
                    // a copy that never completes leaves nothing more to wait for
                    atomicCAS(p.status, 0, STATUS_TIMEOUT);
                    *abort = 1;
                }
            }
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        // One thread issues every tcgen05 operation; the rest of the warp only takes
        // part in the TMEM allocation and release.
        if (lane == 0) {
            int it = 0, tcount = 0;
            bool issued = false;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
                if (!mbar_wait(tmem_empty, ((uint32_t)tcount & 1u) ^ 1u, p.timeout_ns, abort)) {
                    gemm_fail(p, abort);
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % GEMM_STAGES;
                    const uint32_t ph = (uint32_t)(it / GEMM_STAGES) & 1u;
                    if (!mbar_wait(&full[s], ph, p.timeout_ns, abort)) {
                        gemm_fail(p, abort);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int k_elems = min(C::BK, K - kb * C::BK);
                    const int n_atoms = k_elems / (C::G * 4);
                    const int n_mma = k_elems / C::MMA_K;
                    const uint32_t sf_col = GEMM_ACC_COLS + (uint32_t)(it & 1) * C::SF_COLS;
                    const uint32_t tsfa = tmem_base + sf_col;
                    const uint32_t tsfb = tmem_base + sf_col + C::ATOMS * 4;
                    for (int a = 0; a < n_atoms; ++a) {
                        tmem_cp_sf_atom(tsfa + a * 4, smem_desc(smem_u32(sSFA + s * C::SFA_BYTES + a * 512), 0, 128, 0));
#pragma unroll
                        for (int rb = 0; rb < 2; ++rb)
                            tmem_cp_sf_atom(
                                tsfb + a * 8 + rb * 4,
                                smem_desc(smem_u32(sSFB + s * C::SFB_BYTES + (rb * C::ATOMS + a) * 512), 0, 128, 0));
                    }
                    const uint32_t a_base = smem_u32(sA + s * C::A_BYTES);
                    const uint32_t b_base = smem_u32(sB + s * C::B_BYTES);
                    for (int k = 0; k < n_mma; ++k) {
                        // scale-factor selection: which atom (TMEM column group) and which byte
                        int atom, sf_id;
                        if (KIND == G_MXFP4) {
                            atom = k >> 1;
                            sf_id = (k & 1) * 2;
                        } else if (KIND == G_NVFP4) {
                            atom = k;
                            sf_id = 0;
                        } else {
                            atom = 0;
                            sf_id = k;
                        }
                        const uint32_t idesc = C::IDESC | ((uint32_t)sf_id << 29) | ((uint32_t)sf_id << 4);
                        const uint64_t adesc = smem_desc(a_base + k * 32, 0, 1024, 2);
                        const uint64_t bdesc = smem_desc(b_base + k * 32, 0, 1024, 2);
                        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
                        if (KIND == G_MXFP4)
                            mma_mxf4nvf4_block32(tmem_base, adesc, bdesc, idesc, acc, tsfa + atom * 4, tsfb + atom * 8);
                        else if (KIND == G_NVFP4)
                            mma_mxf4nvf4_block16(tmem_base, adesc, bdesc, idesc, acc, tsfa + atom * 4, tsfb + atom * 8);
                        else
                            mma_mxf8f6f4_block32(tmem_base, adesc, bdesc, idesc, acc, tsfa + atom * 4, tsfb + atom * 8);
                    }
                    tc_commit(&empty[s]);
                    issued = true;
                }
                if (!ok) break;
                tc_commit(tmem_full);
            }
            // drain: no MMA may still be writing TMEM when it is freed
            if (issued) {
                tc_commit(mma_done);
                if (!mbar_wait_drain(mma_done, 0, p.timeout_ns)) gemm_fail(p, abort);
            }
        }
        __syncwarp();
    } else {
        // ============================================================ epilogue
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int h = (warp - 2) >> 2;       // column half of the 256-wide tile
        float gs = 1.0f;
        if (KIND == G_NVFP4) gs = __fmul_rn(*p.g_a, *p.g_w);
        int tcount = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
            const int mb = tile / num_n, nb = tile % num_n;
            // the decision must be warp-uniform: tcgen05.ld below is .sync.aligned
            const bool got = mbar_wait(tmem_full, (uint32_t)tcount & 1u, p.timeout_ns, abort);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) gemm_fail(p, abort);
                break;
            }
            tc_fence_after();
            uint32_t acc[4][32];
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * 128);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(taddr + c * 32, acc[c]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tmem_empty);

            const int row = mb * GEMM_BM + q * 32 + lane;
            const int col0 = nb * GEMM_BN + h * 128;
            if (row < M && col0 < N) {
                float ur[32];
                if (KIND == G_W4A8) {
                    const float4* up = reinterpret_cast<const float4*>(p.u + (size_t)row * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 t = up[i];
                        ur[4 * i] = t.x, ur[4 * i + 1] = t.y, ur[4 * i + 2] = t.z, ur[4 * i + 3] = t.w;
                    }
                }
                __nv_bfloat16* yrow = p.y + (size_t)row * N + col0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        const int col = col0 + c * 32 + j;
                        float v[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(acc[c][j + i]) * gs;
                        if (KIND == G_W4A8) {
#pragma unroll
                            for (int r = 0; r < 32; ++r) {
                                const uint4 lv = *reinterpret_cast<const uint4*>(p.l2 + (size_t)r * N + col);
                                const uint32_t lw[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    v[2 * i] = __fmaf_rn(ur[r], __uint_as_float(lw[i] << 16), v[2 * i]);
                                    v[2 * i + 1] = __fmaf_rn(ur[r], __uint_as_float(lw[i] & 0xFFFF0000u), v[2 * i + 1]);
                                }
                            }
                        }
                        if (p.bias) {
                            const uint4 bv = *reinterpret_cast<const uint4*>(p.bias + col);
                            const __half2* bh = reinterpret_cast<const __half2*>(&bv);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float2 bf = __half22float2(bh[i]);
                                v[2 * i] += bf.x;
                                v[2 * i + 1] += bf.y;
                            }
                        }
                        uint4 o;
                        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
                            ow[i] = *reinterpret_cast<uint32_t*>(&b2);
                        }
                        *reinterpret_cast<uint4*>(yrow + c * 32 + j) = o;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
    }
}

}  // namespace fp4
