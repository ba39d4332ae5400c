// gemm.cuh -- persistent block-scaled GEMMs for sm_100a (tcgen05 + TMA), fused epilogues.
//
//   y[m, n] = bf16_rn( gs * sum_k deq(a[m, k]) * deq(w[n, k]) (+ u[m,:] L2[:, n]) + bias[n] )
//
// Two kernels:
//   gemm2_kernel  (default for M > 128, and every W4A8 / W4A4-SVDQuant / fused-activation
//                 call) -- a cta_group::2 pair of CTAs computes a 256 x 256 tile; see the
//                 block comment above Gemm2Cfg for its warp roles, TMEM layout and schedule.
//   gemm_kernel   (M <= 128, or forced) -- one CTA per SM, 128 x 256 tiles, described below.
// Per K-stage the operands take one 128-byte swizzle atom per row:
//   FP4 x FP4 (kind::mxf4nvf4): 256 packed E2M1 values, 4 MMAs of K = 64
//   W4A8 (kind::mxf8f6f4): 128 E4M3 / unpacked E2M1 values, 4 MMAs of K = 32
// gemm_kernel warp roles (320 threads):
//   warp 0      TMA producer: A/B tiles (tensor maps) + scale-factor atoms (bulk copies)
//   warp 1      TMEM owner and MMA issuer: tcgen05.cp scale atoms into TMEM, then
//               tcgen05.mma block_scale into a 128 x 256 fp32 accumulator in TMEM
//   warps 2..9  epilogue: drain the accumulator to registers (freeing TMEM for the next
//               tile's MMAs at once), then scale, add bias, round to bf16 and store
// Every mbarrier wait is bounded; a wait that runs out sets the device status word and
// the shared abort flag, and all roles leave their loops, drain in-flight copies/MMAs and
// free TMEM before the CTA exits.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gelu.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace fp4 {

// G_SVD4: W4A4 SVDQuant, MXFP4 activations x MXFP4 residual (the MXFP4 main loop) plus the
// low-rank stage of the 2-CTA kernel, like G_W4A8.
enum GemmKind { G_MXFP4 = 0, G_NVFP4 = 1, G_W4A8 = 2, G_SVD4 = 3 };

constexpr int GEMM_THREADS = 320;
constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_STAGES = 4;
constexpr int GEMM_ACC_COLS = 256;
constexpr int GEMM_TMEM_COLS = 512;

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
    uint8_t* h_codes;         // fused GELU + quantize output: FP4 codes [M, N/2]
    uint8_t* h_sf;            //   and scale bytes (128x4 atoms over [M, N])
    const float* g_h;         //   NVFP4 global of that output (device scalar) or null
    int seg_max;              // stream-K (2-CTA kernel): partial slabs per tile in `partials`
    float* partials;          //   fp32 [tiles][seg_max][256][256] partial sums of split tiles
    int* counters;            //   [tiles][16] arrivals per 32 x 128 region (zero before launch)
    uint64_t timeout_ns;
    int skip_iter;            // test hook: producer skips this k-iteration (-1: none)
    int* status;              // device status word
};

FP4_DEV void gemm_fail(const GemmParams& p, volatile int* abort) {
    *abort = 1;
    atomicCAS(p.status, 0, STATUS_TIMEOUT);
}

// Scale, add bias and round to bf16 NC x 32 columns of one output row held in registers
// (acc[c][j] = column col0 + 32c + j, fp32 bits; row < M).  The W4A8 low-rank term is
// already in the accumulator (a tensor-core stage of the pair kernel).
// On return acc[c][w], w < 16, holds columns 32c + 2w and 32c + 2w + 1 as a bf16 pair.
template <int KIND, int NC>
FP4_DEV void epilogue_pack(const GemmParams& p, uint32_t (&acc)[NC][32], int row, int col0, float gs) {
#pragma unroll
    for (int c = 0; c < NC; ++c) {
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(acc[c][j + i]) * gs;
            if (p.bias) {
                const uint4 bv = *reinterpret_cast<const uint4*>(p.bias + col0 + c * 32 + j);
                const __half2* bh = reinterpret_cast<const __half2*>(&bv);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 bf = __half22float2(bh[i]);
                    v[2 * i] += bf.x;
                    v[2 * i + 1] += bf.y;
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
                acc[c][j / 2 + i] = *reinterpret_cast<uint32_t*>(&b2);
            }
        }
    }
}

// Pack one row's NC 32-column chunks and store them straight to global memory (1-CTA kernel).
template <int KIND, int NC>
FP4_DEV void epilogue_store(const GemmParams& p, uint32_t (&acc)[NC][32], int row, int col0, float gs) {
    if (row >= p.M || col0 >= p.N) return;
    epilogue_pack<KIND, NC>(p, acc, row, col0, gs);
    __nv_bfloat16* yrow = p.y + (size_t)row * p.N + col0;
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int g = 0; g < 4; ++g)
            *reinterpret_cast<uint4*>(yrow + c * 32 + g * 8) =
                make_uint4(acc[c][4 * g], acc[c][4 * g + 1], acc[c][4 * g + 2], acc[c][4 * g + 3]);
}

// Which TMEM scale atom and which byte of it MMA number k of a stage reads.
template <int KIND>
FP4_DEV void sf_select(int k, int& atom, int& sf_id) {
    if (KIND == G_MXFP4 || KIND == G_SVD4) {  // 2 E8M0 scales (K = 64) per MMA: byte pair 0-1 or 2-3
        atom = k >> 1;
        sf_id = (k & 1) * 2;
    } else if (KIND == G_NVFP4) {  // 4 E4M3 scales (K = 64) per MMA: the whole word
        atom = k;
        sf_id = 0;
    } else {  // W4A8: 1 E8M0 scale (K = 32) per MMA
        atom = 0;
        sf_id = k;
    }
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
                    // the stage's MMAs, unrolled with every operand a constant offset (the issuing
                    // thread's own latency sets the MMA rate); MMA k reads 32 bytes at k * 32 of
                    // every 128-byte row, and a last stage of K % 256 = 128 holds two MMAs
                    const uint64_t adesc = smem_desc(smem_u32(sA + s * C::A_BYTES), 0, 1024, 2);
                    const uint64_t bdesc = smem_desc(smem_u32(sB + s * C::B_BYTES), 0, 1024, 2);
                    const uint32_t acc0 = kb > 0 ? 1u : 0u;
                    static_assert(C::BK / C::MMA_K == 4, "four MMAs per stage");
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if (k >= n_mma) break;
                        // scale-factor selection: which atom (TMEM column group) and which byte
                        int atom, sf_id;
                        sf_select<KIND>(k, atom, sf_id);
                        const uint32_t idesc = C::IDESC | ((uint32_t)sf_id << 29) | ((uint32_t)sf_id << 4);
                        const uint64_t ad = adesc + (uint64_t)(k * 2), bd = bdesc + (uint64_t)(k * 2);
                        const uint32_t acc = k > 0 ? 1u : acc0;
                        if (KIND == G_MXFP4)
                            mma_mxf4nvf4_block32(tmem_base, ad, bd, idesc, acc, tsfa + atom * 4, tsfb + atom * 8);
                        else if (KIND == G_NVFP4)
                            mma_mxf4nvf4_block16(tmem_base, ad, bd, idesc, acc, tsfa + atom * 4, tsfb + atom * 8);
                        else
                            mma_mxf8f6f4_block32(tmem_base, ad, bd, idesc, acc, tsfa + atom * 4, tsfb + atom * 8);
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

            epilogue_store<KIND, 4>(p, acc, mb * GEMM_BM + q * 32 + lane, nb * GEMM_BN + h * 128, gs);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
    }
}

// =======================================================================================
// 2-CTA variant (cta_group::2): a cluster of two CTAs on an SM pair computes a 256 x 256
// tile with M = 256 MMAs issued by the pair leader (CTA rank 0).  Each CTA loads its own
// 128 rows of A and 128 of the 256 B rows; the tensor core combines both halves of B.
// Per SM and K stage that is 256 operand rows instead of 384 for a 1-CTA 128 x 256
// tile, so both the L2 -> shared-memory stream and the shared-memory reads of the MMA
// shrink by a third.
//
// Scale factors go to TMEM without tcgen05.cp: four "scale writer" warps, one per 32-lane
// TMEM quarter, read the raw 512-byte atoms from shared memory and store them with
// tcgen05.st in the layout the MMA reads: lane 32q+i, column xa+4a+g holds word g of row i
// of A atom a (the scales of A row 32g+i), and column xb+8a+4rb+g holds word g of row i of
// B atom a in row block rb, in every quarter q.  The tensor pipe then runs MMAs only, and
// shared memory sees only the raw atoms.  Both CTAs hold the scales of all 256 B rows.
// The writers load a stage's words before waiting for its TMEM buffer to be free, so only
// the TMEM store and the arrive follow that wait.  A scale-ring slot goes back to the scale
// producer only after the TMEM stores have consumed its words: handed back as soon as the
// shared-memory loads were issued, a slot was refilled by the next TMA load before those
// loads had read it whenever the writers then waited long for their TMEM buffer (the MMA
// stalled behind the fused GELU epilogue), and stages ran with the wrong scales.
//
// Accumulators: two 256-column accumulators overlapping by 96 columns ([0,256),
// [160,416)), or by 64 for the W4A8 kernel and the fused GELU epilogues ([192,448)); the
// epilogue drains the shared columns first, so the next tile's MMAs wait for that part
// only.  The TMEM scale buffers follow the second accumulator: four for the plain-output
// kinds with two scale atoms per stage (MXFP4, W4A4 SVDQuant) and for W4A8 (one atom), two
// for NVFP4 (four atoms) and for the fused GELU epilogues.
//
// Warps (512 threads, four warpgroups): 0 operand TMA producer, 1 TMEM owner + MMA issuer
// (leader), 2 stage coordinator (leader), 3 scale TMA producer, 4-7 scale writers, 8-15
// epilogue.  The control warpgroups (0-7) drop to REG_LO registers per thread with setmaxnreg and the
// epilogue warpgroups rise to REG_HI: the fused epilogues run without spilling, and an
// NVFP4 overlap holder can copy its whole 128-column share before converting any.
// The tensor pipe queues very little ahead of the issuing thread, so every cycle that
// thread spends between two MMAs is a bubble.  The MMA warp therefore tests no mbarrier:
// the coordinator does the waits and hands each stage over with a hardware named barrier
// (bar.arrive / bar.sync), which does not touch shared memory.
// Synchronization:
//   full[s]      (leader)  A/B bytes of both CTAs; the leader alone expects them
//   empty[s]     (both)    the leader's commit (MMAs of stage s done)
//   sc_full[j]   (local)   this CTA's raw scale atoms in scale-ring slot j
//   sc_empty[j]  (local)   slot j stored into TMEM by this CTA's 4 writer warps (separate scale ring;
//                          NVFP4's scale slots ride in the operand ring and are recycled
//                          with empty[s], loaded by the operand producer)
//   sf_ready[t]  (leader)  scale buffer t written in both CTAs (8 writer warps)
//   tmem_full[b] (both)    accumulator b complete
//   acc_free[b]  (leader)  accumulator b fully drained by both CTAs (16 warps)
//   ovl_free     (leader)  overlap columns of the last tile drained (8 warps)
// =======================================================================================
// named barrier of the 8 epilogue warps (the MMA hand-off ring uses ids 1 .. TB <= 4)
constexpr uint32_t EPI_TABLE_BAR = 8;

template <int KIND, int OUTQ = 0>
struct Gemm2Cfg {
    using C1 = GemmCfg<KIND>;
    // 128-byte operand rows (128-byte swizzle) for every kind: with 64-byte rows (64-byte
    // swizzle) a 256x256x64 MMA was measured at ~290 cycles instead of ~160
    static constexpr int BK = C1::BK;
    static constexpr int G = C1::G, MMA_K = C1::MMA_K;
    static constexpr int ATOMS = BK / (G * 4);  // scale atoms per stage: MX 2, NV 4, W4A8 1
    static constexpr int ROW_BYTES = 128;       // per operand row per stage
    static constexpr uint32_t SWZ = 2u;         // descriptor layout: 128-byte swizzle
    static constexpr int SBO = 8 * ROW_BYTES;
    static constexpr int N_MMA = BK / MMA_K;
    static_assert(N_MMA == 4, "the MMA warp issues a stage as four unrolled MMAs");
    static constexpr int A_BYTES = 128 * ROW_BYTES;
    static constexpr int B_BYTES = 128 * ROW_BYTES;  // this CTA's half of the 256 B rows
    static constexpr int RSFA_BYTES = ATOMS * 512;    // raw atoms, this CTA's 128 A rows
    static constexpr int RSFB_BYTES = 2 * ATOMS * 512;  // raw atoms, all 256 B rows
    // Two rings.  The operand ring (A and B tiles of a stage) is refilled when the MMAs of
    // the stage it held are done; the scale ring (the raw scale atoms of a stage) is
    // refilled as soon as the scale writers have read a slot into registers, so the scale
    // atoms run ahead of the operands and their slots cost no operand-ring space.
    // Operand tiles arrive over a TMA path whose latency under this load (~2000 cycles,
    // measured) makes the number of stages in flight the limit: the operand ring takes five
    // stages (32 KB each), six for W4A8, whose epilogue's per-warp Y staging tile is then
    // 32 x 32 bf16 (64-byte rows, 64-byte swizzle) to make room.
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int SC_BYTES = RSFA_BYTES + RSFB_BYTES;
    // NVFP4 (four atoms per stage, two TMEM scale buffers) measured 10 % slower with the
    // separate scale ring, so its scale atoms ride in the operand ring as before: the
    // operand producer loads them with the stage's tiles (SC_STAGES == STAGES, slot s of the
    // scale area belongs to operand stage s and is recycled with it).
    static constexpr bool SEP_SC = (KIND != G_NVFP4);
    static constexpr int STAGES = (KIND == G_W4A8) ? 6 : 5;
    static constexpr int SC_STAGES = SEP_SC ? 4 : STAGES;
    static constexpr int EPI_COLS = (STAGES == 6) ? 32 : 64;
    static constexpr int EPI_TILE = 32 * EPI_COLS * 2;
    static constexpr int EPI_BYTES = 8 * EPI_TILE;
    // the dynamic shared array is declared 1024-byte aligned (checked at run time), so the
    // layout needs no alignment slack
    // + barriers; NVFP4 also keeps the fused epilogue's 128-entry reciprocal table after them
    static constexpr int SMEM_BYTES =
        STAGES * STAGE_BYTES + EPI_BYTES + SC_STAGES * SC_BYTES + 512 + (KIND == G_NVFP4 ? 512 : 0);
    static constexpr uint32_t AB_TX = A_BYTES + ((KIND == G_W4A8) ? B_BYTES / 2 : B_BYTES);
    static constexpr uint32_t SF_TX = RSFA_BYTES + RSFB_BYTES;
    // TMEM columns: two accumulators overlapping by OVL columns, the shared columns drained
    // first.  NVFP4 stages carry 4 scale atoms (48 columns), so its accumulators overlap by
    // 96 to leave room for two scale buffers; the others overlap by 64, which the holders
    // drain as their first 64-column pair.  A 96-column overlap spans both pairs: with
    // plain bf16 output (HOLD_ALL) its holders copy all four chunks to registers before
    // converting any, so the overlap is released after the copy rather than after a pair
    // has been written; the fused epilogues need those registers for their arithmetic.
    // The plain-output MXFP4 and W4A4 SVDQuant kernels (two atoms, 24 columns per scale
    // buffer) overlap by 96 too, which leaves room for four scale buffers: the writers then
    // refill a buffer four stages after its MMAs were issued rather than two.  The fused
    // GELU epilogues keep a 64-column overlap (their holders convert before releasing it)
    // and two buffers; W4A8 (one atom, 12 columns) fits four buffers beside a 64 overlap.
    static constexpr int ACC1_COL = (KIND == G_NVFP4) ? 160 : (KIND == G_W4A8 || OUTQ != 0) ? 192 : 160;
    static constexpr int SF_COL0 = ACC1_COL + 256;
    static constexpr int OVL = 256 - ACC1_COL;
    static constexpr bool HOLD_ALL = (OUTQ == 0) && (OVL > 64);
    static constexpr int SFA_COLS = 4 * ATOMS;        // A: 4 columns per atom
    static constexpr int SF_COLS = SFA_COLS + 8 * ATOMS;  // B: 8 columns per atom
    static constexpr int TB = ((GEMM_TMEM_COLS - SF_COL0) / SF_COLS) >= 4 ? 4 : ((GEMM_TMEM_COLS - SF_COL0) / SF_COLS);
    // 16 warps in four warpgroups; the two control warpgroups (warps 0-7) hand registers to
    // the two epilogue warpgroups (8-15).  Launched with 128 registers per thread.
    static constexpr int THREADS = 512;
    static constexpr uint32_t REG_LAUNCH = 128, REG_LO = 80, REG_HI = 176;
    static_assert(256 * REG_LO + 256 * REG_HI == THREADS * REG_LAUNCH, "register split must match the launch");
    // W4A8 low-rank stage (one per tile, after the K stages): A = the u pair, 128 rows x 64
    // bf16 (128-byte rows, 128-byte swizzle, K-major); B = L2 as stored, [rank = 32][N] bf16,
    // read MN-major: this CTA's 128 columns as two 64-column blocks of 32 K rows x 128 bytes
    // (128-byte swizzle; K rows 8 at a time 1024 bytes apart, the second block 4096 bytes
    // on); four kind::f16 MMAs of K = 16 (u_hi x L2, then u_lo x L2), B transposed (bit 16).
    static constexpr uint32_t LR_TX = 128 * 128 + 2 * 32 * 128;
    static constexpr uint32_t LR_B_LBO = 32 * 128, LR_B_SBO = 8 * 128;
    static constexpr uint32_t IDESC_LR = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
    static constexpr uint32_t IDESC = (C1::A_FMT << 7) | (C1::B_FMT << 10) | ((uint32_t)(256 >> 3) << 17) |
                                      (C1::SCALE_FMT << 23) | ((uint32_t)(256 >> 4) << 24);
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert((STAGES * (A_BYTES + B_BYTES)) % 1024 == 0, "staging tiles 1024-byte aligned");
    static_assert(TB >= 2 && SF_COL0 + TB * SF_COLS <= GEMM_TMEM_COLS, "TMEM budget");
    static_assert(OVL == 64 || OVL == 96, "epilogue overlap handling");
};

// Pair-kernel epilogue: pack one row's 64 columns and write them, as 128 bytes, into row
// `r` of the warp's 32 x 128-byte staging tile in the 128-byte-swizzled layout the output
// tensor map reads (16-byte granule g of row r at granule g ^ (r % 8)).  Rows at or beyond
// M are not computed; the TMA store clips them.
template <int KIND>
FP4_DEV void epilogue_stage(const GemmParams& p, uint32_t (&acc)[2][32], int row, int col0, float gs, uint8_t* tile,
                            int r) {
    if (row >= p.M) return;
    epilogue_pack<KIND, 2>(p, acc, row, col0, gs);
    const uint32_t base = smem_u32(tile) + (uint32_t)r * 128u;
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
            const uint32_t g = (uint32_t)(c * 4 + g4) ^ ((uint32_t)r & 7u);
            st_shared_v4(base + g * 16u, acc[c][4 * g4], acc[c][4 * g4 + 1], acc[c][4 * g4 + 2], acc[c][4 * g4 + 3]);
        }
}

// 32 packed bf16 columns of row r (16 words, from epilogue_pack) into a 32 x 32 staging
// tile with 64-byte rows under the 64-byte swizzle: 16-byte chunk g of row r lands in slot
// g ^ ((r >> 1) & 3), so each group of 8 lanes covers all 32 banks
FP4_DEV void epilogue_stage_32(const uint32_t (&w)[32], uint8_t* tile, int r) {
    const uint32_t base = smem_u32(tile) + (uint32_t)r * 64u;
#pragma unroll
    for (int g4 = 0; g4 < 4; ++g4) {
        const uint32_t g = (uint32_t)g4 ^ (((uint32_t)r >> 1) & 3u);
        st_shared_v4(base + g * 16u, w[4 * g4], w[4 * g4 + 1], w[4 * g4 + 2], w[4 * g4 + 3]);
    }
}

// Fused down-projection input (OUTQ 1: MXFP4, 2: NVFP4).  Columns col0 .. col0+63 of one
// row, rounded to bf16 z by epilogue_pack, become h = bf16_rn(gelu_tanh(z)) (gelu.cuh) and
// are quantized in the output format's groups along N (MXFP4: 2 groups of 32 with an E8M0
// scale, NVFP4: 4 groups of 16 with an E4M3 scale under the global g_h) by the same steps
// as quant_kernel: codes to h_codes[row][col / 2], scale bytes into the 128x4 atoms of the
// [M, N] activation.  Each thread owns its row, so no group spans threads.  Rows in
// [M, Mpad) store zero scale bytes (the layout's padding), rows >= Mpad nothing.
template <int KIND, int OUTQ>
FP4_DEV void epilogue_gelu_quant(const GemmParams& p, uint32_t (&acc)[2][32], int row, int col0, float gs, float g_h,
                                 float six_g_h, const float* rcp_tab) {
    const int Mpad = (p.M + 127) & ~127;
    if (row >= Mpad || col0 >= p.N) return;
    constexpr int G = (OUTQ == 1) ? 32 : 16;
    const int64_t apr = p.N / (G * 4);                 // scale atoms per 128-row block
    const int j0 = col0 / G;                           // first group of the 64 columns
    uint8_t* word = p.h_sf + sf_word_offset(row, j0 >> 2, apr);
    uint32_t sfw = 0;                                  // this pair's scale bytes in their word slots
    if (row < p.M) {
        epilogue_pack<KIND, 2>(p, acc, row, col0, gs);  // acc[c][w], w < 16: bf16 pairs of z
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float h[32];
#pragma unroll
            for (int w = 0; w < 16; ++w)
                gelu_bf16_x2(__uint_as_float(acc[c][w] << 16), __uint_as_float(acc[c][w] & 0xFFFF0000u), h[2 * w],
                             h[2 * w + 1]);
            uint32_t cw[4];
#pragma unroll
            for (int g = 0; g < 32 / G; ++g) {
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < G; ++i) amax = fmaxf(amax, fabsf(h[g * G + i]));
                uint32_t sfb;
                if (OUTQ == 1) {
                    sfb = mx_scale_byte<2>(amax);
                    const float inv = mx_inv_scale(sfb);
#pragma unroll
                    for (int i = 0; i < G; ++i) h[g * G + i] = __fmul_rn(h[g * G + i], inv);
                } else {
                    sfb = cvt_e4m3x2(__fdiv_rn(amax, six_g_h), 0.0f) & 0xFFu;
                    // 1 / (e4m3(sfb) * g_h), tabulated per E4M3 code; 0 marks a zero scale
                    const float r = rcp_tab[sfb & 0x7Fu];
#pragma unroll
                    for (int i = 0; i < G; ++i) h[g * G + i] = (r == 0.0f) ? 0.0f : __fmul_rn(h[g * G + i], r);
                }
                sfw |= sfb << (8 * ((j0 + c * (32 / G) + g) & 3));
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) cw[q] = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(h + 8 * q));
            *reinterpret_cast<uint4*>(p.h_codes + (size_t)row * (p.N / 2) + col0 / 2 + 16 * c) =
                make_uint4(cw[0], cw[1], cw[2], cw[3]);
        }
    }
    if (OUTQ == 1)  // groups j0, j0 + 1: one half of the atom word
        *reinterpret_cast<uint16_t*>(word + (j0 & 3)) = (uint16_t)(sfw >> (8 * (j0 & 3)));
    else            // groups j0 .. j0 + 3: the whole word
        *reinterpret_cast<uint32_t*>(word) = sfw;
}

// Work schedule of the 2-CTA kernel.  Whole tiles round-robin over the pairs, or (stream-K,
// for problems with fewer tiles than two rounds of pairs) each pair takes an equal,
// contiguous share of the flattened (tile, K block) space, cut at tile ends into units.
// A tile split over several pairs is summed through fp32 partial slabs (epilogue).
struct Sched {
    int num_tiles, num_kb, num_pairs, pair;
    bool sk;
    int lo, hi, t;
    FP4_DEV int kstart(int p) const { return (int)((int64_t)p * num_tiles * num_kb / num_pairs); }
    // the pair whose share contains flattened K block k
    FP4_DEV int pair_of(int k) const {
        int q = (int)(((int64_t)k * num_pairs) / ((int64_t)num_tiles * num_kb));
        while (q + 1 < num_pairs && kstart(q + 1) <= k) ++q;
        while (q > 0 && kstart(q) > k) --q;
        return q;
    }
    FP4_DEV void begin() {
        if (sk) {
            lo = kstart(pair);
            hi = kstart(pair + 1);
        } else {
            t = pair;
        }
    }
    FP4_DEV bool get(int& tile, int& kb0, int& kb1) const {
        if (sk) {
            if (lo >= hi) return false;
            tile = lo / num_kb;
            kb0 = lo - tile * num_kb;
            kb1 = min(num_kb, kb0 + (hi - lo));
            return true;
        }
        if (t >= num_tiles) return false;
        tile = t;
        kb0 = 0;
        kb1 = num_kb;
        return true;
    }
    FP4_DEV void step(int kb0, int kb1) {
        if (sk) lo += kb1 - kb0;
        else t += num_pairs;
    }
};

FP4_DEV void gemm2_fail(const GemmParams& p, volatile int* abort, uint32_t peer_abort) {
    *abort = 1;
    st_cluster_u32(peer_abort, 1u);
    atomicCAS(p.status, 0, STATUS_TIMEOUT);
}

// Arrive on a barrier of the pair leader: a local arrive in the leader, a remote relaxed
// arrive in the follower (used after TMEM loads/stores that tcgen05.wait has completed, so
// no memory write needs publishing; a release.cluster arrive would fence every call).
FP4_DEV void arrive_leader_relaxed(uint64_t* bar, uint32_t rank) {
    if (rank == 0)
        mbar_arrive(bar);
    else
        mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(bar), 0));
}

// OUTQ 0: bf16 output through the TMA-store epilogue; 1 / 2: the fused GELU + MXFP4 /
// NVFP4 quantize epilogue (epilogue_gelu_quant) in place of the bf16 output.
// SK: the stream-K schedule (small problems, opt-in); a separate instantiation so the
// default kernel carries none of its registers.
template <int KIND, int OUTQ = 0, bool SK = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Gemm2Cfg<KIND>::THREADS, 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                 const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmU,
                 const __grid_constant__ CUtensorMap tmL, GemmParams p) {
    using C = Gemm2Cfg<KIND, OUTQ>;
    constexpr int S = C::STAGES;
    constexpr int TB = C::TB;
    extern __shared__ __align__(1024) uint8_t smem2_raw[];
    // 128-byte-swizzled operand tiles need 1024-byte alignment; both CTAs see the same
    // layout, so both leave here together, before any barrier
    // and the launch must have provided the whole layout: a kernel launched with less
    // dynamic shared memory than its configuration needs writes nothing and reports it
    uint32_t dyn_smem;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_smem));
    if ((smem_u32(smem2_raw) & 1023u) != 0 || dyn_smem < (uint32_t)C::SMEM_BYTES) {
        if (threadIdx.x == 0) atomicCAS(p.status, 0, STATUS_LAYOUT);
        return;
    }
    uint8_t* sA = smem2_raw;
    uint8_t* sB = sA + S * C::A_BYTES;
    uint8_t* sEpi = sB + S * C::B_BYTES;                  // 8 per-warp Y staging tiles
    uint8_t* sSC = sEpi + C::EPI_BYTES;                   // scale ring: per slot A atoms, then B atoms
    constexpr int SJ = C::SC_STAGES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sSC + SJ * C::SC_BYTES);
    // fused NVFP4 epilogue: reciprocals of the decoded scales, 128 floats after the barriers
    float* rcp_tab = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 512);
    uint64_t* full = bars;
    uint64_t* empty = full + S;
    uint64_t* sc_full = empty + S;                        // [SJ] scale ring slot loaded (local)
    uint64_t* sc_empty = sc_full + SJ;                    // [SJ] scale ring slot read by the 4 writers (local)
    uint64_t* sf_ready = sc_empty + SJ;                   // [TB]
    uint64_t* tmem_full = sf_ready + TB;                  // [2]
    uint64_t* acc_free = tmem_full + 2;                   // [2]
    uint64_t* ovl_free = acc_free + 2;
    uint64_t* mma_done = ovl_free + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t peer_abort = mapa_shared(smem_u32((const void*)abort), rank ^ 1u);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < SJ; ++j) {
            mbar_init(&sc_full[j], 1);
            mbar_init(&sc_empty[j], 4);
        }
        for (int t = 0; t < TB; ++t) mbar_init(&sf_ready[t], 8);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 1);
            mbar_init(&acc_free[b], 16);
        }
        mbar_init(ovl_free, 8);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmSFA);
        prefetch_tmap(&tmSFB);
        prefetch_tmap(&tmY);
        if (KIND == G_W4A8 || KIND == G_SVD4) {
            prefetch_tmap(&tmU);
            prefetch_tmap(&tmL);
        }
    }
    __syncwarp();
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, GEMM_TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncwarp();  // the cluster barrier is .aligned: every warp converged
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int M = p.M, N = p.N, K = p.K;
    const int num_m = (M + 255) / 256;
    const int num_n = (N + 255) / 256;
    const int num_tiles = num_m * num_n;
    const int num_kb = (K + C::BK - 1) / C::BK;
    // stages per unit: its K blocks, then (W4A8, W4A4 SVDQuant) the low-rank stage kb == num_kb
    // (those kinds always run whole tiles)
    constexpr bool HAS_LR = (KIND == G_W4A8 || KIND == G_SVD4);
    const int apr = K / (C::G * 4);  // scale atoms per 128-row block
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const Sched sched0{num_tiles, num_kb, num_pairs, pair, SK, 0, 0, 0};

    if (warp >= 8) {
        // the two epilogue warpgroups take the registers the control warps give up
        setmaxnreg_inc<C::REG_HI>();
        // ============================================================ epilogue (both CTAs)
        // Epilogue warp ew = warp - 8 drains TMEM lane quarter warp % 4 (the only quarter a
        // warp can reach) and column half ew / 4 of every tile: 32 rows x 128 columns.
        const int ew = warp - 8;
        const int q = warp & 3;
        const int h = ew >> 2;
        uint8_t* stile = sEpi + ew * C::EPI_TILE;
        // Y is streamed out (2 GB at the FFN shape): evict-first lines drain to DRAM during
        // the GEMM instead of being written back while the next kernel streams its input
        const uint64_t pol_y = policy_evict_first();
        // acc: the 64-column pair being written; acc2: an overlap holder's second pair (HOLD_ALL)
        uint32_t acc[2][32], acc2[2][32];
        float gs = 1.0f;
        if (KIND == G_NVFP4) gs = __fmul_rn(*p.g_a, *p.g_w);
        float g_h = 1.0f, six_g_h = 6.0f;
        if (OUTQ == 2) {
            g_h = *p.g_h;
            six_g_h = __fmul_rn(6.0f, g_h);
            // the decoded group scale d = e4m3(sf) * g_h has at most 127 values: tabulate 1 / d
            // once (0 for d = 0) by the operations the quantizer uses, then sync the 8 warps
            const int et = ew * 32 + lane;
            if (et < 128) {
                const float d = __fmul_rn(e4m3_to_f32((uint32_t)et), g_h);
                rcp_tab[et] = d == 0.0f ? 0.0f : __frcp_rn(d);
            }
            named_bar_sync(EPI_TABLE_BAR, 256u);
        }
        int tcount = 0;
        Sched sc = sched0;
        sc.begin();
        int tile, kb0, kb1;
        for (; sc.get(tile, kb0, kb1); sc.step(kb0, kb1), ++tcount) {
            const int mb = tile / num_n, nb = tile % num_n;
            const int b = tcount & 1;
            const bool got = mbar_wait(&tmem_full[b], ((uint32_t)tcount >> 1) & 1u, p.timeout_ns, abort);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) gemm2_fail(p, abort, peer_abort);
                break;
            }
            tc_fence_after();
            const uint32_t taddr =
                tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::ACC1_COL) + (uint32_t)(h * 128);
            const int row0 = mb * 256 + (int)rank * 128 + q * 32;
            const int row = row0 + lane;
            const int col0 = nb * GEMM_BN + h * 128;
            // stream-K: the tile's segments (pairs whose share meets it) and this unit's index
            int nseg = 1, seg = 0;
            if constexpr (SK) {
                const int pf = sc.pair_of(tile * num_kb);
                nseg = sc.pair_of(tile * num_kb + num_kb - 1) - pf + 1;
                seg = pair - pf;
            }
            // this warp's 32 x 128 region of the tile's fp32 partial slabs, stored lane-major
            // (float4 (chunk, j4, lane) at ((chunk * 8 + j4) * 32 + lane) * 4) so every warp
            // instruction writes or reads 512 contiguous bytes; the summing warp has the same
            // rows and lanes, so only it needs to know the layout
            float* slab0 = p.partials + (size_t)tile * p.seg_max * 65536 + ((int)rank * 8 + ew) * 4096 + lane * 4;
            // pack 64 columns into the staging tile and hand them to one TMA store (which
            // clips rows at or beyond M); the tile is reused once the previous store has read it
            auto emit = [&](uint32_t (&a)[2][32], int chunk) {
                if (OUTQ != 0) {
                    epilogue_gelu_quant<KIND, OUTQ>(p, a, row, col0 + chunk * 32, gs, g_h, six_g_h, rcp_tab);
                    return;
                }
                if (col0 >= p.N) return;
                if constexpr (C::EPI_COLS == 64) {
                    if (lane == 0) bulk_wait_group_read0();
                    __syncwarp();
                    epilogue_stage<KIND>(p, a, row, col0 + chunk * 32, gs, stile, lane);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && row0 < p.M) {
                        tma_store_2d_hint(&tmY, stile, col0 + chunk * 32, row0, pol_y);
                        bulk_commit_group();
                    }
                } else {
                    // one 32-column store per chunk through the half-size tile
                    if (row < p.M) epilogue_pack<KIND, 2>(p, a, row, col0 + chunk * 32, gs);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        if (lane == 0) bulk_wait_group_read0();
                        __syncwarp();
                        if (row < p.M) epilogue_stage_32(a[c], stile, lane);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0 && row0 < p.M) {
                            tma_store_2d_hint(&tmY, stile, col0 + (chunk + c) * 32, row0, pol_y);
                            bulk_commit_group();
                        }
                    }
                }
            };
            // a split tile: this segment's fp32 sums of the 64 columns go to its slab
            auto stage_store = [&](uint32_t (&a)[2][32], int chunk) {
                if (!SK || nseg == 1) {
                    emit(a, chunk);
                    return;
                }
                float* dst = slab0 + (size_t)seg * 65536;
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(dst + (((chunk + c) * 8 + j / 4) * 32) * 4) =
                            make_float4(__uint_as_float(a[c][j]), __uint_as_float(a[c][j + 1]),
                                        __uint_as_float(a[c][j + 2]), __uint_as_float(a[c][j + 3]));
            };
            // the OVL columns shared by both accumulators are the last OVL tile columns of
            // accumulator 0 (half 1) or the first OVL of accumulator 1 (half 0): their holders
            // drain them first and release them -- after the first chunk pair when OVL = 64,
            // after copying all four chunks with HOLD_ALL, else after both pairs
            const bool holds_overlap = (h == (b == 0 ? 1 : 0));
            const int first = holds_overlap ? (b == 0 ? 2 : 0) : 0;
            const int second = 2 - first;
            tmem_ld_32x32b_x32(taddr + first * 32, acc[0]);
            tmem_ld_32x32b_x32(taddr + (first + 1) * 32, acc[1]);
            if (C::HOLD_ALL && holds_overlap) {
                tmem_ld_32x32b_x32(taddr + second * 32, acc2[0]);
                tmem_ld_32x32b_x32(taddr + (second + 1) * 32, acc2[1]);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    arrive_leader_relaxed(ovl_free, rank);
                    arrive_leader_relaxed(&acc_free[b], rank);
                }
                stage_store(acc, first);
                stage_store(acc2, second);
            } else {
                tmem_wait_ld();
                if (holds_overlap && C::OVL <= 64) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) arrive_leader_relaxed(ovl_free, rank);
                }
                stage_store(acc, first);
                tmem_ld_32x32b_x32(taddr + second * 32, acc[0]);
                tmem_ld_32x32b_x32(taddr + (second + 1) * 32, acc[1]);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (holds_overlap && C::OVL > 64 && lane == 0) arrive_leader_relaxed(ovl_free, rank);
                if (lane == 0) arrive_leader_relaxed(&acc_free[b], rank);
                stage_store(acc, second);
            }
            if (SK && nseg > 1) {
                // the last of the tile's segments to arrive sums the slabs in segment order
                // (a fixed order, so the result does not depend on which one is last) and
                // runs the epilogue; nobody waits for anybody
                __threadfence();
                __syncwarp();
                int last = 0;
                if (lane == 0) last = atomicAdd(p.counters + tile * 16 + (int)rank * 8 + ew, 1) == nseg - 1;
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __threadfence();
#pragma unroll 1
                    for (int pr = 0; pr < 4; pr += 2) {
                        // segment-outer: 16 independent float4 loads per segment in flight
#pragma unroll 1
                        for (int sg = 0; sg < nseg; ++sg) {
                            const float* src = slab0 + (size_t)sg * 65536;
#pragma unroll
                            for (int c = 0; c < 2; ++c)
#pragma unroll
                                for (int j = 0; j < 32; j += 4) {
                                    const float4 v =
                                        __ldcg(reinterpret_cast<const float4*>(src + (((pr + c) * 8 + j / 4) * 32) * 4));
                                    if (sg == 0) {
                                        acc[c][j] = __float_as_uint(v.x), acc[c][j + 1] = __float_as_uint(v.y);
                                        acc[c][j + 2] = __float_as_uint(v.z), acc[c][j + 3] = __float_as_uint(v.w);
                                    } else {
                                        acc[c][j] = __float_as_uint(__fadd_rn(__uint_as_float(acc[c][j]), v.x));
                                        acc[c][j + 1] = __float_as_uint(__fadd_rn(__uint_as_float(acc[c][j + 1]), v.y));
                                        acc[c][j + 2] = __float_as_uint(__fadd_rn(__uint_as_float(acc[c][j + 2]), v.z));
                                        acc[c][j + 3] = __float_as_uint(__fadd_rn(__uint_as_float(acc[c][j + 3]), v.w));
                                    }
                                }
                        }
                        emit(acc, pr);
                    }
                }
            }
        }
        // the staging tile must outlive the stores that read it
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
    } else {
        // warps 0-7: operand producer, MMA issuer, coordinator, scale producer and the scale writers
        setmaxnreg_dec<C::REG_LO>();
        if (warp == 0) {
            // ============================================================ producer (both CTAs)
            if (lane == 0) {
                // the activations may come from the kernel just before us (programmatic launch)
                griddep_wait();
                const uint64_t pol_a = policy_evict_normal();
                const uint64_t pol_b = policy_evict_last();
                int it = 0;
                bool ok = true;
                Sched sc = sched0;
                sc.begin();
                int tile, kb0, kb1;
                while (ok && sc.get(tile, kb0, kb1)) {
                    const int mb = tile / num_n, nb = tile % num_n;
                    for (int kb = kb0; kb < kb1 + (HAS_LR ? 1 : 0); ++kb, ++it) {
                        const int s = it % S;
                        const uint32_t ph = (uint32_t)(it / S) & 1u;
                        if (!mbar_wait(&empty[s], ph ^ 1u, p.timeout_ns, abort)) {
                            gemm2_fail(p, abort, peer_abort);
                            ok = false;
                            break;
                        }
                        if (it == p.skip_iter) continue;  // test hook: this stage is never filled
                        // A/B of both CTAs land on the leader's barrier; only the leader expects them
                        const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
                        if (HAS_LR && kb == num_kb) {
                            // low-rank stage: u pair rows and the L2 columns
                            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::LR_TX);
                            tma_load_2d_pair(sA + s * C::A_BYTES, &tmU, bar, 0, mb * 256 + (int)rank * 128, pol_a);
                            // L2 [32][N]: this CTA's 128 columns as two 64-column boxes of 32 rows
                            tma_load_2d_pair(sB + s * C::B_BYTES, &tmL, bar, nb * 256 + (int)rank * 128, 0, pol_b);
                            tma_load_2d_pair(sB + s * C::B_BYTES + C::LR_B_LBO, &tmL, bar,
                                             nb * 256 + (int)rank * 128 + 64, 0, pol_b);
                            continue;
                        }
                        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::AB_TX);
                        // x: bytes of the row for packed FP4 and E4M3, elements for the W4A8 unpacking map
                        const int ax = kb * C::ROW_BYTES;
                        const int bx = (KIND == G_W4A8) ? kb * C::BK : kb * C::ROW_BYTES;
                        tma_load_2d_pair(sA + s * C::A_BYTES, &tmA, bar, ax, mb * 256 + (int)rank * 128, pol_a);
                        tma_load_2d_pair(sB + s * C::B_BYTES, &tmB, bar, bx, nb * 256 + (int)rank * 128, pol_b);
                        if constexpr (!C::SEP_SC) {
                            // this CTA's raw scale atoms of the stage, into the stage's scale slot
                            uint8_t* slot = sSC + s * C::SC_BYTES;
                            mbar_arrive_expect_tx(&sc_full[s], C::SF_TX);
                            tma_load_2d(slot, &tmSFA, &sc_full[s], 0, (mb * 2 + (int)rank) * apr + kb * C::ATOMS, pol_a);
    #pragma unroll
                            for (int r = 0; r < 2; ++r)
                                tma_load_2d(slot + C::RSFA_BYTES + r * C::ATOMS * 512, &tmSFB, &sc_full[s], 0,
                                            (nb * 2 + r) * apr + kb * C::ATOMS, pol_b);
                        }
                    }
                    sc.step(kb0, kb1);
                }
                // drain what was issued into this pair's ring: (leader) both CTAs' A/B, and the
                // scale atoms when they ride in the operand ring
                for (int j = max(0, it - S); j < it; ++j) {
                    if (j == p.skip_iter) continue;
                    if (!C::SEP_SC && !mbar_wait_drain(&sc_full[j % S], (uint32_t)(j / S) & 1u, p.timeout_ns))
                        gemm2_fail(p, abort, peer_abort);
                    if (rank == 0 && !mbar_wait_drain(&full[j % S], (uint32_t)(j / S) & 1u, p.timeout_ns))
                        gemm2_fail(p, abort, peer_abort);
                }
            }
        } else if (warp == 3) {
            // ============================================================ scale producer (both CTAs)
            // This CTA's raw scale atoms of every stage into the scale ring; a slot is reused
            // once the four writer warps have read it.  The W4A8 / W4A4 SVDQuant low-rank stage
            // has no scales: its slot turn completes with a plain arrive, so the ring counters
            // stay in step with the stages.
            if (C::SEP_SC && lane == 0) {
                griddep_wait();
                const uint64_t pol_a = policy_evict_normal();
                const uint64_t pol_b = policy_evict_last();
                int it = 0;
                bool ok = true;
                Sched sc = sched0;
                sc.begin();
                int tile, kb0, kb1;
                while (ok && sc.get(tile, kb0, kb1)) {
                    const int mb = tile / num_n, nb = tile % num_n;
                    for (int kb = kb0; kb < kb1 + (HAS_LR ? 1 : 0); ++kb, ++it) {
                        const int j = it % SJ;
                        if (!mbar_wait(&sc_empty[j], ((uint32_t)(it / SJ) & 1u) ^ 1u, p.timeout_ns, abort)) {
                            gemm2_fail(p, abort, peer_abort);
                            ok = false;
                            break;
                        }
                        if (HAS_LR && kb == num_kb) {
                            mbar_arrive(&sc_full[j]);
                            continue;
                        }
                        uint8_t* slot = sSC + j * C::SC_BYTES;
                        mbar_arrive_expect_tx(&sc_full[j], C::SF_TX);
                        tma_load_2d(slot, &tmSFA, &sc_full[j], 0, (mb * 2 + (int)rank) * apr + kb * C::ATOMS, pol_a);
    #pragma unroll
                        for (int r = 0; r < 2; ++r)
                            tma_load_2d(slot + C::RSFA_BYTES + r * C::ATOMS * 512, &tmSFB, &sc_full[j], 0,
                                        (nb * 2 + r) * apr + kb * C::ATOMS, pol_b);
                    }
                    sc.step(kb0, kb1);
                }
                // drain this CTA's scale loads still in flight
                for (int q = max(0, it - SJ); q < it; ++q)
                    if (!mbar_wait_drain(&sc_full[q % SJ], (uint32_t)(q / SJ) & 1u, p.timeout_ns))
                        gemm2_fail(p, abort, peer_abort);
            }
        } else if (warp >= 4) {
            // ============================================================ scale writers (both CTAs)
            const int quarter = warp & 3;
            const uint32_t tlane = tmem_base + ((uint32_t)(quarter * 32) << 16);
            int it = 0;
            bool ok = true;
            Sched sc = sched0;
            sc.begin();
            int tile, kb0, kb1;
            while (ok && sc.get(tile, kb0, kb1)) {
                for (int kb = kb0; kb < kb1 + (HAS_LR ? 1 : 0); ++kb, ++it) {
                    const int j = it % SJ;
                    const int t = it % TB;
                    bool got = mbar_wait(&sc_full[j], (uint32_t)(it / SJ) & 1u, p.timeout_ns, abort);
                    if (!__all_sync(0xffffffffu, got)) {
                        if (lane == 0) gemm2_fail(p, abort, peer_abort);
                        ok = false;
                        break;
                    }
                    const uint4* rsfa = reinterpret_cast<const uint4*>(sSC + j * C::SC_BYTES);
                    const uint4* rsfb = reinterpret_cast<const uint4*>(sSC + j * C::SC_BYTES + C::RSFA_BYTES);
                    // lane i takes row i of every atom: words 0-3 = the scales of rows i, 32+i, 64+i, 96+i
                    uint32_t va[4 * C::ATOMS];
                    uint32_t vb[8 * C::ATOMS];
    #pragma unroll
                    for (int a = 0; a < C::ATOMS; ++a) {
                        const uint4 w = rsfa[a * 32 + lane];
                        va[4 * a] = w.x, va[4 * a + 1] = w.y, va[4 * a + 2] = w.z, va[4 * a + 3] = w.w;
    #pragma unroll
                        for (int rb = 0; rb < 2; ++rb) {
                            const uint4 z = rsfb[(rb * C::ATOMS + a) * 32 + lane];
                            vb[8 * a + 4 * rb] = z.x, vb[8 * a + 4 * rb + 1] = z.y;
                            vb[8 * a + 4 * rb + 2] = z.z, vb[8 * a + 4 * rb + 3] = z.w;
                        }
                    }
                    // buffer t is free once the MMAs of iteration it - TB (same buffer) are done
                    got = it < TB || mbar_wait(&empty[(it - TB) % S], (uint32_t)((it - TB) / S) & 1u, p.timeout_ns, abort);
                    if (!__all_sync(0xffffffffu, got)) {
                        if (lane == 0) gemm2_fail(p, abort, peer_abort);
                        ok = false;
                        break;
                    }
                    // order the TMEM stores after the MMAs that read the buffer (their commit,
                    // observed through the mbarrier)
                    tc_fence_after();
                    const uint32_t xa = C::SF_COL0 + (uint32_t)(t * C::SF_COLS);
                    const uint32_t xb = xa + C::SFA_COLS;
                    // the W4A8 low-rank stage reads no scales: its buffer turn passes unwritten
                    if (HAS_LR && kb == num_kb) {
                    } else if constexpr (C::ATOMS == 4) {
                        tmem_st_32x32b_x16(tlane + xa, *reinterpret_cast<const uint32_t(*)[16]>(va));
                        tmem_st_32x32b_x16(tlane + xb, *reinterpret_cast<const uint32_t(*)[16]>(vb));
                        tmem_st_32x32b_x16(tlane + xb + 16, *reinterpret_cast<const uint32_t(*)[16]>(vb + 16));
                    } else if constexpr (C::ATOMS == 2) {
                        tmem_st_32x32b_x8(tlane + xa, va);
                        tmem_st_32x32b_x16(tlane + xb, vb);
                    } else {
                        tmem_st_32x32b_x4(tlane + xa, va);
                        tmem_st_32x32b_x8(tlane + xb, vb);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) arrive_leader_relaxed(&sf_ready[t], rank);
                    // the slot's words have been consumed by the TMEM stores: hand the slot back
                    // to the scale producer (a slot that rides in the operand ring is recycled
                    // with its stage instead)
                    if (C::SEP_SC && lane == 0) mbar_arrive(&sc_empty[j]);
                }
                sc.step(kb0, kb1);
            }
        } else if (warp == 1) {
            // ============================================================ MMA issuer (leader)
            // The whole warp runs the loop so that it can take the named barrier each stage;
            // lane 0 issues.  Per stage it touches no shared memory at all: the coordinator
            // warp has checked everything the stage needs before releasing it, and the abort
            // flag is read once per tile (the coordinator releases every stage of a tile even
            // after a failure, so the warp always reaches that check).
            // The issuing thread's own latency decides the MMA rate: with the stage's four MMAs
            // unrolled and every operand a running value or a constant offset, a stage issues
            // at the tensor pipe's 128 cycles per 256x256x64 MMA; recomputing descriptors,
            // scale ids and slot indices per MMA was measured at ~150.
            if (rank == 0) {
                uint32_t it = 0;
                int tcount = 0;
                bool issued = false, ok = true;
                int s = 0, t = 0;  // it % S and it % TB
                const uint64_t adesc0 = smem_desc(smem_u32(sA), 0, C::SBO, C::SWZ);
                const uint64_t bdesc0 = smem_desc(smem_u32(sB), 0, C::SBO, C::SWZ);
                Sched sc = sched0;
                sc.begin();
                int tile, kb0, kb1;
                for (; ok && sc.get(tile, kb0, kb1); sc.step(kb0, kb1), ++tcount) {
                    const int b = tcount & 1;
                    const uint32_t dacc = tmem_base + (uint32_t)(b * C::ACC1_COL);
                    for (int kb = kb0; kb < kb1 + (HAS_LR ? 1 : 0); ++kb, ++it) {
                        named_bar_sync(1u + (uint32_t)t, 64u);
                        if (lane == 0 && HAS_LR && kb == num_kb) {
                            // low-rank stage: acc += u_hi L2 + u_lo L2 (bf16 x bf16 -> fp32)
                            tc_fence_after();
                            const uint32_t a_base = smem_u32(sA + s * C::A_BYTES);
                            const uint32_t b_base = smem_u32(sB + s * C::B_BYTES);
    #pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const uint64_t adesc = smem_desc(a_base + k * 32, 0, 1024, 2u);
                                const uint64_t bdesc =
                                    smem_desc(b_base + (k & 1) * 2 * C::LR_B_SBO, C::LR_B_LBO, C::LR_B_SBO, 2u);
                                mma2_f16(dacc, adesc, bdesc, C::IDESC_LR, 1u);
                            }
                            tc_commit_pair(&empty[s], 0x3);
                        } else if (lane == 0) {
                            tc_fence_after();
                            // slot s's descriptors: slot 0's plus s * bytes / 16 in the start-address
                            // field; MMA k reads the 32 bytes at k * 32 of every 128-byte row
                            const uint64_t adesc = adesc0 + (uint64_t)(s * (C::A_BYTES >> 4));
                            const uint64_t bdesc = bdesc0 + (uint64_t)(s * (C::B_BYTES >> 4));
                            const uint32_t tsfa = tmem_base + C::SF_COL0 + (uint32_t)(t * C::SF_COLS);
                            const uint32_t tsfb = tsfa + C::SFA_COLS;
                            const uint32_t acc0 = kb > kb0 ? 1u : 0u;
                            // a last stage of K % BK = 128 (FP4 kinds) holds two MMAs
                            const bool half = (KIND != G_W4A8) && (K - kb * C::BK < C::BK);
    #pragma unroll
                            for (int k = 0; k < C::N_MMA; ++k) {
                                if (k >= 2 && half) break;
                                int atom, sf_id;
                                sf_select<KIND>(k, atom, sf_id);
                                const uint32_t idesc = C::IDESC | ((uint32_t)sf_id << 29) | ((uint32_t)sf_id << 4);
                                const uint32_t acc = k > 0 ? 1u : acc0;
                                const uint64_t ad = adesc + (uint64_t)(k * 2), bd = bdesc + (uint64_t)(k * 2);
                                if (KIND == G_MXFP4 || KIND == G_SVD4)
                                    mma2_mxf4nvf4_block32(dacc, ad, bd, idesc, acc, tsfa + atom * 4, tsfb + atom * 8);
                                else if (KIND == G_NVFP4)
                                    mma2_mxf4nvf4_block16(dacc, ad, bd, idesc, acc, tsfa + atom * 4, tsfb + atom * 8);
                                else
                                    mma2_mxf8f6f4_block32(dacc, ad, bd, idesc, acc, tsfa + atom * 4, tsfb + atom * 8);
                            }
                            tc_commit_pair(&empty[s], 0x3);
                        }
                        __syncwarp();
                        issued = true;
                        if (++s == S) s = 0;
                        if (++t == TB) t = 0;
                    }
                    if (lane == 0) tc_commit_pair(&tmem_full[b], 0x3);
                    __syncwarp();
                    if (__any_sync(0xffffffffu, *abort != 0)) ok = false;
                }
                if (issued) {
                    if (lane == 0) tc_commit_pair(mma_done, 0x1);
                    __syncwarp();
                    const bool drained = mbar_wait_drain(mma_done, 0, p.timeout_ns);
                    if (!__all_sync(0xffffffffu, drained) && lane == 0) gemm2_fail(p, abort, peer_abort);
                }
            }
            __syncwarp();
        } else if (warp == 2) {
            // ============================================================ stage coordinator (leader)
            // Waits, in the MMA warp's order, for everything a stage needs (the accumulator
            // and the overlap at a tile's first stage; A/B bytes of both CTAs; both CTAs'
            // scale buffer) and then releases the stage with named barrier 1 + it % TB.  After
            // a failure it still releases the remaining stages of that tile without waiting,
            // so the MMA warp, which checks the abort flag at the end of each tile, never
            // waits on a barrier that nobody arrives at.  The ring of TB barrier ids cannot be lapped:
            // the scale buffer of stage it + TB is free only after the MMA warp has passed
            // stage it.
            if (rank == 0) {
                uint32_t it = 0;
                int tcount = 0;
                bool ok = true;
                Sched sc = sched0;
                sc.begin();
                int tile, kb0, kb1;
                for (; ok && sc.get(tile, kb0, kb1); sc.step(kb0, kb1), ++tcount) {
                    const int b = tcount & 1;
                    // accumulator b drained (unit tcount-2) and the overlap of unit tcount-1 drained
                    bool got = mbar_wait(&acc_free[b], (((uint32_t)tcount >> 1) & 1u) ^ 1u, p.timeout_ns, abort);
                    if (got && tcount > 0) got = mbar_wait(ovl_free, (uint32_t)(tcount - 1) & 1u, p.timeout_ns, abort);
                    for (int kb = kb0; kb < kb1 + (HAS_LR ? 1 : 0); ++kb, ++it) {
                        if (got) got = mbar_wait(&full[it % S], (it / S) & 1u, p.timeout_ns, abort);
                        if (got) got = mbar_wait(&sf_ready[it % TB], (it / TB) & 1u, p.timeout_ns, abort);
                        got = __all_sync(0xffffffffu, got);
                        if (!got && ok) {
                            if (lane == 0) gemm2_fail(p, abort, peer_abort);
                            ok = false;
                        }
                        __syncwarp();
                        named_bar_arrive(1u + it % TB, 64u);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncwarp();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, GEMM_TMEM_COLS);
    }
}

}  // namespace fp4
