// attn_fused.cuh -- one head of FP4 attention (MXFP4 or NVFP4) in one kernel: S, the softmax
// weights and their quantization stay on the SM (TMEM and shared memory), O accumulates in TMEM.
//
// Reading (the Wan2.2-Animate-14B MXFP4 card, "Results", names SageAttention v3 as Blackwell
// microscaling FP4 attention; no page gives its algorithm): the keys are taken in blocks of
// 256.  For block j and each query row, S_j = deq(Q) deq(K_j)^T (fp32, in TMEM), the running
// maximum m_j = max(m_{j-1}, max_k fl(s_k c)) (c = scale log2 e; NVFP4 folds the scores'
// globals in, c' = fl(c fl(g_q g_k))), the weights P~_j = 2^(fl(fl(s c) - m_j)) quantized in
// groups of G keys by the activation rule (MXFP4: 32, E8M0; NVFP4: 16, E4M3 under P~'s global),
// O_j = O_{j-1} 2^(m_{j-1} - m_j) + deq(P~_j) deq(V_j) (fp32, in TMEM) and
// l_j = l_{j-1} 2^(m_{j-1} - m_j) + sum P~_j; the output is bf16_rn(O / l) (NVFP4: times
// fl(g_p g_v)).  The weights are thus quantized against the running maximum of the blocks
// seen so far, as a streaming (flash) attention must, not against the row's final maximum as
// the separate-kernel path (fp4_attn_softmax_quant) does.
//
// One CTA per 128 query rows of one head; 640 threads: warp 0 TMA producer, warp 1 TMEM
// owner and MMA issuer, warps 2-3 idle, warps 4-19 the softmax (a thread is one query row,
// its TMEM lane, in one quarter of the key block: warp w takes keys 64 qq .. 64 qq + 63 with
// qq = (w - 4) / 4, four warps per SM sub-partition to hide the latency of TMEM loads and exp2).
// Per key block: S_j = Q K_j^T (two 128x256x64 block32 MMAs); each softmax thread reads its
// quarter of S_j from TMEM twice (the quarter's maximum, exchanged with the other quarters
// through shared memory and a bounded mbarrier; then the weights), rescales its 32 columns of
// O in TMEM when the maximum grew (after the previous P~ V is done), writes its P~_j codes into
// a 128-byte-swizzled shared tile and its two scale bytes into the P~ atom; then
// O += P~_j V_j (four 128x128x64 MMAs, the P~ atoms copied into TMEM by tcgen05.cp).  Each
// quarter keeps its own l (scaled by the same factors); they are added at the end.  K_j, V_j
// and their atoms come through a two-slot TMA ring.  Every wait is bounded (status
// FP4_ERR_TIMEOUT).
#pragma once
#include <cuda_bf16.h>

#include <type_traits>

#include "ptx.cuh"
#include "quant.cuh"

namespace fp4 {

struct AttnParams {
    int64_t T_q, T_kv, tq_pad, tk_pad;
    int head, nblk;  // head index; key blocks of 256 (the last may hold 128 padded keys)
    float c;         // scale * log2(e), fp32
    const uint8_t* q_sf;  // this head's Q scale atoms (query tile t at t * Q_SF)
    const uint8_t* k_sf;  // this head's K scale atoms (key block j at j * KV_SF)
    const uint8_t* v_sf;  // this head's V^T scale atoms (key block j at j * KV_SF)
    // NVFP4: the fp32 globals of Q, K, V and P~ (device scalars); MXFP4: null
    const float* g_q;
    const float* g_k;
    const float* g_v;
    const float* g_p;
    __nv_bfloat16* o;     // [T_q][128]
    float2* stats;        // [T_q] (final running maximum, l) or null
    // test hook (null in the product path): for query tile trace_tile only, per key block j
    // the running maximum m_j of each of its 128 rows ([nblk][128] floats), the P~_j codes
    // ([nblk][128][128 bytes]) and scale bytes ([nblk][128][256 / G]), padding rows included
    int trace_tile;
    float* dbg_m;
    uint8_t* dbg_codes;
    uint8_t* dbg_sf;
    uint64_t timeout_ns;
    int* status;
};

constexpr int ATT_THREADS = 640;
constexpr int ATT_Q_BYTES = 128 * 128;  // 128 rows x 128 bytes (the 64 bytes of a head, zero-filled to 128)
constexpr int ATT_K_BYTES = 256 * 128;
constexpr int ATT_V_BYTES = 128 * 128;
constexpr int ATT_P_BYTES = 128 * 128;
constexpr int ATT_OFF_K = ATT_Q_BYTES;
constexpr int ATT_OFF_V = ATT_OFF_K + 2 * ATT_K_BYTES;
constexpr int ATT_OFF_P = ATT_OFF_V + 2 * ATT_V_BYTES;
// scale atoms: G = 32 (MXFP4) or 16 (NVFP4) elements per scale, 4 scales per atom row; the
// regions below are sized for NVFP4 (twice MXFP4's atoms) in both formats
constexpr int ATT_OFF_QSF = ATT_OFF_P + ATT_P_BYTES;  // one query tile's atoms, <= 1024
constexpr int ATT_OFF_KSF = ATT_OFF_QSF + 1024;       // [2 slots] x 2048
constexpr int ATT_OFF_VSF = ATT_OFF_KSF + 4096;       // [2 slots] x 2048
constexpr int ATT_OFF_PSF = ATT_OFF_VSF + 4096;       // one block's P~ atoms, <= 2048
constexpr int ATT_OFF_RCP = ATT_OFF_PSF + 2048;       // NVFP4: 1 / (dec(s) g_p) for the 128 E4M3 bytes
constexpr int ATT_OFF_RED = ATT_OFF_RCP + 512;        // [2][4][128] floats
constexpr int ATT_OFF_BAR = ATT_OFF_RED + 4096;
constexpr int ATT_SMEM = ATT_OFF_BAR + 256;
static_assert(ATT_OFF_QSF % 1024 == 0, "operand tiles 1024-byte aligned");
// TMEM columns: S [0, 256), O [256, 384), then the scale buffers (an atom = 4 columns; B
// operands of N = 256 take two atoms side by side, rows 0-127 then 128-255)
constexpr uint32_t ATT_T_S = 0, ATT_T_O = 256;
constexpr uint32_t ATT_T_QSF = 384;  // atom a at +4a
constexpr uint32_t ATT_T_KSF = 392;  // [2 slots] x 16: dims atom a at +8a, key row block rb at +4rb
constexpr uint32_t ATT_T_VSF = 424;  // [2 slots] x 16: key atom u at +4u
constexpr uint32_t ATT_T_PSF = 456;  // [2 buffers] x 16: key atom u at +4u

template <bool NV>
struct AttnCfg {
    static constexpr int G = NV ? 16 : 32;
    static constexpr int AR = NV ? 2 : 1;   // atoms per 128 rows of Q or K (128 dims), and per 128 keys of V^T or P~
    static constexpr int Q_SF = AR * 512;   // bytes of one query tile's atoms
    static constexpr int KV_SF = 2 * AR * 512;  // bytes of one 256-key block's atoms of K, and of V^T
    static constexpr int SFB_ROW = 256 / G;     // scale bytes of one row of one block
    // instruction descriptor: E2M1 x E2M1, scale format (UE8M0 = 1, UE4M3 = 0), M = 128; N added per MMA
    static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((NV ? 0u : 1u) << 23) | ((uint32_t)(128 >> 4) << 24);
    static constexpr uint32_t IDESC_S = IDESC | ((uint32_t)(256 >> 3) << 17);
    static constexpr uint32_t IDESC_PV = IDESC | ((uint32_t)(128 >> 3) << 17);
};

FP4_DEV void attn_fail(const AttnParams& p, volatile int* abort) {
    *abort = 1;
    atomicCAS(p.status, 0, STATUS_TIMEOUT);
}

template <bool NV>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attn_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, AttnParams p) {
    extern __shared__ __align__(1024) uint8_t sm[];
    uint32_t dyn_smem;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_smem));
    if ((smem_u32(sm) & 1023u) != 0 || dyn_smem < (uint32_t)ATT_SMEM) {
        if (threadIdx.x == 0) atomicCAS(p.status, 0, STATUS_LAYOUT);
        return;
    }
    uint8_t* sQ = sm;
    uint8_t* sK = sm + ATT_OFF_K;
    uint8_t* sV = sm + ATT_OFF_V;
    uint8_t* sP = sm + ATT_OFF_P;
    uint8_t* sQSF = sm + ATT_OFF_QSF;
    uint8_t* sKSF = sm + ATT_OFF_KSF;
    uint8_t* sVSF = sm + ATT_OFF_VSF;
    uint8_t* sPSF = sm + ATT_OFF_PSF;
    float* nv_rcp = reinterpret_cast<float*>(sm + ATT_OFF_RCP);
    using C = AttnCfg<NV>;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + ATT_OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;   // [2]
    uint64_t* kv_empty = bars + 3;  // [2]
    uint64_t* s_full = bars + 5;    // S_j in TMEM (MMA commit)
    uint64_t* s_free = bars + 6;    // S_j read by the 4 softmax warps
    uint64_t* p_full = bars + 7;    // P~_j tile and atoms written (4 softmax warps)
    uint64_t* o_done = bars + 8;    // P~_j V_j done (MMA commit)
    uint64_t* mma_done = bars + 9;
    uint64_t* pair_bar = bars + 10;  // [4]: the four softmax warps on rows 32 q .. 32 q + 31
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 14);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = blockIdx.x, nb = p.nblk;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, 16);
        mbar_init(p_full, 16);
        for (int i = 0; i < 4; ++i) mbar_init(&pair_bar[i], 4);
        mbar_init(o_done, 1);
        mbar_init(mma_done, 1);
        *abort = 0;
        fence_mbar_init();
    }
    // the scale slots of a partial last key block are not all loaded: start them at zero
    for (int i = threadIdx.x; i < (4096 + 4096) / 16; i += ATT_THREADS)
        *reinterpret_cast<uint4*>(sKSF + i * 16) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    // NVFP4: the reciprocal of each decoded P~ scale times P~'s global, as the activation
    // quantizer takes it (0 for a zero scale)
    if (NV && threadIdx.x < 128) {
        const float d = __fmul_rn(e4m3_to_f32(threadIdx.x), *p.g_p);
        nv_rcp[threadIdx.x] = d == 0.0f ? 0.0f : __frcp_rn(d);
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ============================================================ producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_normal();
            mbar_arrive_expect_tx(q_full, ATT_Q_BYTES + C::Q_SF);
            tma_load_2d(sQ, &tmQ, q_full, 0, (int)(p.head * p.tq_pad + (int64_t)qt * 128), pol);
            bulk_load(sQSF, p.q_sf + (int64_t)qt * C::Q_SF, C::Q_SF, q_full, pol);
            int j = 0;
            for (; j < nb; ++j) {
                const int s = j & 1;
                if (!mbar_wait(&kv_empty[s], (uint32_t)((j >> 1) & 1) ^ 1u, p.timeout_ns, abort)) {
                    attn_fail(p, abort);
                    break;
                }
                const int64_t key0 = (int64_t)j * 256;
                const int rbs = (key0 + 128 < p.tk_pad) ? 2 : 1;  // 128-key units present
                const int sfb = rbs * C::AR * 512;                  // their atoms' bytes, K and V^T each
                mbar_arrive_expect_tx(&kv_full[s], ATT_K_BYTES + ATT_V_BYTES + 2 * sfb);
                tma_load_2d(sK + s * ATT_K_BYTES, &tmK, &kv_full[s], 0, (int)(p.head * p.tk_pad + key0), pol);
                bulk_load(sKSF + s * 2048, p.k_sf + (int64_t)j * C::KV_SF, sfb, &kv_full[s], pol);
                tma_load_2d(sV + s * ATT_V_BYTES, &tmV, &kv_full[s], j * 128, p.head * 128, pol);
                bulk_load(sVSF + s * 2048, p.v_sf + (int64_t)j * C::KV_SF, sfb, &kv_full[s], pol);
            }
            // every copy issued must land before the CTA exits
            for (int i = max(0, j - 2); i < j; ++i)
                if (!mbar_wait_drain(&kv_full[i & 1], (uint32_t)((i >> 1) & 1), p.timeout_ns)) attn_fail(p, abort);
            if (!mbar_wait_drain(q_full, 0, p.timeout_ns)) attn_fail(p, abort);
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            bool ok = mbar_wait(q_full, 0, p.timeout_ns, abort);
            tc_fence_after();
            if (ok)
                for (int a = 0; a < C::AR; ++a)
                    tmem_cp_sf_atom(tmem + ATT_T_QSF + 4 * a, smem_desc(smem_u32(sQSF + 512 * a), 0, 128, 0));
            const uint64_t qdesc = smem_desc(smem_u32(sQ), 0, 1024, 2);
            const uint64_t pdesc = smem_desc(smem_u32(sP), 0, 1024, 2);
            auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc, uint32_t sfa,
                           uint32_t sfb) {
                if (NV)
                    mma_mxf4nvf4_block16(d, ad, bd, idesc, acc, sfa, sfb);
                else
                    mma_mxf4nvf4_block32(d, ad, bd, idesc, acc, sfa, sfb);
            };
            auto issue_s = [&](int j) -> bool {
                const int s = j & 1;
                if (!mbar_wait(&kv_full[s], (uint32_t)((j >> 1) & 1), p.timeout_ns, abort)) return false;
                tc_fence_after();
                const uint32_t tk = tmem + ATT_T_KSF + s * 16, tv = tmem + ATT_T_VSF + s * 16;
                for (int rb = 0; rb < 2; ++rb)
                    for (int a = 0; a < C::AR; ++a)
                        tmem_cp_sf_atom(tk + 8 * a + 4 * rb,
                                        smem_desc(smem_u32(sKSF + s * 2048 + (rb * C::AR + a) * 512), 0, 128, 0));
                for (int u = 0; u < 2 * C::AR; ++u)
                    tmem_cp_sf_atom(tv + 4 * u, smem_desc(smem_u32(sVSF + s * 2048 + u * 512), 0, 128, 0));
                const uint64_t kdesc = smem_desc(smem_u32(sK + s * ATT_K_BYTES), 0, 1024, 2);
                // K = 128 dims: MMA k reads bytes 32 k .. 32 k + 31 of each row; MXFP4: scale bytes
                // 2k, 2k + 1 of the single atom, NVFP4: the whole word of atom k
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint32_t sf_id = NV ? 0u : (uint32_t)k * 2u;
                    const int a = NV ? k : 0;
                    mma(tmem + ATT_T_S, qdesc + (uint64_t)(k * 2), kdesc + (uint64_t)(k * 2),
                        C::IDESC_S | (sf_id << 29) | (sf_id << 4), k > 0 ? 1u : 0u, tmem + ATT_T_QSF + 4 * a,
                        tk + 8 * a);
                }
                tc_commit(s_full);
                return true;
            };
            auto issue_pv = [&](int j) -> bool {
                const int s = j & 1;
                if (!mbar_wait(p_full, (uint32_t)(j & 1), p.timeout_ns, abort)) return false;
                tc_fence_after();
                const uint32_t tp = tmem + ATT_T_PSF + s * 16, tv = tmem + ATT_T_VSF + s * 16;
                for (int u = 0; u < 2 * C::AR; ++u)
                    tmem_cp_sf_atom(tp + 4 * u, smem_desc(smem_u32(sPSF + u * 512), 0, 128, 0));
                const uint64_t vdesc = smem_desc(smem_u32(sV + s * ATT_V_BYTES), 0, 1024, 2);
                // K = 256 keys: MMA k reads keys 64 k .. 64 k + 63; MXFP4: atom k / 2, bytes
                // 2 (k % 2), +1; NVFP4: the whole word of atom k
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int atom = NV ? k : (k >> 1);
                    const uint32_t sf_id = NV ? 0u : (uint32_t)(k & 1) * 2u;
                    mma(tmem + ATT_T_O, pdesc + (uint64_t)(k * 2), vdesc + (uint64_t)(k * 2),
                        C::IDESC_PV | (sf_id << 29) | (sf_id << 4), (j > 0 || k > 0) ? 1u : 0u, tp + 4 * atom,
                        tv + 4 * atom);
                }
                tc_commit(o_done);
                tc_commit(&kv_empty[s]);
                return true;
            };
            // from the scale copy on, tensor-core work may be in flight: drain it before exit
            const bool issued = ok;
            if (ok) ok = issue_s(0);
            for (int j = 0; ok && j < nb; ++j) {
                if (j + 1 < nb) {
                    // S_{j+1} overwrites S_j: the softmax warps must have read it
                    ok = mbar_wait(s_free, (uint32_t)(j & 1), p.timeout_ns, abort);
                    if (ok) tc_fence_after();
                    if (ok) ok = issue_s(j + 1);
                }
                if (ok) ok = issue_pv(j);
            }
            if (!ok) attn_fail(p, abort);
            if (issued) {
                tc_commit(mma_done);
                if (!mbar_wait_drain(mma_done, 0, p.timeout_ns)) attn_fail(p, abort);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ============================================================ softmax
        // warps 4-19: warp w takes keys 64 qq .. 64 qq + 63 of every block (qq = (w - 4) / 4)
        // for the 32 query rows of TMEM lanes 32 (w % 4) ..; a thread is one query row in one
        // quarter.  The four warps on the same rows exchange their maxima and, at the end,
        // their sums through shared memory and a bounded mbarrier.
        const int q4 = warp & 3;
        const int qq = (warp - 4) >> 2;
        const int r = q4 * 32 + lane;
        const int64_t row = (int64_t)qt * 128 + r;
        const bool real = row < p.T_q;
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        const uint32_t t_s = tl + ATT_T_S + (uint32_t)qq * 64u;  // this quarter's S columns
        const uint32_t t_o = tl + ATT_T_O + (uint32_t)qq * 32u;  // this quarter's O columns
        float* red = reinterpret_cast<float*>(sm + ATT_OFF_RED);  // [2 phases][4 quarters][128 rows]
        uint64_t* pair = &pair_bar[q4];
        // the exponent multiplier; NVFP4 folds the scores' globals in: c' = fl(c fl(g_q g_k))
        const float c = NV ? __fmul_rn(p.c, __fmul_rn(*p.g_q, *p.g_k)) : p.c;
        const float six_g = NV ? __fmul_rn(6.0f, *p.g_p) : 6.0f;
        const bool tracing = p.dbg_m != nullptr && qt == p.trace_tile;
        float m_run = -INFINITY, l = 0.0f;  // l: this quarter's sum
        bool ok = true;
        for (int j = 0; j < nb && ok; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(s_full, (uint32_t)(j & 1), p.timeout_ns, abort));
            if (!ok) break;
            tc_fence_after();
            const int64_t k0 = (int64_t)j * 256 + qq * 64;  // this quarter's first key
            const int nvalid = (int)(p.T_kv - k0 >= 64 ? 64 : (p.T_kv > k0 ? p.T_kv - k0 : 0));
            // pass 1: the quarter's maximum of s over its valid keys; c > 0, so the block's
            // max fl(s c) is fl(max s * c)
            float mx = -INFINITY;
            {
                uint32_t v[32], w[32];
                tmem_ld_32x32b_x32(t_s, v);
                tmem_ld_32x32b_x32(t_s + 32, w);
                tmem_wait_ld();
                tmem_tie(v);
                tmem_tie(w);
                float t[32];
                if (nvalid == 64) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) t[i] = fmaxf(__uint_as_float(v[i]), __uint_as_float(w[i]));
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        t[i] = fmaxf(i < nvalid ? __uint_as_float(v[i]) : -INFINITY,
                                     32 + i < nvalid ? __uint_as_float(w[i]) : -INFINITY);
                }
#pragma unroll
                for (int n = 16; n >= 1; n >>= 1)
#pragma unroll
                    for (int i = 0; i < n; ++i) t[i] = fmaxf(t[i], t[i + n]);
                mx = t[0];
            }
            red[((j & 1) * 4 + qq) * 128 + r] = mx;
            __syncwarp();
            if (lane == 0) mbar_arrive(pair);
            ok = __all_sync(0xffffffffu, mbar_wait(pair, (uint32_t)(j & 1), p.timeout_ns, abort));
            if (!ok) break;
            const float* rj = red + (j & 1) * 512 + r;
            const float mb = fmaxf(fmaxf(rj[0], rj[128]), fmaxf(rj[256], rj[384]));
            const float m_new = fmaxf(m_run, __fmul_rn(mb, c));
            // P~_{j-1} V_{j-1} must be done before the P~ tile, its atoms or O are touched
            if (j > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(o_done, (uint32_t)((j - 1) & 1), p.timeout_ns, abort));
                if (!ok) break;
                tc_fence_after();
            }
            // O and l follow the new maximum: O *= 2^(m_prev - m_new) (whole warp, a factor of 1
            // for rows whose maximum did not grow); each quarter rescales its 32 columns of O
            const bool grow = (j > 0) && (m_new > m_run);
            const bool warp_grow = __any_sync(0xffffffffu, grow);
            if (warp_grow) {
                const float f = grow ? exp2f(__fsub_rn(m_run, m_new)) : 1.0f;
                l = __fmul_rn(l, f);
                uint32_t o[32];
                tmem_ld_32x32b_x32(t_o, o);
                tmem_wait_ld();
                tmem_tie(o);
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__fmul_rn(__uint_as_float(o[i]), f));
                tmem_st_32x32b_x16(t_o, *reinterpret_cast<const uint32_t(*)[16]>(o));
                tmem_st_32x32b_x16(t_o + 16, *reinterpret_cast<const uint32_t(*)[16]>(o + 16));
            }
            // pass 2: P~ = exp2(fl(fl(s c) - m_new)), groups of G keys, into row r of the
            // 128-byte-swizzled P~ tile (16-byte granule g at g ^ (r % 8))
            uint32_t sfw = 0u;  // this quarter's scale bytes, in atom-word order
            float lb = 0.0f;
            const uint32_t prow = smem_u32(sP) + (uint32_t)r * 128u;
            auto chunk = [&](int ch, auto full_tag) {
                constexpr bool FULL = decltype(full_tag)::value;
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_s + ch * 32, v);
                tmem_wait_ld();
                tmem_tie(v);
                if (ch == 1) {
                    // the quarter's last read of S_j has landed: the MMA warp may compute S_{j+1}
                    // while this chunk's weights are made
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s_free);
                }
                float pv[32], part[16], mxp[16];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const bool valid = FULL || ch * 32 + i < nvalid;
                    pv[i] = valid ? exp2f(__fsub_rn(__fmul_rn(__uint_as_float(v[i]), c), m_new)) : 0.0f;
                }
                // the 32 weights summed as a pairwise tree, then added to the quarter's block sum
                // in order; their maximum by the same tree
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    part[i] = __fadd_rn(pv[2 * i], pv[2 * i + 1]);
                    mxp[i] = fmaxf(pv[2 * i], pv[2 * i + 1]);
                }
#pragma unroll
                for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                    for (int i = 0; i < w; ++i) {
                        part[i] = __fadd_rn(part[i], part[i + w]);
                        mxp[i] = fmaxf(mxp[i], mxp[i + w]);
                    }
                lb = __fadd_rn(lb, part[0]);
                const int gch = qq * 2 + ch;  // the chunk's 16-byte granule in the 256-key row
                uint32_t cw[4];
                if (NV) {
                    // two groups of 16: each group's maximum, its E4M3 scale s = e4m3(amax / (6 g_p))
                    // and codes e2m1(p * fl(1 / fl(dec(s) g_p)))
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        float gm[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) gm[i] = fmaxf(pv[16 * g + 2 * i], pv[16 * g + 2 * i + 1]);
#pragma unroll
                        for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                            for (int i = 0; i < w; ++i) gm[i] = fmaxf(gm[i], gm[i + w]);
                        const uint32_t sfb = cvt_e4m3x2(__fdiv_rn(gm[0], six_g), 0.0f) & 0xFFu;
                        const float rr = nv_rcp[sfb & 0x7Fu];
#pragma unroll
                        for (int i = 0; i < 16; ++i) pv[16 * g + i] = rr == 0.0f ? 0.0f : __fmul_rn(pv[16 * g + i], rr);
                        sfw |= sfb << (8 * (2 * ch + g));
                        if (tracing) p.dbg_sf[((int64_t)j * 128 + r) * C::SFB_ROW + gch * 2 + g] = (uint8_t)sfb;
                    }
                } else {
                    const uint32_t sfb = mx_scale_byte<2>(mxp[0]);
                    const float inv = mx_inv_scale(sfb);
#pragma unroll
                    for (int i = 0; i < 32; ++i) pv[i] = __fmul_rn(pv[i], inv);
                    sfw |= sfb << (8 * ch);
                    if (tracing) p.dbg_sf[((int64_t)j * 128 + r) * C::SFB_ROW + gch] = (uint8_t)sfb;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) cw[q] = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(pv + 8 * q));
                st_shared_v4(prow + (uint32_t)((gch ^ (r & 7)) * 16), cw[0], cw[1], cw[2], cw[3]);
                if (tracing) {
                    const int64_t d = (int64_t)j * 128 + r;
                    *reinterpret_cast<uint4*>(p.dbg_codes + d * 128 + gch * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                }
            };
            if (nvalid == 64) {
                chunk(0, std::true_type{});
                chunk(1, std::true_type{});
            } else {
                chunk(0, std::false_type{});
                chunk(1, std::false_type{});
            }
            l = __fadd_rn(l, lb);
            // the row's scale bytes into the P~ atoms: MXFP4 bytes 2 (qq % 2), +1 of the row's
            // word in atom qq / 2 (128 keys per atom); NVFP4 the whole word of atom qq (64 keys)
            if (NV)
                *reinterpret_cast<uint32_t*>(sPSF + qq * 512 + (r & 31) * 16 + (r >> 5) * 4) = sfw;
            else
                *reinterpret_cast<uint16_t*>(sPSF + (qq >> 1) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (qq & 1) * 2) =
                    (uint16_t)sfw;
            if (warp_grow) tmem_wait_st();
            if (tracing && qq == 0) p.dbg_m[(int64_t)j * 128 + r] = m_new;
            // the tile and atoms are written by threads and read by the tensor core
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
            m_run = m_new;
        }
        // the four quarters' sums added in a fixed order, then O / l rounded once to bf16
        if (ok) {
            red[((nb & 1) * 4 + qq) * 128 + r] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(pair);
            ok = __all_sync(0xffffffffu, mbar_wait(pair, (uint32_t)(nb & 1), p.timeout_ns, abort));
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (uint32_t)((nb - 1) & 1), p.timeout_ns, abort));
        if (ok) {
            tc_fence_after();
            const float* rl = red + (nb & 1) * 512 + r;
            const float lt = __fadd_rn(__fadd_rn(rl[0], rl[128]), __fadd_rn(rl[256], rl[384]));
            // NVFP4: O also carries the globals of P~ and V: o = O fl(fl(g_p g_v) fl(1 / l))
            const float inv_l = NV ? __fmul_rn(__fmul_rn(*p.g_p, *p.g_v), __frcp_rn(lt)) : __frcp_rn(lt);
            uint32_t o[32];
            tmem_ld_32x32b_x32(t_o, o);
            tmem_wait_ld();
            tmem_tie(o);
            if (real) {
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(o[2 * i]), inv_l),
                                                             __fmul_rn(__uint_as_float(o[2 * i + 1]), inv_l));
                    w[i] = *reinterpret_cast<uint32_t*>(&b);
                }
                uint4* dst = reinterpret_cast<uint4*>(p.o + row * 128 + qq * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            }
            if (p.stats != nullptr && real && qq == 0) p.stats[row] = make_float2(m_run, lt);
        } else if (lane == 0) {
            attn_fail(p, abort);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace fp4
