// fp4bsa.cu -- the C ABI (include/fp4bsa.h): argument validation, TMA descriptors,
// kernel launches and the device status word.  One translation unit holds every
// kernel, so the status word is a plain __device__ variable.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "fp4bsa.h"
#include "attn.cuh"
#include "attn_fused.cuh"
#include "gemm.cuh"
#include "quant.cuh"

using namespace fp4;

__device__ int g_fp4_status = 0;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;
uint64_t g_timeout_ns = kDefaultTimeoutNs;
int g_skip_iter = -1;  // test hook, see fp4bsa_test_skip_iteration
int g_gemm_ctas = 0;   // tuning hook: 0 auto (2-CTA kernel for M > 128), 1 or 2 to force

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceState {
    bool ready = false;
    bool arch_ok = false;
    int sm_count = 0;
    int pairs[4] = {0, 0, 0, 0};  // co-resident CTA pairs of gemm2_kernel<kind>
    int quant_occ[3] = {1, 1, 1};  // resident CTAs per SM of quant_kernel<kind>
    int* status = nullptr;
};

// The pair kernels move registers between warpgroups with setmaxnreg; the split is sized
// for exactly Gemm2Cfg::REG_LAUNCH registers per thread at launch, and with fewer the
// epilogue warps' increase could never be satisfied.  Checked before any pair launch.
bool launch_regs_are(const void* kernel, int want) {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.numRegs == want;
}

template <int KIND>
int max_pairs(int sm_count) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sm_count & ~1);
    cfg.blockDim = dim3(Gemm2Cfg<KIND>::THREADS);
    cfg.dynamicSmemBytes = Gemm2Cfg<KIND>::SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void*)gemm2_kernel<KIND>, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = sm_count / 2;
    }
    return n;
}

std::mutex g_mu;
DeviceState g_dev[64];
EncodeTiledFn g_encode = nullptr;

fp4_status_t device_state(DeviceState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& s = g_dev[dev];
    if (!s.ready) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&s.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FP4_ERR_CUDA;
        s.arch_ok = (major == 10 && minor == 0);
        if (s.arch_ok) {
            if (cudaGetSymbolAddress(reinterpret_cast<void**>(&s.status), g_fp4_status) != cudaSuccess)
                return FP4_ERR_CUDA;
            if (cudaFuncSetAttribute(gemm_kernel<G_MXFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     GemmCfg<G_MXFP4>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(gemm_kernel<G_NVFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     GemmCfg<G_NVFP4>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(gemm2_kernel<G_MXFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Gemm2Cfg<G_MXFP4>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(gemm2_kernel<G_NVFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Gemm2Cfg<G_NVFP4>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(gemm2_kernel<G_W4A8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Gemm2Cfg<G_W4A8>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(gemm2_kernel<G_SVD4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Gemm2Cfg<G_SVD4>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(gemm2_kernel<G_MXFP4, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Gemm2Cfg<G_MXFP4, 1>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(gemm2_kernel<G_NVFP4, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Gemm2Cfg<G_NVFP4, 2>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(gemm2_kernel<G_MXFP4, 0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Gemm2Cfg<G_MXFP4>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(gemm2_kernel<G_NVFP4, 0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Gemm2Cfg<G_NVFP4>::SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(attn_fused_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     ATT_SMEM) != cudaSuccess ||
                cudaFuncSetAttribute(attn_fused_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     ATT_SMEM) != cudaSuccess)
                return FP4_ERR_CUDA;
            {
                constexpr int R = (int)Gemm2Cfg<G_MXFP4>::REG_LAUNCH;
                const void* pair_kernels[] = {
                    (const void*)gemm2_kernel<G_MXFP4>,          (const void*)gemm2_kernel<G_NVFP4>,
                    (const void*)gemm2_kernel<G_W4A8>,           (const void*)gemm2_kernel<G_SVD4>,
                    (const void*)gemm2_kernel<G_MXFP4, 1>,       (const void*)gemm2_kernel<G_NVFP4, 2>,
                    (const void*)gemm2_kernel<G_MXFP4, 0, true>, (const void*)gemm2_kernel<G_NVFP4, 0, true>};
                for (const void* k : pair_kernels)
                    if (!launch_regs_are(k, R)) return FP4_ERR_ARCH;
            }
            if (cudaFuncSetAttribute(lowrank_down_kernel<Q_MXFP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     LR_SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(lowrank_down_kernel<LR_NO_QUANT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     LR_SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(lowrank_down_kernel<Q_MXFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     LR_SMEM_BYTES) != cudaSuccess)
                return FP4_ERR_CUDA;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&s.quant_occ[Q_MXFP4], quant_kernel<Q_MXFP4>,
                                                              QUANT_THREADS, 0) != cudaSuccess ||
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&s.quant_occ[Q_NVFP4], quant_kernel<Q_NVFP4>,
                                                              QUANT_THREADS, 0) != cudaSuccess ||
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&s.quant_occ[Q_MXFP8], quant_kernel<Q_MXFP8>,
                                                              QUANT_THREADS, 0) != cudaSuccess)
                return FP4_ERR_CUDA;
            s.pairs[G_MXFP4] = max_pairs<G_MXFP4>(s.sm_count);
            s.pairs[G_NVFP4] = max_pairs<G_NVFP4>(s.sm_count);
            s.pairs[G_W4A8] = max_pairs<G_W4A8>(s.sm_count);
            s.pairs[G_SVD4] = max_pairs<G_SVD4>(s.sm_count);
        }
        if (!g_encode) {
            cudaDriverEntryPointQueryResult q;
            void* fn = nullptr;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return FP4_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        s.ready = true;
    }
    if (!s.arch_ok) return FP4_ERR_ARCH;
    *out = &s;
    return FP4_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int group_of(fp4_fmt_t fmt) { return fmt == FP4_FMT_MXFP4 ? 32 : 16; }
inline bool fmt_ok(fp4_fmt_t fmt) { return fmt == FP4_FMT_MXFP4 || fmt == FP4_FMT_NVFP4; }
constexpr int64_t kMaxDim = (int64_t)1 << 30;

fp4_status_t check_shape(int64_t M, int64_t K, int64_t N) {
    if (M < 1) return FP4_ERR_INVALID_ARG;
    if (K < 128 || K % 128 != 0 || N < 128 || N % 128 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (M >= kMaxDim || K >= kMaxDim || N >= kMaxDim) return FP4_ERR_UNSUPPORTED_SHAPE;
    // the quantizer numbers 128-element units with 32-bit indices
    if ((M + 127) / 128 * 128 * (K / 128) >= ((int64_t)1 << 31)) return FP4_ERR_UNSUPPORTED_SHAPE;
    return FP4_OK;
}

fp4_status_t launched() { return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA; }

// One resident wave of quantize CTAs, each taking a contiguous range of 128-element units.
int quant_blocks(const DeviceState* ds, int kind, int64_t M, int64_t K) {
    const int64_t Mpad = (M + 127) & ~int64_t(127);
    const int64_t units = Mpad * (K / 128);
    const int64_t span = (QUANT_THREADS / 16) * QUANT_UNROLL;
    int64_t blocks = (units + span - 1) / span;
    const int64_t cap = (int64_t)ds->sm_count * (ds->quant_occ[kind] > 0 ? ds->quant_occ[kind] : 1);
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

// gelu: quantize bf16_rn(gelu_tanh(x)) instead of x (MXFP4 / NVFP4 only)
// heads: x is [M tokens, K = heads x 128], written head-major (MXFP4 / NVFP4 only)
fp4_status_t launch_quant(const DeviceState* ds, int kind, const void* x, int64_t M, int64_t K, const float* g,
                          uint8_t* out, uint8_t* sf, cudaStream_t st, bool gelu = false, bool heads = false) {
    const int blocks = quant_blocks(ds, kind, M, K);
    const uint4* xv = static_cast<const uint4*>(x);
    if (heads && kind == Q_MXFP4)
        quant_kernel<Q_MXFP4, false, true><<<blocks, QUANT_THREADS, 0, st>>>(xv, M, K, g, out, sf);
    else if (heads)
        quant_kernel<Q_NVFP4, false, true><<<blocks, QUANT_THREADS, 0, st>>>(xv, M, K, g, out, sf);
    else if (gelu && kind == Q_MXFP4)
        quant_kernel<Q_MXFP4, true><<<blocks, QUANT_THREADS, 0, st>>>(xv, M, K, g, out, sf);
    else if (gelu)
        quant_kernel<Q_NVFP4, true><<<blocks, QUANT_THREADS, 0, st>>>(xv, M, K, g, out, sf);
    else if (kind == Q_MXFP4)
        quant_kernel<Q_MXFP4><<<blocks, QUANT_THREADS, 0, st>>>(xv, M, K, g, out, sf);
    else if (kind == Q_NVFP4)
        quant_kernel<Q_NVFP4><<<blocks, QUANT_THREADS, 0, st>>>(xv, M, K, g, out, sf);
    else
        quant_kernel<Q_MXFP8><<<blocks, QUANT_THREADS, 0, st>>>(xv, M, K, g, out, sf);
    return launched();
}

// Encoded tensor maps are cached per host thread, keyed by every encode argument: a map
// holds only an address, a shape and a box (no memory contents), so a cached map stays
// valid for as long as the same arguments are passed, and encoding (a driver call of a
// few microseconds) happens once per distinct buffer and shape.
struct TmapKey {
    const void* ptr;
    uint64_t inner, rows, row_bytes;
    uint32_t box_inner, box_rows;
    int dt, swz;
    bool operator==(const TmapKey& o) const {
        return ptr == o.ptr && inner == o.inner && rows == o.rows && row_bytes == o.row_bytes &&
               box_inner == o.box_inner && box_rows == o.box_rows && dt == o.dt && swz == o.swz;
    }
};
constexpr int kTmapCache = 64;
struct TmapCache {
    TmapKey key[kTmapCache];
    CUtensorMap map[kTmapCache];
    int n = 0, next = 0;
};
thread_local TmapCache t_tmaps;

fp4_status_t encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t rows,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                       CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    const TmapKey key{ptr, inner, rows, row_bytes, box_inner, box_rows, (int)dt, (int)swz};
    TmapCache& c = t_tmaps;
    for (int i = 0; i < c.n; ++i)
        if (c.key[i] == key) {
            *m = c.map[i];
            return FP4_OK;
        }
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return FP4_ERR_CUDA;
    const int slot = (c.n < kTmapCache) ? c.n++ : (c.next++ % kTmapCache);
    c.key[slot] = key;
    c.map[slot] = *m;
    return FP4_OK;
}

template <int KIND>
fp4_status_t launch_gemm(const DeviceState* ds, const CUtensorMap& ta, const CUtensorMap& tb, GemmParams& p,
                         cudaStream_t st) {
    const int tiles = ((p.M + GEMM_BM - 1) / GEMM_BM) * ((p.N + GEMM_BN - 1) / GEMM_BN);
    const int grid = tiles < ds->sm_count ? tiles : ds->sm_count;
    p.timeout_ns = g_timeout_ns;
    p.skip_iter = g_skip_iter;
    p.status = ds->status;
    gemm_kernel<KIND><<<grid, GEMM_THREADS, GemmCfg<KIND>::SMEM_BYTES, st>>>(ta, tb, p);
    return launched();
}

// Scale-factor buffer seen by TMA as rows of 512-byte atoms (128 x u32), `atoms` per box.
fp4_status_t encode_sf(CUtensorMap* m, const uint8_t* sf, int64_t rows, int64_t K, int group, int atoms) {
    const uint64_t total_atoms = (uint64_t)((rows + 127) / 128) * (uint64_t)(K / (group * 4));
    return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, sf, 128, total_atoms, 512, 128, (uint32_t)atoms,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
}

// ---------------------------------------------------------------- stream-K plan (small M)
// With fewer 256x256 tiles than two rounds of pairs, the 2-CTA kernel can spread the
// flattened (tile, K block) space evenly over the pairs (stream-K); tiles split between
// pairs are summed through fp32 slabs in the linear's workspace.  The workspace is sized
// for kPlanPairs (a B200's 148 SMs); a device whose pair count needs more slabs per tile
// runs whole tiles instead.
constexpr int kPlanPairs = 74;
int g_stream_k = 0;  // tuning / test hook: 0 default (off), 1 never, 2 whenever the workspace allows
int g_pdl = 1;       // tuning hook: programmatic launch of fp4_linear's short GEMMs after the quantize (1 on, 0 off)

int64_t sk_kstart(int64_t p, int64_t total, int P) { return p * total / P; }
int64_t sk_pair_of(int64_t k, int64_t total, int P) {
    int64_t q = k * P / total;
    while (q + 1 < P && sk_kstart(q + 1, total, P) <= k) ++q;
    while (q > 0 && sk_kstart(q, total, P) > k) --q;
    return q;
}
// largest number of pairs sharing one tile
int sk_seg_max(int64_t tiles, int64_t num_kb, int P) {
    const int64_t total = tiles * num_kb;
    int64_t m = 1;
    for (int64_t t = 0; t < tiles; ++t)
        m = std::max(m, sk_pair_of(t * num_kb + num_kb - 1, total, P) - sk_pair_of(t * num_kb, total, P) + 1);
    return (int)m;
}
// K blocks of the 2-CTA MXFP4 / NVFP4 kernel (256 K per stage, the last may be half)
int64_t sk_num_kb(int64_t K) { return (K + 255) / 256; }

// Low-rank down-projection u = x L1 (W4A8 / W4A4 SVDQuant): with few 128-row blocks (the
// 4290-token W4A8 shape has 34) K is split over up to 8 blocks per row block, whose fp32
// partial sums a second kernel adds in split order.  Only the full linears, which own a
// workspace, split; the split is a function of (M, K) alone, so the workspace size is too.
constexpr int kLowrankFuseBlocks = 64;  // row blocks from which one pass streams X at full speed
int lr_split(int64_t M, int64_t K) {
    const int64_t blocks = (M + LR_ROWS - 1) / LR_ROWS, nkc = K / LR_KC;
    if (blocks >= kLowrankFuseBlocks) return 1;
    for (int sp : {8, 4, 2})
        if (nkc % sp == 0 && nkc / sp >= 2) return sp;
    return 1;
}
size_t lr_partial_bytes(int64_t M, int64_t K) {
    const int sp = lr_split(M, K);
    const int64_t mpad = (M + LR_ROWS - 1) / LR_ROWS * LR_ROWS;
    return sp > 1 ? align256((size_t)sp * mpad * 32 * sizeof(float)) : 0;
}
// X -> (codes, scales) in format QK and u = X L1, in one pass over X.  With few row blocks
// and no room for a K split (the standalone quantize calls take no workspace), the
// 34-odd blocks of one pass cannot stream X fast enough, so the quantizer runs as its own
// grid first (at 4290 x 3072: 42 us for the two launches against 53 us fused).
template <int QK>
fp4_status_t launch_lowrank(const DeviceState* ds, const void* x_bf16, const void* l1_bf16, int64_t M, int64_t K,
                            void* u_pair, float* partial, uint8_t* codes, uint8_t* sf, cudaStream_t st) {
    const int blocks = (int)((M + LR_ROWS - 1) / LR_ROWS);
    const auto x = static_cast<const __nv_bfloat16*>(x_bf16);
    const auto l1 = static_cast<const __nv_bfloat16*>(l1_bf16);
    const auto u = static_cast<__nv_bfloat16*>(u_pair);
    const int sp = partial ? lr_split(M, K) : 1;
    if (sp == 1 && blocks < kLowrankFuseBlocks) {
        fp4_status_t s = launch_quant(ds, QK, x_bf16, M, K, nullptr, codes, sf, st);
        if (s != FP4_OK) return s;
        lowrank_down_kernel<LR_NO_QUANT><<<blocks, LR_THREADS, LR_SMEM_BYTES, st>>>(x, l1, (int)M, (int)K, u,
                                                                                   nullptr, 0, nullptr, nullptr);
        return launched();
    }
    if (sp == 1) {
        lowrank_down_kernel<QK><<<blocks, LR_THREADS, LR_SMEM_BYTES, st>>>(x, l1, (int)M, (int)K, u, nullptr, 0,
                                                                          codes, sf);
        return launched();
    }
    lowrank_down_kernel<QK><<<dim3(blocks, sp), LR_THREADS, LR_SMEM_BYTES, st>>>(
        x, l1, (int)M, (int)K, u, partial, (int)(K / LR_KC / sp), codes, sf);
    lowrank_reduce_kernel<<<(int)((M * 32 + 255) / 256), 256, 0, st>>>(partial, (int)M, blocks * LR_ROWS, sp, u);
    return launched();
}
// Every pair's share must hold at least one K block (tiles * K blocks >= pairs): a pair
// with an empty share would be counted among a tile's segments without ever arriving.
// Only on request (hook): measured on B200, the small problems it targets are bound by
// the kernel's fixed launch / prologue / pipeline-fill cost, and the slab round trip and
// unit hand-offs made stream-K slower than whole tiles for every text-token shape tried.
bool sk_wanted(int64_t M, int64_t K, int64_t N) {
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    if (g_stream_k == 1 || sk_num_kb(K) < 4 || tiles * sk_num_kb(K) < kPlanPairs) return false;
    return g_stream_k == 2;
}
size_t sk_bytes(int64_t M, int64_t K, int64_t N) {
    if (!sk_wanted(M, K, N)) return 0;
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    return align256((size_t)tiles * sk_seg_max(tiles, sk_num_kb(K), kPlanPairs) * 65536 * 4) +
           align256((size_t)tiles * 64);
}

// 2-CTA GEMM: A box 128 rows, B box 128 rows (half of the 256-wide N tile) per CTA.
// tu / tl: the W4A8 low-rank operands (u pair, L2 [rank, N]); other kinds pass any map.
// OUTQ != 0: the fused GELU + quantize output (p.h_codes / p.h_sf) instead of p.y.
// pdl: launch with programmatic stream serialization, so the kernel's launch and prologue
// overlap the previous kernel on the stream (its producer waits before reading A); used
// right after our own quantize kernel, which does not touch the GEMM's output.
template <int KIND, int OUTQ = 0, bool SK = false>
fp4_status_t launch_gemm2(const DeviceState* ds, const CUtensorMap& ta, const CUtensorMap& tb, const uint8_t* sfa,
                          const uint8_t* sfb, GemmParams& p, cudaStream_t st, const CUtensorMap* tu = nullptr,
                          const CUtensorMap* tl = nullptr, bool pdl = false) {
    // the launch's shared-memory size is the kernel's own configuration (kind and output)
    using C = Gemm2Cfg<KIND, OUTQ>;
    CUtensorMap tsa, tsb;
    fp4_status_t s;
    if ((s = encode_sf(&tsa, sfa, p.M, p.K, C::G, C::ATOMS)) != FP4_OK) return s;
    if ((s = encode_sf(&tsb, sfb, p.N, p.K, C::G, C::ATOMS)) != FP4_OK) return s;
    // output: bf16 [M, N], stored by the epilogue in 32-row boxes of EPI_COLS columns (64:
    // 128-byte swizzle, 32: 64-byte swizzle)
    CUtensorMap ty = ta;
    if (OUTQ == 0 && (s = encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.y, (uint64_t)p.N, (uint64_t)p.M,
                                    (uint64_t)p.N * 2, C::EPI_COLS, 32,
                                    C::EPI_COLS == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B)) != FP4_OK)
        return s;
    const int tiles = ((p.M + 255) / 256) * ((p.N + 255) / 256);
    // stream-K keeps every pair busy; whole tiles need no more pairs than tiles
    const int pairs = (SK || tiles >= ds->pairs[KIND]) ? ds->pairs[KIND] : tiles;
    p.timeout_ns = g_timeout_ns;
    p.skip_iter = g_skip_iter;
    p.status = ds->status;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, gemm2_kernel<KIND, OUTQ, SK>, ta, tb, tsa, tsb, ty, tu ? *tu : ta, tl ? *tl : tb, p) !=
        cudaSuccess)
        return FP4_ERR_CUDA;
    return launched();
}

}  // namespace

extern "C" {

size_t fp4_codes_bytes(fp4_fmt_t fmt, int64_t rows, int64_t K) {
    if (!fmt_ok(fmt) || rows < 0 || K < 0 || (K & 1)) return 0;
    return (size_t)rows * (size_t)(K / 2);
}

size_t fp4_sf_bytes(fp4_fmt_t fmt, int64_t rows, int64_t K) {
    if (!fmt_ok(fmt) || rows < 0 || K < 0 || K % 128 != 0) return 0;
    const int64_t rp = (rows + 127) / 128 * 128;
    return (size_t)rp * (size_t)(K / group_of(fmt));
}

size_t fp4_linear_workspace_bytes(fp4_fmt_t fmt, int64_t M, int64_t K, int64_t N) {
    if (!fmt_ok(fmt) || check_shape(M, K, N) != FP4_OK) return 0;
    // quantized activations, then (small M) the stream-K partial slabs and counters
    return align256(fp4_codes_bytes(fmt, M, K)) + align256(fp4_sf_bytes(fmt, M, K)) + sk_bytes(M, K, N);
}

size_t w4a8_workspace_bytes(int64_t M, int64_t K, int64_t N, int rank) {
    if (rank != 32 || check_shape(M, K, N) != FP4_OK) return 0;
    // E4M3 codes, E8M0 scales, u pair (M x 2 rank bf16), split-K partials of u
    return align256((size_t)M * K) + align256(fp4_sf_bytes(FP4_FMT_MXFP4, M, K)) + align256((size_t)M * rank * 4) +
           lr_partial_bytes(M, K);
}

size_t w4a4_workspace_bytes(int64_t M, int64_t K, int64_t N, int rank) {
    if (rank != 32 || check_shape(M, K, N) != FP4_OK) return 0;
    // MXFP4 codes, E8M0 scales, u pair (M x 2 rank bf16), split-K partials of u
    return align256(fp4_codes_bytes(FP4_FMT_MXFP4, M, K)) + align256(fp4_sf_bytes(FP4_FMT_MXFP4, M, K)) +
           align256((size_t)M * rank * 4) + lr_partial_bytes(M, K);
}

fp4_status_t fp4_tensor_amax(const void* x_bf16, int64_t n, float* amax_out, void* stream) {
    if (!x_bf16 || !amax_out || n < 1) return FP4_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(amax_out) & 3u)) return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    fp4_status_t s = device_state(&ds);
    if (s != FP4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(amax_out, 0, sizeof(float), st) != cudaSuccess) return FP4_ERR_CUDA;
    int64_t blocks = (n / 8 + 255) / 256;
    if (blocks > ds->sm_count * 8) blocks = ds->sm_count * 8;
    if (blocks < 1) blocks = 1;
    amax_kernel<<<(int)blocks, 256, 0, st>>>(static_cast<const uint16_t*>(x_bf16), n,
                                             reinterpret_cast<unsigned int*>(amax_out));
    return launched();
}

fp4_status_t fp4_calibrate_act_global(const void* x_bf16, int64_t n, float* amax_inout, float* g_out,
                                      void* stream) {
    if (!x_bf16 || !amax_inout || !g_out || n < 1) return FP4_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(amax_inout) & 3u) ||
        (reinterpret_cast<uintptr_t>(g_out) & 3u))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    fp4_status_t s = device_state(&ds);
    if (s != FP4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int64_t blocks = (n / 8 + 255) / 256;
    if (blocks > ds->sm_count * 8) blocks = ds->sm_count * 8;
    if (blocks < 1) blocks = 1;
    // the running amax is raised in place (max is order-independent), then g = T / 2688
    amax_kernel<<<(int)blocks, 256, 0, st>>>(static_cast<const uint16_t*>(x_bf16), n,
                                             reinterpret_cast<unsigned int*>(amax_inout));
    if ((s = launched()) != FP4_OK) return s;
    nv_global_from_kernel<<<1, 1, 0, st>>>(amax_inout, g_out);
    return launched();
}

fp4_status_t fp4_quantize_act(fp4_fmt_t fmt, const void* x_bf16, int64_t M, int64_t K, const float* a_global,
                              uint8_t* x_codes, uint8_t* x_sf, void* stream) {
    if (!fmt_ok(fmt) || !x_bf16 || !x_codes || !x_sf) return FP4_ERR_INVALID_ARG;
    if ((fmt == FP4_FMT_NVFP4) != (a_global != nullptr)) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, 128);
    if (s != FP4_OK) return s;
    if (!aligned16(x_bf16) || !aligned16(x_codes) || !aligned16(x_sf) || !aligned16(a_global))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    return launch_quant(ds, fmt == FP4_FMT_MXFP4 ? Q_MXFP4 : Q_NVFP4, x_bf16, M, K, a_global, x_codes, x_sf,
                        static_cast<cudaStream_t>(stream));
}

fp4_status_t fp4_gelu_quantize_act(fp4_fmt_t fmt, const void* z_bf16, int64_t M, int64_t K,
                                   const float* a_global, uint8_t* x_codes, uint8_t* x_sf, void* stream) {
    if (!fmt_ok(fmt) || !z_bf16 || !x_codes || !x_sf) return FP4_ERR_INVALID_ARG;
    if ((fmt == FP4_FMT_NVFP4) != (a_global != nullptr)) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, 128);
    if (s != FP4_OK) return s;
    if (!aligned16(z_bf16) || !aligned16(x_codes) || !aligned16(x_sf) || (reinterpret_cast<uintptr_t>(a_global) & 3u))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    return launch_quant(ds, fmt == FP4_FMT_MXFP4 ? Q_MXFP4 : Q_NVFP4, z_bf16, M, K, a_global, x_codes, x_sf,
                        static_cast<cudaStream_t>(stream), true);
}

size_t fp4_heads_codes_bytes(fp4_fmt_t fmt, int64_t T, int64_t H, int64_t D) {
    if (!fmt_ok(fmt) || T < 0 || H < 0 || D != FP4_HEAD_DIM) return 0;
    return (size_t)H * (size_t)((T + 127) / 128 * 128) * (size_t)(D / 2);
}

size_t fp4_heads_sf_bytes(fp4_fmt_t fmt, int64_t T, int64_t H, int64_t D) {
    if (!fmt_ok(fmt) || T < 0 || H < 0 || D != FP4_HEAD_DIM) return 0;
    return (size_t)H * fp4_sf_bytes(fmt, T, D);
}

fp4_status_t fp4_quantize_heads(fp4_fmt_t fmt, const void* x_bf16, int64_t T, int64_t H, int64_t D,
                                const float* g, uint8_t* codes, uint8_t* sf, void* stream) {
    if (!fmt_ok(fmt) || !x_bf16 || !codes || !sf || T < 1 || H < 1) return FP4_ERR_INVALID_ARG;
    if ((fmt == FP4_FMT_NVFP4) != (g != nullptr)) return FP4_ERR_INVALID_ARG;
    if (D != FP4_HEAD_DIM || H >= kMaxDim / D) return FP4_ERR_UNSUPPORTED_SHAPE;
    fp4_status_t s = check_shape(T, H * D, 128);
    if (s != FP4_OK) return s;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(sf) || (reinterpret_cast<uintptr_t>(g) & 3u))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    return launch_quant(ds, fmt == FP4_FMT_MXFP4 ? Q_MXFP4 : Q_NVFP4, x_bf16, T, H * D, g, codes, sf,
                        static_cast<cudaStream_t>(stream), false, true);
}

fp4_status_t fp4_pack_weight(fp4_fmt_t fmt, const void* w_bf16, int64_t N, int64_t K, uint8_t* w_codes,
                             uint8_t* w_sf, float* w_global, void* stream) {
    if (!fmt_ok(fmt) || !w_bf16 || !w_codes || !w_sf) return FP4_ERR_INVALID_ARG;
    if ((fmt == FP4_FMT_NVFP4) != (w_global != nullptr)) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(N, K, 128);
    if (s != FP4_OK) return s;
    if (!aligned16(w_bf16) || !aligned16(w_codes) || !aligned16(w_sf) || !aligned16(w_global))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (fmt == FP4_FMT_NVFP4) {
        if ((s = fp4_tensor_amax(w_bf16, N * K, w_global, stream)) != FP4_OK) return s;
        nv_global_kernel<<<1, 1, 0, st>>>(w_global);
        if ((s = launched()) != FP4_OK) return s;
    }
    return launch_quant(ds, fmt == FP4_FMT_MXFP4 ? Q_MXFP4 : Q_NVFP4, w_bf16, N, K, w_global, w_codes, w_sf, st);
}

}  // extern "C"

namespace {
// fp4_gemm, optionally with a stream-K workspace (sk_ws: slabs then counters, sk_ws_bytes
// as sized by sk_bytes) that fp4_linear passes for small M.
fp4_status_t gemm_impl(fp4_fmt_t fmt, const uint8_t* a_codes, const uint8_t* a_sf, int64_t M, int64_t K, int64_t N,
                       const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global, const float* a_global,
                       const void* bias_f16, void* y_bf16, void* stream, uint8_t* sk_ws, size_t sk_ws_bytes,
                       bool pdl = false) {
    if (!fmt_ok(fmt) || !a_codes || !a_sf || !w_codes || !w_sf || !y_bf16) return FP4_ERR_INVALID_ARG;
    const bool nv = (fmt == FP4_FMT_NVFP4);
    if (nv != (w_global != nullptr) || nv != (a_global != nullptr)) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, N);
    if (s != FP4_OK) return s;
    if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(w_codes) || !aligned16(w_sf) || !aligned16(y_bf16) ||
        !aligned16(bias_f16) || (reinterpret_cast<uintptr_t>(w_global) & 3u) ||
        (reinterpret_cast<uintptr_t>(a_global) & 3u))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    // stream-K over the 2-CTA kernel when the linear provided its workspace and the pair
    // count of this device fits the slabs it was sized for
    bool sk = false;
    int seg_max = 1;
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    if (sk_ws && sk_ws_bytes > 0 && g_gemm_ctas != 1) {
        const int P = ds->pairs[nv ? G_NVFP4 : G_MXFP4];
        if (tiles * sk_num_kb(K) >= P) {
            seg_max = sk_seg_max(tiles, sk_num_kb(K), P);
            sk = (size_t)tiles * seg_max * 65536 * 4 + (size_t)tiles * 64 <= sk_ws_bytes;
        }
    }
    // 2-CTA 256x256 tiles (faster at every M measured) unless M fits one 128-row tile or
    // the 1-CTA kernel is forced (tuning hook)
    const bool pair = sk || (g_gemm_ctas != 1 && M > GEMM_BM);
    CUtensorMap ta, tb;
    if ((s = encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, K / 2, M, K / 2, 128, GEMM_BM)) != FP4_OK)
        return s;
    if ((s = encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, 128, pair ? 128 : GEMM_BN)) !=
        FP4_OK)
        return s;
    GemmParams p{};
    p.M = (int)M, p.N = (int)N, p.K = (int)K;
    p.sfa = a_sf, p.sfb = w_sf, p.g_a = a_global, p.g_w = w_global;
    p.bias = static_cast<const __half*>(bias_f16);
    p.y = static_cast<__nv_bfloat16*>(y_bf16);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (sk) {
        const size_t slab_bytes = align256((size_t)tiles * seg_max * 65536 * 4);
        p.seg_max = seg_max;
        p.partials = reinterpret_cast<float*>(sk_ws);
        p.counters = reinterpret_cast<int*>(sk_ws + slab_bytes);
        if (cudaMemsetAsync(p.counters, 0, (size_t)tiles * 64, st) != cudaSuccess) return FP4_ERR_CUDA;
    }
    if (sk)
        return nv ? launch_gemm2<G_NVFP4, 0, true>(ds, ta, tb, a_sf, w_sf, p, st, nullptr, nullptr, pdl)
                  : launch_gemm2<G_MXFP4, 0, true>(ds, ta, tb, a_sf, w_sf, p, st, nullptr, nullptr, pdl);
    if (pair)
        return nv ? launch_gemm2<G_NVFP4>(ds, ta, tb, a_sf, w_sf, p, st, nullptr, nullptr, pdl)
                  : launch_gemm2<G_MXFP4>(ds, ta, tb, a_sf, w_sf, p, st, nullptr, nullptr, pdl);
    return nv ? launch_gemm<G_NVFP4>(ds, ta, tb, p, st) : launch_gemm<G_MXFP4>(ds, ta, tb, p, st);
}
}  // namespace

extern "C" {

fp4_status_t fp4_gemm(fp4_fmt_t fmt, const uint8_t* a_codes, const uint8_t* a_sf, int64_t M, int64_t K, int64_t N,
                      const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global, const float* a_global,
                      const void* bias_f16, void* y_bf16, void* stream) {
    return gemm_impl(fmt, a_codes, a_sf, M, K, N, w_codes, w_sf, w_global, a_global, bias_f16, y_bf16, stream,
                     nullptr, 0);
}

size_t fp4_heads_vt_codes_bytes(fp4_fmt_t fmt, int64_t T, int64_t H, int64_t D) {
    if (!fmt_ok(fmt) || T < 0 || H < 0 || D != FP4_HEAD_DIM) return 0;
    return (size_t)H * (size_t)D * (size_t)((T + 127) / 128 * 128 / 2);
}

size_t fp4_heads_vt_sf_bytes(fp4_fmt_t fmt, int64_t T, int64_t H, int64_t D) {
    if (!fmt_ok(fmt) || T < 0 || H < 0 || D != FP4_HEAD_DIM) return 0;
    return (size_t)H * fp4_sf_bytes(fmt, D, (T + 127) / 128 * 128);
}

fp4_status_t fp4_quantize_heads_vt(fp4_fmt_t fmt, const void* v_bf16, int64_t T, int64_t H, int64_t D,
                                   const float* g, uint8_t* codes, uint8_t* sf, void* stream) {
    if (!fmt_ok(fmt) || !v_bf16 || !codes || !sf || T < 1 || H < 1) return FP4_ERR_INVALID_ARG;
    if ((fmt == FP4_FMT_NVFP4) != (g != nullptr)) return FP4_ERR_INVALID_ARG;
    if (D != FP4_HEAD_DIM || H >= kMaxDim / D || T >= kMaxDim || H >= 65536) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(v_bf16) || !aligned16(codes) || !aligned16(sf) || (reinterpret_cast<uintptr_t>(g) & 3u))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    fp4_status_t s = device_state(&ds);
    if (s != FP4_OK) return s;
    const int64_t tpad = (T + 127) / 128 * 128;
    const dim3 grid((unsigned)(tpad / 128), (unsigned)H);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (fmt == FP4_FMT_NVFP4)
        quant_vt_kernel<Q_NVFP4><<<grid, 128, 0, cs>>>(static_cast<const __nv_bfloat16*>(v_bf16), T, (int)H, tpad, g,
                                                       codes, sf);
    else
        quant_vt_kernel<Q_MXFP4><<<grid, 128, 0, cs>>>(static_cast<const __nv_bfloat16*>(v_bf16), T, (int)H, tpad,
                                                       nullptr, codes, sf);
    return launched();
}

fp4_status_t fp4_attn_softmax_quant(fp4_fmt_t fmt, const void* s_bf16, int64_t T_q, int64_t T_kv, float scale,
                                    const float* p_global, void* stats, uint8_t* p_codes, uint8_t* p_sf,
                                    void* stream) {
    if (!fmt_ok(fmt) || !s_bf16 || !stats || !p_codes || !p_sf || T_q < 1 || T_kv < 1) return FP4_ERR_INVALID_ARG;
    if ((fmt == FP4_FMT_NVFP4) != (p_global != nullptr)) return FP4_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(p_global) & 3u) return FP4_ERR_MISALIGNED;
    if (!(scale > 0.0f) || !(scale < 3.0e38f)) return FP4_ERR_INVALID_ARG;
    if (T_q >= kMaxDim || T_kv >= kMaxDim || T_q >= (int64_t)1 << 31) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(s_bf16) || !aligned16(stats) || !aligned16(p_codes) || !aligned16(p_sf))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    fp4_status_t st = device_state(&ds);
    if (st != FP4_OK) return st;
    const int64_t kpad = (T_kv + 127) / 128 * 128, qpad = (T_q + 127) / 128 * 128;
    // c = scale * log2(e), rounded once to fp32; both kernels take exp2 of fl(fl(s c) - m)
    const float c = (float)((double)scale * 1.4426950408889634);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    softmax_max_kernel<<<(unsigned)T_q, SOFTMAX_THREADS, 0, cs>>>(static_cast<const __nv_bfloat16*>(s_bf16), kpad,
                                                                   T_kv, c, static_cast<float2*>(stats));
    if ((st = launched()) != FP4_OK) return st;
    const auto sb = static_cast<const __nv_bfloat16*>(s_bf16);
    const auto sp = static_cast<float2*>(stats);
    if (fmt == FP4_FMT_NVFP4)
        softmax_quant_kernel<Q_NVFP4><<<(unsigned)qpad, SOFTMAX_THREADS, 0, cs>>>(sb, T_q, kpad, T_kv, c, sp, p_global,
                                                                                 p_codes, p_sf);
    else
        softmax_quant_kernel<Q_MXFP4><<<(unsigned)qpad, SOFTMAX_THREADS, 0, cs>>>(sb, T_q, kpad, T_kv, c, sp, nullptr,
                                                                                 p_codes, p_sf);
    return launched();
}

fp4_status_t fp4_attn_pv(fp4_fmt_t fmt, const uint8_t* p_codes, const uint8_t* p_sf, const float* p_global,
                         int64_t T_q, int64_t T_kv, const uint8_t* vt_codes, const uint8_t* vt_sf, const float* v_global,
                         int64_t H, int64_t D, int64_t head, const void* stats, void* o_bf16, void* stream) {
    if (!fmt_ok(fmt) || !p_codes || !p_sf || !vt_codes || !vt_sf || !o_bf16) return FP4_ERR_INVALID_ARG;
    if (!aligned16(stats)) return FP4_ERR_MISALIGNED;
    if (T_q < 1 || T_kv < 1 || H < 1 || head < 0 || head >= H) return FP4_ERR_INVALID_ARG;
    if (D != FP4_HEAD_DIM) return FP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t kpad = (T_kv + 127) / 128 * 128;
    // head `head` of V^T: D rows of kpad keys, its scale atoms after the previous heads'
    const uint8_t* vc = vt_codes + (size_t)head * D * (kpad / 2);
    const uint8_t* vs = vt_sf + (size_t)head * fp4_sf_bytes(fmt, D, kpad);
    // O = P V_h: P is the activation operand (M = T_q, K = the padded keys), V_h^T the weight
    // (NVFP4: the epilogue applies g_P g_V; gemm_impl checks that both are given)
    fp4_status_t s = gemm_impl(fmt, p_codes, p_sf, T_q, kpad, D, vc, vs, v_global, p_global, nullptr, o_bf16, stream,
                               nullptr, 0);
    if (s != FP4_OK || !stats) return s;
    // then each row of O divided by its softmax sum
    const int64_t vecs = T_q * (D / 8);
    attn_row_scale_kernel<<<(unsigned)((vecs + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<__nv_bfloat16*>(o_bf16), T_q, (int)D, static_cast<const float2*>(stats));
    return launched();
}

fp4_status_t fp4_attn_scores(fp4_fmt_t fmt, const uint8_t* q_codes, const uint8_t* q_sf, int64_t T_q,
                             const uint8_t* k_codes, const uint8_t* k_sf, int64_t T_kv, int64_t H, int64_t D,
                             int64_t head, const float* g_q, const float* g_k, void* s_bf16, void* stream) {
    if (!fmt_ok(fmt) || !q_codes || !q_sf || !k_codes || !k_sf || !s_bf16) return FP4_ERR_INVALID_ARG;
    if (T_q < 1 || T_kv < 1 || H < 1 || head < 0 || head >= H) return FP4_ERR_INVALID_ARG;
    if (D != FP4_HEAD_DIM) return FP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t tq_pad = (T_q + 127) / 128 * 128, tk_pad = (T_kv + 127) / 128 * 128;
    // head `head` of the head-major buffers: its codes, then its scale atoms
    const uint8_t* qc = q_codes + (size_t)head * tq_pad * (D / 2);
    const uint8_t* kc = k_codes + (size_t)head * tk_pad * (D / 2);
    const uint8_t* qs = q_sf + (size_t)head * fp4_sf_bytes(fmt, T_q, D);
    const uint8_t* ks = k_sf + (size_t)head * fp4_sf_bytes(fmt, T_kv, D);
    // S = Q_h K_h^T: Q_h is the activation operand (M = T_q), K_h the weight operand over
    // all T_kv_pad key rows (padding keys have zero codes, so their columns hold 0)
    return gemm_impl(fmt, qc, qs, T_q, D, tk_pad, kc, ks, g_k, g_q, nullptr, s_bf16, stream, nullptr, 0);
}

}  // extern "C"

namespace {
fp4_status_t attn_fused_impl(fp4_fmt_t fmt, const uint8_t* q_codes, const uint8_t* q_sf, int64_t T_q,
                             const uint8_t* k_codes, const uint8_t* k_sf, int64_t T_kv, const uint8_t* vt_codes,
                             const uint8_t* vt_sf, int64_t H, int64_t D, int64_t head, float scale,
                             const float* g_q, const float* g_k, const float* g_v, const float* p_global,
                             void* stats, void* o_bf16, int64_t trace_tile, float* trace_m, uint8_t* trace_codes,
                             uint8_t* trace_sf, void* stream) {
    if (!fmt_ok(fmt) || !q_codes || !q_sf || !k_codes || !k_sf || !vt_codes || !vt_sf || !o_bf16)
        return FP4_ERR_INVALID_ARG;
    const bool nv = fmt == FP4_FMT_NVFP4;
    // NVFP4 takes all four globals, MXFP4 none
    if ((nv && (!g_q || !g_k || !g_v || !p_global)) || (!nv && (g_q || g_k || g_v || p_global)))
        return FP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(g_q) | reinterpret_cast<uintptr_t>(g_k) | reinterpret_cast<uintptr_t>(g_v) |
         reinterpret_cast<uintptr_t>(p_global)) & 3u)
        return FP4_ERR_MISALIGNED;
    if (T_q < 1 || T_kv < 1 || H < 1 || head < 0 || head >= H) return FP4_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || !(scale < 3.0e38f)) return FP4_ERR_INVALID_ARG;
    if (D != FP4_HEAD_DIM) return FP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t tq_pad = (T_q + 127) / 128 * 128, tk_pad = (T_kv + 127) / 128 * 128;
    // TMA row coordinates are 32-bit: every head's padded rows must stay below 2^31
    if (T_q >= kMaxDim || T_kv >= kMaxDim || H * tq_pad >= ((int64_t)1 << 31) || H * tk_pad >= ((int64_t)1 << 31))
        return FP4_ERR_UNSUPPORTED_SHAPE;
    const bool tracing = trace_m || trace_codes || trace_sf;
    if (tracing && (!trace_m || !trace_codes || !trace_sf || trace_tile < 0 || trace_tile >= tq_pad / 128))
        return FP4_ERR_INVALID_ARG;
    if (!aligned16(q_codes) || !aligned16(q_sf) || !aligned16(k_codes) || !aligned16(k_sf) || !aligned16(vt_codes) ||
        !aligned16(vt_sf) || !aligned16(stats) || !aligned16(o_bf16) || !aligned16(trace_m) ||
        !aligned16(trace_codes) || !aligned16(trace_sf))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    fp4_status_t s = device_state(&ds);
    if (s != FP4_OK) return s;
    // Q and K: all heads' rows of 64 bytes (zero-filled to the 128-byte box); V^T: H * 128
    // rows of T_kv_pad / 2 bytes, one 256-key box per block
    CUtensorMap tq, tk, tv;
    if ((s = encode_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_codes, D / 2, (uint64_t)(H * tq_pad), D / 2, 128, 128)) !=
        FP4_OK)
        return s;
    if ((s = encode_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_codes, D / 2, (uint64_t)(H * tk_pad), D / 2, 128, 256)) !=
        FP4_OK)
        return s;
    if ((s = encode_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, vt_codes, (uint64_t)(tk_pad / 2), (uint64_t)(H * D),
                       (uint64_t)(tk_pad / 2), 128, 128)) != FP4_OK)
        return s;
    AttnParams p{};
    p.T_q = T_q, p.T_kv = T_kv, p.tq_pad = tq_pad, p.tk_pad = tk_pad;
    p.head = (int)head;
    p.nblk = (int)((tk_pad + 255) / 256);
    p.c = (float)((double)scale * 1.4426950408889634);
    p.q_sf = q_sf + (size_t)head * fp4_sf_bytes(fmt, T_q, D);
    p.k_sf = k_sf + (size_t)head * fp4_sf_bytes(fmt, T_kv, D);
    p.v_sf = vt_sf + (size_t)head * fp4_sf_bytes(fmt, D, tk_pad);
    p.o = static_cast<__nv_bfloat16*>(o_bf16);
    p.stats = static_cast<float2*>(stats);
    p.g_q = g_q, p.g_k = g_k, p.g_v = g_v, p.g_p = p_global;
    p.trace_tile = tracing ? (int)trace_tile : -1;
    p.dbg_m = trace_m, p.dbg_codes = trace_codes, p.dbg_sf = trace_sf;
    p.timeout_ns = g_timeout_ns;
    p.status = ds->status;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (nv)
        attn_fused_kernel<true><<<(unsigned)(tq_pad / 128), ATT_THREADS, ATT_SMEM, cs>>>(tq, tk, tv, p);
    else
        attn_fused_kernel<false><<<(unsigned)(tq_pad / 128), ATT_THREADS, ATT_SMEM, cs>>>(tq, tk, tv, p);
    return launched();
}
}  // namespace

extern "C" {

fp4_status_t fp4_attn_fused(fp4_fmt_t fmt, const uint8_t* q_codes, const uint8_t* q_sf, int64_t T_q,
                            const uint8_t* k_codes, const uint8_t* k_sf, int64_t T_kv, const uint8_t* vt_codes,
                            const uint8_t* vt_sf, int64_t H, int64_t D, int64_t head, float scale, const float* g_q,
                            const float* g_k, const float* g_v, const float* p_global, void* stats, void* o_bf16,
                            void* stream) {
    return attn_fused_impl(fmt, q_codes, q_sf, T_q, k_codes, k_sf, T_kv, vt_codes, vt_sf, H, D, head, scale, g_q, g_k,
                           g_v, p_global, stats, o_bf16, -1, nullptr, nullptr, nullptr, stream);
}

fp4_status_t fp4_attn_fused_trace(fp4_fmt_t fmt, const uint8_t* q_codes, const uint8_t* q_sf, int64_t T_q,
                                  const uint8_t* k_codes, const uint8_t* k_sf, int64_t T_kv, const uint8_t* vt_codes,
                                  const uint8_t* vt_sf, int64_t H, int64_t D, int64_t head, float scale,
                                  const float* g_q, const float* g_k, const float* g_v, const float* p_global,
                                  void* stats, void* o_bf16, int64_t trace_tile, float* trace_m,
                                  uint8_t* trace_codes, uint8_t* trace_sf, void* stream) {
    return attn_fused_impl(fmt, q_codes, q_sf, T_q, k_codes, k_sf, T_kv, vt_codes, vt_sf, H, D, head, scale, g_q, g_k,
                           g_v, p_global, stats, o_bf16, trace_tile, trace_m, trace_codes, trace_sf, stream);
}

fp4_status_t fp4_linear(fp4_fmt_t fmt, const void* x_bf16, int64_t M, int64_t K, int64_t N, const uint8_t* w_codes,
                        const uint8_t* w_sf, const float* w_global, const float* a_global, const void* bias_f16,
                        void* y_bf16, void* workspace, size_t ws_bytes, void* stream) {
    if (!fmt_ok(fmt) || !x_bf16 || !workspace) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, N);
    if (s != FP4_OK) return s;
    if (ws_bytes < fp4_linear_workspace_bytes(fmt, M, K, N)) return FP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    uint8_t* codes = static_cast<uint8_t*>(workspace);
    uint8_t* sf = codes + align256(fp4_codes_bytes(fmt, M, K));
    // validate the GEMM's arguments before launching anything
    const bool nv = (fmt == FP4_FMT_NVFP4);
    if (!w_codes || !w_sf || !y_bf16 || nv != (w_global != nullptr) || nv != (a_global != nullptr))
        return FP4_ERR_INVALID_ARG;
    if ((s = fp4_quantize_act(fmt, x_bf16, M, K, a_global, codes, sf, stream)) != FP4_OK) return s;
    // small M: the stream-K slabs follow the quantized activations
    const size_t sk = sk_bytes(M, K, N);
    uint8_t* sk_ws = sk ? sf + align256(fp4_sf_bytes(fmt, M, K)) : nullptr;
    // short GEMMs (at most two rounds of 256x256 tiles on a B200) overlap their launch and
    // prologue with the quantize kernel; measured 5-7 % faster there, and no gain on long ones
    const bool pdl = g_pdl != 0 && ((M + 255) / 256) * ((N + 255) / 256) <= 2 * kPlanPairs;
    return gemm_impl(fmt, codes, sf, M, K, N, w_codes, w_sf, w_global, a_global, bias_f16, y_bf16, stream, sk_ws, sk,
                     pdl);
}

fp4_status_t fp4_gemm_gelu_quant(fp4_fmt_t fmt, const uint8_t* a_codes, const uint8_t* a_sf, int64_t M, int64_t K,
                                 int64_t N, const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global,
                                 const float* a_global, const void* bias_f16, const float* h_global,
                                 uint8_t* h_codes, uint8_t* h_sf, void* stream) {
    if (!fmt_ok(fmt) || !a_codes || !a_sf || !w_codes || !w_sf || !h_codes || !h_sf) return FP4_ERR_INVALID_ARG;
    const bool nv = fmt == FP4_FMT_NVFP4;
    if (nv != (w_global != nullptr) || nv != (a_global != nullptr) || nv != (h_global != nullptr))
        return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, N);
    if (s != FP4_OK) return s;
    if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(w_codes) || !aligned16(w_sf) || !aligned16(bias_f16) ||
        !aligned16(h_codes) || !aligned16(h_sf) || (reinterpret_cast<uintptr_t>(w_global) & 3u) ||
        (reinterpret_cast<uintptr_t>(a_global) & 3u) || (reinterpret_cast<uintptr_t>(h_global) & 3u))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    // always the 2-CTA kernel (its epilogue warps each own 64 columns of a row)
    CUtensorMap ta, tb;
    if ((s = encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, K / 2, M, K / 2, 128, GEMM_BM)) != FP4_OK)
        return s;
    if ((s = encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, 128, 128)) != FP4_OK) return s;
    GemmParams p{};
    p.M = (int)M, p.N = (int)N, p.K = (int)K;
    p.sfa = a_sf, p.sfb = w_sf, p.g_a = a_global, p.g_w = w_global;
    p.bias = static_cast<const __half*>(bias_f16);
    p.h_codes = h_codes, p.h_sf = h_sf, p.g_h = h_global;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return nv ? launch_gemm2<G_NVFP4, 2>(ds, ta, tb, a_sf, w_sf, p, st)
              : launch_gemm2<G_MXFP4, 1>(ds, ta, tb, a_sf, w_sf, p, st);
}

fp4_status_t fp4_linear_gelu_quant(fp4_fmt_t fmt, const void* x_bf16, int64_t M, int64_t K, int64_t N,
                                   const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global,
                                   const float* a_global, const void* bias_f16, const float* h_global,
                                   uint8_t* h_codes, uint8_t* h_sf, void* workspace, size_t ws_bytes, void* stream) {
    if (!fmt_ok(fmt) || !x_bf16 || !workspace) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, N);
    if (s != FP4_OK) return s;
    if (ws_bytes < fp4_linear_workspace_bytes(fmt, M, K, N)) return FP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    uint8_t* codes = static_cast<uint8_t*>(workspace);
    uint8_t* sf = codes + align256(fp4_codes_bytes(fmt, M, K));
    const bool nv = fmt == FP4_FMT_NVFP4;
    if (!w_codes || !w_sf || !h_codes || !h_sf || nv != (w_global != nullptr) || nv != (a_global != nullptr) ||
        nv != (h_global != nullptr))
        return FP4_ERR_INVALID_ARG;
    if ((s = fp4_quantize_act(fmt, x_bf16, M, K, a_global, codes, sf, stream)) != FP4_OK) return s;
    return fp4_gemm_gelu_quant(fmt, codes, sf, M, K, N, w_codes, w_sf, w_global, a_global, bias_f16, h_global,
                               h_codes, h_sf, stream);
}

}  // extern "C"
namespace {
fp4_status_t w4a8_quantize_impl(const void* x_bf16, int64_t M, int64_t K, const void* l1_bf16, int rank,
                               uint8_t* x_e4m3, uint8_t* x_sf, void* u_pair, float* partial, void* stream) {
    if (!x_bf16 || !l1_bf16 || !x_e4m3 || !x_sf || !u_pair || rank != 32) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, 128);
    if (s != FP4_OK) return s;
    if (!aligned16(x_bf16) || !aligned16(l1_bf16) || !aligned16(x_e4m3) || !aligned16(x_sf) || !aligned16(u_pair))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launch_lowrank<Q_MXFP8>(ds, x_bf16, l1_bf16, M, K, u_pair, partial, x_e4m3, x_sf, st);
}
}  // namespace
extern "C" {
fp4_status_t w4a8_quantize_act(const void* x_bf16, int64_t M, int64_t K, const void* l1_bf16, int rank,
                               uint8_t* x_e4m3, uint8_t* x_sf, void* u_pair, void* stream) {
    return w4a8_quantize_impl(x_bf16, M, K, l1_bf16, rank, x_e4m3, x_sf, u_pair, nullptr, stream);
}

fp4_status_t w4a8_gemm(const uint8_t* x_e4m3, const uint8_t* x_sf, const void* u_pair, int64_t M, int64_t K,
                       int64_t N, const uint8_t* r_codes, const uint8_t* r_sf, const void* l2_bf16, int rank,
                       const void* bias_f16, void* y_bf16, void* stream) {
    if (!x_e4m3 || !x_sf || !u_pair || !r_codes || !r_sf || !l2_bf16 || !y_bf16 || rank != 32)
        return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, N);
    if (s != FP4_OK) return s;
    // the unpacking tensor map needs a 32-byte aligned residual-weight base
    if (!aligned16(x_e4m3) || !aligned16(x_sf) || !aligned16(u_pair) || (reinterpret_cast<uintptr_t>(r_codes) & 31u) ||
        !aligned16(r_sf) || !aligned16(l2_bf16) || !aligned16(bias_f16) || !aligned16(y_bf16))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    // always the 2-CTA kernel: its low-rank stage runs on the tensor core
    CUtensorMap ta, tb, tu, tl;
    if ((s = encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, x_e4m3, K, M, K, 128, GEMM_BM)) != FP4_OK) return s;
    // packed E2M1 in global memory, unpacked to one 16-byte slot per 16 values in shared memory
    if ((s = encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, r_codes, K, N, K / 2, 128, 128)) != FP4_OK)
        return s;
    // u pair [M, 64] bf16 (128-byte rows) and L2 [32, N] bf16 as stored, in 64-column boxes
    if ((s = encode_2d(&tu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, u_pair, 2 * (uint64_t)rank, M, 4 * (uint64_t)rank,
                       2 * rank, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != FP4_OK)
        return s;
    if ((s = encode_2d(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, l2_bf16, (uint64_t)N, (uint64_t)rank, 2 * (uint64_t)N, 64,
                       (uint32_t)rank, CU_TENSOR_MAP_SWIZZLE_128B)) != FP4_OK)
        return s;
    GemmParams p{};
    p.M = (int)M, p.N = (int)N, p.K = (int)K;
    p.sfa = x_sf, p.sfb = r_sf;
    p.bias = static_cast<const __half*>(bias_f16);
    p.y = static_cast<__nv_bfloat16*>(y_bf16);
    return launch_gemm2<G_W4A8>(ds, ta, tb, x_sf, r_sf, p, static_cast<cudaStream_t>(stream), &tu, &tl);
}

fp4_status_t w4a8_svd_linear(const void* x_bf16, int64_t M, int64_t K, int64_t N, const uint8_t* r_codes,
                             const uint8_t* r_sf, const void* l1_bf16, const void* l2_bf16, int rank,
                             const void* bias_f16, void* y_bf16, void* workspace, size_t ws_bytes, void* stream) {
    if (!workspace || rank != 32) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, N);
    if (s != FP4_OK) return s;
    if (ws_bytes < w4a8_workspace_bytes(M, K, N, rank)) return FP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    if (!r_codes || !r_sf || !l2_bf16 || !y_bf16) return FP4_ERR_INVALID_ARG;
    uint8_t* xe = static_cast<uint8_t*>(workspace);
    uint8_t* xs = xe + align256((size_t)M * K);
    uint8_t* u = xs + align256(fp4_sf_bytes(FP4_FMT_MXFP4, M, K));
    float* partial = lr_partial_bytes(M, K) ? reinterpret_cast<float*>(u + align256((size_t)M * rank * 4)) : nullptr;
    if ((s = w4a8_quantize_impl(x_bf16, M, K, l1_bf16, rank, xe, xs, u, partial, stream)) != FP4_OK) return s;
    return w4a8_gemm(xe, xs, u, M, K, N, r_codes, r_sf, l2_bf16, rank, bias_f16, y_bf16, stream);
}

}  // extern "C"
namespace {
fp4_status_t w4a4_quantize_impl(const void* x_bf16, int64_t M, int64_t K, const void* l1_bf16, int rank,
                               uint8_t* x_codes, uint8_t* x_sf, void* u_pair, float* partial, void* stream) {
    if (!x_bf16 || !l1_bf16 || !x_codes || !x_sf || !u_pair || rank != 32) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, 128);
    if (s != FP4_OK) return s;
    if (!aligned16(x_bf16) || !aligned16(l1_bf16) || !aligned16(x_codes) || !aligned16(x_sf) || !aligned16(u_pair))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launch_lowrank<Q_MXFP4>(ds, x_bf16, l1_bf16, M, K, u_pair, partial, x_codes, x_sf, st);
}
}  // namespace
extern "C" {
fp4_status_t w4a4_quantize_act(const void* x_bf16, int64_t M, int64_t K, const void* l1_bf16, int rank,
                               uint8_t* x_codes, uint8_t* x_sf, void* u_pair, void* stream) {
    return w4a4_quantize_impl(x_bf16, M, K, l1_bf16, rank, x_codes, x_sf, u_pair, nullptr, stream);
}

fp4_status_t w4a4_gemm(const uint8_t* x_codes, const uint8_t* x_sf, const void* u_pair, int64_t M, int64_t K,
                       int64_t N, const uint8_t* r_codes, const uint8_t* r_sf, const void* l2_bf16, int rank,
                       const void* bias_f16, void* y_bf16, void* stream) {
    if (!x_codes || !x_sf || !u_pair || !r_codes || !r_sf || !l2_bf16 || !y_bf16 || rank != 32)
        return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, N);
    if (s != FP4_OK) return s;
    if (!aligned16(x_codes) || !aligned16(x_sf) || !aligned16(u_pair) || !aligned16(r_codes) || !aligned16(r_sf) ||
        !aligned16(l2_bf16) || !aligned16(bias_f16) || !aligned16(y_bf16))
        return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    CUtensorMap ta, tb, tu, tl;
    if ((s = encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, x_codes, K / 2, M, K / 2, 128, GEMM_BM)) != FP4_OK)
        return s;
    if ((s = encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, r_codes, K / 2, N, K / 2, 128, 128)) != FP4_OK) return s;
    if ((s = encode_2d(&tu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, u_pair, 2 * (uint64_t)rank, M, 4 * (uint64_t)rank,
                       2 * rank, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != FP4_OK)
        return s;
    if ((s = encode_2d(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, l2_bf16, (uint64_t)N, (uint64_t)rank, 2 * (uint64_t)N, 64,
                       (uint32_t)rank, CU_TENSOR_MAP_SWIZZLE_128B)) != FP4_OK)
        return s;
    GemmParams p{};
    p.M = (int)M, p.N = (int)N, p.K = (int)K;
    p.sfa = x_sf, p.sfb = r_sf;
    p.bias = static_cast<const __half*>(bias_f16);
    p.y = static_cast<__nv_bfloat16*>(y_bf16);
    return launch_gemm2<G_SVD4>(ds, ta, tb, x_sf, r_sf, p, static_cast<cudaStream_t>(stream), &tu, &tl);
}

fp4_status_t w4a4_svd_linear(const void* x_bf16, int64_t M, int64_t K, int64_t N, const uint8_t* r_codes,
                             const uint8_t* r_sf, const void* l1_bf16, const void* l2_bf16, int rank,
                             const void* bias_f16, void* y_bf16, void* workspace, size_t ws_bytes, void* stream) {
    if (!workspace || rank != 32) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, N);
    if (s != FP4_OK) return s;
    if (ws_bytes < w4a4_workspace_bytes(M, K, N, rank)) return FP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FP4_ERR_MISALIGNED;
    if (!r_codes || !r_sf || !l2_bf16 || !y_bf16) return FP4_ERR_INVALID_ARG;
    uint8_t* xc = static_cast<uint8_t*>(workspace);
    uint8_t* xs = xc + align256(fp4_codes_bytes(FP4_FMT_MXFP4, M, K));
    uint8_t* u = xs + align256(fp4_sf_bytes(FP4_FMT_MXFP4, M, K));
    float* partial = lr_partial_bytes(M, K) ? reinterpret_cast<float*>(u + align256((size_t)M * rank * 4)) : nullptr;
    if ((s = w4a4_quantize_impl(x_bf16, M, K, l1_bf16, rank, xc, xs, u, partial, stream)) != FP4_OK) return s;
    return w4a4_gemm(xc, xs, u, M, K, N, r_codes, r_sf, l2_bf16, rank, bias_f16, y_bf16, stream);
}

fp4_status_t fp4_sync_status(void* stream) {
    DeviceState* ds;
    fp4_status_t s = device_state(&ds);
    if (s != FP4_OK) return s;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP4_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_fp4_status, sizeof(int)) != cudaSuccess) return FP4_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fp4_status, &zero, sizeof(int)) != cudaSuccess) return FP4_ERR_CUDA;
    return word == 0 ? FP4_OK : static_cast<fp4_status_t>(word);
}

const char* fp4_status_string(fp4_status_t status) {
    switch (status) {
        case FP4_OK: return "FP4_OK";
        case FP4_ERR_INVALID_ARG: return "FP4_ERR_INVALID_ARG";
        case FP4_ERR_UNSUPPORTED_SHAPE: return "FP4_ERR_UNSUPPORTED_SHAPE";
        case FP4_ERR_MISALIGNED: return "FP4_ERR_MISALIGNED";
        case FP4_ERR_WORKSPACE: return "FP4_ERR_WORKSPACE";
        case FP4_ERR_ARCH: return "FP4_ERR_ARCH";
        case FP4_ERR_CUDA: return "FP4_ERR_CUDA";
        case FP4_ERR_TIMEOUT: return "FP4_ERR_TIMEOUT";
    }
    return "FP4_ERR_UNKNOWN";
}

void fp4_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns = ns ? ns : kDefaultTimeoutNs; }

// ---------------------------------------------------------------------------------------
// Allocation-free variant of fp4_linear.  Some callers cannot call cudaMalloc: code that
// runs inside another framework's memory pool or a plugin whose host forbids device
// allocations, or a real-time loop where an allocation could block.  For them the
// quantized activations live in this library's own device array instead of a
// caller-provided workspace.  The array is FP4_NOALLOC_SCRATCH_BYTES on every GPU that
// loads the library, for the life of the process; all calls share it, so calls that
// overlap on the GPU (different streams, or different host threads on one device) race.
// Nothing in it needs clearing: the quantizer rewrites every byte the GEMM reads.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FP4_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};
}  // namespace

fp4_status_t fp4_linear_noalloc(fp4_fmt_t fmt, const void* x_bf16, int64_t M, int64_t K, int64_t N,
                                const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global,
                                const float* a_global, const void* bias_f16, void* y_bf16, void* stream) {
    if (!fmt_ok(fmt)) return FP4_ERR_INVALID_ARG;
    fp4_status_t s = check_shape(M, K, N);
    if (s != FP4_OK) return s;
    if (fp4_linear_workspace_bytes(fmt, M, K, N) > (size_t)FP4_NOALLOC_SCRATCH_BYTES) return FP4_ERR_WORKSPACE;
    DeviceState* ds;
    if ((s = device_state(&ds)) != FP4_OK) return s;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP4_ERR_CUDA;
    void* scratch = nullptr;
    {
        // once per device, with that device current: the array's name is only a host-side
        // stand-in, so its device address has to be looked up
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        if (!g_scratch_addr[dev]) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FP4_ERR_CUDA;
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    return fp4_linear(fmt, x_bf16, M, K, N, w_codes, w_sf, w_global, a_global, bias_f16, y_bf16, scratch,
                      (size_t)FP4_NOALLOC_SCRATCH_BYTES, stream);
}

// Tuning hook (not in the public header): 1 forces the 1-CTA 128x256 kernel; 0 (default)
// and 2 use the 2-CTA 256x256 kernel whenever M > 128.
void fp4bsa_set_gemm_ctas(int ctas) { g_gemm_ctas = (ctas == 1 || ctas == 2) ? ctas : 0; }

// Tuning / test hook (not in the public header): stream-K for fp4_linear: 0 default (off),
// 1 never, 2 whenever the workspace allows (tiles x K blocks >= pairs).  The workspace
// size query follows the same setting.
void fp4bsa_set_stream_k(int mode) { g_stream_k = (mode == 1 || mode == 2) ? mode : 0; }

// Tuning hook (not in the public header): 1 (default) launches fp4_linear's 2-CTA GEMM with
// programmatic dependent launch after its quantize kernel, 0 with a plain launch.
void fp4bsa_set_pdl(int on) { g_pdl = on ? 1 : 0; }

// Test hook (not in the public header): the GEMM producer skips the given k-iteration of
// its ring, so the MMA warp's bounded wait runs out.  -1 disables it.
void fp4bsa_test_skip_iteration(int it) { g_skip_iter = it; }

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Test hook (not in the public header): the fp32 GELU-tanh value, before its bf16 rounding,
// that the fused epilogue and fp4_gelu_quantize_act compute for each bf16 input, so the
// tests can hold it against its stated error bound.  z_bf16 [n] and g_f32 [n] are device
// arrays; n even.
__global__ void gelu_probe_kernel(const uint32_t* z2, int64_t pairs, float2* g2) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < pairs; i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t w = z2[i];
        float g0, g1;
        gelu_f32_x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u), g0, g1);
        g2[i] = make_float2(g0, g1);
    }
}

// ---------------------------------------------------------------------------------------
// Measurement hook (not in the public header): each block's first thread records its SM id,
// that SM's cycle counter and the global nanosecond timer: out[3 b + 0..2].  Two probes
// around a timed region give every SM's average clock over it (cycles / nanoseconds), which
// nvidia-smi's periodic samples can miss when the clock moves within a short region.
__global__ void clock_probe_kernel(unsigned long long* out) {
    if (threadIdx.x == 0) {
        unsigned int sm;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
        out[3 * blockIdx.x + 0] = sm;
        out[3 * blockIdx.x + 1] = (unsigned long long)clock64();
        out[3 * blockIdx.x + 2] = globaltimer();
    }
}

extern "C" fp4_status_t fp4bsa_clock_probe(uint64_t* out, int blocks, void* stream) {
    if (!out || blocks < 1 || blocks > 4096) return FP4_ERR_INVALID_ARG;
    clock_probe_kernel<<<blocks, 32, 0, (cudaStream_t)stream>>>(reinterpret_cast<unsigned long long*>(out));
    return launched();
}

extern "C" fp4_status_t fp4bsa_test_gelu_f32(const void* z_bf16, int64_t n, float* g_f32, void* stream) {
    if (!z_bf16 || !g_f32 || n < 2 || (n & 1)) return FP4_ERR_INVALID_ARG;
    if (((uintptr_t)z_bf16 & 3u) || ((uintptr_t)g_f32 & 7u)) return FP4_ERR_MISALIGNED;
    DeviceState* ds;
    fp4_status_t s = device_state(&ds);
    if (s != FP4_OK) return s;
    if (!ds->arch_ok) return FP4_ERR_ARCH;
    const int64_t pairs = n / 2;
    const int blocks = (int)std::min<int64_t>((pairs + 255) / 256, (int64_t)ds->sm_count * 8);
    gelu_probe_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(static_cast<const uint32_t*>(z_bf16), pairs,
                                                               reinterpret_cast<float2*>(g_f32));
    return launched();
}
