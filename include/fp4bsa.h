/*
 * fp4bsa.h -- C ABI of the block-scaled FP4 quantized linear for NVIDIA B200 (sm_100a).
 *
 * The operation is the quantized linear layer of the Wan2.2 diffusion transformers:
 * bf16 activations are quantized on the fly to FP4 E2M1 with per-block scales and
 * multiplied against pre-packed FP4 weights; an fp16 bias is added and the output is
 * bf16.  Two FP4 formats are supported:
 *
 *   MXFP4  E2M1 values, two per byte, one E8M0 scale per 32 values along K
 *          (Wan2.2-I2V-A14B-Lightning-Diffusers-MXFP4-AutoRound, "Quantization Details":
 *           group_size 32, act_dynamic, weights "packed FP4 E2M1 (two FP4 values per
 *           byte) with per-32 E8M0 scales"; biases kept F16).
 *   NVFP4  E2M1 values, one FP8 E4M3 scale per 16 values, one FP32 global scale per
 *          tensor; activations use dynamic block scales under a static, calibrated
 *          global (Wan2.2-T2V-A14B-Diffusers-NVFP4-AutoRound, "Model Details").
 *
 * and a W4A8 SVDQuant linear: MXFP4 residual weight, dynamic MXFP8 (E4M3, per-32
 * E8M0) activations, and a rank-32 low-rank correction x L1 L2 added in the epilogue
 * (wan2.2-ti2v-w4a8-svd README, opening paragraph).
 *
 * ---------------------------------------------------------------------------------
 * Conventions (apply to every call)
 *   - Pointers marked (device) are CUDA device pointers; (host) are host pointers.
 *     All device pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Every call that launches work is asynchronous on `stream`; no call synchronizes
 *     except fp4_sync_status.
 *   - Ownership: the caller allocates and frees every buffer, including workspaces.
 *     The library allocates no device memory.  It keeps a process-wide cache of TMA
 *     descriptors keyed by (pointer, shape) and a device status word per GPU.
 *   - Shapes: M >= 1 (any value), K and N multiples of 128, all < 2^31 / 2.
 *   - Errors: arguments are validated on the host before any launch; an invalid call
 *     returns a status and launches nothing.  Launch failures return FP4_ERR_CUDA.  A
 *     device-side wait that runs out of time records FP4_ERR_TIMEOUT in the status
 *     word (read it with fp4_sync_status).  No C++ exception crosses this ABI.
 *
 * Layouts (part of the ABI; exactly what the CPU oracle in oracle/ produces):
 *   codes  [rows][K/2] bytes, row-major; element 2i in bits 3:0, element 2i+1 in
 *          bits 7:4 of byte i of its row.
 *   sf     one byte per group (G = 32 for MXFP4/MXFP8, 16 for NVFP4) in 128-row x
 *          4-group atoms of 512 bytes, rows padded to a multiple of 128:
 *            off(r, j) = ((r/128)*(Kg/4) + j/4)*512 + (r%32)*16 + ((r%128)/32)*4 + j%4
 *          with Kg = K/G.  Padding bytes are written as 0.
 *   e4m3 elements (MXFP8) [rows][K] bytes, row-major.
 *   Rounding: E2M1 and E4M3 round to nearest, ties to even, saturating (E2M1 at 6,
 *   E4M3 at 448); the sign of zero is kept.  MX scale = 2^(floor(log2 amax) - 2)
 *   (MXFP8: - 8) stored as E8M0; an all-zero group stores 0x00.  NVFP4:
 *   g = T/2688 (T = tensor amax, 2688 = 6*448; T = 0 gives g = 1),
 *   s = amax/(6 g) -> E4M3, codes = e2m1(x * (1/(dec(s) g))), each step one fp32
 *   IEEE operation; a block whose scale is 0 stores zero codes.
 * ---------------------------------------------------------------------------------
 */
#ifndef FP4BSA_H
#define FP4BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { FP4_FMT_MXFP4 = 0, FP4_FMT_NVFP4 = 1 } fp4_fmt_t;

typedef enum {
    FP4_OK = 0,
    FP4_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, M < 1, rank != 32 */
    FP4_ERR_UNSUPPORTED_SHAPE = 2, /* K or N not a multiple of 128, sizes too large */
    FP4_ERR_MISALIGNED = 3,        /* a device pointer not 16-byte aligned */
    FP4_ERR_WORKSPACE = 4,         /* workspace smaller than the size query returned */
    FP4_ERR_ARCH = 5,              /* current device is not sm_100 */
    FP4_ERR_CUDA = 6,              /* a CUDA runtime or driver call failed */
    FP4_ERR_TIMEOUT = 7            /* a device-side wait ran out of time (see fp4_sync_status) */
} fp4_status_t;

/* ----------------------------------------------------------------- size queries (host) */

/* Bytes of packed E2M1 codes for a [rows, K] operand: rows * K / 2 (MXFP4 card, Quantization
 * Details: two FP4 E2M1 values per byte).  0 if K is odd. */
size_t fp4_codes_bytes(fp4_fmt_t fmt, int64_t rows, int64_t K);

/* Bytes of the scale-factor buffer of a [rows, K] operand in the 128x4 atom layout:
 * ceil(rows/128)*128 * K/G (G = 32 MXFP4, one E8M0 per 32 values, MXFP4 card Quantization
 * Details; G = 16 NVFP4, one E4M3 per 16 values, NVFP4 card Model Details).  0 on a bad fmt
 * or K % 128 != 0. */
size_t fp4_sf_bytes(fp4_fmt_t fmt, int64_t rows, int64_t K);

/* Workspace fp4_linear needs: the dynamically quantized activations (MXFP4 card: act_dynamic;
 * NVFP4 card: dynamic block scales), codes then scales, each 256-byte aligned.  0 on
 * invalid arguments. */
size_t fp4_linear_workspace_bytes(fp4_fmt_t fmt, int64_t M, int64_t K, int64_t N);

/* Workspace w4a8_svd_linear needs (W4A8 README, W4A8 format): MXFP8 elements [M,K], their scales, the low-rank
 * projection u = x L1 as its bf16 pair [M, 2 rank] and, when x has fewer than 64 blocks of
 * 128 rows, fp32 partial sums of u for a K-split projection; each 256-byte aligned. */
size_t w4a8_workspace_bytes(int64_t M, int64_t K, int64_t N, int rank);

/* ----------------------------------------------------------------- quantization */

/* Per-tensor amax: *amax_out (device fp32) = max |x_i| over n bf16 values (device).
 * Used for the NVFP4 weight global and for calibrating the static activation global
 * (NVFP4 card, Model Details: the activation globals are static, set by calibration).
 * The result is order-independent. */
fp4_status_t fp4_tensor_amax(const void* x_bf16, int64_t n, float* amax_out, void* stream);

/* Static activation global for NVFP4, from calibration (NVFP4 card, Model Details: the
 * activation global scales are static, set once from calibration data, while the block
 * scales stay dynamic).  Call it once per calibration batch of the layer's input:
 *   x_bf16      (device) n bf16 values of one calibration batch
 *   amax_inout  (device, in/out) one fp32: the running tensor amax over the batches seen so
 *               far; set it to 0 before the first batch.  Raised to max(amax_inout, max|x_i|).
 *   g_out       (device, out) one fp32: g_a = amax_inout / 2688 in fp32 (1 if it is 0), the
 *               a_global that fp4_quantize_act and fp4_linear take.
 * The result is order-independent (a max) and bit-exact with the format rule above. */
fp4_status_t fp4_calibrate_act_global(const void* x_bf16, int64_t n, float* amax_inout, float* g_out,
                                      void* stream);

/* Offline weight pre-pack (MXFP4 / NVFP4 cards: weights stored as packed E2M1 with
 * block scales; NVFP4 adds an FP32 global from the tensor amax).
 *   w_bf16    (device) [N, K] bf16, torch Linear layout (out_features x in_features)
 *   w_codes   (device, out) fp4_codes_bytes(fmt, N, K) bytes
 *   w_sf      (device, out) fp4_sf_bytes(fmt, N, K) bytes
 *   w_global  (device, out) NVFP4: one fp32, g_w = max|W| / 2688; MXFP4: must be NULL
 * Same rounding as the activation quantizer; deterministic. */
fp4_status_t fp4_pack_weight(fp4_fmt_t fmt, const void* w_bf16, int64_t N, int64_t K,
                             uint8_t* w_codes, uint8_t* w_sf, float* w_global, void* stream);

/* Dynamic activation quantization (MXFP4 card: act_dynamic, act_group_size 32; NVFP4
 * card: dynamic block scales with a calibrated static global).
 *   x_bf16    (device) [M, K] bf16 row-major
 *   a_global  (device) NVFP4: the static activation global g_a (one fp32); MXFP4: NULL
 *   x_codes   (device, out) fp4_codes_bytes(fmt, M, K) bytes
 *   x_sf      (device, out) fp4_sf_bytes(fmt, M, K) bytes (padding rows zeroed) */
fp4_status_t fp4_quantize_act(fp4_fmt_t fmt, const void* x_bf16, int64_t M, int64_t K,
                              const float* a_global, uint8_t* x_codes, uint8_t* x_sf,
                              void* stream);

/* ----------------------------------------------------------------- GEMM */

/* Block-scaled FP4 x FP4 GEMM with fused epilogue on pre-quantized activations (the
 * MXFP4 card runs its W4A4 linears on a block-scaled FP4 matmul; the NVFP4 card, How to
 * Use, stresses that real FP4 GEMMs run, not a quantize-dequantize emulation):
 *   y[m,n] = bf16_rn( gs * sum_k deq(a[m,k]) deq(w[n,k]) + bias[n] )
 * with gs = g_a * g_w for NVFP4 and 1 for MXFP4; the sum accumulates in fp32.
 *   a_codes, a_sf       (device) quantized activations as fp4_quantize_act writes them
 *   w_codes, w_sf       (device) packed weight as fp4_pack_weight writes it
 *   w_global, a_global  (device) NVFP4 globals; both NULL for MXFP4
 *   bias_f16            (device) [N] fp16, or NULL for no bias
 *   y_bf16              (device, out) [M, N] bf16 row-major */
fp4_status_t fp4_gemm(fp4_fmt_t fmt, const uint8_t* a_codes, const uint8_t* a_sf, int64_t M,
                      int64_t K, int64_t N, const uint8_t* w_codes, const uint8_t* w_sf,
                      const float* w_global, const float* a_global, const void* bias_f16,
                      void* y_bf16, void* stream);

/* The W4A4 quantized linear, one call per linear layer (MXFP4 card, Quantization Details: the
 * transformer blocks' linears run with W4A4 MXFP4; NVFP4 card, Model Details): fp4_quantize_act
 * into `workspace`, then fp4_gemm.
 *   x_bf16     (device) [M, K] bf16
 *   workspace  (device) at least fp4_linear_workspace_bytes(fmt, M, K, N) bytes; its
 *              contents on return are the quantized activations (codes, then scales)
 * Other arguments as fp4_gemm. */
fp4_status_t fp4_linear(fp4_fmt_t fmt, const void* x_bf16, int64_t M, int64_t K, int64_t N,
                        const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global,
                        const float* a_global, const void* bias_f16, void* y_bf16,
                        void* workspace, size_t ws_bytes, void* stream);

/* Size of the device array fp4_linear_noalloc uses in place of a workspace. */
#define FP4_NOALLOC_SCRATCH_BYTES (16u << 20)

/* fp4_linear for callers that cannot allocate device memory (a plugin whose host owns
 * every allocation, code running under another framework's memory pool, a real-time
 * loop that must not block in an allocator).  The model-card pages this library follows
 * have no counterpart to it: it is a packaging variant of fp4_linear, not part of the method.
 *   Same arguments and result as fp4_linear, minus the workspace: the quantized
 *   activations go to a library-owned device array of FP4_NOALLOC_SCRATCH_BYTES
 *   (16 MiB) that exists on every GPU that loads the library until the process exits.
 *   The call allocates nothing (no cudaMalloc/cudaFree, no allocating library routine).
 *   The first call on a device looks up that array's device address (with the device
 *   current); make that first call before any stream capture.
 *   Returns FP4_ERR_WORKSPACE, launching nothing, when
 *   fp4_linear_workspace_bytes(fmt, M, K, N) exceeds FP4_NOALLOC_SCRATCH_BYTES
 *   (e.g. MXFP4 with K = 5120 fits up to 6161 rows: 6161 x 2560 code bytes plus
 *   49 x 128 x 160 scale bytes = 16,775,680 bytes).
 *   Every call shares the one array, and it keeps the last call's contents: calls that
 *   overlap on the GPU (other streams, other host threads on the same device) race and
 *   must be serialized by the caller.  No part of the array needs clearing between calls. */
fp4_status_t fp4_linear_noalloc(fp4_fmt_t fmt, const void* x_bf16, int64_t M, int64_t K, int64_t N,
                                const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global,
                                const float* a_global, const void* bias_f16, void* y_bf16,
                                void* stream);

/* ----------------------------------------------------------------- fused FFN activation */

/* The Wan2.2 FFN applies GELU-tanh between its two quantized linears (ffn.net.0.proj ->
 * ffn.net.2, MXFP4 card Quantization Details coverage list).  These calls produce the
 * down projection's quantized input, h = bf16_rn(gelu_tanh(z)) with z the bf16
 * up-projection output, without writing z to memory, where
 *   gelu_tanh(z) = 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))).
 * The library evaluates it in fp32 as z / (1 + 2^t), t = -2 sqrt(2/pi) (z + 0.044715 z^3) / ln 2:
 * 2^t by rounding t to an integer n and a degree-6 Taylor polynomial of 2^(t - n), the
 * reciprocal by three Newton-Raphson steps from a guess taken from the bits of 1 + 2^t; for
 * t > 125 the result is a zero of z's sign.  Its error against the exact value is at most
 * (2 |a| + 16) 2^-23 |gelu(z)| + 2^-126 with a = t ln 2, and h is its nearest bf16, so h is
 * the correctly rounded bf16 of gelu_tanh(z) except where that value lies within the bound
 * of a rounding midpoint, where h may be the other neighbour (a few in a thousand inputs).
 * The evaluation is deterministic: the same z always gives the same h.  h is then quantized
 * exactly as fp4_quantize_act quantizes x (same formats, layouts and NVFP4 global rule). */

/* Standalone: z_bf16 [M, K] bf16 (the up-projection output) -> codes [M, K/2] and scale
 * factors of h in `fmt`; a_global is the down projection's static activation global
 * (NVFP4) or NULL (MXFP4). */
fp4_status_t fp4_gelu_quantize_act(fp4_fmt_t fmt, const void* z_bf16, int64_t M, int64_t K,
                                   const float* a_global, uint8_t* x_codes, uint8_t* x_sf,
                                   void* stream);

/* The up projection with the activation fused into its epilogue: same operands as
 * fp4_gemm (a_codes, a_sf [M, K]; w_codes, w_sf [N, K]; NVFP4 globals; bias [N] or NULL),
 * but instead of y it writes z = bf16_rn(acc (g_a g_w) + bias), h = bf16_rn(gelu_tanh(z)),
 * quantized in the same format `fmt`:
 *   h_global (device) NVFP4: the down projection's static activation global; MXFP4: NULL
 *   h_codes  (device, out) [M, N/2];  h_sf (device, out) fp4_sf_bytes(fmt, M, N) bytes
 * i.e. exactly the x_codes / x_sf that fp4_quantize_act would produce from h, ready as the
 * A operand of the down projection (K' = N).  Always the 2-CTA kernel. */
fp4_status_t fp4_gemm_gelu_quant(fp4_fmt_t fmt, const uint8_t* a_codes, const uint8_t* a_sf,
                                 int64_t M, int64_t K, int64_t N, const uint8_t* w_codes,
                                 const uint8_t* w_sf, const float* w_global,
                                 const float* a_global, const void* bias_f16,
                                 const float* h_global, uint8_t* h_codes, uint8_t* h_sf,
                                 void* stream);

/* fp4_quantize_act of x into `workspace` (fp4_linear_workspace_bytes), then
 * fp4_gemm_gelu_quant. */
fp4_status_t fp4_linear_gelu_quant(fp4_fmt_t fmt, const void* x_bf16, int64_t M, int64_t K,
                                   int64_t N, const uint8_t* w_codes, const uint8_t* w_sf,
                                   const float* w_global, const float* a_global,
                                   const void* bias_f16, const float* h_global,
                                   uint8_t* h_codes, uint8_t* h_sf, void* workspace,
                                   size_t ws_bytes, void* stream);

/* ----------------------------------------------------------------- W4A8 SVDQuant */

/* Activation side of the W4A8 SVDQuant linear (W4A8 README, W4A8 format: the activations
 * are quantized to MXFP8 at run time and a rank-32 low-rank branch, which reads the
 * unquantized input, corrects the product):
 *   x_bf16   (device) [M, K] bf16
 *   l1_bf16  (device) [K, rank] bf16 (proj_down with 1/s folded in)
 *   x_e4m3   (device, out) [M, K] E4M3 bytes
 *   x_sf     (device, out) fp4_sf_bytes(FP4_FMT_MXFP4, M, K) bytes (E8M0, per 32)
 *   u_pair   (device, out) [M, 2 * rank] bf16: u = x L1 accumulated in fp32, stored as
 *            hi = bf16_rn(u) in columns [0, rank) and lo = bf16_rn(u - hi) in columns
 *            [rank, 2 rank), so hi + lo equals u within 2^-18 |u| (M * rank * 4 bytes,
 *            the size of an fp32 [M, rank] array). */
fp4_status_t w4a8_quantize_act(const void* x_bf16, int64_t M, int64_t K, const void* l1_bf16,
                               int rank, uint8_t* x_e4m3, uint8_t* x_sf, void* u_pair,
                               void* stream);

/* W4A8 GEMM with low-rank epilogue (W4A8 README, W4A8 format: MXFP4 residual times MXFP8
 * activations plus the rank-32 correction):
 *   y = bf16_rn( sum_k deq8(x) deq4(r) + u L2 + bias ).
 *   r_codes, r_sf  (device) MXFP4-packed residual weight [N, K] (fp4_pack_weight);
 *                  r_codes must be 32-byte aligned
 *   u_pair         (device) [M, 2 * rank] bf16 from w4a8_quantize_act
 *   l2_bf16        (device) [rank, N] bf16, the low-rank up-projection (proj_up) as stored,
 *                  row-major; read as it is, with no packing step
 *   bias_f16       (device) [N] fp16 or NULL;  y_bf16 (device, out) [M, N] bf16
 * The low-rank product is accumulated on the tensor core into the same fp32 accumulator,
 * as (u_hi L2 + u_lo L2), before the bias and the bf16 rounding. */
fp4_status_t w4a8_gemm(const uint8_t* x_e4m3, const uint8_t* x_sf, const void* u_pair, int64_t M,
                       int64_t K, int64_t N, const uint8_t* r_codes, const uint8_t* r_sf,
                       const void* l2_bf16, int rank, const void* bias_f16, void* y_bf16,
                       void* stream);

/* The full W4A8 SVDQuant linear (W4A8 README, opening paragraph and W4A8 format):
 * w4a8_quantize_act into `workspace` (with few rows, u = x L1 split over K into the
 * workspace's partial sums, added in a fixed order), then w4a8_gemm.
 *   x_bf16 [M, K]; r_codes, r_sf: the MXFP4 residual [N, K]; l1_bf16 [K, rank] (proj_down,
 *   1/s folded in); l2_bf16 [rank, N] (proj_up); rank must be 32; bias [N] fp16 or NULL;
 *   workspace of at least w4a8_workspace_bytes(M, K, N, rank) bytes. */
fp4_status_t w4a8_svd_linear(const void* x_bf16, int64_t M, int64_t K, int64_t N,
                             const uint8_t* r_codes, const uint8_t* r_sf, const void* l1_bf16,
                             const void* l2_bf16, int rank, const void* bias_f16, void* y_bf16,
                             void* workspace, size_t ws_bytes, void* stream);

/* ----------------------------------------------------------------- W4A4 SVDQuant */

/* The W4A8 README's experimental W4A4 variant (Quick start: MXFP4 activations):
 * the same calibrated factors (MXFP4 residual R, rank-32 L1 / L2), with the activations
 * quantized to MXFP4 instead of MXFP8; the low-rank branch still reads the unquantized
 * input.  y = bf16_rn( sum_k deq4(x) deq4(r) + u L2 + bias ). */

/* Workspace for w4a4_svd_linear: MXFP4 codes + scales of x, the u pair and, when x has
 * fewer than 64 blocks of 128 rows, fp32 partial sums of u for a K-split u = x L1 (0 if
 * invalid). */
size_t w4a4_workspace_bytes(int64_t M, int64_t K, int64_t N, int rank);

/* Activation side: MXFP4 codes and scales of x (exactly fp4_quantize_act with
 * FP4_FMT_MXFP4) and the u pair of x L1 (exactly as w4a8_quantize_act writes it).
 *   x_codes  (device, out) [M, K/2]; x_sf (device, out) fp4_sf_bytes(FP4_FMT_MXFP4, M, K)
 *   u_pair   (device, out) [M, 2 * rank] bf16 */
fp4_status_t w4a4_quantize_act(const void* x_bf16, int64_t M, int64_t K, const void* l1_bf16,
                               int rank, uint8_t* x_codes, uint8_t* x_sf, void* u_pair,
                               void* stream);

/* W4A4 SVDQuant GEMM: MXFP4 x MXFP4 block-scaled main loop plus the tensor-core low-rank
 * stage (u_hi L2 + u_lo L2) into the same fp32 accumulator, + bias, bf16 out.
 *   r_codes, r_sf  MXFP4-packed residual [N, K] (fp4_pack_weight)
 *   l2_bf16        [rank, N] bf16 up-projection, as stored */
fp4_status_t w4a4_gemm(const uint8_t* x_codes, const uint8_t* x_sf, const void* u_pair, int64_t M,
                       int64_t K, int64_t N, const uint8_t* r_codes, const uint8_t* r_sf,
                       const void* l2_bf16, int rank, const void* bias_f16, void* y_bf16,
                       void* stream);

/* The full W4A4 SVDQuant linear: w4a4_quantize_act into `workspace`, then w4a4_gemm. */
fp4_status_t w4a4_svd_linear(const void* x_bf16, int64_t M, int64_t K, int64_t N,
                             const uint8_t* r_codes, const uint8_t* r_sf, const void* l1_bf16,
                             const void* l2_bf16, int rank, const void* bias_f16, void* y_bf16,
                             void* workspace, size_t ws_bytes, void* stream);

/* ----------------------------------------------------------------- FP4 attention operands */

/* First slice of microscaling FP4 attention: the attention backends the Wan2.2-Animate-14B
 * MXFP4 card compares ("Results") include SageAttention v3, which it describes as
 * Blackwell microscaling FP4 attention.  The card gives no algorithm; this library reads
 * it as Q and K quantized per token and head in blocks along head_dim by the same MXFP4 /
 * NVFP4 rules as the linear's activations, and the scores S = deq(Q_h) deq(K_h)^T of one
 * head computed by the block-scaled GEMM (fp32 accumulation, bf16 out).  Softmax and the
 * P V product are not part of this interface.
 *
 * Head-major layout of a quantized [T tokens, H heads x D] tensor (D = FP4_HEAD_DIM):
 *   codes  [H][Tpad][D/2] bytes, Tpad = T rounded up to 128; tokens in [T, Tpad) hold
 *          zero codes;
 *   sf     H consecutive blocks of fp4_sf_bytes(fmt, T, D) bytes: head h's scales in the
 *          sf layout above for a [T, D] matrix (K = D).
 * Head h's codes and scales are thus exactly fp4_quantize_act of columns h*D .. h*D+D-1
 * of x (with T rows), the codes padded to Tpad rows with zeros. */
#define FP4_HEAD_DIM 128

/* Bytes of the head-major codes / scales of a [T, H x D] tensor (0 if invalid: D must be
 * FP4_HEAD_DIM). */
size_t fp4_heads_codes_bytes(fp4_fmt_t fmt, int64_t T, int64_t H, int64_t D);
size_t fp4_heads_sf_bytes(fp4_fmt_t fmt, int64_t T, int64_t H, int64_t D);

/* Quantize x_bf16 (device) [T, H*D] bf16, row-major (token-major, heads contiguous within
 * a token, as a linear projection writes them), into the head-major layout above.
 *   g      (device) NVFP4: the tensor's fp32 global (e.g. fp4_calibrate_act_global over x
 *          itself); MXFP4: must be NULL
 *   codes  (device, out) fp4_heads_codes_bytes(fmt, T, H, D)
 *   sf     (device, out) fp4_heads_sf_bytes(fmt, T, H, D)
 * D other than FP4_HEAD_DIM returns FP4_ERR_UNSUPPORTED_SHAPE. */
fp4_status_t fp4_quantize_heads(fp4_fmt_t fmt, const void* x_bf16, int64_t T, int64_t H, int64_t D,
                                const float* g, uint8_t* codes, uint8_t* sf, void* stream);

/* Scores of head `head`: s_bf16 (device, out) [T_q][T_kv_pad] bf16, row-major, T_kv_pad =
 * T_kv rounded up to 128, s[i][j] = bf16_rn( sum_d deq(q)[i][d] deq(k)[j][d] ) with the
 * NVFP4 globals g_q g_k applied (device fp32, NULL for MXFP4); columns j >= T_kv are 0.
 * q_codes / q_sf and k_codes / k_sf are the whole head-major buffers of fp4_quantize_heads
 * (T_q resp. T_kv tokens, H heads).  No softmax scaling is applied. */
fp4_status_t fp4_attn_scores(fp4_fmt_t fmt, const uint8_t* q_codes, const uint8_t* q_sf, int64_t T_q,
                             const uint8_t* k_codes, const uint8_t* k_sf, int64_t T_kv, int64_t H,
                             int64_t D, int64_t head, const float* g_q, const float* g_k, void* s_bf16,
                             void* stream);

/* The rest of one head's attention, read the same way: per query row the unnormalized
 * softmax weights P~_j = 2^(s_j c - max) over the T_kv keys (c = scale * log2 e; the largest
 * is exactly 1), quantized in blocks of G consecutive keys, and their sum l; V of the head
 * quantized per head-dim channel in blocks of G consecutive tokens; O = deq(P~) deq(V) by
 * the block-scaled GEMM, whose K is then the key axis, each row then divided by its l.
 * MXFP4: G = 32; NVFP4: G = 16 with E4M3 scales under one fp32 global per tensor (V: from its
 * amax, e.g. fp4_calibrate_act_global over v; P~: a constant the caller provides, 1/2688 =
 * 1/(6*448) since p <= 1).
 * fp4_attn_scores, fp4_attn_softmax_quant and fp4_attn_pv in sequence give one head's
 * attention output.
 *
 * Head-major layout of V^T, quantized from v [T tokens, H heads x D]:
 *   codes  [H][D][Tpad/2] bytes (head h, channel d: its Tpad tokens as packed E2M1; padding
 *          tokens hold zero codes);
 *   sf     H consecutive blocks of fp4_sf_bytes(fmt, D, Tpad) bytes: head h's scales in the
 *          sf layout above for the [D, Tpad] matrix (rows = channels, K = tokens). */
size_t fp4_heads_vt_codes_bytes(fp4_fmt_t fmt, int64_t T, int64_t H, int64_t D);
size_t fp4_heads_vt_sf_bytes(fp4_fmt_t fmt, int64_t T, int64_t H, int64_t D);

/* Quantize v_bf16 (device) [T, H*D] bf16, row-major, into the V^T layout above (codes and
 * sf device, out).  g (device): NVFP4, V's fp32 global; MXFP4, must be NULL.  D must be
 * FP4_HEAD_DIM (else FP4_ERR_UNSUPPORTED_SHAPE); H < 65536. */
fp4_status_t fp4_quantize_heads_vt(fp4_fmt_t fmt, const void* v_bf16, int64_t T, int64_t H, int64_t D,
                                   const float* g, uint8_t* codes, uint8_t* sf, void* stream);

/* Softmax weights of scores and their quantization.
 *   s_bf16  (device) [T_q][T_kv_pad] bf16 scores (fp4_attn_scores' output; columns >= T_kv
 *           are ignored)
 *   scale   the softmax scale (e.g. 1/sqrt(D)), > 0 and finite; the kernels use
 *           c = fp32(scale * log2 e), m = max_j fl(s_j c) over j < T_kv, t_j = fl(fl(s_j c)
 *           - m), p~_j = exp2(t_j) with CUDA's exp2f (within 2 ulp), so p~ is 2^(s_j c - max)
 *           within a relative 2 (ln2 * 4 max|s c| + 4) 2^-24; and l = sum_j p~_j in fp32 (each
 *           of a row's 256 threads adds its keys in order, then a fixed tree), within a
 *           relative (8 ceil(T_kv_pad / 2048) + 12) 2^-24 more of the sum of the p~ it adds
 *   p_global (device) NVFP4: P's fp32 global (1/2688 for p <= 1); MXFP4: must be NULL
 *   stats   (device, out) [T_q] pairs of fp32 (m, l)
 *   p_codes (device, out) [T_q][T_kv_pad/2]; p_sf (device, out) fp4_sf_bytes(fmt, T_q,
 *           T_kv_pad): p~ quantized by the format's rules above; keys >= T_kv hold 0 and
 *           padding rows zero scale bytes. */
fp4_status_t fp4_attn_softmax_quant(fp4_fmt_t fmt, const void* s_bf16, int64_t T_q, int64_t T_kv, float scale,
                                    const float* p_global, void* stats, uint8_t* p_codes, uint8_t* p_sf,
                                    void* stream);

/* O for head `head`: bf16 [T_q][D] = deq(P~) deq(V_head) by the block-scaled GEMM with
 * K = T_kv_pad, then, when stats is given, each row o = bf16_rn(o * fl(1 / l)).
 *   p_codes, p_sf      fp4_attn_softmax_quant's output (T_q rows); p_global its NVFP4 global
 *   vt_codes, vt_sf    fp4_quantize_heads_vt's output (T_kv tokens, H heads); v_global its
 *                      NVFP4 global (both globals device pointers, NULL for MXFP4)
 *   stats   (device) fp4_attn_softmax_quant's (m, l) pairs, or NULL for the unnormalized
 *           product
 *   o_bf16  (device, out) [T_q][D] bf16 */
fp4_status_t fp4_attn_pv(fp4_fmt_t fmt, const uint8_t* p_codes, const uint8_t* p_sf, const float* p_global,
                         int64_t T_q, int64_t T_kv, const uint8_t* vt_codes, const uint8_t* vt_sf,
                         const float* v_global, int64_t H, int64_t D, int64_t head, const void* stats,
                         void* o_bf16, void* stream);

/* One head's FP4 attention in one kernel, in the streaming (flash) form of the reading
 * above (the Wan2.2-Animate-14B MXFP4 card, "Results": FP4 attention on Blackwell with
 * microscaling; the page gives no algorithm).  The keys are taken in blocks of 256; per
 * query row and block j: s = deq(q) deq(k)^T in fp32 (never rounded to bf16), the running
 * maximum m_j = max(m_{j-1}, max fl(s c)) over the block's keys < T_kv (c = fp32(scale *
 * log2 e)), the weights p~ = exp2(fl(fl(s c) - m_j)) quantized in groups of G keys (MXFP4:
 * 32, E8M0 scales; NVFP4: 16, E4M3 scales under P~'s global p_global, 1/2688 for p <= 1),
 * O_j = O_{j-1} f_j + deq(P~_j) deq(V_j) with f_j = exp2(fl(m_{j-1} - m_j)) (1 when the
 * maximum did not grow); the sum is kept per quarter block (keys 64 q .. 64 q + 63 of every
 * block): l_q = fl(fl(l_q f_j) + the quarter's two pairwise-tree sums of 32 weights, added in
 * key order), and l = fl(fl(l_0 + l_1) + fl(l_2 + l_3)).  The output is
 * o = bf16_rn(O fl(1 / l)).  The weights are thus quantized against the running maximum,
 * not the row's final one as fp4_attn_softmax_quant does, and S stays in fp32.
 *   q_codes / q_sf, k_codes / k_sf   fp4_quantize_heads' buffers (T_q resp. T_kv tokens)
 *   vt_codes / vt_sf                 fp4_quantize_heads_vt's buffers (T_kv tokens)
 *   scale   the softmax scale, > 0 and finite
 *   g_q, g_k, g_v, p_global  (device) NVFP4: the fp32 globals of Q, K, V and P~; the scores'
 *           pair is folded into the exponent multiplier, c' = fl(c fl(g_q g_k)) and
 *           fl(s c) = fl(acc c') for the raw block-scaled product acc, and the output is
 *           o = bf16_rn(O fl(fl(p_global g_v) fl(1 / l))); MXFP4: all four must be NULL
 *   stats   (device, out) [T_q] pairs of fp32 (final running maximum, l), or NULL
 *   o_bf16  (device, out) [T_q][D] bf16
 * Globals given for MXFP4 or missing for NVFP4 return FP4_ERR_INVALID_ARG.  D = FP4_HEAD_DIM;
 * H times T_q or T_kv rounded up to 128 must stay below 2^31 (else FP4_ERR_UNSUPPORTED_SHAPE).
 * One CTA per 128 query rows; a wait that runs out of time records FP4_ERR_TIMEOUT. */
fp4_status_t fp4_attn_fused(fp4_fmt_t fmt, const uint8_t* q_codes, const uint8_t* q_sf, int64_t T_q,
                            const uint8_t* k_codes, const uint8_t* k_sf, int64_t T_kv, const uint8_t* vt_codes,
                            const uint8_t* vt_sf, int64_t H, int64_t D, int64_t head, float scale, const float* g_q,
                            const float* g_k, const float* g_v, const float* p_global, void* stats, void* o_bf16,
                            void* stream);

/* fp4_attn_fused that also records, for the 128 query rows of tile trace_tile (rows
 * 128 trace_tile ...), every block's intermediate values: trace_m [nblk][128] fp32 running
 * maxima, trace_codes [nblk][128][128] the P~_j codes (256 keys per row, two per byte, low
 * nibble first), trace_sf [nblk][128][256 / G] their scale bytes; nblk = ceil(T_kv_pad / 256).
 * A test hook with no counterpart on the pages: all three device pointers or none (then it
 * is fp4_attn_fused), 0 <= trace_tile < T_q_pad / 128. */
fp4_status_t fp4_attn_fused_trace(fp4_fmt_t fmt, const uint8_t* q_codes, const uint8_t* q_sf, int64_t T_q,
                                  const uint8_t* k_codes, const uint8_t* k_sf, int64_t T_kv, const uint8_t* vt_codes,
                                  const uint8_t* vt_sf, int64_t H, int64_t D, int64_t head, float scale,
                                  const float* g_q, const float* g_k, const float* g_v, const float* p_global,
                                  void* stats, void* o_bf16, int64_t trace_tile, float* trace_m,
                                  uint8_t* trace_codes, uint8_t* trace_sf, void* stream);

/* ----------------------------------------------------------------- status */

/* The status calls below are part of this library's error model, not of the method: the
 * model-card pages describe no library interface, so they have no counterpart there. */

/* Synchronizes `stream`, then returns and clears the device status word of the current
 * GPU: FP4_ERR_TIMEOUT if a kernel's bounded wait ran out since the last call,
 * FP4_ERR_ARCH if a GEMM kernel found its shared memory placed without the 1024-byte
 * alignment it is built for, or smaller than its layout (it then wrote no output),
 * FP4_ERR_CUDA if the synchronization failed, FP4_OK otherwise. */
fp4_status_t fp4_sync_status(void* stream);

/* Static, human-readable name of a status code. */
const char* fp4_status_string(fp4_status_t status);

/* Test hook: limit, in nanoseconds, of every device-side wait in kernels launched
 * after this call on this process (default 2e9 = 2 s).  0 restores the default. */
void fp4_set_wait_timeout_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* FP4BSA_H */
