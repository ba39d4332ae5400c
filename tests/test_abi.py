"""The C ABI on the host (no GPU): the library loads, exports every symbol the header
declares, answers size queries, and rejects invalid calls before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fb():
    import fp4_block_scaled_act_b200 as fb

    fb.build()
    return fb


def header_symbols():
    text = open(os.path.join(ROOT, "include", "fp4bsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:fp4|w4a8|w4a4)_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_header_symbol(fb):
    syms = header_symbols()
    assert len(syms) >= 15
    L = ctypes.CDLL(os.path.join(ROOT, "fp4_block_scaled_act_b200", "libfp4bsa.so"))
    for s in syms:
        assert hasattr(L, s), s
    assert sorted(fb.EXPORTS) == syms


def test_size_queries(fb):
    MX, NV = fb.MXFP4, fb.NVFP4
    assert fb.fp4_codes_bytes(MX, 75600, 5120) == 75600 * 2560
    assert fb.fp4_sf_bytes(MX, 75600, 5120) == 75648 * 160     # rows padded to 128
    assert fb.fp4_sf_bytes(NV, 75600, 5120) == 75648 * 320
    assert fb.fp4_sf_bytes(MX, 1, 128) == 128 * 4
    assert fb.fp4_sf_bytes(MX, 10, 100) == 0                    # K % 128 != 0
    assert fb.lib().fp4_sf_bytes(7, 10, 128) == 0               # bad format
    ws = fb.fp4_linear_workspace_bytes(MX, 75600, 5120, 13824)
    assert ws == 193536000 + 12103680
    assert fb.fp4_linear_workspace_bytes(MX, 0, 5120, 13824) == 0
    assert fb.w4a8_workspace_bytes(4290, 3072, 14336, 32) > 4290 * 3072
    assert fb.w4a8_workspace_bytes(4290, 3072, 14336, 16) == 0
    # W4A4 SVDQuant: MXFP4 codes + scales + the u pair, each 256-byte aligned, and (34 row
    # blocks of 128 < 64: u = x L1 split 8 ways over K = 3072) fp32 partials of u for 8 splits
    # of the 4352 padded rows
    a256 = lambda n: (n + 255) // 256 * 256
    assert fb.w4a4_workspace_bytes(4290, 3072, 14336, 32) == (
        a256(4290 * 1536) + a256(fb.fp4_sf_bytes(MX, 4290, 3072)) + a256(4290 * 32 * 4) + a256(8 * 4352 * 32 * 4))
    # 591 row blocks: no split, no partials
    assert fb.w4a4_workspace_bytes(75600, 5120, 13824, 32) == (
        a256(75600 * 2560) + a256(fb.fp4_sf_bytes(MX, 75600, 5120)) + a256(75600 * 32 * 4))
    assert fb.w4a4_workspace_bytes(4290, 3072, 14336, 16) == 0
    # head-major attention operands: [H][Tpad][64] codes, H blocks of [Tpad, 128] scales
    assert fb.fp4_heads_codes_bytes(MX, 75600, 40) == 40 * 75648 * 64
    assert fb.fp4_heads_sf_bytes(MX, 75600, 40) == 40 * fb.fp4_sf_bytes(MX, 75600, 128) == 40 * 75648 * 4
    assert fb.fp4_heads_sf_bytes(NV, 130, 3) == 3 * 256 * 8
    assert fb.fp4_heads_codes_bytes(MX, 130, 3, 64) == 0                # head_dim 128 only
    # V^T: [H][128][Tpad/2] codes, H blocks of [128, Tpad] scales (along the tokens)
    assert fb.fp4_heads_vt_codes_bytes(MX, 75600, 40) == 40 * 128 * 75648 // 2
    assert fb.fp4_heads_vt_sf_bytes(MX, 75600, 40) == 40 * fb.fp4_sf_bytes(MX, 128, 75648) == 40 * 128 * 75648 // 32
    assert fb.fp4_heads_vt_sf_bytes(NV, 130, 3) == 3 * 128 * 256 // 16


def test_bytes_per_weight_match_format(fb):
    """Packed FP4 + scales = 0.5 + 1/32 (MXFP4) or 0.5 + 1/16 (NVFP4) bytes per weight for
    every Wan2.2 A14B linear shape (N multiple of 128: no padding)."""
    for N, K in ((5120, 5120), (13824, 5120), (5120, 13824)):
        mx = fb.fp4_codes_bytes(fb.MXFP4, N, K) + fb.fp4_sf_bytes(fb.MXFP4, N, K)
        nv = fb.fp4_codes_bytes(fb.NVFP4, N, K) + fb.fp4_sf_bytes(fb.NVFP4, N, K)
        assert mx * 32 == N * K * 17
        assert nv * 16 == N * K * 9


def test_status_strings(fb):
    for i, name in enumerate(fb.STATUS):
        assert fb.fp4_status_string(i) == name


def test_invalid_calls_rejected_before_launch(fb):
    """Fake (never dereferenced) pointers: validation must fail first."""
    L = fb.lib()
    P = ctypes.c_void_p
    A = 1 << 20          # 16-byte aligned fake address
    bad = A + 8          # misaligned
    st = P(0)
    # bad format
    assert L.fp4_quantize_act(5, A, 16, 256, None, A, A, st) == 1
    # K not a multiple of 128
    assert L.fp4_quantize_act(0, A, 16, 200, None, A, A, st) == 2
    # M < 1
    assert L.fp4_quantize_act(0, A, 0, 256, None, A, A, st) == 1
    # NVFP4 without an activation global / MXFP4 with one
    assert L.fp4_quantize_act(1, A, 16, 256, None, A, A, st) == 1
    assert L.fp4_quantize_act(0, A, 16, 256, A, A, A, st) == 1
    # misaligned pointer
    assert L.fp4_quantize_act(0, bad, 16, 256, None, A, A, st) == 3
    # null output
    assert L.fp4_quantize_act(0, A, 16, 256, None, None, A, st) == 1
    # GEMM: N not a multiple of 128
    assert L.fp4_gemm(0, A, A, 16, 256, 200, A, A, None, None, None, A, st) == 2
    assert L.fp4_gemm(0, A, A, 16, 256, 256, A, A, None, None, bad, A, st) == 3
    # linear: workspace too small
    assert L.fp4_linear(0, A, 16, 256, 256, A, A, None, None, None, A, A, 10, st) == 4
    # W4A8: rank must be 32
    assert L.w4a8_svd_linear(A, 16, 256, 256, A, A, A, A, 16, None, A, A, 1 << 30, st) == 1
    assert L.w4a8_gemm(A, A, A, 16, 256, 384, A, A, A, 32, None, bad, st) == 3
    # W4A4 SVDQuant: rank, shape, alignment, workspace
    assert L.w4a4_svd_linear(A, 16, 256, 256, A, A, A, A, 16, None, A, A, 1 << 30, st) == 1
    assert L.w4a4_gemm(A, A, A, 16, 256, 200, A, A, A, 32, None, A, st) == 2
    assert L.w4a4_gemm(A, A, A, 16, 256, 384, A, A, A, 32, None, bad, st) == 3
    assert L.w4a4_svd_linear(A, 16, 256, 256, A, A, A, A, 32, None, A, A, 10, st) == 4
    assert L.w4a4_quantize_act(A, 16, 256, A, 32, A, A, None, st) == 1
    # fused GELU + quantize: NVFP4 needs the output global, MXFP4 must not get one
    assert L.fp4_gemm_gelu_quant(1, A, A, 16, 256, 256, A, A, A, A, None, None, A, A, st) == 1
    assert L.fp4_gemm_gelu_quant(0, A, A, 16, 256, 256, A, A, None, None, None, A, A, A, st) == 1
    assert L.fp4_gemm_gelu_quant(0, A, A, 16, 256, 200, A, A, None, None, None, None, A, A, st) == 2
    assert L.fp4_gemm_gelu_quant(0, A, A, 16, 256, 256, A, A, None, None, None, None, bad, A, st) == 3
    assert L.fp4_linear_gelu_quant(0, A, 16, 256, 256, A, A, None, None, None, None, A, A, A, 10, st) == 4
    assert L.fp4_gelu_quantize_act(1, A, 16, 256, None, A, A, st) == 1
    assert L.fp4_gelu_quantize_act(0, A, 16, 200, None, A, A, st) == 2
    # weight pack: MXFP4 must not get a global
    assert L.fp4_pack_weight(0, A, 256, 256, A, A, A, st) == 1
    assert L.fp4_tensor_amax(A, 0, A, st) == 1
    # FP4 attention operands: head_dim, format / global pairing, alignment, head index
    assert L.fp4_quantize_heads(0, A, 16, 2, 64, None, A, A, st) == 2
    assert L.fp4_quantize_heads(1, A, 16, 2, 128, None, A, A, st) == 1
    assert L.fp4_quantize_heads(0, A, 16, 2, 128, A, A, A, st) == 1
    assert L.fp4_quantize_heads(0, bad, 16, 2, 128, None, A, A, st) == 3
    assert L.fp4_quantize_heads(0, A, 0, 2, 128, None, A, A, st) == 1
    assert L.fp4_attn_scores(0, A, A, 16, A, A, 16, 2, 128, 2, None, None, A, st) == 1
    assert L.fp4_attn_scores(0, A, A, 16, A, A, 16, 2, 64, 0, None, None, A, st) == 2
    assert L.fp4_attn_scores(1, A, A, 16, A, A, 16, 2, 128, 0, None, None, A, st) == 1
    assert L.fp4_attn_scores(0, A, A, 16, A, A, 16, 2, 128, 0, None, None, bad, st) == 3
    # V^T, softmax + P quantize, P V: format / global pairing, shape, alignment, head index
    assert L.fp4_quantize_heads_vt(1, A, 16, 2, 128, None, A, A, st) == 1
    assert L.fp4_quantize_heads_vt(0, A, 16, 2, 128, A, A, A, st) == 1
    assert L.fp4_quantize_heads_vt(0, A, 16, 2, 96, None, A, A, st) == 2
    assert L.fp4_quantize_heads_vt(0, A, 16, 70000, 128, None, A, A, st) == 2
    assert L.fp4_quantize_heads_vt(0, bad, 16, 2, 128, None, A, A, st) == 3
    assert L.fp4_attn_softmax_quant(1, A, 16, 16, 0.1, None, A, A, A, st) == 1
    assert L.fp4_attn_softmax_quant(0, A, 16, 16, 0.0, None, A, A, A, st) == 1
    assert L.fp4_attn_softmax_quant(0, A, 0, 16, 0.1, None, A, A, A, st) == 1
    assert L.fp4_attn_softmax_quant(0, A, 16, 16, 0.1, None, A, bad, A, st) == 3
    assert L.fp4_attn_pv(0, A, A, None, 16, 16, A, A, None, 2, 128, 2, None, A, st) == 1
    assert L.fp4_attn_pv(1, A, A, None, 16, 16, A, A, A, 2, 128, 0, None, A, st) == 1
    assert L.fp4_attn_pv(0, A, A, None, 16, 16, A, A, None, 2, 64, 0, None, A, st) == 2
    assert L.fp4_attn_pv(0, A, A, None, 16, 16, A, A, None, 2, 128, 0, bad, A, st) == 3
    F = ctypes.c_float
    # fused head: globals all (NVFP4) or none (MXFP4), head < H, D = 128, scale > 0, aligned,
    # 32-bit TMA rows
    N4 = (None, None, None, None)
    G4 = (A, A, A, A)
    assert L.fp4_attn_fused(1, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.1), *N4, None, A, st) == 1
    assert L.fp4_attn_fused(1, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.1), A, A, A, None, None, A, st) == 1
    assert L.fp4_attn_fused(0, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.1), *G4, None, A, st) == 1
    assert L.fp4_attn_fused(1, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.1), A, A, A, A + 2, None, A, st) == 3
    assert L.fp4_attn_fused(0, A, A, 16, A, A, 16, A, A, 2, 128, 2, F(0.1), *N4, None, A, st) == 1
    assert L.fp4_attn_fused(0, A, A, 16, A, A, 16, A, A, 2, 64, 0, F(0.1), *N4, None, A, st) == 2
    assert L.fp4_attn_fused(0, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.0), *N4, None, A, st) == 1
    assert L.fp4_attn_fused(0, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.1), *N4, None, bad, st) == 3
    assert L.fp4_attn_fused(0, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.1), *N4, bad, A, st) == 3
    assert L.fp4_attn_fused(0, A, A, 16, A, A, 60000, A, A, 40000, 128, 0, F(0.1), *N4, None, A, st) == 2
    # trace: all three buffers or none, the tile inside the query rows
    assert L.fp4_attn_fused_trace(0, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.1), *N4, None, A, 1, A, A, A, st) == 1
    assert L.fp4_attn_fused_trace(0, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.1), *N4, None, A, 0, A, None, A,
                                  st) == 1
    assert L.fp4_attn_fused_trace(0, A, A, 16, A, A, 16, A, A, 2, 128, 0, F(0.1), *N4, None, A, 0, A, A, bad,
                                  st) == 3


def test_product_path_has_no_oracle_import():
    """The package never imports or loads the oracle."""
    pkg = os.path.join(ROOT, "fp4_block_scaled_act_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                for pat in ("import oracle", "from oracle", "liboracle", "fp4_oracle"):
                    assert pat not in text, (f, pat)
