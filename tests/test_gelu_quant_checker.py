"""CPU check of the validity test used for the fused GELU + quantize GEMM epilogue
(tests/gpu_helpers.check_gelu_quant): an output built by the oracle from its own GEMM
result passes, and planted mistakes in it (a code or a scale byte out of range, a
nonzero padding byte) are caught."""
import numpy as np
import pytest

import oracle
import synth
from tests import gpu_helpers as H


def _case(fmt, M=130, K=256, N=256, seed=5):
    x = synth.activation(seed, M, K, "lognormal")
    w = synth.weight(seed + 1, N, K)
    b = synth.bias(seed + 2, N)
    g_a = oracle.nv_global(oracle.tensor_amax(x)) if fmt == oracle.NV else None
    rows = np.arange(M)
    Y, S = oracle.fp4_linear_rows(fmt, x, w, b, rows, g_a=g_a)
    zb = H._bf16_bracket(Y)
    z = np.where(np.abs(H._bf16_f64(zb[0]) - Y) <= np.abs(H._bf16_f64(zb[1]) - Y), zb[0], zb[1]).astype(np.uint16)
    g_h = oracle.nv_global(oracle.tensor_amax(oracle.gelu_bf16(z))) if fmt == oracle.NV else None
    codes, sf = oracle.gelu_quantize(fmt, z, g_h)
    return codes, sf, Y, S, rows, M, N, g_h


@pytest.mark.parametrize("fmt", [oracle.MX, oracle.NV])
def test_checker_accepts_the_oracle_output_and_catches_planted_mistakes(fmt):
    import torch

    codes, sf, Y, S, rows, M, N, g_h = _case(fmt)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    assert H.check_gelu_quant(fmt, t(codes), t(sf), Y, S, rows, M, N, g_h, "oracle output") == 1.0
    # a code far from its admissible range: the largest magnitude with the opposite sign
    bad = codes.copy()
    r, c = 17, 40
    lo = bad[r, c // 2] & 0x0F if c % 2 == 0 else bad[r, c // 2] >> 4
    flipped = (0x7 if (lo & 0x8) else 0xF)
    bad[r, c // 2] = (bad[r, c // 2] & 0xF0) | flipped if c % 2 == 0 else (bad[r, c // 2] & 0x0F) | (flipped << 4)
    with pytest.raises(AssertionError, match="codes outside"):
        H.check_gelu_quant(fmt, t(bad), t(sf), Y, S, rows, M, N, g_h, "planted code")
    # a scale byte three steps too large
    G = 32 if fmt == oracle.MX else 16
    bad_sf = sf.copy()
    off = oracle.sf_offset(3, 2, N // G)
    bad_sf[off] = min(int(bad_sf[off]) + 3, 0x7E if fmt == oracle.NV else 250)
    with pytest.raises(AssertionError, match="scale bytes"):
        H.check_gelu_quant(fmt, t(codes), t(bad_sf), Y, S, rows, M, N, g_h, "planted scale")
    # a padding-row scale byte
    pad_sf = sf.copy()
    pad_sf[oracle.sf_offset(M + 1, 0, N // G)] = 1
    with pytest.raises(AssertionError, match="padding"):
        H.check_gelu_quant(fmt, t(codes), t(pad_sf), Y, S, rows, M, N, g_h, "planted padding")


@pytest.mark.parametrize("fmt", [oracle.MX, oracle.NV])
def test_exact_z_checker_accepts_bounded_perturbation_and_catches_mistakes(fmt):
    """check_gelu_quant_exact: the oracle's own output passes with no differing rows; an
    output computed from gelu values moved anywhere inside the library's stated bound (so
    that h lands on the other bf16 neighbour where the exact value is near a midpoint)
    passes; a planted code or scale outside the admissible range fails."""
    import torch
    from oracle import oracle_np as onp

    rng = np.random.default_rng(8)
    M, K = 64, 256
    z = synth.f32_to_bf16_bits(rng.normal(0.0, 2.5, (M, K)).astype(np.float32))
    g_h = oracle.nv_global(oracle.tensor_amax(oracle.gelu_bf16(z))) if fmt == oracle.NV else None
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    codes, sf = oracle.gelu_quantize(fmt, z, g_h)
    assert H.check_gelu_quant_exact(fmt, t(codes), t(sf), z, g_h, "oracle") == 0.0
    # a simulated fp32 evaluation at the edges of the bound
    zf = synth.bf16_bits_to_f32(z).astype(np.float64)
    g, e, cut = H.gelu_error_bound(zf)
    sim = g + e * np.where(rng.random(g.shape) < 0.5, -0.999, 0.999)
    h = onp.f64_to_bf16_rn(sim)
    c2, s2 = oracle.quantize(fmt, h, g_h)
    frac = H.check_gelu_quant_exact(fmt, t(c2), t(s2), z, g_h, "bounded perturbation")
    assert 0.0 <= frac <= 1.0
    # a code far outside its range
    bad = codes.copy()
    bad[5, 7] ^= 0x70 if (bad[5, 7] >> 4) & 0x7 < 4 else 0x30
    with pytest.raises(AssertionError, match="codes outside|scale bytes"):
        H.check_gelu_quant_exact(fmt, t(bad), t(sf), z, g_h, "planted code")
    G = 32 if fmt == oracle.MX else 16
    bad_sf = sf.copy()
    off = oracle.sf_offset(9, 1, K // G)
    bad_sf[off] = min(int(bad_sf[off]) + 3, 0x7E if fmt == oracle.NV else 250)
    with pytest.raises(AssertionError, match="scale bytes"):
        H.check_gelu_quant_exact(fmt, t(codes), t(bad_sf), z, g_h, "planted scale")
