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
