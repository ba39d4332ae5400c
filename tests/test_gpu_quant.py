"""GPU parity of the quantization kernels against the CPU oracle.

Codes and the whole scale-factor buffer (padding rows included) must match the
oracle byte for byte; the NVFP4 weight global must match bit for bit.  The one
exception is the GELU-tanh quantizer, whose fp32 GELU is judged against the fp64
definition within its stated bound (see the GELU section below).
"""
import numpy as np
import pytest

import oracle
import synth
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

MX, NV = oracle.MX, oracle.NV


@pytest.fixture(scope="module")
def fb():
    import fp4_block_scaled_act_b200 as fb

    fb.build()
    return fb


def _quant_dev(fb, fmt, x_bits, g=None):
    import torch

    x = H.dev_bf16(x_bits)
    ga = H.dev_f32([g]) if fmt == NV else None
    codes, sf = fb.quantize_act(x, fmt, ga)
    torch.cuda.synchronize()
    return H.host_u8(codes), H.host_u8(sf)


def _assert_quant(fb, orc, fmt, x_bits, g=None):
    c_ref, s_ref = orc.quantize(fmt, x_bits, g)
    c, s = _quant_dev(fb, fmt, x_bits, g)
    assert c.shape == c_ref.shape and s.shape == s_ref.shape
    if not np.array_equal(c, c_ref):
        i = np.argwhere(c != c_ref)[0]
        raise AssertionError(f"codes differ at {tuple(i)}: gpu {c[tuple(i)]:#04x} oracle {c_ref[tuple(i)]:#04x}")
    if not np.array_equal(s, s_ref):
        i = int(np.argwhere(s != s_ref)[0][0])
        raise AssertionError(f"scale byte {i} differs: gpu {s[i]:#04x} oracle {s_ref[i]:#04x}")


# ------------------------------------------------------------------ converter sweeps
def test_e2m1_conversion_sweep(fb, orc):
    """Every finite bf16 value in (-8, 8) through the device E2M1 path, scale fixed at 1.

    Each 32-group holds a 6.0 so the MX scale is 2^0 and the codes are e2m1(x) itself."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = synth.bf16_bits_to_f32(allbits)
    keep = np.isfinite(vals) & (np.abs(vals) < 8.0)
    xs = allbits[keep]
    n_per_group = 31
    groups = -(-xs.size // n_per_group)
    pad = np.zeros(groups * n_per_group, dtype=np.uint16)
    pad[: xs.size] = xs
    body = pad.reshape(groups, n_per_group)
    six = np.full((groups, 1), synth.f32_to_bf16_bits(np.float32(6.0)), dtype=np.uint16)
    flat = np.concatenate([six, body], axis=1).reshape(-1)
    K = 512
    rows = -(-flat.size // K)
    x = np.zeros(rows * K, dtype=np.uint16)
    x[: flat.size] = flat
    _assert_quant(fb, orc, MX, x.reshape(rows, K))


@pytest.mark.parametrize("min_rows", [0, 8200], ids=["separate-kernels", "fused-with-lowrank"])
def test_e4m3_conversion_sweep(fb, orc, min_rows):
    """Every finite bf16 value in (-512, 512) through the device E4M3 path (MXFP8 with a
    300.0 in each group, so the scale is 2^0 and the elements are e4m3(x)).  Padded with zero
    rows to 8200 (65 blocks of 128), the call quantizes inside the low-rank projection's pass
    instead of in its own kernel."""
    import torch

    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = synth.bf16_bits_to_f32(allbits)
    xs = allbits[np.isfinite(vals) & (np.abs(vals) < 512.0)]
    n_per_group = 31
    groups = -(-xs.size // n_per_group)
    pad = np.zeros(groups * n_per_group, dtype=np.uint16)
    pad[: xs.size] = xs
    big = np.full((groups, 1), synth.f32_to_bf16_bits(np.float32(300.0)), dtype=np.uint16)
    flat = np.concatenate([big, pad.reshape(groups, n_per_group)], axis=1).reshape(-1)
    K = 512
    rows = max(-(-flat.size // K), min_rows)
    x = np.zeros(rows * K, dtype=np.uint16)
    x[: flat.size] = flat
    x = x.reshape(rows, K)
    e_ref, s_ref = orc.quantize_mxfp8(x)
    l1 = torch.zeros((K, 32), dtype=torch.bfloat16, device="cuda")
    xe = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    xs_ = torch.empty(fb.fp4_sf_bytes(MX, rows, K), dtype=torch.uint8, device="cuda")
    u = torch.empty((rows, 64), dtype=torch.bfloat16, device="cuda")
    fb.w4a8_quantize_act(H.dev_bf16(x), rows, K, l1, 32, xe, xs_, u)
    torch.cuda.synchronize()
    e = H.host_u8(xe)
    if not np.array_equal(e, e_ref):
        i = np.argwhere(e != e_ref)[0]
        raise AssertionError(f"e4m3 differs at {tuple(i)}: input {synth.bf16_bits_to_f32(x[tuple(i)])!r} "
                             f"gpu {e[tuple(i)]:#04x} oracle {e_ref[tuple(i)]:#04x}")
    np.testing.assert_array_equal(H.host_u8(xs_), s_ref)


# ------------------------------------------------------------------ shapes and formats
SHAPES = [(1, 128), (7, 256), (128, 512), (129, 384), (256, 512), (300, 640), (1000, 1280)]


@pytest.mark.parametrize("M,K", SHAPES)
def test_mxfp4_quant(fb, orc, M, K):
    x = synth.activation(100 + M, M, K, "lognormal")
    _assert_quant(fb, orc, MX, x)


@pytest.mark.parametrize("M,K", SHAPES)
def test_nvfp4_quant(fb, orc, M, K):
    x = synth.activation(200 + M, M, K, "lognormal")
    cal = synth.activation(300 + M, 256, K, "lognormal")
    g = orc.nv_global(orc.tensor_amax(cal))     # static global from a different batch
    _assert_quant(fb, orc, NV, x, g)


# 8300 rows = 65 blocks of 128 (the last ragged): one pass quantizes and projects
@pytest.mark.parametrize("M,K", [(1, 128), (130, 256), (4290 // 10, 3072), (8300, 384)])
def test_mxfp8_quant_and_lowrank(fb, orc, M, K):
    import torch

    x = synth.activation(400 + M, M, K, "lognormal")
    f = synth.svdquant_factors(500 + K, 256, K, calib_tokens=256)
    e_ref, s_ref = orc.quantize_mxfp8(x)
    xe = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    xs = torch.empty(fb.fp4_sf_bytes(MX, M, K), dtype=torch.uint8, device="cuda")
    u = torch.empty((M, 64), dtype=torch.bfloat16, device="cuda")
    fb.w4a8_quantize_act(H.dev_bf16(x), M, K, H.dev_bf16(f["l1_bf16"]), 32, xe, xs, u)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(H.host_u8(xe), e_ref)
    np.testing.assert_array_equal(H.host_u8(xs), s_ref)
    # u = x L1 accumulated in fp32, carried as the bf16 pair hi + lo: against fp64, within
    # the fp32 accumulation error of sum_k |x_k l1_k| plus the pair's 2^-18 |u|
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    l1 = synth.bf16_bits_to_f32(f["l1_bf16"]).astype(np.float64)
    u_ref = xf @ l1
    mag = np.abs(xf) @ np.abs(l1)
    pair = u.float().cpu().numpy().astype(np.float64)
    hi, lo = pair[:, :32], pair[:, 32:]
    err = np.abs(hi + lo - u_ref)
    assert np.all(err <= 4 * K * 2.0 ** -24 * mag + 2.0 ** -17 * np.abs(u_ref) + 1e-30)
    # a valid split: lo is below half an ulp of hi (bf16: 2^-8 relative)
    assert np.all(np.abs(lo) <= 2.0 ** -8 * np.abs(hi) + 1e-30)


def test_edge_values(fb, orc):
    """Zeros, negative zeros, huge and tiny magnitudes, and mixed-sign groups."""
    K = 256
    rows = []
    rows.append(np.zeros(K, dtype=np.float32))
    rows.append(np.full(K, -0.0, dtype=np.float32))
    rows.append(np.linspace(-3e38, 3e38, K).astype(np.float32))
    rows.append((np.linspace(-1, 1, K) * 1e-38).astype(np.float32))
    r = np.zeros(K, dtype=np.float32)
    r[::2] = 1e-30
    r[1::2] = -7.0
    rows.append(r)
    rows.append(np.where(np.arange(K) % 17 == 0, 1e4, -1e-4).astype(np.float32))
    x = synth.f32_to_bf16_bits(np.stack(rows))
    _assert_quant(fb, orc, MX, x)
    for T in (2688.0, 1.0, 1e-3, 3e38):
        _assert_quant(fb, orc, NV, x, orc.nv_global(T))


# ------------------------------------------------------------------ amax and weight pack
def test_tensor_amax(fb, orc):
    import torch

    for n, seed in ((1, 1), (7, 2), (4096, 3), (1_000_003, 4)):
        x = synth.activation(seed, 1, n, "lognormal")
        xd = H.dev_bf16(x.reshape(-1))
        out = torch.empty(1, dtype=torch.float32, device="cuda")
        fb.fp4_tensor_amax(xd, n, out)
        torch.cuda.synchronize()
        assert out.item() == orc.tensor_amax(x)


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("N,K", [(128, 128), (384, 512), (512, 512)])
def test_pack_weight(fb, orc, fmt, N, K):
    import torch

    w = synth.weight(600 + N + K, N, K)
    c_ref, s_ref, g_ref = orc.pack_weight(fmt, w)
    pw = fb.pack_weight(H.dev_bf16(w), fmt)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(H.host_u8(pw.codes), c_ref)
    np.testing.assert_array_equal(H.host_u8(pw.sf), s_ref)
    if fmt == NV:
        assert np.float32(pw.w_global.item()) == np.float32(g_ref)


def test_quant_determinism(fb):
    import torch

    x = H.dev_bf16(synth.activation(7, 513, 1024, "lognormal"))
    a = fb.quantize_act(x, MX)
    b = fb.quantize_act(x, MX)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ------------------------------------------------------------------ NVFP4 activation calibration
def test_calibrate_act_global(fb, orc):
    """fp4_calibrate_act_global over one and over several batches (a running max), and an
    all-zero batch (g = 1): bit-exact against the oracle's global of the same values."""
    import torch

    K = 5120
    s = synth.seeds_for(2)
    b1 = synth.activation(s["calib"], 4096, K, "lognormal", gain_seed=s["gain"])
    b2 = synth.activation(s["calib"] + 1, 1000, K, "lognormal", gain_seed=s["gain"])
    b3 = (b2.astype(np.uint32) & 0x807F).astype(np.uint16)      # small values (exponent field 0)
    g, amax = fb.calibrate_act_global(H.dev_bf16(b1))
    torch.cuda.synchronize()
    assert amax.item() == orc.tensor_amax(b1)
    assert g.item() == orc.nv_global(orc.tensor_amax(b1))
    g, amax = fb.calibrate_act_global([H.dev_bf16(b) for b in (b3, b2, b1)])
    torch.cuda.synchronize()
    allb = np.concatenate([b1.ravel(), b2.ravel(), b3.ravel()])
    assert amax.item() == orc.tensor_amax(allb) and g.item() == orc.nv_global(orc.tensor_amax(allb))
    z = np.zeros((3, 128), dtype=np.uint16)
    g, amax = fb.calibrate_act_global(H.dev_bf16(z))
    torch.cuda.synchronize()
    assert amax.item() == 0.0 and g.item() == 1.0


# ------------------------------------------------------------------ full size (the bench workload)
@pytest.mark.parametrize("fmt", [MX, NV])
def test_full_size_quant(fb, orc, fmt):
    """M = 75600 tokens, K = 5120: every code and scale byte, in the bench's launch shape."""
    M, K = 75600, 5120
    s = synth.seeds_for(2 if fmt == NV else 1)
    x = synth.activation(s["x"], M, K, "lognormal", gain_seed=s["gain"])
    g = None
    if fmt == NV:
        cal = synth.activation(s["calib"], synth.CALIB_TOKENS, K, "lognormal", gain_seed=s["gain"])
        g = orc.nv_global(orc.tensor_amax(cal))
    _assert_quant(fb, orc, fmt, x, g)


@pytest.mark.parametrize("M,K", [(130, 512), (300, 1024), (8300, 384)])
def test_w4a4_quantize_act(fb, orc, M, K):
    """W4A4 SVDQuant activation side: MXFP4 codes and scales bit-exact, the u pair as in W4A8."""
    import torch

    x = synth.activation(900 + M, M, K, "lognormal")
    f = synth.svdquant_factors(901 + K, 256, K, calib_tokens=256)
    c_ref, s_ref = orc.quantize(MX, x)
    xc = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    xs = torch.empty(fb.fp4_sf_bytes(MX, M, K), dtype=torch.uint8, device="cuda")
    u = torch.empty((M, 64), dtype=torch.bfloat16, device="cuda")
    fb.w4a4_quantize_act(H.dev_bf16(x), M, K, H.dev_bf16(f["l1_bf16"]), 32, xc, xs, u)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(H.host_u8(xc), c_ref)
    np.testing.assert_array_equal(H.host_u8(xs), s_ref)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    l1 = synth.bf16_bits_to_f32(f["l1_bf16"]).astype(np.float64)
    u_ref = xf @ l1
    mag = np.abs(xf) @ np.abs(l1)
    pair = u.float().cpu().numpy().astype(np.float64)
    err = np.abs(pair[:, :32] + pair[:, 32:] - u_ref)
    assert np.all(err <= 4 * K * 2.0 ** -24 * mag + 2.0 ** -17 * np.abs(u_ref) + 1e-30)


# ------------------------------------------------------------------ GELU-tanh + quantize (R10)
# The oracle's h is bf16_rn(gelu(z)) with gelu in fp64; the library evaluates gelu in fp32
# under a stated error bound (gelu.cuh), so its h may be the other bf16 neighbour where gelu(z)
# sits within that bound of a rounding midpoint.  The bound itself is checked first, on every
# finite bf16 z; the quantized outputs are then compared with the oracle row by row, and the
# rows that differ must be admissible for the bound (gpu_helpers.check_gelu_quant_exact).
def _finite_bf16():
    z = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    return z[((z >> 7) & 0xFF) != 0xFF]


def test_gelu_f32_error_bound_every_bf16(fb, orc):
    """The library's fp32 GELU against the fp64 definition, for every finite bf16 input:
    |g - gelu(z)| <= (2|a| + 16) 2^-23 |gelu(z)| + 2^-126 (a = -2v), a signed zero past the
    cut-off a/ln2 > 125, and its bf16 rounding within the interval the tests accept."""
    import torch

    z = _finite_bf16()
    z = np.concatenate([z, np.zeros(z.size % 2, dtype=np.uint16)])
    g_dev = torch.empty(z.size, dtype=torch.float32, device="cuda")
    fb.fp4bsa_test_gelu_f32(H.dev_bf16(z), z.size, g_dev)
    torch.cuda.synchronize()
    g = g_dev.cpu().numpy().astype(np.float64)
    zf = synth.bf16_bits_to_f32(z).astype(np.float64)
    ref, bound, cut = H.gelu_error_bound(zf)
    err = np.abs(g - ref)
    ok = (err <= bound) | (cut & (g == 0.0) & (np.signbit(g) == np.signbit(zf)))
    if not ok.all():
        i = int(np.argwhere(~ok)[0][0])
        raise AssertionError(f"{(~ok).sum()} inputs outside the bound; first z={zf[i]!r} gpu={g[i]!r} "
                             f"ref={ref[i]!r} bound={bound[i]!r}")
    assert np.all(~cut | (g == 0.0))               # past the cut-off: a zero, as stated
    # h = bf16_rn(g) lies in the accepted interval; count where it differs from the oracle's h
    from oracle import oracle_np as onp

    h = onp.f64_to_bf16_rn(g)
    hmin, hmax = H.gelu_h_interval(z, z)
    hv = synth.bf16_bits_to_f32(h).astype(np.float64)
    assert np.all((hv >= hmin) & (hv <= hmax))
    differ = int((synth.bf16_bits_to_f32(orc.gelu_bf16(z)) != synth.bf16_bits_to_f32(h)).sum())
    assert differ <= z.size // 200, differ          # a rounding-midpoint effect, not a drift
    print(f"gelu: {differ} of {z.size} bf16 inputs round to the other neighbour of the oracle's h")


def _gelu_sweep_bits():
    """Every bf16 value with |z| <= 16, both signs, in rows of 256 (zero padded)."""
    pos = np.arange(0x0000, 0x4181, dtype=np.uint16)  # 0x4180 = 16.0
    z = np.concatenate([pos, pos | np.uint16(0x8000)])
    pad = (-z.size) % 256
    return np.concatenate([z, np.zeros(pad, dtype=np.uint16)]).reshape(-1, 256)


def _gelu_case(fb, orc, fmt, z, max_rows_differ=0.05):
    import torch

    g = orc.nv_global(orc.tensor_amax(orc.gelu_bf16(z))) if fmt == NV else None
    codes, sf = fb.gelu_quantize_act(H.dev_bf16(z), fmt, H.dev_f32([g]) if fmt == NV else None)
    torch.cuda.synchronize()
    frac = H.check_gelu_quant_exact(fmt, codes, sf, z, g, f"gelu quantize fmt={fmt} shape={z.shape}")
    assert frac <= max_rows_differ, frac
    return frac


@pytest.mark.parametrize("fmt", [MX, NV])
def test_gelu_quantize_act_every_bf16_in_range(fb, orc, fmt):
    """Every bf16 |z| <= 16: rows equal to the oracle's, or admissible for the GELU bound."""
    _gelu_case(fb, orc, fmt, _gelu_sweep_bits(), max_rows_differ=0.25)


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("M,K,sigma", [(1, 256, 0.3), (130, 512, 1.0), (300, 13824, 3.0)])
def test_gelu_quantize_act_shapes(fb, orc, fmt, M, K, sigma):
    rng = np.random.default_rng(M + K)
    z = synth.f32_to_bf16_bits((rng.normal(0.0, sigma, (M, K))).astype(np.float32))
    _gelu_case(fb, orc, fmt, z, max_rows_differ=1.0 if K >= 13824 else 0.25)


def test_gelu_quantize_act_full_size_nvfp4(fb, orc):
    """The ffn down projection's input at the full shape (M = 75600, K = 13824), NVFP4."""
    z = synth.activation(7100, 75600, 13824, "lognormal")
    _gelu_case(fb, orc, NV, z, max_rows_differ=1.0)
