"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: the format definitions
on the model-card pages, hand-worked examples (tests/golden), exact closed-form
cases, invariants the pages state (per-tensor independence, byte counts), the
independent NumPy restatement on tiny shapes, and a loose statistical check of the
MXFP4 error the W4A8 README reports.
"""
import json
import math
import os

import numpy as np
import pytest

import synth
from oracle import oracle_np as onp

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def bf16(vals):
    return synth.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


# ------------------------------------------------------------------ codecs
def test_e2m1_table(orc):
    t = GOLD["e2m1_table"]
    for c, v in zip(t["codes"], t["values"]):
        assert orc.e2m1_decode(c) == v and math.copysign(1, orc.e2m1_decode(c)) == math.copysign(1, v)
        assert onp.e2m1_decode(np.uint8(c)) == v
        # every grid value encodes back to its own code
        assert orc.e2m1_encode(v) == c


@pytest.mark.parametrize("v,code,why", GOLD["e2m1_rounding"]["cases"])
def test_e2m1_rounding(orc, v, code, why):
    assert orc.e2m1_encode(v) == code, why
    assert int(onp.e2m1_encode(np.float32(v))) == code, why


def test_e2m1_monotone_dense_sweep(orc):
    # encode is monotone non-decreasing in |v| and every result is a nearest grid value
    vals = np.linspace(0, 7, 2801, dtype=np.float32)
    mags = [orc.e2m1_decode(orc.e2m1_encode(float(v))) for v in vals]
    assert all(b >= a for a, b in zip(mags, mags[1:]))
    grid = np.array(GOLD["e2m1_table"]["values"][:8])
    for v, m in zip(vals, mags):
        d = np.abs(grid - min(float(v), 6.0))
        assert abs(m - min(float(v), 6.0)) == d.min()


def test_e4m3_decode_structure(orc):
    for b, v in GOLD["e4m3"]["decode"]:
        assert orc.e4m3_decode(b) == v
    pos = [orc.e4m3_decode(b) for b in range(0x7F)]
    assert all(b > a for a, b in zip(pos, pos[1:])), "positive codes strictly increasing"
    assert pos[-1] == 448.0 and pos[1] == 2.0 ** -9 and pos[8] == 2.0 ** -6
    assert math.isnan(orc.e4m3_decode(0x7F)) and math.isnan(orc.e4m3_decode(0xFF))
    for b in range(0x80):
        if b != 0x7F:
            assert orc.e4m3_decode(b | 0x80) == -orc.e4m3_decode(b)
    np.testing.assert_array_equal(onp.e4m3_decode(np.arange(0x7F, dtype=np.uint8)), np.array(pos))


@pytest.mark.parametrize("v,code,why", GOLD["e4m3"]["encode"])
def test_e4m3_encode(orc, v, code, why):
    assert orc.e4m3_encode(v) == code, why
    assert int(onp.e4m3_encode(np.float32(v))) == code, why


def test_e4m3_encode_exhaustive_vs_numpy(orc):
    # every fp32 value on a dense log grid spanning the E4M3 range, plus all midpoints
    codes = np.arange(0x7F, dtype=np.uint8)
    vals = onp.e4m3_decode(codes)
    mids = (vals[:-1] + vals[1:]) / 2
    xs = np.concatenate([vals, mids, np.geomspace(1e-4, 600, 4000)]).astype(np.float32)
    xs = np.concatenate([xs, -xs])
    c_np = onp.e4m3_encode(xs)
    c_c = np.array([orc.e4m3_encode(float(x)) for x in xs], dtype=np.uint8)
    np.testing.assert_array_equal(c_c, c_np)


def test_e8m0_decode(orc):
    assert orc.e8m0_decode(127) == 1.0
    assert orc.e8m0_decode(0) == 2.0 ** -127
    assert orc.e8m0_decode(254) == 2.0 ** 127
    for b in range(254):
        assert orc.e8m0_decode(b + 1) == 2 * orc.e8m0_decode(b)
    assert math.isnan(orc.e8m0_decode(255))


# ------------------------------------------------------------------ worked groups
def _group(vals, G):
    row = np.zeros((1, 128), dtype=np.float32)
    row[0, : len(vals)] = vals
    return bf16(row)


@pytest.mark.parametrize("case", GOLD["mxfp4_groups"]["cases"], ids=lambda c: c["why"][:30])
def test_mxfp4_worked(orc, case):
    x = _group(case["x"], 32)
    for codes, sf in (orc.quantize(orc.MX, x), onp.quant_mxfp4(x)):
        assert sf[orc.sf_offset(0, 0, 4)] == case["sf"], case["why"]
        un = onp.unpack_nibbles(codes)[0]
        assert list(un[: len(case["codes"])]) == case["codes"], case["why"]
        assert not un[len(case["codes"]):32].any()


@pytest.mark.parametrize("case", GOLD["mxfp8_groups"]["cases"], ids=lambda c: c["why"][:30])
def test_mxfp8_worked(orc, case):
    x = _group(case["x"], 32)
    for elems, sf in (orc.quantize_mxfp8(x), onp.quant_mxfp8(x)):
        assert sf[orc.sf_offset(0, 0, 4)] == case["sf"], case["why"]
        assert list(elems[0, : len(case["codes"])]) == case["codes"], case["why"]
        assert not elems[0, len(case["codes"]):32].any()


@pytest.mark.parametrize("case", GOLD["nvfp4_blocks"]["cases"], ids=lambda c: c["why"][:30])
def test_nvfp4_worked(orc, case):
    x = _group(case["x"], 16)
    g = orc.nv_global(case["T"])
    assert g == np.float32(np.float32(case["T"]) / np.float32(2688.0))
    for codes, sf in (orc.quantize(orc.NV, x, g), onp.quant_nvfp4(x, g)):
        assert sf[orc.sf_offset(0, 0, 8)] == case["sf"], case["why"]
        un = onp.unpack_nibbles(codes)[0]
        assert list(un[: len(case["codes"])]) == case["codes"], case["why"]


def test_nv_global_zero_tensor(orc):
    assert orc.nv_global(0.0) == 1.0
    x = np.zeros((3, 128), dtype=np.uint16)
    c, s = orc.quantize(orc.NV, x, orc.nv_global(orc.tensor_amax(x)))
    assert not c.any() and not s.any()


def test_nvfp4_static_global_saturation(orc):
    # a runtime block above the calibrated amax: scale saturates at 448, codes clip at +-6
    g = orc.nv_global(1.0)
    x = _group([20.0, -20.0, 1.0], 16)
    c, s = orc.quantize(orc.NV, x, g)
    assert s[0] == 0x7E
    un = onp.unpack_nibbles(c)[0]
    assert list(un[:2]) == [7, 15]


# ------------------------------------------------------------------ layouts
@pytest.mark.parametrize("rows,Kg", [(1, 4), (128, 4), (129, 8), (300, 12), (256, 160)])
def test_sf_layout_bijection(orc, rows, Kg):
    rp = -(-rows // 128) * 128
    offs = np.array([[orc.sf_offset(r, j, Kg) for j in range(Kg)] for r in range(rp)])
    assert sorted(offs.ravel().tolist()) == list(range(rp * Kg))
    assert orc.sf_bytes(rows, Kg) == rp * Kg
    # independent construction (reshape/transpose into 128x4 atoms)
    sfm = (np.arange(rows * Kg) % 251).astype(np.uint8).reshape(rows, Kg)
    flat = onp.swizzle_sf(sfm)
    for r in range(rows):
        for j in range(Kg):
            assert flat[offs[r, j]] == sfm[r, j]
    np.testing.assert_array_equal(onp.unswizzle_sf(flat, rows, Kg), sfm)


def test_sf_layout_hand_values(orc):
    # 128x4 atom: 32-row stripes 16 bytes apart, 4 stripes interleaved at 4-byte steps
    assert orc.sf_offset(0, 0, 8) == 0
    assert orc.sf_offset(0, 3, 8) == 3
    assert orc.sf_offset(1, 0, 8) == 16
    assert orc.sf_offset(31, 0, 8) == 496
    assert orc.sf_offset(32, 0, 8) == 4
    assert orc.sf_offset(127, 3, 8) == 31 * 16 + 3 * 4 + 3
    assert orc.sf_offset(0, 4, 8) == 512          # next group-of-4 atom along K
    assert orc.sf_offset(128, 0, 8) == 1024       # next 128-row block after Kg/4 atoms


def test_nibble_order_and_roundtrip(orc):
    # element 2i in the low nibble, 2i+1 in the high nibble (reading R5)
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 0] = 6.0   # code 7 (scale 1: amax 6 -> e = 0)
    x[0, 1] = -1.0  # code 0xA
    c, s = orc.quantize(orc.MX, bf16(x))
    assert c[0, 0] == (0xA << 4) | 0x7
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 16, size=(7, 256), dtype=np.uint8)
    np.testing.assert_array_equal(onp.unpack_nibbles(onp.pack_nibbles(codes)), codes)


# ------------------------------------------------------------------ cross-check (brute force)
@pytest.mark.parametrize("K", [128, 256, 384])
def test_c_oracle_matches_numpy_oracle(orc, K):
    rng = np.random.default_rng(K)
    for M in range(1, 9):
        x = bf16(rng.standard_normal((M, K)) * rng.lognormal(0, 2, size=K))
        c1, s1 = orc.quantize(orc.MX, x)
        c2, s2 = onp.quant_mxfp4(x)
        np.testing.assert_array_equal(c1, c2)
        np.testing.assert_array_equal(s1, s2)
        g = orc.nv_global(orc.tensor_amax(x))
        c1, s1 = orc.quantize(orc.NV, x, g)
        c2, s2 = onp.quant_nvfp4(x, g)
        np.testing.assert_array_equal(c1, c2)
        np.testing.assert_array_equal(s1, s2)
        e1, s1 = orc.quantize_mxfp8(x)
        e2, s2 = onp.quant_mxfp8(x)
        np.testing.assert_array_equal(e1, e2)
        np.testing.assert_array_equal(s1, s2)
        for N in (1, 3, 8):
            w = bf16(rng.standard_normal((N, K)) * 0.02)
            b = synth.f32_to_f16_bits(rng.standard_normal(N).astype(np.float32) * 0.01)
            for fmt, name in ((orc.MX, "mx"), (orc.NV, "nv")):
                ga = None if fmt == orc.MX else orc.nv_global(orc.tensor_amax(x))
                Y, S = orc.fp4_linear_rows(fmt, x, w, b, np.arange(M), g_a=ga)
                if fmt == orc.MX:
                    (ac, asf), (wc, wsf), gw, gaa = onp.quant_mxfp4(x), onp.quant_mxfp4(w), 1.0, 1.0
                else:
                    gw = onp.nv_global(np.abs(onp.bf16_to_f32(w)).max())
                    (ac, asf), (wc, wsf), gaa = onp.quant_nvfp4(x, ga), onp.quant_nvfp4(w, gw), ga
                Y2, S2 = onp.linear_fp64(onp.dequant_fp4(name, ac, asf, M, K, gaa),
                                         onp.dequant_fp4(name, wc, wsf, N, K, gw), b)
                # different summation orders: compare against the magnitude sum
                assert np.all(np.abs(Y - Y2) <= 1e-12 * S2)
                np.testing.assert_allclose(S, S2, rtol=1e-12, atol=1e-300)


# ------------------------------------------------------------------ GEMM closed forms
def _grid_matrix(rng, rows, K):
    """Values on the E2M1 grid, every 32-group holding a +-6 so the MX scale is exactly 1."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)
    v = grid[rng.integers(0, 8, size=(rows, K))] * np.where(rng.random((rows, K)) < 0.5, -1, 1)
    v[:, ::32] = 6.0
    return v.astype(np.float32)


def test_gemm_exact_on_grid(orc):
    rng = np.random.default_rng(11)
    M, N, K = 5, 7, 256
    a = _grid_matrix(rng, M, K)
    w = _grid_matrix(rng, N, K)
    b = synth.f32_to_f16_bits(np.array([0.5, -0.25, 0, 1, 2, -3, 0.125], dtype=np.float32))
    Y, S = orc.fp4_linear_rows(orc.MX, bf16(a), bf16(w), b, np.arange(M))
    exact = a.astype(np.float64) @ w.astype(np.float64).T + synth.f16_bits_to_f32(b).astype(np.float64)
    np.testing.assert_array_equal(Y, exact)
    np.testing.assert_array_equal(S, np.abs(a).astype(np.float64) @ np.abs(w).astype(np.float64).T)


def test_gemm_selector_weight(orc):
    # W row n has one 4.0 at column (3n) % K: Y[:, n] picks out A[:, (3n) % K] * 4 / 4 ... exactly
    rng = np.random.default_rng(12)
    M, N, K = 6, 9, 128
    a = _grid_matrix(rng, M, K)
    w = np.zeros((N, K), dtype=np.float32)
    cols = (3 * np.arange(N)) % K
    w[np.arange(N), cols] = 4.0      # amax 4 -> e = 0 -> code for 4 exact
    Y, _ = orc.fp4_linear_rows(orc.MX, bf16(a), bf16(w), None, np.arange(M))
    np.testing.assert_array_equal(Y, 4.0 * a[:, cols].astype(np.float64))


def test_gemm_nvfp4_exact_on_grid(orc):
    rng = np.random.default_rng(13)
    M, N, K = 4, 5, 128
    a = _grid_matrix(rng, M, K)
    a[:, ::16] = 6.0
    w = _grid_matrix(rng, N, K)
    w[:, ::16] = 6.0
    # T = 2688 gives g = 1, block amax 6 gives scale 1: all values exact
    ga = orc.nv_global(2688.0)
    assert ga == 1.0
    wc, ws = orc.quantize(orc.NV, bf16(w), 1.0)
    Y, _ = orc.fp4_linear_rows(orc.NV, bf16(a), None, None, np.arange(M), g_a=ga, packed_w=(wc, ws, 1.0))
    np.testing.assert_array_equal(Y, a.astype(np.float64) @ w.astype(np.float64).T)


def test_gemm_constant_rows(orc):
    M, N, K = 3, 4, 256
    a = np.full((M, K), 1.5, dtype=np.float32)
    w = np.full((N, K), -0.5, dtype=np.float32)
    Y, _ = orc.fp4_linear_rows(orc.MX, bf16(a), bf16(w), None, np.arange(M))
    # 1.5 -> amax 1.5, e=-2 -> code for 6 -> 1.5 exactly; -0.5 -> e=-3, -4 -> -0.5 exactly
    np.testing.assert_array_equal(Y, np.full((M, N), -0.75 * K))


def test_tolerance_formula(orc):
    # 1 bf16 ulp: y in [1, 2) -> 2^-7; y in [256, 512) -> 2
    t = orc.tolerance(np.array([1.0, 1.99, 300.0, 0.0]), np.zeros(4))
    assert list(t[:3]) == [2.0 ** -7, 2.0 ** -7, 2.0] and t[3] == 2.0 ** -133


# ------------------------------------------------------------------ invariants from the pages
def test_per_tensor_independence(orc):
    """Sharded conversion gives identical output (the NVFP4 ctq card, 'Why per-shard quantization')."""
    w = synth.weight(77, 384, 256)
    c, s = orc.quantize(orc.MX, w)
    parts = [orc.quantize(orc.MX, w[i:i + 128]) for i in range(0, 384, 128)]
    np.testing.assert_array_equal(np.concatenate([p[0] for p in parts]), c)
    np.testing.assert_array_equal(np.concatenate([p[1] for p in parts]), s)
    g = orc.nv_global(orc.tensor_amax(w))
    c, s = orc.quantize(orc.NV, w, g)
    parts = [orc.quantize(orc.NV, w[i:i + 128], g) for i in range(0, 384, 128)]
    np.testing.assert_array_equal(np.concatenate([p[0] for p in parts]), c)
    np.testing.assert_array_equal(np.concatenate([p[1] for p in parts]), s)


def test_determinism(orc):
    x = synth.activation(5, 300, 512, "lognormal")
    a = orc.quantize(orc.MX, x)
    b = orc.quantize(orc.MX, x)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_mxfp4_error_matches_reported_scale(orc):
    """The W4A8 README reports an MXFP4 residual relative error of ~11.6%; RTN on a
    Gaussian-like residual should land in the same neighbourhood (loose: 9-14%)."""
    f = synth.svdquant_factors(3001, 512, 3072, calib_tokens=512)
    r = f["r_bf16"]
    c, s = orc.quantize(orc.MX, r)
    deq = orc.dequant_fp4(orc.MX, c, s, r.shape[1])
    ref = synth.bf16_bits_to_f32(r).astype(np.float64)
    rel = np.linalg.norm(deq - ref) / np.linalg.norm(ref)
    assert 0.09 < rel < 0.14, rel


def test_w4a8_fold_identity():
    """X W0^T = X R^T + (X L1) L2 in fp64 before any rounding (the exporter folds 1/s
    into the residual and proj_down so the checkpoint is self-contained)."""
    f = synth.svdquant_factors(3002, 256, 384, rank=32, calib_tokens=256)
    x = synth.bf16_bits_to_f32(synth.activation(9, 16, 384, "lognormal")).astype(np.float64)
    lhs = x @ f["w0"].T
    rhs = x @ f["r"].T + (x @ f["l1"]) @ f["l2"]
    np.testing.assert_allclose(rhs, lhs, rtol=1e-9, atol=1e-12)


def test_lowrank_oracle_matches_numpy(orc):
    f = synth.svdquant_factors(3003, 128, 256, rank=32, calib_tokens=128)
    x = synth.activation(10, 6, 256, "lognormal")
    LR, LS = orc.lowrank_fp64(x, np.arange(6), f["l1_bf16"], f["l2_bf16"])
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    l1 = synth.bf16_bits_to_f32(f["l1_bf16"]).astype(np.float64)
    l2 = synth.bf16_bits_to_f32(f["l2_bf16"]).astype(np.float64)
    u = xf @ l1
    np.testing.assert_allclose(LR, u @ l2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(LS, np.abs(u) @ np.abs(l2), rtol=1e-10, atol=1e-12)


def test_wan_a14b_byte_count():
    """400 quantized linears per transformer (MXFP4 card, Coverage); packed FP4 + per-32
    E8M0 scales take 0.5 + 1/32 bytes per weight.  The card quotes about 7.45 GiB; the
    exact figure below (7.46e9 bytes) matches it when read as decimal gigabytes."""
    per_block = 8 * 5120 * 5120 + 2 * 5120 * 13824
    params = 40 * per_block
    assert len(range(40)) * 10 == 400
    assert params == 14_050_918_400
    mx_bytes = params // 2 + params // 32
    assert mx_bytes == 7_464_550_400
    assert abs(mx_bytes / 1e9 - 7.45) < 0.02


# ------------------------------------------------------------------ GELU-tanh (R10)
# The activation between ffn.net.0.proj and ffn.net.2 (the MXFP4 cards' coverage lists):
# 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))).  The oracle evaluates it in fp32 in a
# fixed order with its own exp; these pins tie that evaluation to the definition.
def _f32(v):
    return float(np.float32(v))


def _gelu_arg(z):
    """a = -2 sqrt(2/pi) (z + 0.044715 z^3), the exp argument of the fp32 evaluation."""
    return -2.0 * math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)


def test_exp2_f32_against_math(orc):
    """floor reduction + degree-6 Taylor in ln2 f (fma Horner): within 2^-21.5 relative of
    2^t over [-126, 127], and exact at integers (f = 0 gives the polynomial's 1)."""
    rng = np.random.default_rng(11)
    pts = np.concatenate([np.linspace(-126.0, 127.0, 20001), rng.uniform(-126.0, 127.0, 5000),
                          [0.0, -0.0, 1e-8, -1e-8, 0.5, -0.5, 0.49999997, -0.49999997]]).astype(np.float32)
    worst = 0.0
    for t in pts:
        t = float(t)
        ref = 2.0 ** t
        worst = max(worst, abs(orc.exp2_f32(t) - ref) / ref)
    assert worst <= 2.0 ** -21.5, worst
    for n in range(-126, 128):
        assert orc.exp2_f32(float(n)) == 2.0 ** n


def test_recip_f32_newton(orc):
    """Newton-Raphson 1/d from the exponent-bit guess: within 2^-23 relative over
    [1, 2^125], and exact where 1/d is a power of two reached by the iteration."""
    rng = np.random.default_rng(14)
    ds = np.concatenate([np.exp2(np.linspace(0.0, 125.0, 50001)), rng.uniform(1.0, 4.0, 5000),
                         [1.0, 1.5, 2.0, 3.0, 1.0000001, 1.9999999]]).astype(np.float32)
    worst = max(abs(orc.recip_f32(float(d)) * float(d) - 1.0) for d in ds)
    assert worst <= 2.0 ** -23, worst
    for k in range(0, 126, 5):
        assert orc.recip_f32(2.0 ** k) == 2.0 ** -k


def test_gelu_f32_against_tanh_definition(orc):
    """Where 1 + tanh(v) does not cancel in fp64 (z >= -5) the plain definition is the
    reference; the fp32 evaluation is within (2|a| + 16) 2^-23 relative of it."""
    for z in np.linspace(-5.0, 14.0, 19001).astype(np.float32):
        z = float(z)
        ref = orc.gelu_f64(z)
        got = orc.gelu_f32(z)
        tol = (2.0 * abs(_gelu_arg(z)) + 16.0) * 2.0 ** -23 * abs(ref) + 2.0 ** -126
        assert abs(got - ref) <= tol, (z, got, ref)


def test_gelu_f32_against_library_gelu(orc):
    """PyTorch's own tanh-approximated GELU in fp64 (a library routine) on random bf16
    inputs of both signs, within the same bound."""
    import torch

    rng = np.random.default_rng(12)
    z = np.concatenate([rng.normal(0.0, 2.0, 4000), rng.uniform(-5.0, 12.0, 2000)])
    zb = synth.f32_to_bf16_bits(z.astype(np.float32))
    zf = synth.bf16_bits_to_f32(zb).astype(np.float64)
    ref = torch.nn.functional.gelu(torch.from_numpy(zf), approximate="tanh").numpy()
    for zi, ri in zip(zf, ref):
        if zi < -5.0:
            continue  # fp64 cancellation in 1 + tanh
        got = orc.gelu_f32(float(zi))
        tol = (2.0 * abs(_gelu_arg(zi)) + 16.0) * 2.0 ** -23 * abs(ri) + 2.0 ** -126
        assert abs(got - ri) <= tol, (zi, got, ri)


def test_gelu_f32_tail_against_sigmoid_identity(orc):
    """On the negative tail the fp64 reference is the exact identity
    0.5 (1 + tanh(v)) = 1 / (1 + exp(-2v)), itself checked against tanh where both are
    accurate; the fp32 result is a signed zero once 2^t passes 2^125 (true value below
    2^-118 |z|)."""
    for z in np.linspace(-5.0, 5.0, 1001):
        v = math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)
        assert abs(0.5 * (1.0 + math.tanh(v)) - 1.0 / (1.0 + math.exp(-2.0 * v))) <= 1e-15
    for z in np.linspace(-10.02, -5.0, 5021).astype(np.float32):
        z = float(z)
        a = _gelu_arg(z)
        got = orc.gelu_f32(z)
        if got == 0.0:
            assert math.copysign(1.0, got) == -1.0 and a > 86.6  # t = a / ln2 > 125
            assert abs(z / (1.0 + math.exp(a))) < 2.0 ** -118 * abs(z)
            continue
        ref = z / (1.0 + math.exp(a))
        assert abs(got - ref) <= (2.0 * abs(a) + 16.0) * 2.0 ** -23 * abs(ref), (z, got, ref)
    assert math.copysign(1.0, orc.gelu_f32(-11.0)) == -1.0 and orc.gelu_f32(-11.0) == 0.0
    assert orc.gelu_f32(-3.0e38) == 0.0


def test_gelu_f32_special_values(orc):
    assert orc.gelu_f32(0.0) == 0.0
    for z in (12.0, 20.0, 1000.0, 3.0e38):  # sigmoid(2v) rounds to 1 in fp32
        assert orc.gelu_f32(z) == _f32(z)
    # GELU-tanh(1) = 0.84119199... (the tanh-approximation's value, fp64 definition)
    assert abs(orc.gelu_f32(1.0) - 0.8411919906082768) <= 2.0 ** -21
    # odd part: gelu(z) - gelu(-z) = z
    for z in (0.25, 0.75, 1.5, 2.5, 4.0):
        assert abs(orc.gelu_f32(z) - orc.gelu_f32(-z) - z) <= 2.0 ** -20 * z


def test_gelu_bf16_rounding(orc):
    """gelu_bf16 rounds the fp32 result to nearest even bf16, brute-forced on small inputs."""
    import struct

    def bf16_rn(f):
        u = struct.unpack("<I", struct.pack("<f", f))[0]
        lower = u & 0xFFFF
        hi = u >> 16
        if lower > 0x8000 or (lower == 0x8000 and (hi & 1)):
            hi += 1
        return hi & 0xFFFF

    rng = np.random.default_rng(13)
    z = synth.f32_to_bf16_bits(rng.normal(0.0, 3.0, 3000).astype(np.float32))
    h = orc.gelu_bf16(z)
    zf = synth.bf16_bits_to_f32(z)
    for zi, hi in zip(zf, h):
        assert int(hi) == bf16_rn(orc.gelu_f32(float(zi)))
    # the composition used for the fused path: GELU, bf16, then the MXFP4 quantizer
    zz = z[:2 * 128].reshape(2, 128)
    c1, s1 = orc.gelu_quantize(orc.MX, zz)
    c2, s2 = orc.quantize(orc.MX, orc.gelu_bf16(zz))
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)
