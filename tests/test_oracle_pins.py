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


@pytest.mark.parametrize("case", GOLD["mxfp8_groups"]["cases"], ids=lambda c: c["why"][:30])
def test_mxfp8_dequant_worked(orc, case):
    """orc_dequant_mxfp8 (and the NumPy restatement) turn the worked groups' bytes back into
    the hand-computed values."""
    x = _group(case["x"], 32)
    elems, sf = orc.quantize_mxfp8(x)
    n = len(case["dequant"])
    got = orc.dequant_mxfp8(elems, sf, 128)[0]
    assert list(got[:n]) == case["dequant"], case["why"]
    assert not got[n:32].any()
    assert list(onp.dequant_mxfp8(elems, sf, 1, 128)[0, :n]) == case["dequant"]


def test_mxfp8_dequant_matches_numpy(orc):
    """orc_dequant_mxfp8 against the NumPy restatement on random bytes (every E4M3 code but
    NaN, every scale byte from 100 to 154), selected rows included."""
    rng = np.random.default_rng(31)
    rows, K = 300, 256
    codes = rng.integers(0, 256, size=(rows, K), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0
    sfm = rng.integers(100, 155, size=(rows, K // 32), dtype=np.uint8)
    sf = onp.swizzle_sf(sfm)
    ref = onp.dequant_mxfp8(codes, sf, rows, K)
    np.testing.assert_array_equal(orc.dequant_mxfp8(codes, sf, K), ref)
    sel = np.array([0, 5, 127, 128, 299])
    np.testing.assert_array_equal(orc.dequant_mxfp8(codes, sf, K, rows=sel), ref[sel])


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


@pytest.mark.parametrize("K", [128, 256])
def test_svd_linear_oracle_brute_force(orc, K):
    """The composed SVDQuant oracle (W4A8: MXFP8 activations, W4A4: MXFP4 activations, MXFP4
    residual, rank-32 low-rank term on the unquantized input, bias) against the same steps
    composed from the NumPy restatement, for every M, N in 1..8."""
    rng = np.random.default_rng(K + 7)
    rank = 32
    for M in range(1, 9):
        for N in range(1, 9):
            x = bf16(rng.standard_normal((M, K)) * rng.lognormal(0, 1.5, size=K))
            r = bf16(rng.standard_normal((N, K)) * 0.02)
            l1 = bf16(rng.standard_normal((K, rank)) * 0.05)
            l2 = bf16(rng.standard_normal((rank, N)) * 0.05)
            b = synth.f32_to_f16_bits(rng.standard_normal(N).astype(np.float32) * 0.01)
            rc, rs, _ = orc.pack_weight(orc.MX, r)
            xf = onp.bf16_to_f32(x).astype(np.float64)
            lr = (xf @ onp.bf16_to_f32(l1).astype(np.float64)) @ onp.bf16_to_f32(l2).astype(np.float64)
            lrs = np.abs(xf @ onp.bf16_to_f32(l1).astype(np.float64)) @ np.abs(onp.bf16_to_f32(l2).astype(np.float64))
            wc, wsf = onp.quant_mxfp4(r)
            w = onp.dequant_fp4("mx", wc, wsf, N, K)
            for act in ("mxfp8", "mxfp4"):
                Y, S = orc.svd_linear_rows(act, x, (rc, rs), l1, l2, b, np.arange(M))
                if act == "mxfp8":
                    e, sf = onp.quant_mxfp8(x)
                    a = onp.dequant_mxfp8(e, sf, M, K)
                else:
                    c, sf = onp.quant_mxfp4(x)
                    a = onp.dequant_fp4("mx", c, sf, M, K)
                Y2, S2 = onp.linear_fp64(a, w, b)
                Y2, S2 = Y2 + lr, S2 + lrs
                assert np.all(np.abs(Y - Y2) <= 1e-12 * S2 + 1e-300), (act, M, N)
                np.testing.assert_allclose(S, S2, rtol=1e-12, atol=1e-300)


def test_svd_linear_oracle_selects_rows(orc):
    """Rows selected out of order give the same values as the full result."""
    f = synth.svdquant_factors(3004, 128, 256, rank=32, calib_tokens=128)
    x = synth.activation(11, 40, 256, "lognormal")
    rc, rs, _ = orc.pack_weight(orc.MX, f["r_bf16"])
    b = synth.bias(5, 128)
    for act in ("mxfp8", "mxfp4"):
        Y, S = orc.svd_linear_rows(act, x, (rc, rs), f["l1_bf16"], f["l2_bf16"], b, np.arange(40))
        sel = np.array([39, 0, 17, 17, 3])
        Ys, Ss = orc.svd_linear_rows(act, x, (rc, rs), f["l1_bf16"], f["l2_bf16"], b, sel)
        np.testing.assert_array_equal(Ys, Y[sel])
        np.testing.assert_array_equal(Ss, S[sel])


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
# gelu(z) = 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))).  The oracle is that definition
# in fp64 (the exp identity where 1 + tanh cancels), rounded to the nearest bf16.  These
# pins tie it to a library GELU, to the independent NumPy route, to exact identities, and
# the bf16 rounding to exact rational arithmetic.
def _gelu_erf(z):
    """The exact GELU, z Phi(z), that the tanh form approximates."""
    return 0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0)))


def test_gelu_f64_against_library_gelu(orc):
    """PyTorch's tanh-approximated GELU in fp64 (a library routine) where its 1 + tanh does
    not cancel (z >= -5: 1 + tanh(v) >= 1e-7, so its own relative error stays below 1e-8)."""
    import torch

    rng = np.random.default_rng(12)
    z = np.concatenate([np.linspace(-5.0, 14.0, 19001), rng.normal(0.0, 2.0, 4000).clip(-5.0, None)])
    ref = torch.nn.functional.gelu(torch.from_numpy(z), approximate="tanh").numpy()
    got = np.array([orc.gelu_f64(float(v)) for v in z])
    tol = np.where(z >= -2.0, 1e-14, 1e-8) * np.abs(ref) + 1e-300
    assert np.all(np.abs(got - ref) <= tol), np.max(np.abs(got - ref) / (np.abs(ref) + 1e-300))


def test_gelu_f64_matches_numpy_route_every_bf16(orc):
    """Every finite bf16 z: the C oracle's tanh / exp split and the NumPy logaddexp route
    agree to 1e-12 relative (normal doubles), and give the same bf16 h for every z."""
    z = np.arange(65536, dtype=np.uint16)
    exp_field = (z >> 7) & 0xFF
    z = z[exp_field != 0xFF]                            # finite values only
    zf = synth.bf16_bits_to_f32(z).astype(np.float64)
    g_np = onp.gelu_f64(zf)
    g_c = np.array([orc.gelu_f64(float(v)) for v in zf[::5]])
    # relative agreement where the values are normal doubles; fp64 subnormals (|g| < 2^-1022,
    # z below about -26) carry fewer bits and both round to a zero bf16
    normal = np.abs(g_np[::5]) >= 2.0 ** -1000
    rel = np.abs(g_c - g_np[::5])[normal] / np.abs(g_np[::5])[normal]
    assert rel.max() <= 1e-12, rel.max()
    assert np.all(np.abs(g_c - g_np[::5])[~normal] <= 2.0 ** -1000)
    np.testing.assert_array_equal(orc.gelu_bf16(z), onp.f64_to_bf16_rn(g_np))


def test_gelu_f64_identities(orc):
    """gelu(z) - gelu(-z) = z (the two sides take different branches for z != 0); gelu(0) = 0;
    gelu(z) = z once tanh(v) rounds to 1; a signed zero once e^{-2v} overflows; within 1e-3
    of the exact GELU z Phi(z) that the tanh form approximates."""
    for z in np.linspace(0.0, 30.0, 3001)[1:]:
        assert abs(orc.gelu_f64(z) - orc.gelu_f64(-z) - z) <= 4e-16 * z, z
    assert orc.gelu_f64(0.0) == 0.0
    for z in (20.0, 100.0, 3.0e38):
        assert orc.gelu_f64(z) == z
    for z in (-40.0, -1e3, -3.0e38):
        g = orc.gelu_f64(z)
        assert g == 0.0 and math.copysign(1.0, g) == -1.0
    for z in np.linspace(-8.0, 8.0, 1601):
        assert abs(orc.gelu_f64(z) - _gelu_erf(z)) <= 1e-3, z
    # worked values of the definition: gelu(1) = 0.5 (1 + tanh(sqrt(2/pi) 1.044715)), gelu(-1) = gelu(1) - 1
    assert abs(orc.gelu_f64(1.0) - 0.8411919906082768) <= 1e-15
    assert abs(orc.gelu_f64(-1.0) + 0.15880800939172324) <= 1e-15


def test_f64_to_bf16_rn_exact(orc):
    """Nearest bf16 with ties to the even code, against exact rational arithmetic, on random
    doubles, exact midpoints, subnormals, the smallest normal and the largest finite value."""
    from fractions import Fraction

    def bf16_value(b):
        return Fraction(float(synth.bf16_bits_to_f32(np.array([b], dtype=np.uint16))[0]))

    def nearest(x):
        xf = Fraction(x)
        a = abs(xf)
        best = None
        t = int(np.float32(abs(x)).view(np.uint32) >> 16) if abs(x) < 3.4e38 else 0x7F7F
        for c in range(max(0, t - 2), min(0x7F7F, t + 3) + 1):
            d = abs(bf16_value(c) - a)
            if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
                best = (d, c)
        return best[1] | (0x8000 if math.copysign(1.0, x) < 0 else 0)

    rng = np.random.default_rng(21)
    xs = list(rng.normal(0, 1, 300) * np.exp2(rng.integers(-140, 120, 300)))
    for b in rng.integers(1, 0x7F7E, 200):                 # exact midpoints between neighbours
        lo, hi = bf16_value(int(b)), bf16_value(int(b) + 1)
        xs.append(float((lo + hi) / 2))
        xs.append(-float((lo + hi) / 2))
    xs += [2.0 ** -133, 3 * 2.0 ** -134, 2.0 ** -134, 2.0 ** -126, float.fromhex("0x1.fep127"), float.fromhex("0x1.fdp127"), 1.0, -0.0, 0.0]
    for x in xs:
        got = orc.f64_to_bf16_rn(float(x))
        assert got == nearest(float(x)), (x, hex(got), hex(nearest(float(x))))
        assert got == int(onp.f64_to_bf16_rn(np.array([x]))[0]), x
    assert orc.f64_to_bf16_rn(float.fromhex("0x1.ffp127")) == 0x7F80       # the tie above the largest finite value


def test_gelu_quantize_composition(orc):
    """gelu_quantize is gelu_bf16 then the format's quantizer."""
    rng = np.random.default_rng(13)
    z = synth.f32_to_bf16_bits(rng.normal(0.0, 3.0, 512).astype(np.float32)).reshape(2, 256)
    for fmt in (orc.MX, orc.NV):
        g = None if fmt == orc.MX else orc.nv_global(orc.tensor_amax(orc.gelu_bf16(z)))
        c1, s1 = orc.gelu_quantize(fmt, z, g)
        c2, s2 = orc.quantize(fmt, orc.gelu_bf16(z), g)
        np.testing.assert_array_equal(c1, c2)
        np.testing.assert_array_equal(s1, s2)
