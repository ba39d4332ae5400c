"""Shared helpers for the GPU parity tests: device copies of seeded inputs and the
oracle comparison of GEMM outputs."""
from __future__ import annotations

import numpy as np

import oracle
import synth


def torch_mod():
    import torch

    return torch


def dev_bf16(bits: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f16(bits: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.float16).cuda()


def dev_f32(vals):
    torch = torch_mod()
    return torch.tensor(np.asarray(vals, dtype=np.float32).reshape(-1), device="cuda")


def host_u8(t) -> np.ndarray:
    return t.contiguous().cpu().view(torch_mod().uint8).numpy()


def host_bf16_as_f64(y) -> np.ndarray:
    bits = y.contiguous().cpu().view(torch_mod().int16).numpy().view(np.uint16)
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def sample_rows(M: int, n_random: int = 64, seed: int = 0) -> np.ndarray:
    """First rows, seeded random rows and every row of the ragged last 128-row tile."""
    rng = np.random.default_rng(seed)
    tail0 = (M // 128) * 128
    if tail0 == M:
        tail0 = max(0, M - 128)
    rows = set(range(min(8, M)))
    rows |= set(rng.integers(0, M, size=min(n_random, M)).tolist())
    rows |= set(range(tail0, M))
    return np.array(sorted(rows), dtype=np.int64)


def check_linear(y_dev, Y_ref: np.ndarray, S: np.ndarray, rows: np.ndarray, what: str):
    """|y - y_ref| <= ulp_bf16(y_ref) + 1e-5 * sum_k |a_k w_k| on the given rows."""
    y = host_bf16_as_f64(y_dev)[rows]
    tol = oracle.tolerance(Y_ref, S)
    err = np.abs(y - Y_ref)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {bad.sum()} / {bad.size} elements out of tolerance; first at row {rows[i[0]]} col {i[1]}: "
            f"gpu {y[tuple(i)]!r} ref {Y_ref[tuple(i)]!r} tol {tol[tuple(i)]!r}; max err/tol {(err / tol).max():.3g}")
    return float((err / tol).max())


# ------------------------------------------------------------------ fused GELU + quantize
# The library evaluates GELU-tanh in fp32 (gelu.cuh) and rounds it to bf16; the oracle takes
# the definition in fp64 and rounds that.  The library states the bound
#   |gelu_f32(z) - gelu(z)| <= (2 |a| + 16) 2^-23 |gelu(z)| + 2^-126,  a = -2 sqrt(2/pi) (z + 0.044715 z^3)
# and returns a zero of z's sign once a / ln2 > 125; test_gelu_f32_error_bound checks that bound
# on the GPU for every finite bf16 z.  Its h may therefore be any bf16 between the roundings of
# the bound's two ends; the checks below accept exactly those values.
def _ordered(bits):
    """bf16 bits -> integers in value order (+0 and -0 both 0)."""
    b = np.asarray(bits).astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def _from_ordered(o):
    o = np.asarray(o).astype(np.int32)
    return np.where(o < 0, 0x8000 | (-o), o).astype(np.uint16)


def _bf16_f64(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


def gelu_error_bound(zf):
    """The library's stated bound on its fp32 GELU at the (exact) inputs zf, and whether the
    input is past its cut-off (a / ln2 > 125, where it returns a signed zero)."""
    from oracle import oracle_np as onp

    zf = np.asarray(zf, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        a = 2.0 * np.sqrt(2.0 / np.pi) * (zf + 0.044715 * zf ** 3) * -1.0
        g = onp.gelu_f64(zf)
        e = (2.0 * np.abs(a) + 16.0) * 2.0 ** -23 * np.abs(g) + 2.0 ** -126
    cut = a / np.log(2.0) > 124.99
    return g, e, cut


_TAB = None


def _gelu_h_tables():
    """Over the ordered bf16 domain o in [-32767, 32767] (index o + 32767): the smallest and
    largest bf16 value of h the library may return for input z(o), and sparse tables for
    range minima / maxima over runs of consecutive z."""
    global _TAB
    if _TAB is None:
        from oracle import oracle_np as onp

        o = np.arange(-32767, 32768)
        zb = _from_ordered(o)
        fin = ((zb >> 7) & 0xFF) != 0xFF
        zf0 = np.where(fin, _bf16_f64(np.where(fin, zb, 0)), 0.0)
        g, e, cut = gelu_error_bound(zf0)
        lo = np.where(cut, np.minimum(g - e, 0.0), g - e)
        hi = np.where(cut, np.maximum(g + e, 0.0), g + e)
        with np.errstate(over="ignore"):
            h_lo = _bf16_f64(onp.f64_to_bf16_rn(lo))
            h_hi = _bf16_f64(onp.f64_to_bf16_rn(hi))
        h_lo = np.where(fin, h_lo, -np.inf)
        h_hi = np.where(fin, h_hi, np.inf)
        mins, maxs = [h_lo], [h_hi]
        k = 1
        while k < h_lo.size:
            pm, px = mins[-1], maxs[-1]
            mins.append(np.minimum(pm[:-k], pm[k:]))
            maxs.append(np.maximum(px[:-k], px[k:]))
            k *= 2
        _TAB = (mins, maxs)
    return _TAB


def gelu_h_interval(z_lo_bits, z_hi_bits):
    """For brackets [z_lo, z_hi] of bf16 inputs (bits, z_lo <= z_hi in value): the smallest and
    largest h the library may return for any z in the bracket."""
    mins, maxs = _gelu_h_tables()
    l = _ordered(z_lo_bits) + 32767
    r = _ordered(z_hi_bits) + 32767
    n = r - l + 1
    assert np.all(n >= 1)
    k = np.floor(np.log2(n)).astype(np.int64)
    hmin = np.empty(l.shape)
    hmax = np.empty(l.shape)
    for kk in np.unique(k):
        m = k == kk
        w = 1 << int(kk)
        hmin[m] = np.minimum(mins[kk][l[m]], mins[kk][r[m] - w + 1])
        hmax[m] = np.maximum(maxs[kk][l[m]], maxs[kk][r[m] - w + 1])
    return hmin, hmax


def _bf16_bracket(v):
    """(largest bf16 <= v, smallest bf16 >= v) as bf16 bits, for finite float64 v."""
    t = (np.asarray(v, dtype=np.float64).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    o = _ordered(t)
    lo_v = np.full(v.shape, -np.inf)
    hi_v = np.full(v.shape, np.inf)
    lo_b = np.zeros(v.shape, dtype=np.uint16)
    hi_b = np.zeros(v.shape, dtype=np.uint16)
    for d in (-2, -1, 0, 1, 2):
        b = _from_ordered(o + d)
        val = _bf16_f64(b)
        m = (val <= v) & (val > lo_v)
        lo_v, lo_b = np.where(m, val, lo_v), np.where(m, b, lo_b)
        m = (val >= v) & (val < hi_v)
        hi_v, hi_b = np.where(m, val, hi_v), np.where(m, b, hi_b)
    return lo_b, hi_b


def check_quant_of_interval(fmt, codes, sf_rows, hmin, hmax, g_h, what, row_ids=None):
    """Codes [R, N/2] and scale bytes [R, N/G] (unswizzled) of R rows are admissible for some h
    with hmin <= h <= hmax element-wise: each group's scale byte lies between the scales of the
    smallest and largest admissible group amax, and each code lies, given that scale, between
    the codes of hmin and hmax."""
    from oracle import oracle_np as onp

    G = 32 if fmt == oracle.MX else 16
    R, N = hmin.shape
    mag_lo = np.where((hmin <= 0) & (hmax >= 0), 0.0, np.minimum(np.abs(hmin), np.abs(hmax)))
    mag_hi = np.maximum(np.abs(hmin), np.abs(hmax))
    a_lo = mag_lo.reshape(R, N // G, G).max(-1)
    a_hi = mag_hi.reshape(R, N // G, G).max(-1)
    sf = sf_rows.astype(np.int64)
    rid = np.arange(R) if row_ids is None else np.asarray(row_ids)

    def scaled(h, per_group):
        return (h.reshape(R, N // G, G) * per_group[..., None]).reshape(R, N)

    if fmt == oracle.MX:
        def byte(a):
            _, e = np.frexp(np.where(a > 0, a, 1.0))
            return np.where(a > 0, np.clip(e - 1 - 2 + 127, 0, 254), 0)
        b_lo, b_hi = byte(a_lo), byte(a_hi)
        inv = np.ldexp(1.0, (127 - sf).astype(np.int64))           # exact powers of two
        s_lo = scaled(hmin, inv).astype(np.float32)
        s_hi = scaled(hmax, inv).astype(np.float32)
        zero = np.zeros((R, N), dtype=bool)
    else:
        six_g = np.float32(6.0) * np.float32(g_h)
        b_lo = onp.e4m3_encode(a_lo.astype(np.float32) / six_g).astype(np.int64)
        b_hi = onp.e4m3_encode(a_hi.astype(np.float32) / six_g).astype(np.int64)
        d = onp.e4m3_decode(sf).astype(np.float32) * np.float32(g_h)
        r = np.where(d != 0, np.float32(1.0) / np.where(d != 0, d, np.float32(1.0)), np.float32(0.0)).astype(np.float32)
        s_lo = (hmin.astype(np.float32).reshape(R, N // G, G) * r[..., None]).reshape(R, N)
        s_hi = (hmax.astype(np.float32).reshape(R, N // G, G) * r[..., None]).reshape(R, N)
        zero = np.repeat(d == 0, G, axis=1)
    bad_sf = (sf < b_lo) | (sf > b_hi)
    if bad_sf.any():
        i = tuple(np.argwhere(bad_sf)[0])
        raise AssertionError(f"{what}: {bad_sf.sum()} scale bytes outside their admissible range; first at row "
                             f"{rid[i[0]]} group {i[1]}: byte {sf[i]} range [{b_lo[i]}, {b_hi[i]}]")
    q = onp.e2m1_decode(onp.unpack_nibbles(codes))
    q_lo = np.where(zero, 0.0, onp.e2m1_decode(onp.e2m1_encode(s_lo)))
    q_hi = np.where(zero, 0.0, onp.e2m1_decode(onp.e2m1_encode(s_hi)))
    bad = (q < q_lo) | (q > q_hi)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} / {bad.size} codes outside their admissible range; first at "
                             f"row {rid[i[0]]} col {i[1]}: code value {q[i]} range [{q_lo[i]}, {q_hi[i]}]")


def check_gelu_quant(fmt, codes_dev, sf_dev, Y_ref, S, rows, M, N, g_h, what):
    """Validity of the fused up-projection output h = quant(bf16(gelu(z))), z the bf16 GEMM
    result.  z is only known to the GEMM tolerance (|z - Y| <= ulp_bf16(Y) + 1e-5 S), so for
    every element the admissible bf16 z form a bracket, mapped through the library's GELU
    bound (gelu_h_interval) to an interval [h_min, h_max]; the codes and scales must be
    admissible for it (check_quant_of_interval).  Padding rows' scale bytes must be zero.
    Returns the fraction of codes equal to the oracle's quantization of bf16(gelu(bf16(Y)))."""
    from oracle import oracle_np as onp

    G = 32 if fmt == oracle.MX else 16
    T = oracle.tolerance(Y_ref, S)
    zl = _bf16_bracket(Y_ref - T)[1]
    zh = _bf16_bracket(Y_ref + T)[0]
    hmin, hmax = gelu_h_interval(zl, zh)
    R = len(rows)
    Mpad = -(-M // 128) * 128
    sf_all = onp.unswizzle_sf(host_u8(sf_dev), Mpad, N // G)
    assert np.all(sf_all[M:] == 0), f"{what}: nonzero scale bytes in padding rows"
    codes = host_u8(codes_dev)[rows]
    check_quant_of_interval(fmt, codes, sf_all[rows], hmin, hmax, g_h, what, row_ids=rows)
    # agreement with the oracle's own choice z = bf16(Y)
    zb = _bf16_bracket(Y_ref)
    zn = np.where(np.abs(_bf16_f64(zb[0]) - Y_ref) <= np.abs(_bf16_f64(zb[1]) - Y_ref), zb[0], zb[1])
    c_ref, _ = oracle.gelu_quantize(fmt, zn.reshape(R, N), g_h)
    return float((onp.unpack_nibbles(c_ref) == onp.unpack_nibbles(codes)).mean())


def check_gelu_quant_exact(fmt, codes_dev, sf_dev, z_bits, g_h, what, chunk=4096):
    """fp4_gelu_quantize_act of an exactly known bf16 z [M, K]: rows whose codes and scale bytes
    equal the oracle's (bf16(gelu_f64(z)) quantized) pass at once; every other row must be
    admissible for the library's GELU bound (check_quant_of_interval).  Padding rows' scale
    bytes must be zero.  Returns the fraction of rows that differ from the oracle."""
    from oracle import oracle_np as onp

    M, K = z_bits.shape
    G = 32 if fmt == oracle.MX else 16
    Mpad = -(-M // 128) * 128
    codes = host_u8(codes_dev).reshape(M, K // 2)
    sf_all = onp.unswizzle_sf(host_u8(sf_dev), Mpad, K // G)
    assert np.all(sf_all[M:] == 0), f"{what}: nonzero scale bytes in padding rows"
    differ = 0
    for r0 in range(0, M, chunk):
        r1 = min(M, r0 + chunk)
        c_ref, s_ref = oracle.gelu_quantize(fmt, z_bits[r0:r1], g_h)
        s_ref = onp.unswizzle_sf(s_ref, r1 - r0, K // G)
        bad = np.nonzero((c_ref != codes[r0:r1]).any(1) | (s_ref != sf_all[r0:r1]).any(1))[0]
        if bad.size:
            differ += bad.size
            zb = z_bits[r0 + bad]
            hmin, hmax = gelu_h_interval(zb, zb)
            check_quant_of_interval(fmt, codes[r0 + bad], sf_all[r0 + bad], hmin, hmax, g_h, what,
                                    row_ids=r0 + bad)
    return differ / M
