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
def _ordered(bits):
    """bf16 bits -> integers in value order (+0 and -0 both 0)."""
    b = np.asarray(bits).astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def _from_ordered(o):
    o = np.asarray(o).astype(np.int32)
    return np.where(o < 0, 0x8000 | (-o), o).astype(np.uint16)


def _bf16_f64(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


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


def check_gelu_quant(fmt, codes_dev, sf_dev, Y_ref, S, rows, M, N, g_h, what):
    """Validity of the fused up-projection output h = quant(bf16(gelu(z))), z the bf16 GEMM
    result.  z is only known to the GEMM tolerance (|z - Y| <= ulp_bf16(Y) + 1e-5 S), so
    for every element the oracle brackets the admissible bf16 z, maps the bracket through
    the oracle's bf16 GELU (monotone on each side of its minimum near z = -0.752, whose
    value is included when the bracket straddles it) to an interval [h_min, h_max], and
    requires: each group's scale byte lies between the scales of the smallest and largest
    admissible group amax, and each code lies, given the GPU's own scale, between the codes
    of h_min and h_max.  Padding rows' scale bytes must be zero.  Returns the fraction of
    codes equal to the quantization of the oracle's own bf16(gelu(bf16(Y)))."""
    from oracle import oracle_np as onp

    G = 32 if fmt == oracle.MX else 16
    T = oracle.tolerance(Y_ref, S)
    zl = _bf16_bracket(Y_ref - T)[1]
    zh = _bf16_bracket(Y_ref + T)[0]
    hl = _bf16_f64(oracle.gelu_bf16(zl))
    hh = _bf16_f64(oracle.gelu_bf16(zh))
    hmin, hmax = np.minimum(hl, hh), np.maximum(hl, hh)
    # the bf16 GELU's minimum region
    o0, o1 = _ordered(_bf16_bracket(np.array([-0.80]))[0])[0], _ordered(_bf16_bracket(np.array([-0.70]))[1])[0]
    zt_b = _from_ordered(np.arange(o0, o1 + 1))
    zt, ht = _bf16_f64(zt_b), _bf16_f64(oracle.gelu_bf16(zt_b))
    zlv, zhv = _bf16_f64(zl), _bf16_f64(zh)
    span = (zlv <= zt.max()) & (zhv >= zt.min())
    if span.any():
        idx = np.nonzero(span)
        inside = (zt[None, :] >= zlv[idx][:, None]) & (zt[None, :] <= zhv[idx][:, None])
        hm = np.where(inside, ht[None, :], np.inf).min(axis=1)
        hmin[idx] = np.minimum(hmin[idx], hm)
    mag_lo = np.where((hmin <= 0) & (hmax >= 0), 0.0, np.minimum(np.abs(hmin), np.abs(hmax)))
    mag_hi = np.maximum(np.abs(hmin), np.abs(hmax))
    R = len(rows)
    a_lo = mag_lo.reshape(R, N // G, G).max(-1)
    a_hi = mag_hi.reshape(R, N // G, G).max(-1)
    Mpad = -(-M // 128) * 128
    sf_all = onp.unswizzle_sf(host_u8(sf_dev), Mpad, N // G)
    assert np.all(sf_all[M:] == 0), f"{what}: nonzero scale bytes in padding rows"
    sf = sf_all[rows].astype(np.int64)

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
    assert not bad_sf.any(), (f"{what}: {bad_sf.sum()} scale bytes outside their admissible range; first "
                              f"{np.argwhere(bad_sf)[0]}")
    codes = onp.unpack_nibbles(host_u8(codes_dev)[rows])
    q = onp.e2m1_decode(codes)
    q_lo = np.where(zero, 0.0, onp.e2m1_decode(onp.e2m1_encode(s_lo)))
    q_hi = np.where(zero, 0.0, onp.e2m1_decode(onp.e2m1_encode(s_hi)))
    bad = (q < q_lo) | (q > q_hi)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} / {bad.size} codes outside their admissible range; first at "
                             f"row {rows[i[0]]} col {i[1]}: code value {q[i]} range [{q_lo[i]}, {q_hi[i]}]")
    # agreement with the oracle's own choice z = bf16(Y)
    zb = _bf16_bracket(Y_ref)
    zn = np.where(np.abs(_bf16_f64(zb[0]) - Y_ref) <= np.abs(_bf16_f64(zb[1]) - Y_ref), zb[0], zb[1])
    c_ref, _ = oracle.gelu_quantize(fmt, zn.reshape(R, N), g_h)
    return float((onp.unpack_nibbles(c_ref) == codes).mean())
