"""Independent NumPy oracle for tiny shapes (cross-check of the C oracle).

TEST INFRASTRUCTURE ONLY: imported by the test suite and nothing else.

It restates the same definitions (MXFP4 / NVFP4 / MXFP8 quantization and the fp64
linear) with different algorithms from the C oracle, so a slip in one does not
repeat in the other:
  * E2M1 and E4M3 rounding use arithmetic round-half-to-even (np.rint) on the
    grid spacing of each binade, instead of a nearest-value scan.
  * The scale-factor swizzle is built by reshaping and transposing the [rows, K/G]
    scale matrix into 128x4 atoms, instead of a closed-form offset.
  * The GEMM is a library matmul in float64.
  * GELU-tanh goes through logaddexp, and bf16 rounding picks the nearer of two
    neighbouring codes, instead of the C oracle's tanh / exp split and rint.

Sources: MXFP4 format (Wan2.2-I2V-A14B-Lightning MXFP4 card, Quantization
Details); NVFP4 format (Wan2.2-T2V-A14B NVFP4 card, Model Details); W4A8 SVDQuant
(wan2.2-ti2v-w4a8-svd README).  Readings R1-R7 are the same as in fp4_oracle.c.
"""
from __future__ import annotations

import numpy as np

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def bf16_to_f32(b):
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------- E2M1 ------------
def e2m1_round(a):
    """|v| (float64 array) -> nearest E2M1 magnitude, RNE, saturating at 6."""
    a = np.asarray(a, dtype=np.float64)
    # spacing: 0.5 below 2 (covers the subnormal 0.5 and the [1,2) binade), 1 in [2,4), 2 in [4,8)
    step = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    q = np.rint(a / step) * step          # np.rint rounds half to even
    return np.minimum(q, 6.0)


def e2m1_encode(v):
    v = np.asarray(v, dtype=np.float32)
    mag = e2m1_round(np.abs(v.astype(np.float64)))
    idx = np.searchsorted(E2M1_VALUES, mag)
    assert np.all(E2M1_VALUES[idx] == mag)
    return (np.signbit(v).astype(np.uint8) << 3) | idx.astype(np.uint8)


def e2m1_decode(c):
    c = np.asarray(c, dtype=np.uint8)
    m = E2M1_VALUES[c & 7]
    return np.where(c & 8, -m, m)


# ---------------------------------------------------------------- E4M3 ------------
def e4m3_decode(b):
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    s, e, m = (b >> 7) & 1, (b >> 3) & 15, b & 7
    v = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return np.where(s == 1, -v, v)


def e4m3_encode(v):
    """fp32 -> E4M3 byte: RNE on the binade's 3-bit mantissa grid, saturate to 448."""
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v.astype(np.float64))
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    E = np.maximum(ex - 1, -6)            # below 2^-6 the grid is the subnormal one
    step = 2.0 ** (E - 3.0)
    q = np.minimum(np.rint(a / step) * step, 448.0)
    # back to a code: exponent field and mantissa of q
    _, qex = np.frexp(np.where(q > 0, q, 1.0))
    qE = qex - 1
    normal = (q >= 2.0 ** -6)
    efield = np.where(normal, qE + 7, 0)
    mant = np.where(normal, q / 2.0 ** qE - 1.0, q / 2.0 ** -6) * 8.0
    assert np.all(mant == np.round(mant))
    code = (efield.astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(q == 0, 0, code)
    return ((np.signbit(v).astype(np.int64) << 7) | code).astype(np.uint8)


def e8m0_decode(b):
    return 2.0 ** (np.asarray(b, dtype=np.float64) - 127.0)


# ---------------------------------------------------------------- layouts ---------
def pack_nibbles(codes):
    """[rows, K] 4-bit codes -> [rows, K/2] bytes, even k in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 15
    out[:, 1::2] = packed >> 4
    return out


def swizzle_sf(sfm):
    """[rows, Kg] scale bytes -> flat buffer of 128-row x 4-group atoms (rows padded)."""
    rows, Kg = sfm.shape
    rp = -(-rows // 128) * 128
    pad = np.zeros((rp, Kg), dtype=np.uint8)
    pad[:rows] = sfm
    # row r = rb*128 + rg*32 + r32 ; group j = kb*4 + jj
    t = pad.reshape(rp // 128, 4, 32, Kg // 4, 4)          # (rb, rg, r32, kb, jj)
    t = t.transpose(0, 3, 2, 1, 4)                          # (rb, kb, r32, rg, jj)
    return np.ascontiguousarray(t).reshape(-1)


def unswizzle_sf(flat, rows, Kg):
    rp = -(-rows // 128) * 128
    t = np.asarray(flat, dtype=np.uint8).reshape(rp // 128, Kg // 4, 32, 4, 4)
    t = t.transpose(0, 3, 2, 1, 4).reshape(rp, Kg)
    return t[:rows]


# ---------------------------------------------------------------- quantizers ------
def _groups(x_bf16, G):
    x = bf16_to_f32(x_bf16)
    rows, K = x.shape
    return x, x.reshape(rows, K // G, G)


def quant_mxfp4(x_bf16):
    x, xg = _groups(x_bf16, 32)
    amax = np.abs(xg).max(axis=2).astype(np.float64)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))
    e = np.where(amax > 0, ex - 1 - 2, -127)
    e = np.clip(e, -127, 127)
    q = (xg.astype(np.float64) * 2.0 ** (-e[:, :, None])).astype(np.float32)
    codes = e2m1_encode(q).reshape(x.shape)
    return pack_nibbles(codes), swizzle_sf((e + 127).astype(np.uint8))


def quant_mxfp8(x_bf16):
    x, xg = _groups(x_bf16, 32)
    amax = np.abs(xg).max(axis=2).astype(np.float64)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))
    e = np.clip(np.where(amax > 0, ex - 1 - 8, -127), -127, 127)
    q = (xg.astype(np.float64) * 2.0 ** (-e[:, :, None])).astype(np.float32)
    return e4m3_encode(q).reshape(x.shape), swizzle_sf((e + 127).astype(np.uint8))


def nv_global(T):
    T = np.float32(T)
    return np.float32(1.0) if T == 0 else np.float32(T / np.float32(2688.0))


def quant_nvfp4(x_bf16, g):
    g = np.float32(g)
    x, xg = _groups(x_bf16, 16)
    amax = np.abs(xg).max(axis=2)                              # float32
    s = (amax / (np.float32(6.0) * g)).astype(np.float32)
    sf = e4m3_encode(s)
    d = (e4m3_decode(sf).astype(np.float32) * g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (np.float32(1.0) / d).astype(np.float32)
        q = (xg * r[:, :, None]).astype(np.float32)
    codes = np.where(d[:, :, None] == 0, np.uint8(0), e2m1_encode(np.where(d[:, :, None] == 0, 0, q)))
    return pack_nibbles(codes.reshape(x.shape)), swizzle_sf(sf)


# ---------------------------------------------------------------- GELU-tanh (R10) --
def gelu_f64(z):
    """gelu(z) = 0.5 z (1 + tanh(v)), v = sqrt(2/pi) (z + 0.044715 z^3), written as
    z / (1 + e^{-2v}) = z exp(-log(1 + e^{-2v})) with logaddexp (no cancellation for
    either sign of v): a different route from the C oracle's tanh/exp split."""
    z = np.asarray(z, dtype=np.float64)
    v = np.sqrt(2.0 / np.pi) * (z + 0.044715 * z ** 3)
    return z * np.exp(-np.logaddexp(0.0, -2.0 * v))


def f64_to_bf16_rn(x):
    """Nearest bf16 (ties to the even code) to each finite double: take the two bf16
    neighbours of x from its fp32 bits (truncation and the next code up) and keep the
    closer one.  The differences are exact (Sterbenz), so the choice is exact."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    t = (a.astype(np.float32).view(np.uint32) >> 16).astype(np.int64)
    # a.astype(float32) may have rounded up past a: step down while the candidate exceeds a
    lo = t.copy()
    for _ in range(2):
        lo = np.where(bf16_to_f32(lo.astype(np.uint16)).astype(np.float64) > a, lo - 1, lo)
    hi = lo + 1
    vlo = bf16_to_f32(lo.astype(np.uint16)).astype(np.float64)
    vhi = bf16_to_f32(np.minimum(hi, 0x7F80).astype(np.uint16)).astype(np.float64)
    dlo, dhi = a - vlo, vhi - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (lo % 2 == 1))
    mag = np.where(a == 0, 0, np.where(pick_hi, hi, lo))
    return (mag | (np.signbit(x).astype(np.int64) << 15)).astype(np.uint16)


# ---------------------------------------------------------------- dequant + GEMM --
def dequant_fp4(fmt, codes, sf_flat, rows, K, g=1.0):
    G = 32 if fmt == "mx" else 16
    c = unpack_nibbles(codes)
    sfm = unswizzle_sf(sf_flat, rows, K // G)
    scale = e8m0_decode(sfm) if fmt == "mx" else e4m3_decode(sfm) * float(g)
    return e2m1_decode(c) * np.repeat(scale, G, axis=1)


def dequant_mxfp8(elems, sf_flat, rows, K):
    sfm = unswizzle_sf(sf_flat, rows, K // 32)
    return e4m3_decode(elems) * np.repeat(e8m0_decode(sfm), 32, axis=1)


def linear_fp64(a_deq, w_deq, bias_f16=None):
    y = a_deq @ w_deq.T
    s = np.abs(a_deq) @ np.abs(w_deq).T
    if bias_f16 is not None:
        y = y + np.asarray(bias_f16, dtype=np.uint16).view(np.float16).astype(np.float64)[None, :]
    return y, s
