"""CPU oracle for the block-scaled FP4 quantized linear.

TEST INFRASTRUCTURE ONLY.  The test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only users; the CUDA library never loads it.

`fp4_oracle.c` is the oracle proper (plain C, fp32 steps as IEEE operations where the
format fixes them, fp64 GELU and GEMM, OpenMP over rows).  This module builds it with gcc and exposes it through
ctypes with numpy arrays.  `oracle_np.py` is an independent NumPy restatement used
to cross-check it on tiny shapes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

MX, NV = 0, 1


def build(force: bool = False) -> str:
    """Compile fp4_oracle.c into liboracle.so (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                               "-shared", "-fPIC", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I64, F, D, U8, U16 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_double,
                                  ctypes.c_uint8, ctypes.c_uint16)
        sig = {
            "orc_e2m1_decode": (D, [U8]), "orc_e2m1_encode": (U8, [F]),
            "orc_e4m3_decode": (D, [U8]), "orc_e4m3_encode": (U8, [F]),
            "orc_e8m0_decode": (D, [U8]), "orc_bf16_to_f32": (F, [U16]),
            "orc_f16_to_double": (D, [U16]),
            "orc_sf_offset": (I64, [I64, I64, I64]), "orc_sf_bytes": (I64, [I64, I64]),
            "orc_tensor_amax": (F, [P, I64]), "orc_nv_global": (F, [F]),
            "orc_quant_mxfp4": (None, [P, I64, I64, P, P]),
            "orc_quant_nvfp4": (None, [P, I64, I64, F, P, P]),
            "orc_quant_mxfp8": (None, [P, I64, I64, P, P]),
            "orc_dequant_fp4": (None, [ctypes.c_int, P, P, I64, D, P, I64, P]),
            "orc_dequant_mxfp8": (None, [P, P, I64, P, I64, P]),
            "orc_linear_fp64": (None, [P, I64, P, I64, I64, P, P, P]),
            "orc_lowrank_fp64": (None, [P, I64, P, I64, P, P, I64, I64, P, P]),
            "orc_num_threads": (ctypes.c_int, []),
            "orc_gelu_f64": (D, [D]), "orc_f64_to_bf16_rn": (U16, [D]),
            "orc_gelu_bf16": (None, [P, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------------------- codecs
def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(float(v))


def e2m1_decode(c: int) -> float:
    return lib().orc_e2m1_decode(int(c))


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(float(v))


def e4m3_decode(b: int) -> float:
    return lib().orc_e4m3_decode(int(b))


def e8m0_decode(b: int) -> float:
    return lib().orc_e8m0_decode(int(b))


def sf_offset(r: int, j: int, Kg: int) -> int:
    return lib().orc_sf_offset(r, j, Kg)


def sf_bytes(rows: int, Kg: int) -> int:
    return lib().orc_sf_bytes(rows, Kg)


def group_size(fmt: int) -> int:
    return 32 if fmt == MX else 16


# ----------------------------------------------------------------------------- quantizers
def tensor_amax(x_bf16: np.ndarray) -> float:
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    return lib().orc_tensor_amax(_p(x), x.size)


def nv_global(T: float) -> float:
    return lib().orc_nv_global(float(T))


def quantize(fmt: int, x_bf16: np.ndarray, g: float | None = None):
    """bf16 [rows, K] -> (codes [rows, K/2] uint8, sf flat uint8) in format fmt."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, K = x.shape
    G = group_size(fmt)
    codes = np.zeros((rows, K // 2), dtype=np.uint8)
    sf = np.zeros(sf_bytes(rows, K // G), dtype=np.uint8)
    if fmt == MX:
        lib().orc_quant_mxfp4(_p(x), rows, K, _p(codes), _p(sf))
    else:
        lib().orc_quant_nvfp4(_p(x), rows, K, float(g), _p(codes), _p(sf))
    return codes, sf


def gelu_f64(z: float) -> float:
    """Plain GELU-tanh definition in fp64 (R10)."""
    return lib().orc_gelu_f64(float(z))


def f64_to_bf16_rn(x: float) -> int:
    """Bits of the bf16 nearest to the double x (ties to even, subnormals kept)."""
    return int(lib().orc_f64_to_bf16_rn(float(x)))


def gelu_bf16(z_bf16: np.ndarray) -> np.ndarray:
    """h = bf16_rn(gelu(z)) element-wise, gelu in fp64; bf16 bits in and out (R10)."""
    z = np.ascontiguousarray(z_bf16, dtype=np.uint16)
    h = np.zeros_like(z)
    lib().orc_gelu_bf16(_p(z), z.size, _p(h))
    return h


def gelu_quantize(fmt: int, z_bf16: np.ndarray, g: float | None = None):
    """The down projection's input from the bf16 up-projection output z: GELU-tanh,
    bf16 rounding, then the format's quantizer (R10 then c-3 / c-4)."""
    return quantize(fmt, gelu_bf16(z_bf16), g)


def quantize_mxfp8(x_bf16: np.ndarray):
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, K = x.shape
    elems = np.zeros((rows, K), dtype=np.uint8)
    sf = np.zeros(sf_bytes(rows, K // 32), dtype=np.uint8)
    lib().orc_quant_mxfp8(_p(x), rows, K, _p(elems), _p(sf))
    return elems, sf


def pack_weight(fmt: int, w_bf16: np.ndarray):
    """Offline weight pack: (codes, sf, global).  NVFP4 global from the tensor amax."""
    if fmt == MX:
        c, s = quantize(MX, w_bf16)
        return c, s, None
    g = nv_global(tensor_amax(w_bf16))
    c, s = quantize(NV, w_bf16, g)
    return c, s, g


# ----------------------------------------------------------------------------- dequant
def dequant_fp4(fmt: int, codes, sf, K: int, g: float = 1.0, rows=None) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    ids = np.arange(codes.shape[0], dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((ids.size, K), dtype=np.float64)
    lib().orc_dequant_fp4(fmt, _p(codes), _p(sf), K, float(g), _p(ids), ids.size, _p(out))
    return out


def dequant_mxfp8(elems, sf, K: int, rows=None) -> np.ndarray:
    elems = np.ascontiguousarray(elems, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    ids = np.arange(elems.shape[0], dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((ids.size, K), dtype=np.float64)
    lib().orc_dequant_mxfp8(_p(elems), _p(sf), K, _p(ids), ids.size, _p(out))
    return out


def linear_fp64(a_deq: np.ndarray, w_deq: np.ndarray, bias_f16=None):
    """(Y, S): Y = a w^T + bias in fp64, S = |a| |w|^T."""
    a = np.ascontiguousarray(a_deq, dtype=np.float64)
    w = np.ascontiguousarray(w_deq, dtype=np.float64)
    nrows, K = a.shape
    N = w.shape[0]
    Y = np.empty((nrows, N), dtype=np.float64)
    S = np.empty((nrows, N), dtype=np.float64)
    b = None if bias_f16 is None else np.ascontiguousarray(bias_f16, dtype=np.uint16)
    lib().orc_linear_fp64(_p(a), nrows, _p(w), N, K, None if b is None else _p(b), _p(Y), _p(S))
    return Y, S


def lowrank_fp64(x_bf16, rows, l1_bf16, l2_bf16):
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    l1 = np.ascontiguousarray(l1_bf16, dtype=np.uint16)
    l2 = np.ascontiguousarray(l2_bf16, dtype=np.uint16)
    ids = np.ascontiguousarray(rows, dtype=np.int64)
    K, rank = l1.shape
    N = l2.shape[1]
    assert rank <= 256
    LR = np.empty((ids.size, N), dtype=np.float64)
    LS = np.empty((ids.size, N), dtype=np.float64)
    lib().orc_lowrank_fp64(_p(x), K, _p(ids), ids.size, _p(l1), _p(l2), rank, N, _p(LR), _p(LS))
    return LR, LS


def fp4_linear_rows(fmt, x_bf16, w_bf16, bias_f16, rows, g_a=None, packed_w=None):
    """End-to-end oracle of the W4A4 linear for selected rows of x.

    Returns (Y, S) in fp64.  For NVFP4, g_a is the static activation global."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    K = x.shape[1]
    wc, ws, gw = packed_w if packed_w is not None else pack_weight(fmt, w_bf16)
    xs = np.ascontiguousarray(x[np.asarray(rows)])
    ac, asf = quantize(fmt, xs, g_a)
    a = dequant_fp4(fmt, ac, asf, K, 1.0 if fmt == MX else g_a)
    w = dequant_fp4(fmt, wc, ws, K, 1.0 if fmt == MX else gw)
    return linear_fp64(a, w, bias_f16)


def svd_linear_rows(act: str, x_bf16, r_packed, l1_bf16, l2_bf16, bias_f16, rows):
    """End-to-end oracle of the SVDQuant linear (W4A8 README) for selected rows of x:
    the activations quantized dynamically (act = "mxfp8" for W4A8, "mxfp4" for the W4A4
    variant) and dequantized, times the dequantized MXFP4 residual r_packed = (codes, sf)
    in fp64, plus the low-rank term (x L1) L2 on the unquantized x (R7) and the bias.
    Returns (Y, S): S sums |a_k r_k| and |u_r L2[r, n]| for the tolerance."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    K = x.shape[1]
    rows = np.asarray(rows)
    xs = np.ascontiguousarray(x[rows])
    if act == "mxfp8":
        e, sf = quantize_mxfp8(xs)
        a = dequant_mxfp8(e, sf, K)
    elif act == "mxfp4":
        c, sf = quantize(MX, xs)
        a = dequant_fp4(MX, c, sf, K)
    else:
        raise ValueError(act)
    rc, rs = r_packed
    w = dequant_fp4(MX, rc, rs, K)
    Y, S = linear_fp64(a, w, bias_f16)
    LR, LS = lowrank_fp64(x, rows, l1_bf16, l2_bf16)
    return Y + LR, S + LS


# ----------------------------------------------------------------------------- FP4 attention operands
# Wan2.2-Animate-14B MXFP4 card, "Results": SageAttention v3 is Blackwell microscaling FP4
# attention.  The card gives no algorithm; the reading followed here quantizes Q and K per
# token and head in blocks of G along head_dim with the activation rules above (a head of
# D = 128 is a whole number of groups, so no group spans two heads) and takes the scores
# of one head as the fp64 product of the dequantized operands.
def quantize_heads(fmt: int, x_bf16: np.ndarray, H: int, g: float | None = None):
    """bf16 [T, H*128] -> head-major (codes [H, Tpad, 64] uint8, sf [H, sf_bytes(Tpad, 128/G)]):
    head h is `quantize` of columns h*128 .. h*128+127, its codes padded with zero rows."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, HD = x.shape
    D = HD // H
    assert D * H == HD and D == 128
    Tpad = (T + 127) // 128 * 128
    codes = np.zeros((H, Tpad, D // 2), dtype=np.uint8)
    sfs = np.zeros((H, sf_bytes(Tpad, D // group_size(fmt))), dtype=np.uint8)
    for h in range(H):
        c, s = quantize(fmt, np.ascontiguousarray(x[:, h * D:(h + 1) * D]), g)
        codes[h, :T] = c
        sfs[h] = s
    return codes, sfs


def attn_scores_rows(fmt: int, q_heads, k_heads, head: int, rows, g_q: float | None = None,
                     g_k: float | None = None):
    """(Y, S) of rows `rows` of head `head`'s scores: Y[i, j] = sum_d deq(q)[i, d] deq(k)[j, d]
    over every key row j of the head-major buffers (padding keys give 0), in fp64;
    S = sum_d |deq(q) deq(k)| for the tolerance."""
    qc, qs = q_heads
    kc, ks = k_heads
    D = 2 * qc.shape[2]
    a = dequant_fp4(fmt, qc[head], qs[head], D, 1.0 if fmt == MX else g_q, rows=rows)
    w = dequant_fp4(fmt, kc[head], ks[head], D, 1.0 if fmt == MX else g_k)
    return linear_fp64(a, w, None)


def quantize_heads_vt(x_bf16: np.ndarray, H: int, fmt: int = MX, g: float | None = None):
    """V bf16 [T, H*128] -> head-major V^T (codes [H, 128, Tpad/2], sf [H, sf_bytes(128, Tpad/G)]):
    head h is `quantize` of the [128, Tpad] matrix whose column t is token t of the head
    (tokens >= T zero), i.e. the scales run along the tokens, the GEMM's K of P V (NVFP4
    under V's global g)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, HD = x.shape
    D = HD // H
    assert D * H == HD and D == 128
    Tpad = (T + 127) // 128 * 128
    codes = np.zeros((H, D, Tpad // 2), dtype=np.uint8)
    sfs = np.zeros((H, sf_bytes(D, Tpad // group_size(fmt))), dtype=np.uint8)
    for h in range(H):
        vt = np.zeros((D, Tpad), dtype=np.uint16)
        vt[:, :T] = x[:, h * D:(h + 1) * D].T
        codes[h], sfs[h] = quantize(fmt, vt, g)
    return codes, sfs


LOG2E = 1.4426950408889634


def softmax_c(scale: float) -> float:
    """The exponent multiplier as the library states it: c = fp32(scale * log2 e)."""
    return float(np.float32(scale * LOG2E))


def softmax_weights(s_bf16, T_kv: int, scale: float):
    """Unnormalized softmax weights of bf16 scores [R, T_kv_pad] over the first T_kv keys, in
    fp64: p~_j = 2^(s_j c - max_k s_k c) with c = softmax_c(scale) (the largest is 1), keys >=
    T_kv 0.  Returns (p~, l, t_max_abs): l[r] = sum_j p~_j, t_max_abs[r] = max_j |s_j c| (for
    the error bounds)."""
    s = synth_bits_to_f64(s_bf16)
    c = softmax_c(scale)
    u = s[:, :T_kv] * c
    m = u.max(axis=1, keepdims=True)
    p = np.zeros_like(s)
    p[:, :T_kv] = np.exp2(u - m)
    return p, p.sum(axis=1), np.abs(u).max(axis=1)


def softmax_weight_bound(t_max_abs):
    """Relative bound on the library's fp32 p~ (per row): the two roundings of fl(fl(s c) - m)
    (terms up to 2 max|s c|, through 2^t: ln2 * 4 max|s c| 2^-24) and exp2f within 2 ulp
    (2^-22); doubled for margin."""
    return 2.0 * (np.log(2.0) * 4.0 * np.asarray(t_max_abs) * 2.0 ** -24 + 2.0 ** -22)


def softmax_sum_bound(T_kv_pad: int, t_max_abs):
    """Relative bound on the library's fp32 l against the exact sum of the exact p~: the
    terms' own error (softmax_weight_bound) plus the fp32 sum of positive terms (each of a
    row's 256 threads adds at most 8 ceil(T_kv_pad / 2048) terms in order, then a 5-step warp
    tree and 7 more additions); doubled for margin."""
    n = 8 * -(-T_kv_pad // 2048) + 12
    return softmax_weight_bound(t_max_abs) + 2.0 * n * 2.0 ** -24


P_GLOBAL_NVFP4 = 1.0 / 2688.0  # the NVFP4 global of P (p <= 1): T / (6 * 448) with T = 1


def pv_rows(p_codes, p_sf, vt_heads, head: int, T_kv_pad: int, rows, fmt: int = MX, g_p: float | None = None,
            g_v: float | None = None):
    """(Y, S) of rows `rows` of O = deq(P) deq(V_head), in fp64 (NVFP4 with the globals g_p, g_v)."""
    vc, vs = vt_heads
    a = dequant_fp4(fmt, p_codes, p_sf, T_kv_pad, 1.0 if fmt == MX else g_p, rows=rows)
    w = dequant_fp4(fmt, vc[head], vs[head], T_kv_pad, 1.0 if fmt == MX else g_v)
    return linear_fp64(a, w, None)


def synth_bits_to_f64(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def num_threads() -> int:
    return lib().orc_num_threads()


def tolerance(Y_ref: np.ndarray, S: np.ndarray) -> np.ndarray:
    """Per-element bound: one bf16 ulp of the exact result + 1e-5 * sum_k |a_k w_k|.

    ulp_bf16(y) = 2^(floor(log2|y|) - 7); for y = 0 the smallest normal bf16 ulp 2^-133."""
    a = np.abs(Y_ref)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    ulp = np.where(a > 0, np.ldexp(1.0, np.maximum(ex - 1 - 7, -133)), 2.0 ** -133)
    return ulp + 1e-5 * S


# ----------------------------------------------------------------------------- streaming attention
# The streaming (flash) form of one head's attention (the Wan2.2-Animate-14B MXFP4 card,
# "Results", names FP4 attention with microscaling on Blackwell; no page gives its
# algorithm): keys in blocks of FLASH_BLOCK; block j's weights are taken against the running
# maximum m_j of the blocks seen so far, and the partial outputs are brought to the final
# maximum by the factors 2^(m_j - m_last).

FLASH_BLOCK = 256
_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def dequant_mx_rows(codes, sf_rows) -> np.ndarray:
    """MXFP4 rows in fp64 from codes [R, K/2] (two E2M1 codes per byte, low nibble first) and
    their E8M0 scale bytes [R, K/32] in row order: value = e2m1(code) 2^(byte - 127)."""
    codes = np.asarray(codes, dtype=np.uint8)
    sf_rows = np.asarray(sf_rows, dtype=np.int64)
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[0], -1)
    vals = _E2M1[nib]
    R, K = vals.shape
    return (vals.reshape(R, K // 32, 32) * np.ldexp(1.0, sf_rows - 127)[..., None]).reshape(R, K)


def dequant_nv_rows(codes, sf_rows, g: float) -> np.ndarray:
    """NVFP4 rows in fp64 from codes [R, K/2] (low nibble first) and their E4M3 scale bytes
    [R, K/16] in row order: value = e2m1(code) dec(byte) g."""
    codes = np.asarray(codes, dtype=np.uint8)
    sf_rows = np.asarray(sf_rows, dtype=np.uint8)
    dec = np.array([e4m3_decode(b) for b in range(256)])
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[0], -1)
    vals = _E2M1[nib]
    R, K = vals.shape
    return (vals.reshape(R, K // 16, 16) * (dec[sf_rows] * float(g))[..., None]).reshape(R, K)


def flash_maxima(s: np.ndarray, T_kv: int, scale: float, block: int = FLASH_BLOCK) -> np.ndarray:
    """Running maxima [R, nblk] (nblk = ceil(T_kv / block)) of exact scores s [R, >= T_kv]:
    m[r, j] = max of s[r, k] c over the keys k < min(T_kv, (j + 1) block), c = softmax_c(scale)."""
    u = np.asarray(s, dtype=np.float64)[:, :T_kv] * softmax_c(scale)
    nb = -(-T_kv // block)
    full = np.full((u.shape[0], nb * block), -np.inf)
    full[:, :T_kv] = u
    return np.maximum.accumulate(full.reshape(u.shape[0], nb, block).max(axis=2), axis=1)


def flash_weights(s: np.ndarray, T_kv: int, scale: float, m: np.ndarray, block: int = FLASH_BLOCK) -> np.ndarray:
    """Block j's weights against its own maximum, fp64 [R, nblk * block]: p[r, k] = 2^(s c - m[r, j])
    for the keys k < T_kv of block j = k // block, 0 for the rest."""
    nb = m.shape[1]
    u = np.asarray(s, dtype=np.float64)[:, :T_kv] * softmax_c(scale)
    p = np.zeros((u.shape[0], nb * block))
    p[:, :T_kv] = np.exp2(u - np.repeat(m, block, axis=1)[:, :T_kv])
    return p


def flash_combine(p_vals: np.ndarray, m: np.ndarray, w: np.ndarray, block: int = FLASH_BLOCK):
    """(Y, S) of the unnormalized streaming output: Y = sum_j 2^(m_j - m_last) P_j W_j^T in fp64,
    P_j block j's columns of p_vals [R, nblk * block], W [N, nblk * block] (columns beyond W's
    width are zero); S the same sum of absolute terms (for the tolerance)."""
    nb = m.shape[1]
    f = np.exp2(m - m[:, -1:])
    a = p_vals[:, :nb * block] * np.repeat(f, block, axis=1)
    wf = np.zeros((w.shape[0], nb * block))
    wf[:, :min(w.shape[1], nb * block)] = w[:, :nb * block]
    return linear_fp64(a, wf, None)


def flash_pv_rows(p_codes, p_sf_rows, m: np.ndarray, vt_heads, head: int, T_kv_pad: int,
                  block: int = FLASH_BLOCK, fmt: int = MX, g_p: float | None = None, g_v: float | None = None):
    """flash_combine of the quantized weights (codes [R, nblk * block / 2], scale bytes
    [R, nblk * block / G] in row order; NVFP4 under the global g_p) with V_head^T dequantized
    from quantize_heads_vt (NVFP4 under g_v)."""
    vc, vs = vt_heads
    w = dequant_fp4(fmt, vc[head], vs[head], T_kv_pad, 1.0 if fmt == MX else g_v)
    a = dequant_mx_rows(p_codes, p_sf_rows) if fmt == MX else dequant_nv_rows(p_codes, p_sf_rows, g_p)
    return flash_combine(a, m, w, block)


def flash_sum(s: np.ndarray, T_kv: int, scale: float, m_last: np.ndarray) -> np.ndarray:
    """l[r] = sum over keys k < T_kv of 2^(s[r, k] c - m_last[r]), fp64: the streaming sum
    sum_j 2^(m_j - m_last) sum_{k in j} 2^(s c - m_j), whose factors telescope."""
    u = np.asarray(s, dtype=np.float64)[:, :T_kv] * softmax_c(scale)
    return np.exp2(u - np.asarray(m_last, dtype=np.float64)[:, None]).sum(axis=1)


def flash_weight_interval(s: np.ndarray, es: np.ndarray, T_kv: int, scale: float, m: np.ndarray,
                          block: int = FLASH_BLOCK, rel: float = 2.0 ** -23):
    """(lo, hi) [R, nblk * block] holding the fp32 weight exp2(fl(fl(s' c) - m_j)) for any fp32
    score s' with |s' - s| <= es (the exponent off by at most c es + rel (|s c| + |m_j|): the
    score's error and the roundings, rel = 2^-23 for the two of fl(fl(s c) - m), 2^-22 when
    the scores' NVFP4 globals are folded into c as well) and exp2f within 2 ulp (relative
    2^-22, taken as 2^-21); keys >= T_kv give [0, 0]."""
    nb = m.shape[1]
    c = softmax_c(scale)
    u = np.asarray(s, dtype=np.float64)[:, :T_kv] * c
    mj = np.repeat(m, block, axis=1)[:, :T_kv]
    d = c * np.asarray(es, dtype=np.float64)[:, :T_kv] + rel * (np.abs(u) + np.abs(mj))
    lo = np.zeros((u.shape[0], nb * block))
    hi = np.zeros((u.shape[0], nb * block))
    lo[:, :T_kv] = np.exp2(u - mj - d) * (1.0 - 2.0 ** -21)
    hi[:, :T_kv] = np.exp2(u - mj + d) * (1.0 + 2.0 ** -21)
    return lo, hi
