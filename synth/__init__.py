"""Seeded synthetic inputs for the W4A4 / W4A8 block-scaled quantized linear.

This module only draws random numbers and stores them in the 16-bit formats the
layer consumes (bf16 activations and weights, fp16 bias).  It contains none of
the quantization or GEMM arithmetic: both the CPU oracle and the CUDA path read
the exact same bytes produced here.

Shapes and distributions follow the Wan2.2 workloads the model cards describe:
tokens of a 21x45x80 latent grid (M = 75600), hidden size 5120, FFN size 13824,
text tokens M = 512, and the TI2V-5B W4A8 linear (M = 4290, K = 3072,
N = 14336, rank 32).  No dataset or trained weight is used: activations are
N(0,1) with per-channel lognormal gains (or a few outlier channels), weights
N(0, 0.02), biases N(0, 0.01).

Generation is chunked along rows; each chunk draws from its own PCG64 stream
spawned from the tensor's seed, so the result does not depend on the number of
threads used.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_CHUNK_ROWS = 2048


# --------------------------------------------------------------------------------------
# 16-bit storage formats (bit-level conversions, round-to-nearest-even)
# --------------------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even.  Inputs are finite."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_f16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> IEEE half bit patterns (uint16), numpy's round-to-nearest-even cast."""
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def f16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(b, dtype=np.uint16).view(np.float16).astype(np.float32)


# --------------------------------------------------------------------------------------
# chunked, thread-count-independent normal draws
# --------------------------------------------------------------------------------------
def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _normal_rows(seed: int, rows: int, cols: int, fill) -> None:
    """Call fill(r0, r1, z) with z ~ N(0,1) float32 [r1-r0, cols] for each row chunk."""
    nchunks = max(1, math.ceil(rows / _CHUNK_ROWS))
    children = np.random.SeedSequence(seed).spawn(nchunks)

    def work(i):
        r0 = i * _CHUNK_ROWS
        r1 = min(rows, r0 + _CHUNK_ROWS)
        g = np.random.Generator(np.random.PCG64(children[i]))
        fill(r0, r1, g.standard_normal((r1 - r0, cols), dtype=np.float32))

    if nchunks == 1:
        work(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nchunks)))


def channel_gains(seed: int, K: int) -> np.ndarray:
    """Per-channel lognormal(0, 1) gains, float32 [K]."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0x6A1])))
    return g.lognormal(0.0, 1.0, size=K).astype(np.float32)


def outlier_channels(seed: int, K: int, count: int = 4) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0x0C7])))
    return np.sort(g.choice(K, size=count, replace=False))


def _gelu_tanh_f32(z: np.ndarray) -> np.ndarray:
    # Input synthesis only: the previous layer's activation, evaluated in fp32.
    c = np.float32(math.sqrt(2.0 / math.pi))
    z3 = z * z * z
    inner = c * (z + np.float32(0.044715) * z3)
    return (np.float32(0.5) * z * (np.float32(1.0) + np.tanh(inner))).astype(np.float32)


def activation(seed: int, M: int, K: int, kind: str, gain_seed: int | None = None) -> np.ndarray:
    """bf16 activation bits [M, K] (uint16).

    kind:
      "outlier"   N(0,1) with 4 seeded channels multiplied by 20
      "lognormal" N(0,1) times a per-channel lognormal(0,1) gain (gain_seed picks the
                  gains, so a calibration batch and the runtime batch of one layer share them)
      "gelu"      GELU-tanh of N(0,1), computed in fp32 then rounded to bf16
    """
    out = np.empty((M, K), dtype=np.uint16)
    if kind == "lognormal":
        gains = channel_gains(seed if gain_seed is None else gain_seed, K)
    elif kind == "outlier":
        chans = outlier_channels(seed if gain_seed is None else gain_seed, K)
        gains = np.ones(K, dtype=np.float32)
        gains[chans] = 20.0
    elif kind == "gelu":
        gains = None
    else:
        raise ValueError(kind)

    def fill(r0, r1, z):
        if kind == "gelu":
            v = _gelu_tanh_f32(z)
        else:
            v = z * gains[None, :]
        out[r0:r1] = f32_to_bf16_bits(v)

    _normal_rows(seed, M, K, fill)
    return out


def weight(seed: int, N: int, K: int, std: float = 0.02) -> np.ndarray:
    """bf16 weight bits [N, K] (torch Linear layout), N(0, std)."""
    out = np.empty((N, K), dtype=np.uint16)

    def fill(r0, r1, z):
        out[r0:r1] = f32_to_bf16_bits(z * np.float32(std))

    _normal_rows(seed, N, K, fill)
    return out


def bias(seed: int, N: int, std: float = 0.01) -> np.ndarray:
    """fp16 bias bits [N], N(0, std)."""
    g = np.random.Generator(np.random.PCG64(seed))
    return f32_to_f16_bits(g.standard_normal(N, dtype=np.float32) * np.float32(std))


# --------------------------------------------------------------------------------------
# Workload catalogue (one entry per linear; seeds = 1000*config + tensor id)
# --------------------------------------------------------------------------------------
CALIB_TOKENS = 8192

LINEARS = {
    # name: (M, K, N, activation kind)
    "tiny_mx": (256, 512, 512, "outlier"),
    "attn_proj": (75600, 5120, 5120, "lognormal"),
    "ffn_up": (75600, 5120, 13824, "lognormal"),
    "ffn_down": (75600, 13824, 5120, "gelu"),
    "text_kv": (512, 5120, 5120, "lognormal"),
    "w4a8_ti2v": (4290, 3072, 14336, "lognormal"),
}


def seeds_for(config: int, layer: int = 0) -> dict:
    base = 1000 * config + 10 * layer
    return {"x": base + 1, "w": base + 2, "bias": base + 3, "calib": base + 4, "gain": base + 5}


def linear_inputs(config: int, M: int, K: int, N: int, kind: str, layer: int = 0,
                  with_calib: bool = False) -> dict:
    """bf16 X [M,K], bf16 W [N,K], fp16 bias [N] (+ an 8192-token calibration batch)."""
    s = seeds_for(config, layer)
    d = {
        "x": activation(s["x"], M, K, kind, gain_seed=s["gain"]),
        "w": weight(s["w"], N, K),
        "bias": bias(s["bias"], N),
    }
    if with_calib:
        d["x_cal"] = activation(s["calib"], CALIB_TOKENS, K, kind, gain_seed=s["gain"])
    return d


# --------------------------------------------------------------------------------------
# W4A8 SVDQuant checkpoint synthesis (offline exporter recipe, untimed)
# --------------------------------------------------------------------------------------
def svdquant_factors(seed: int, N: int, K: int, rank: int = 32, alpha: float = 0.5,
                     calib_tokens: int = CALIB_TOKENS) -> dict:
    """Synthesize a self-contained W4A8 SVDQuant linear from a seeded N(0,0.02) weight.

    SmoothQuant (alpha = 0.5) per-channel s from a seeded calibration batch, exact SVD
    of the smoothed weight, top-`rank` factors, and the 1/s factor folded into the
    residual and the down-projection, as the exporter the W4A8 model card describes.
    Returns float64 W0, R, L1, L2 plus their bf16 bit patterns.
    """
    w0 = bf16_bits_to_f32(weight(seed, N, K)).astype(np.float64)
    xc = bf16_bits_to_f32(activation(seed + 7, calib_tokens, K, "lognormal", gain_seed=seed + 5))
    amax_x = np.abs(xc).max(axis=0).astype(np.float64)
    amax_w = np.abs(w0).max(axis=0)
    s = np.maximum(amax_x, 1e-12) ** alpha / np.maximum(amax_w, 1e-12) ** (1.0 - alpha)
    w_s = w0 * s[None, :]
    u, sig, vt = np.linalg.svd(w_s, full_matrices=False)
    a = u[:, :rank] * sig[None, :rank]            # [N, rank]
    b = vt[:rank, :]                               # [rank, K]
    r = (w_s - a @ b) / s[None, :]                 # [N, K]
    l1 = (b / s[None, :]).T                        # [K, rank]
    l2 = a.T                                       # [rank, N]
    return {
        "w0": w0, "s": s, "r": r, "l1": l1, "l2": l2,
        "r_bf16": f32_to_bf16_bits(r.astype(np.float32)),
        "l1_bf16": f32_to_bf16_bits(l1.astype(np.float32)),
        "l2_bf16": f32_to_bf16_bits(l2.astype(np.float32)),
    }
