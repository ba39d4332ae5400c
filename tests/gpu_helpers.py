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
