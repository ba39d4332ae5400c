"""CPU checks of the constants in the library's fp32 GELU program (gelu.cuh), derived here
from the mathematics rather than taken on trust.  Its error bound against the fp64
definition is checked on the GPU (test_gpu_quant.py::test_gelu_f32_error_bound_every_bf16)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "fp4_block_scaled_act_b200",
                   "csrc", "gelu.cuh")


def _seed_error(K):
    """max |d y0 - 1| over one binade of d, y0 = K - bits(d) read as a float (the error only
    depends on d's mantissa, so one binade covers every d)."""
    m = np.arange(1 << 23, dtype=np.int64)
    bits = (127 << 23) + m
    d = bits.astype(np.uint32).view(np.float32).astype(np.float64)
    y = (np.int64(K) - bits).astype(np.uint32).view(np.float32).astype(np.float64)
    return float(np.abs(d * y - 1.0).max())


def test_reciprocal_seed_is_the_minimax_constant():
    """The kernel's Newton-Raphson seed constant minimizes the worst relative error of the
    exponent-bit guess (its neighbours on both sides are worse), that error is below 0.0506,
    and three Newton steps (each squaring the error) take it below 2^-34."""
    src = open(SRC).read()
    consts = set(re.findall(r"0x7EF3[0-9A-F]{4}u", src))
    assert len(consts) == 1, consts
    K = int(consts.pop()[:-1], 16)
    e0 = _seed_error(K)
    for dk in (1, 2, 4, 16, 256):
        assert _seed_error(K - dk) > e0 and _seed_error(K + dk) > e0, dk
    assert e0 < 0.0506
    assert e0 ** 8 < 2.0 ** -34
    # the first-order model: K = 2^24 (127 - c) with a small bias c (here about 0.0505)
    c = 127.0 - K / 2.0 ** 24
    assert 0.04 < c < 0.06


def test_polynomial_coefficients_are_taylor_terms():
    """The 2^f polynomial's coefficients are (ln 2)^k / k! rounded to fp32."""
    import math

    src = open(SRC).read()
    coef = {k: float.fromhex(v) for v, k in re.findall(r"f2_splat\((0x1\.[0-9a-f]+p-?\d+)f\)+;\s+// \(ln2\)\^(\d)", src)}
    coef = {int(k): v for k, v in coef.items()}
    assert sorted(coef) == [2, 3, 4, 5, 6]
    for k, v in coef.items():
        assert v == float(np.float32(math.log(2.0) ** k / math.factorial(k))), k
    m = re.search(r"f2_splat\((0x1\.[0-9a-f]+p-?\d+)f\)+;\s+// ln2\n", src)
    assert float.fromhex(m.group(1)) == float(np.float32(math.log(2.0)))
