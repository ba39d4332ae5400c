"""GPU parity of the block-scaled GEMM and the end-to-end quantized linear.

Every output element is checked against the fp64 oracle on the dequantized operands
within |y - y_ref| <= ulp_bf16(y_ref) + 1e-5 * sum_k |a_k w_k| for small shapes (several
tiles, ragged M and N tails, odd K stages); at the full Wan2.2 sizes, in the launch
configuration the benchmark times, sampled rows (including every row of the ragged
last tile) are checked the same way.
"""
import contextlib

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


def _run_linear(fb, fmt, x_bits, w_bits, b_bits, g_a=None):
    import torch

    x = H.dev_bf16(x_bits)
    pw = fb.pack_weight(H.dev_bf16(w_bits), fmt)
    bias = H.dev_f16(b_bits) if b_bits is not None else None
    ga = H.dev_f32([g_a]) if fmt == NV else None
    y = fb.linear(x, pw, bias, ga)
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    torch.cuda.synchronize()
    return y


def _oracle(orc, fmt, x_bits, w_bits, b_bits, rows, g_a=None):
    return orc.fp4_linear_rows(fmt, x_bits, w_bits, b_bits, rows, g_a=g_a)


SMALL = [
    (1, 256, 256), (128, 256, 256), (129, 512, 384), (256, 512, 512), (300, 384, 640),
    (77, 1280, 1024), (513, 768, 256),
    # K % 512 = 128 and K = 128: a last (or only) MXFP4 stage of two MMAs
    (300, 640, 384), (260, 128, 256),
]


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("M,K,N", SMALL)
def test_linear_small_all_elements(fb, orc, fmt, M, K, N):
    kind = "outlier" if (M, K, N) == (256, 512, 512) else "lognormal"
    x = synth.activation(10 * M + K, M, K, kind)
    w = synth.weight(20 * N + K, N, K)
    b = synth.bias(N + 3, N)
    g_a = None
    if fmt == NV:
        g_a = orc.nv_global(orc.tensor_amax(synth.activation(30 * M + K, 64, K, kind)))
    y = _run_linear(fb, fmt, x, w, b, g_a)
    rows = np.arange(M)
    Y, S = _oracle(orc, fmt, x, w, b, rows, g_a)
    H.check_linear(y, Y, S, rows, f"fmt={fmt} M={M} K={K} N={N}")


def test_linear_no_bias(fb, orc):
    M, K, N = 200, 512, 384
    x = synth.activation(1, M, K, "lognormal")
    w = synth.weight(2, N, K)
    y = _run_linear(fb, MX, x, w, None)
    Y, S = _oracle(orc, MX, x, w, None, np.arange(M))
    H.check_linear(y, Y, S, np.arange(M), "no bias")


def test_gemm_exact_grid_values(fb, orc):
    """Grid-valued operands with scale 1: the exact product is representable, so y must
    equal bf16(exact) with the error of a single rounding."""
    rng = np.random.default_rng(3)
    M, K, N = 130, 512, 256
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)

    def gm(r, c):
        v = grid[rng.integers(0, 8, size=(r, c))] * np.where(rng.random((r, c)) < 0.5, -1, 1)
        v[:, ::32] = 6.0
        return v.astype(np.float32)

    a, w = gm(M, K), gm(N, K)
    y = _run_linear(fb, MX, synth.f32_to_bf16_bits(a), synth.f32_to_bf16_bits(w), None)
    exact = a.astype(np.float64) @ w.astype(np.float64).T
    got = H.host_bf16_as_f64(y)
    ref_bf16 = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(exact.astype(np.float32))).astype(np.float64)
    np.testing.assert_array_equal(got, ref_bf16)


def test_gemm_selector_weight(fb, orc):
    """W row n holds a single 4.0 at column (5n) % K: y[:, n] = 4 * deq(a)[:, (5n) % K]."""
    M, K, N = 256, 1024, 512
    x = synth.activation(4, M, K, "lognormal")
    w = np.zeros((N, K), dtype=np.float32)
    cols = (5 * np.arange(N)) % K
    w[np.arange(N), cols] = 4.0
    y = _run_linear(fb, MX, x, synth.f32_to_bf16_bits(w), None)
    codes, sf = orc.quantize(MX, x)
    a = orc.dequant_fp4(MX, codes, sf, K)
    exp = 4.0 * a[:, cols]
    np.testing.assert_array_equal(H.host_bf16_as_f64(y),
                                  synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(exp.astype(np.float32))))


def test_gemm_determinism(fb):
    import torch

    M, K, N = 700, 1024, 768
    x = H.dev_bf16(synth.activation(5, M, K, "lognormal"))
    pw = fb.pack_weight(H.dev_bf16(synth.weight(6, N, K)), MX)
    y1 = fb.linear(x, pw)
    y2 = fb.linear(x, pw)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_gemm_entry_matches_linear(fb):
    """fp4_gemm on separately quantized activations == fp4_linear (same kernels)."""
    import torch

    M, K, N = 333, 768, 512
    x = H.dev_bf16(synth.activation(8, M, K, "lognormal"))
    pw = fb.pack_weight(H.dev_bf16(synth.weight(9, N, K)), NV)
    ga = H.dev_f32([0.01])
    codes, sf = fb.quantize_act(x, NV, ga)
    y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fb.fp4_gemm(NV, codes, sf, M, K, N, pw.codes, pw.sf, pw.w_global, ga, None, y1)
    y2 = fb.linear(x, pw, None, ga)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


# ------------------------------------------------------------------ full-size workloads
FULL = [
    # (config, fmt, M, K, N, activation kind)
    (1, MX, 75600, 5120, 5120, "lognormal"),     # attention projection, MXFP4
    (4, MX, 75600, 5120, 13824, "lognormal"),    # ffn up, MXFP4 (the benchmark workload)
    (2, NV, 75600, 5120, 13824, "lognormal"),    # ffn up, NVFP4
    (2, NV, 75600, 13824, 5120, "gelu"),         # ffn down, NVFP4
    (4, MX, 512, 5120, 5120, "lognormal"),       # attn2 k/v on 512 text tokens
    # the rest of the Wan2.2 block's ten linears in both formats
    (4, NV, 75600, 5120, 5120, "lognormal"),     # attn1 q/k/v/out, attn2 q/out, NVFP4
    (4, NV, 512, 5120, 5120, "lognormal"),       # attn2 k/v on 512 text tokens, NVFP4
    (4, MX, 75600, 13824, 5120, "gelu"),         # ffn down, MXFP4
    # the M sweep at 5120 -> 13824 (512 and 4096 are checked on every element below)
    (4, MX, 16384, 5120, 13824, "lognormal"),
    (4, NV, 16384, 5120, 13824, "lognormal"),
]


@pytest.mark.parametrize("cfg,fmt,M,K,N,kind", FULL)
def test_linear_full_size_sampled(fb, orc, cfg, fmt, M, K, N, kind):
    s = synth.seeds_for(cfg, layer=K // 1000 + N // 1000)
    x = synth.activation(s["x"], M, K, kind, gain_seed=s["gain"])
    w = synth.weight(s["w"], N, K)
    b = synth.bias(s["bias"], N)
    g_a = None
    if fmt == NV:
        cal = synth.activation(s["calib"], synth.CALIB_TOKENS, K, kind, gain_seed=s["gain"])
        g_a = orc.nv_global(orc.tensor_amax(cal))
    y = _run_linear(fb, fmt, x, w, b, g_a)
    rows = H.sample_rows(M, n_random=40, seed=cfg)
    Y, S = _oracle(orc, fmt, x, w, b, rows, g_a)
    H.check_linear(y, Y, S, rows, f"full cfg={cfg} fmt={fmt} M={M} K={K} N={N}")


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("M", [512, 4096])
def test_linear_m_sweep_every_element(fb, orc, fmt, M):
    """The M sweep's smaller points at 5120 -> 13824, every element of Y against the oracle."""
    K, N = 5120, 13824
    s = synth.seeds_for(4, layer=K // 1000 + N // 1000)
    x = synth.activation(s["x"] + M, M, K, "lognormal", gain_seed=s["gain"])
    w = synth.weight(s["w"], N, K)
    b = synth.bias(s["bias"], N)
    g_a = None
    if fmt == NV:
        cal = synth.activation(s["calib"], synth.CALIB_TOKENS, K, "lognormal", gain_seed=s["gain"])
        g_a = orc.nv_global(orc.tensor_amax(cal))
    y = _run_linear(fb, fmt, x, w, b, g_a)
    rows = np.arange(M)
    Y, S = _oracle(orc, fmt, x, w, b, rows, g_a)
    H.check_linear(y, Y, S, rows, f"M sweep fmt={fmt} M={M} every element")


# ------------------------------------------------------------------ bounded waits
@pytest.mark.parametrize("M", [128, 256])
def test_bounded_wait_reports_timeout(fb, orc, M):
    """A k-stage that is never filled (test hook) makes the kernel's bounded wait run out
    (M = 128: 1-CTA kernel, M = 256: 2-CTA kernel); the kernel returns, the status word
    reads FP4_ERR_TIMEOUT, and the next call is correct."""
    import torch

    K, N = 512, 256
    x = synth.activation(11, M, K, "lognormal")
    w = synth.weight(12, N, K)
    xd, pw = H.dev_bf16(x), fb.pack_weight(H.dev_bf16(w), MX)
    assert fb.fp4_sync_status() == 0
    L = fb.lib()
    try:
        fb.fp4_set_wait_timeout_ns(2_000_000)  # 2 ms
        L.fp4bsa_test_skip_iteration(1)
        fb.linear(xd, pw)
        st = fb.fp4_sync_status()
    finally:
        L.fp4bsa_test_skip_iteration(-1)
        fb.fp4_set_wait_timeout_ns(0)
    assert fb.fp4_status_string(st) == "FP4_ERR_TIMEOUT"
    y = fb.linear(xd, pw)
    assert fb.fp4_sync_status() == 0
    torch.cuda.synchronize()
    Y, S = orc.fp4_linear_rows(MX, x, w, None, np.arange(M))
    H.check_linear(y, Y, S, np.arange(M), "after timeout")


# ------------------------------------------------------------------ W4A8 SVDQuant linear
def _w4a8_check(fb, orc, M, K, N, seed, rows=None, calib=256):
    import torch

    f = synth.svdquant_factors(seed, N, K, calib_tokens=calib)
    x = synth.activation(seed + 1, M, K, "lognormal", gain_seed=seed + 5)
    b = synth.bias(seed + 2, N)
    rp = fb.pack_weight(H.dev_bf16(f["r_bf16"]), MX)
    y = fb.w4a8_linear(H.dev_bf16(x), rp, H.dev_bf16(f["l1_bf16"]), H.dev_bf16(f["l2_bf16"]), H.dev_f16(b))
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    torch.cuda.synchronize()
    rows = np.arange(M) if rows is None else rows
    rc, rs, _ = orc.pack_weight(MX, f["r_bf16"])
    Y, S = orc.svd_linear_rows("mxfp8", x, (rc, rs), f["l1_bf16"], f["l2_bf16"], b, rows)
    return H.check_linear(y, Y, S, rows, f"w4a8 M={M} K={K} N={N}")


# 8300 rows (65 blocks of 128): the activation side runs as one quantize + project pass
@pytest.mark.parametrize("M,K,N", [(1, 256, 256), (130, 512, 384), (300, 1024, 512), (8300, 256, 256)])
def test_w4a8_small_all_elements(fb, orc, M, K, N):
    _w4a8_check(fb, orc, M, K, N, seed=7000 + M)


def test_w4a8_full_size_sampled(fb, orc):
    """TI2V-5B-shaped W4A8 linear: M = 4290 (11x15x26 tokens), K = 3072, N = 14336, rank 32."""
    M, K, N = 4290, 3072, 14336
    rows = H.sample_rows(M, n_random=48, seed=3)
    _w4a8_check(fb, orc, M, K, N, seed=3001, rows=rows, calib=2048)


def test_w4a8_full_size_every_element(fb, orc):
    """The W4A8 configuration at its full size, every element of Y against the oracle (the
    fp64 oracle of 4290 x 3072 x 14336 takes under a minute on the host)."""
    _w4a8_check(fb, orc, 4290, 3072, 14336, seed=3011, calib=2048)


# ------------------------------------------------------------------ up projection + GELU + quantize
# The FFN's up projection with GELU-tanh and the down projection's quantizer fused into its
# epilogue.  z (the bf16 GEMM result) is only known to the GEMM tolerance, so the output is
# checked for validity (tests/gpu_helpers.check_gelu_quant) and for its agreement rate with
# the oracle's own choice of z.
def _gelu_linear_case(fb, orc, fmt, M, K, N, x, w, b, rows, what):
    import torch

    g_a = orc.nv_global(orc.tensor_amax(x)) if fmt == NV else None
    Y, S = _oracle(orc, fmt, x, w, b, rows, g_a)
    g_h = None
    if fmt == NV:  # the down projection's static global, from the oracle's own output
        zb = H._bf16_bracket(Y)[0]
        g_h = orc.nv_global(orc.tensor_amax(orc.gelu_bf16(zb)))
    pw = fb.pack_weight(H.dev_bf16(w), fmt)
    codes, sf = fb.linear_gelu_quant(H.dev_bf16(x), pw, H.dev_f16(b) if b is not None else None,
                                     H.dev_f32([g_a]) if fmt == NV else None,
                                     H.dev_f32([g_h]) if fmt == NV else None)
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    torch.cuda.synchronize()
    agree = H.check_gelu_quant(fmt, codes, sf, Y, S, rows, M, N, g_h, what)
    assert agree > 0.99, (what, agree)


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("M,K,N", [(1, 256, 256), (129, 512, 384), (300, 768, 512), (600, 1280, 1024)])
def test_linear_gelu_quant_small(fb, orc, fmt, M, K, N):
    x = synth.activation(60 * M + K, M, K, "lognormal")
    w = synth.weight(70 * N + K, N, K)
    b = synth.bias(N + 11, N)
    _gelu_linear_case(fb, orc, fmt, M, K, N, x, w, b, np.arange(M), f"gelu fmt={fmt} M={M} K={K} N={N}")


@pytest.mark.parametrize("cfg,fmt", [(2, NV), (4, MX)])
def test_linear_gelu_quant_full_size_sampled(fb, orc, cfg, fmt):
    """ffn up projection 75600 x 5120 -> 13824 with GELU and the down projection's quantizer."""
    M, K, N = 75600, 5120, 13824
    s = synth.seeds_for(cfg, layer=K // 1000 + N // 1000)
    x = synth.activation(s["x"], M, K, "lognormal", gain_seed=s["gain"])
    w = synth.weight(s["w"], N, K)
    b = synth.bias(s["bias"], N)
    rows = H.sample_rows(M, n_random=24, seed=cfg + 50)
    _gelu_linear_case(fb, orc, fmt, M, K, N, x, w, b, rows, f"gelu full cfg={cfg} fmt={fmt}")


# ------------------------------------------------------------------ W4A4 SVDQuant linear
# The W4A8 README's experimental W4A4 variant: MXFP4 activations on the same factors.
def _w4a4_check(fb, orc, M, K, N, seed, rows=None, calib=256):
    import torch

    f = synth.svdquant_factors(seed, N, K, calib_tokens=calib)
    x = synth.activation(seed + 1, M, K, "lognormal", gain_seed=seed + 5)
    b = synth.bias(seed + 2, N)
    rp = fb.pack_weight(H.dev_bf16(f["r_bf16"]), MX)
    y = fb.w4a4_linear(H.dev_bf16(x), rp, H.dev_bf16(f["l1_bf16"]), H.dev_bf16(f["l2_bf16"]), H.dev_f16(b))
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    torch.cuda.synchronize()
    rows = np.arange(M) if rows is None else rows
    rc, rs, _ = orc.pack_weight(MX, f["r_bf16"])
    Y, S = orc.svd_linear_rows("mxfp4", x, (rc, rs), f["l1_bf16"], f["l2_bf16"], b, rows)
    return H.check_linear(y, Y, S, rows, f"w4a4 M={M} K={K} N={N}")


@pytest.mark.parametrize("M,K,N", [(1, 256, 256), (130, 512, 384), (300, 1024, 512), (8300, 256, 256)])
def test_w4a4_small_all_elements(fb, orc, M, K, N):
    _w4a4_check(fb, orc, M, K, N, seed=8000 + M)


def test_w4a4_full_size_sampled(fb, orc):
    """TI2V-5B-shaped W4A4 SVDQuant linear: M = 4290, K = 3072, N = 14336, rank 32."""
    M, K, N = 4290, 3072, 14336
    rows = H.sample_rows(M, n_random=48, seed=4)
    _w4a4_check(fb, orc, M, K, N, seed=4001, rows=rows, calib=2048)


# ------------------------------------------------------------------ small-M stream-K schedule
# fp4_linear can run small problems as stream-K (a tuning hook turns it on; measured slower
# than whole tiles on B200): tiles shared by pairs are summed through fp32 slabs in a fixed
# segment order.
@contextlib.contextmanager
def _stream_k(fb, mode):
    L = fb.lib()
    L.fp4bsa_set_stream_k(mode)
    try:
        yield L
    finally:
        L.fp4bsa_set_stream_k(0)


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("M,K,N", [(1, 5120, 1024), (77, 2560, 2048), (129, 5120, 1024), (300, 2432, 1024),
                                   (512, 5120, 1280)])
def test_stream_k_all_elements(fb, orc, fmt, M, K, N):
    """Stream-K (forced on) against the oracle on every element, ragged M and K % 256 = 128."""
    x = synth.activation(80 * M + K, M, K, "lognormal")
    w = synth.weight(90 * N + K, N, K)
    b = synth.bias(N + 13, N)
    g_a = orc.nv_global(orc.tensor_amax(x)) if fmt == NV else None
    with _stream_k(fb, 2):
        y = _run_linear(fb, fmt, x, w, b, g_a)
    rows = np.arange(M)
    Y, S = _oracle(orc, fmt, x, w, b, rows, g_a)
    H.check_linear(y, Y, S, rows, f"stream-K fmt={fmt} M={M} K={K} N={N}")


def test_stream_k_deterministic_and_close_to_whole_tiles(fb, orc):
    """Two stream-K runs are bit-identical; whole tiles give the same result within tolerance."""
    import torch

    M, K, N = 512, 5120, 5120  # the attn2 k/v shape (text tokens)
    x = synth.activation(4242, M, K, "lognormal")
    w = synth.weight(4243, N, K)
    b = synth.bias(4244, N)
    with _stream_k(fb, 2):
        y1 = _run_linear(fb, MX, x, w, b)
        y2 = _run_linear(fb, MX, x, w, b)
    assert torch.equal(y1, y2)
    with _stream_k(fb, 1):
        y3 = _run_linear(fb, MX, x, w, b)
    rows = np.arange(M)
    Y, S = _oracle(orc, MX, x, w, b, rows)
    H.check_linear(y1, Y, S, rows, "stream-K attn2 k/v")
    H.check_linear(y3, Y, S, rows, "whole tiles attn2 k/v")


# ------------------------------------------------------------------ each GEMM kernel, forced
# The library picks the cta_group::2 256x256 kernel for M > 128 and the 1-CTA 128x256
# kernel otherwise; a tuning hook forces either, so both stay covered on ragged shapes.
@contextlib.contextmanager
def _gemm_ctas(fb, ctas):
    L = fb.lib()
    L.fp4bsa_set_gemm_ctas(ctas)
    try:
        yield L
    finally:
        L.fp4bsa_set_gemm_ctas(0)


@pytest.mark.parametrize("ctas", [1, 2])
@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("M,K,N", [(129, 512, 384), (300, 768, 512), (600, 1280, 1024)])
def test_each_kernel_all_elements(fb, orc, ctas, fmt, M, K, N):
    x = synth.activation(40 * M + K, M, K, "lognormal")
    w = synth.weight(50 * N + K, N, K)
    b = synth.bias(N + 9, N)
    g_a = orc.nv_global(orc.tensor_amax(x)) if fmt == NV else None
    with _gemm_ctas(fb, ctas):
        y = _run_linear(fb, fmt, x, w, b, g_a)
    rows = np.arange(M)
    Y, S = _oracle(orc, fmt, x, w, b, rows, g_a)
    H.check_linear(y, Y, S, rows, f"ctas={ctas} fmt={fmt} M={M} K={K} N={N}")


@pytest.mark.parametrize("ctas", [1, 2])
def test_w4a8_ignores_the_kernel_hook(fb, orc, ctas):
    """W4A8 always runs the 2-CTA kernel (its low-rank stage is a tensor-core stage there)."""
    with _gemm_ctas(fb, ctas):
        _w4a8_check(fb, orc, 300, 1024, 512, seed=7777)


@pytest.mark.parametrize("ctas", [1, 2])
def test_each_kernel_timeout(fb, orc, ctas):
    """A stage that is never filled makes the kernel's bounded wait run out; the status
    word reads FP4_ERR_TIMEOUT and the next call on the same context is correct."""
    import torch

    M, K, N = 256, 512, 256
    x = synth.activation(13, M, K, "lognormal")
    w = synth.weight(14, N, K)
    xd, pw = H.dev_bf16(x), fb.pack_weight(H.dev_bf16(w), MX)
    assert fb.fp4_sync_status() == 0
    with _gemm_ctas(fb, ctas) as L:
        try:
            fb.fp4_set_wait_timeout_ns(2_000_000)
            L.fp4bsa_test_skip_iteration(1)
            fb.linear(xd, pw)
            st = fb.fp4_sync_status()
            L.fp4bsa_test_skip_iteration(-1)
            fb.fp4_set_wait_timeout_ns(0)
            y = fb.linear(xd, pw)
            st2 = fb.fp4_sync_status()
        finally:
            L.fp4bsa_test_skip_iteration(-1)
            fb.fp4_set_wait_timeout_ns(0)
    assert fb.fp4_status_string(st) == "FP4_ERR_TIMEOUT" and st2 == 0
    torch.cuda.synchronize()
    Y, S = orc.fp4_linear_rows(MX, x, w, None, np.arange(M))
    H.check_linear(y, Y, S, np.arange(M), f"ctas={ctas} after timeout")


# ------------------------------------------------------------------ host-to-host pipeline
@pytest.mark.parametrize("fmt", [MX, NV])
def test_linear_host_chunks(fb, orc, fmt):
    """linear_host: pinned host x -> pinned host y in row chunks (ragged last chunk) with
    overlapped copies, against the oracle on every row."""
    import torch

    M, K, N = 700, 1024, 512
    x = synth.activation(5151 + fmt, M, K, "lognormal")
    w = synth.weight(5152, N, K)
    b = synth.bias(5153, N)
    g_a = orc.nv_global(orc.tensor_amax(x)) if fmt == NV else None
    pw = fb.pack_weight(H.dev_bf16(w), fmt)
    x_host = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()
    pipe = fb.HostPipeline(fmt, 256, K, N)
    y_host = fb.linear_host(x_host, pw, pipe, H.dev_f16(b), H.dev_f32([g_a]) if fmt == NV else None)
    torch.cuda.synchronize()
    assert fb.fp4_sync_status() == 0
    rows = np.arange(M)
    Y, S = _oracle(orc, fmt, x, w, b, rows, g_a)
    H.check_linear(y_host, Y, S, rows, f"linear_host fmt={fmt}")


# ------------------------------------------------------------------ several tiles per CTA pair
# 9 x 17 = 153 output tiles of 256 x 256 for 74 pairs: every pair runs two or three tiles, so
# both accumulators, the hand-over of their shared columns between consecutive tiles and (NVFP4
# with bf16 output) the overlap holders' copy-all release are exercised on every element; M and
# N both end in a ragged tile.
MANY = (2300, 512, 4224)


@pytest.mark.parametrize("fmt", [MX, NV])
def test_pair_kernel_many_tiles_all_elements(fb, orc, fmt):
    M, K, N = MANY
    x = synth.activation(90 * M + K, M, K, "lognormal")
    w = synth.weight(91 * N + K, N, K)
    b = synth.bias(N + 13, N)
    g_a = orc.nv_global(orc.tensor_amax(x)) if fmt == NV else None
    with _gemm_ctas(fb, 2):
        y = _run_linear(fb, fmt, x, w, b, g_a)
    rows = np.arange(M)
    Y, S = _oracle(orc, fmt, x, w, b, rows, g_a)
    H.check_linear(y, Y, S, rows, f"many tiles fmt={fmt}")


def test_w4a8_many_tiles_all_elements(fb, orc):
    _w4a8_check(fb, orc, *MANY, seed=7100)


def test_w4a4_many_tiles_all_elements(fb, orc):
    _w4a4_check(fb, orc, *MANY, seed=8100)


@pytest.mark.parametrize("fmt", [MX, NV])
def test_linear_gelu_quant_many_tiles(fb, orc, fmt):
    M, K, N = MANY
    x = synth.activation(92 * M + K, M, K, "lognormal")
    w = synth.weight(93 * N + K, N, K)
    b = synth.bias(N + 17, N)
    _gelu_linear_case(fb, orc, fmt, M, K, N, x, w, b, np.arange(M), f"gelu many tiles fmt={fmt}")


# ------------------------------------------------------------------ CUDA-graph capture
# The library allocates nothing, synchronizes nothing and copies nothing between host and
# device inside a call, so a quantized linear can be captured once and replayed (the way
# launch-bound text-token calls amortize their fixed cost).  The captured graph holds the
# quantize kernel and the GEMM (with its programmatic launch edge); each replay reads
# whatever the input buffer holds at that moment.
@pytest.mark.parametrize("fmt", [MX, NV])
def test_linear_replays_in_a_cuda_graph(fb, orc, fmt):
    import torch

    M, K, N = 512, 1024, 768
    w = synth.weight(95 * N + K, N, K)
    b = synth.bias(N + 19, N)
    xs = [synth.activation(96 * M + K + i, M, K, "lognormal") for i in range(2)]
    g_a = orc.nv_global(max(orc.tensor_amax(xi) for xi in xs)) if fmt == NV else None
    pw = fb.pack_weight(H.dev_bf16(w), fmt)
    bias = H.dev_f16(b)
    ga = H.dev_f32([g_a]) if fmt == NV else None
    x = H.dev_bf16(xs[0])
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(fb.fp4_linear_workspace_bytes(fmt, M, K, N), dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fb.linear(x, pw, bias, ga, y, ws)  # eager first call: one-time device setup
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        fb.linear(x, pw, bias, ga, y, ws)
    rows = np.arange(M)
    for i, xi in enumerate(xs):
        x.copy_(H.dev_bf16(xi))
        y.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        st = fb.fp4_sync_status()
        assert st == 0, fb.fp4_status_string(st)
        Y, S = _oracle(orc, fmt, xi, w, b, rows, g_a)
        H.check_linear(y, Y, S, rows, f"graph replay {i} fmt={fmt}")
