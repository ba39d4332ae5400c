"""Pins of the FP4 attention-operand oracle (oracle.quantize_heads, oracle.attn_scores_rows).

Reading (Wan2.2-Animate-14B MXFP4 card, "Results": SageAttention v3 is Blackwell
microscaling FP4 attention, no algorithm given): Q and K are quantized per token and head in
blocks of G along head_dim = 128 by the activation rules, stored head-major, and a head's
scores are the fp64 products of the dequantized operands.  These tests pin that oracle to
things other than itself:
  - the head-major result equals the pinned row quantizer run on the whole [T, H*128]
    tensor, bytes re-addressed (a head is a whole number of groups and scale atoms);
  - on inputs every block of which is exactly representable (E2M1 grid values times the
    block's power of two, with the block's amax on 6 * 2^e), quantization is lossless, so
    the scores equal the exact dot products of the original values computed by numpy;
  - padding tokens quantize to zero codes and zero scale bytes, and their score columns
    are 0.
"""
import numpy as np
import pytest

import oracle
import synth

MX, NV = oracle.MX, oracle.NV
D = 128


def _x(seed, T, H):
    return synth.activation(seed, T, H * D, "lognormal")


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("T,H", [(1, 1), (130, 3), (257, 2)])
def test_quantize_heads_is_the_row_quantizer_re_addressed(fmt, T, H):
    x = _x(700 + T + H, T, H)
    g = oracle.nv_global(oracle.tensor_amax(x)) if fmt == NV else None
    codes, sfs = oracle.quantize_heads(fmt, x, H, g)
    full_c, full_s = oracle.quantize(fmt, x, g)
    G = oracle.group_size(fmt)
    Tpad = (T + 127) // 128 * 128
    assert codes.shape == (H, Tpad, D // 2)
    for h in range(H):
        np.testing.assert_array_equal(codes[h, :T], full_c[:, h * D // 2:(h + 1) * D // 2])
        assert not codes[h, T:].any(), "padding tokens must hold zero codes"
        for r in range(Tpad):
            for j in range(D // G):
                assert sfs[h, oracle.sf_offset(r, j, D // G)] == full_s[oracle.sf_offset(r, h * (D // G) + j, H * D // G)]
        assert not any(sfs[h, oracle.sf_offset(r, j, D // G)] for r in range(T, Tpad) for j in range(D // G))


def _representable(rng, T, H, G):
    """Values on the E2M1 grid times 2^e per G-block, each block with an element of
    magnitude 6 * 2^e: MX and NVFP4 (global 1) quantize them without error."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    v = rng.choice(grid, size=(T, H * D)) * rng.choice([-1.0, 1.0], size=(T, H * D))
    e = rng.integers(-3, 4, size=(T, H * D // G)).astype(np.float64)
    v = v.reshape(T, -1, G)
    v[:, :, 0] = 6.0 * rng.choice([-1.0, 1.0], size=v.shape[:2])
    v = v * np.exp2(e)[:, :, None]
    return v.reshape(T, H * D)


@pytest.mark.parametrize("fmt", [MX, NV])
def test_scores_exact_on_representable_blocks(fmt):
    rng = np.random.default_rng(11 + fmt)
    Tq, Tk, H = 5, 131, 2
    G = oracle.group_size(fmt)
    q = _representable(rng, Tq, H, G)
    k = _representable(rng, Tk, H, G)
    qb, kb = synth.f32_to_bf16_bits(q.astype(np.float32)), synth.f32_to_bf16_bits(k.astype(np.float32))
    assert np.array_equal(synth.bf16_bits_to_f32(qb).astype(np.float64), q)  # exact in bf16
    g = 1.0 if fmt == NV else None
    qh = oracle.quantize_heads(fmt, qb, H, g)
    kh = oracle.quantize_heads(fmt, kb, H, g)
    for head in range(H):
        Y, S = oracle.attn_scores_rows(fmt, qh, kh, head, np.arange(Tq), g, g)
        ref = q[:, head * D:(head + 1) * D] @ k[:, head * D:(head + 1) * D].T
        np.testing.assert_array_equal(Y[:, :Tk], ref)
        assert not Y[:, Tk:].any(), "padding key columns must be 0"
        np.testing.assert_array_equal(S[:, :Tk], np.abs(q[:, head * D:(head + 1) * D]) @ np.abs(k[:, head * D:(head + 1) * D]).T)


def test_scores_select_the_head_and_rows():
    """Swapping heads or rows changes the result: the head index and the row selection are
    used as stated (a plausible slip -- head h read at h-1, rows ignored -- fails)."""
    rng = np.random.default_rng(5)
    q = _representable(rng, 4, 3, 32)
    k = _representable(rng, 7, 3, 32)
    qh = oracle.quantize_heads(MX, synth.f32_to_bf16_bits(q.astype(np.float32)), 3)
    kh = oracle.quantize_heads(MX, synth.f32_to_bf16_bits(k.astype(np.float32)), 3)
    rows = np.array([3, 1])
    Y, _ = oracle.attn_scores_rows(MX, qh, kh, 2, rows)
    np.testing.assert_array_equal(Y[:, :7], q[rows, 256:384] @ k[:, 256:384].T)
