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


# ------------------------------------------------------------------ V^T, softmax, P V
@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("T,H", [(1, 1), (130, 2), (257, 3)])
def test_quantize_heads_vt_is_the_row_quantizer_of_the_transpose(fmt, T, H):
    """Head h's V^T is the pinned row quantizer applied to the explicit transpose of its 128
    columns, zero-padded to Tpad tokens: codes and every scale byte (NVFP4 under V's global)."""
    x = _x(900 + T + H, T, H)
    g = oracle.nv_global(oracle.tensor_amax(x)) if fmt == NV else None
    codes, sfs = oracle.quantize_heads_vt(x, H, fmt, g)
    Tpad = (T + 127) // 128 * 128
    assert codes.shape == (H, D, Tpad // 2)
    for h in range(H):
        vt = np.zeros((D, Tpad), dtype=np.uint16)
        for t in range(T):
            for d in range(D):
                vt[d, t] = x[t, h * D + d]
        c, s = oracle.quantize(fmt, vt, g)
        np.testing.assert_array_equal(codes[h], c)
        np.testing.assert_array_equal(sfs[h], s)
        assert not codes[h][:, (T + 1) // 2:].any(), "padding tokens hold zero codes"


def test_quantize_heads_vt_single_token_worked():
    """One token, one head: each channel's first group holds the token's value and 31 zero
    tokens, so its scale comes from |v_d| alone and the code is e2m1(v_d / 2^e)."""
    v = np.array([[6.0, -3.0, 0.5, 0.0] + [1.0] * 124], dtype=np.float32)
    codes, sfs = oracle.quantize_heads_vt(synth.f32_to_bf16_bits(v), 1)
    # channel 0: amax 6 -> e = 0, code 6 = 0x7; channel 1: amax 3 -> e = -1, -3 / 2^-1 = -6 -> 0xF;
    # channel 2: 0.5 -> e = -3, 4 -> 0x6; channel 3: zero group -> byte 0, code 0
    assert [codes[0, d, 0] & 0xF for d in range(4)] == [0x7, 0xF, 0x6, 0x0]
    assert [sfs[0, oracle.sf_offset(d, 0, 128 // 32)] for d in range(4)] == [127, 126, 124, 0]
    assert not codes[0, :, 1:].any(), "padding tokens hold zero codes"


def test_softmax_oracle_against_closed_forms_and_scipy():
    from scipy.special import softmax

    rng = np.random.default_rng(3)
    s = synth.f32_to_bf16_bits(rng.normal(0, 4, size=(5, 384)).astype(np.float32))
    p, l, tmax = oracle.softmax_weights(s, 300, 0.125)
    sf = oracle.synth_bits_to_f64(s)
    c = oracle.softmax_c(0.125)
    ref = softmax(sf[:, :300] * c * np.log(2.0), axis=1)    # 2^(s c) = e^(s c ln 2)
    np.testing.assert_allclose(p[:, :300] / l[:, None], ref, rtol=1e-12, atol=0)
    assert not p[:, 300:].any()
    np.testing.assert_array_equal(p.max(axis=1), 1.0)      # the largest weight is exactly 1
    np.testing.assert_allclose(tmax, np.abs(sf[:, :300] * c).max(axis=1), rtol=0)
    # a constant row: every weight 1, l = T_kv; a row with one score far above the rest: l = 1
    const = np.full((1, 128), synth.f32_to_bf16_bits(np.float32([2.5]))[0], dtype=np.uint16)
    pc, lc, _ = oracle.softmax_weights(const, 100, 1.0)
    assert (pc[0, :100] == 1.0).all() and lc[0] == 100.0
    hot = np.zeros((1, 128), dtype=np.uint16)
    hot[0, 7] = synth.f32_to_bf16_bits(np.float32([1000.0]))[0]
    ph, lh, _ = oracle.softmax_weights(hot, 128, 1.0)
    assert ph[0, 7] == 1.0 and lh[0] == 1.0


def test_softmax_bounds_cover_an_fp32_evaluation():
    """numpy float32 steps as the library states them (fl(fl(s c) - m), exp2, sums per thread
    in the library's key order, then the block tree) stay inside the stated bounds of the
    fp64 weights and sum."""
    rng = np.random.default_rng(4)
    kpad, T_kv = 2048, 1990
    s = synth.f32_to_bf16_bits(rng.normal(0, 6, size=(3, kpad)).astype(np.float32))
    p, l, tmax = oracle.softmax_weights(s, T_kv, 0.088388)
    ew = oracle.softmax_weight_bound(tmax)
    el = oracle.softmax_sum_bound(kpad, tmax)
    c = np.float32(oracle.softmax_c(0.088388))
    sf = oracle.synth_bits_to_f64(s).astype(np.float32)
    for r in range(3):
        u = (sf[r] * c).astype(np.float32)
        m = u[:T_kv].max()
        e = np.zeros(kpad, dtype=np.float32)
        e[:T_kv] = np.exp2((u[:T_kv] - m).astype(np.float32)).astype(np.float32)
        rel = np.abs(e[:T_kv].astype(np.float64) - p[r, :T_kv]) / p[r, :T_kv]
        assert rel.max() <= ew[r], (rel.max(), ew[r])
        # thread t = 32 w + lane takes keys 256 (w + 8 k) + 8 lane .. + 7 in order
        part = np.zeros(256, dtype=np.float32)
        for chunk in range(kpad // 256):
            for lane in range(32):
                t = 32 * (chunk % 8) + lane
                for k in range(8):
                    part[t] = np.float32(part[t] + e[chunk * 256 + lane * 8 + k])
        tot = np.float32(0.0)
        for v in part:
            tot = np.float32(tot + v)
        assert abs(float(tot) - l[r]) <= el[r] * l[r], (abs(float(tot) - l[r]) / l[r], el[r])


def test_pv_oracle_nvfp4_exact_on_representable_blocks():
    """NVFP4 P V on operands exact under global 1 (E2M1 values times the block's power of two,
    each 16-block's amax 6 * 2^e, so the E4M3 block scale is 2^e) equals numpy's product of
    the original values; a P global of 1/2 halves it exactly (the globals are applied)."""
    rng = np.random.default_rng(7)
    Tq, Tk, H = 2, 64, 2
    kpad = 128
    pv = _representable(rng, Tq, 1, 16)[:, :kpad]
    pv[:, Tk:] = 0.0
    pc, ps = oracle.quantize(NV, synth.f32_to_bf16_bits(pv.astype(np.float32)), 1.0)
    vtv = _representable(rng, H * D, 1, 16)[:, :Tk]          # blocks of 16 tokens
    v = np.ascontiguousarray(vtv.T)
    vt = oracle.quantize_heads_vt(synth.f32_to_bf16_bits(v.astype(np.float32)), H, NV, 1.0)
    for head in range(H):
        ref = pv[:, :Tk] @ v[:, head * D:(head + 1) * D]
        Y, _ = oracle.pv_rows(pc, ps, vt, head, kpad, np.arange(Tq), NV, 1.0, 1.0)
        np.testing.assert_array_equal(Y, ref)
        Yh, _ = oracle.pv_rows(pc, ps, vt, head, kpad, np.arange(Tq), NV, 0.5, 1.0)
        np.testing.assert_array_equal(Yh, 0.5 * ref)


def test_pv_oracle_exact_on_representable_blocks():
    """P V on losslessly representable operands (P blocks of 32 keys and V blocks of 32 tokens
    on the E2M1 grid times the block's power of two, each block's amax 6 * 2^e) equals numpy's
    exact product of the original values, for each head; padding keys and tokens give 0."""
    rng = np.random.default_rng(6)
    Tq, Tk, H = 3, 160, 2                                    # 160 tokens = 5 whole groups
    kpad = 256
    pvals = _representable(rng, Tq, 2, 32)[:, :kpad]         # [Tq, 256] exact MX blocks
    pvals[:, Tk:] = 0.0
    pc, ps = oracle.quantize(MX, synth.f32_to_bf16_bits(pvals.astype(np.float32)))
    vtv = _representable(rng, H * D, 2, 32)[:, :Tk]          # [H*128 channels, Tk tokens]: blocks along tokens
    v = np.ascontiguousarray(vtv.T)                          # [Tk, H*128]
    vt = oracle.quantize_heads_vt(synth.f32_to_bf16_bits(v.astype(np.float32)), H)
    for head in range(H):
        Y, _ = oracle.pv_rows(pc, ps, vt, head, kpad, np.arange(Tq))
        np.testing.assert_array_equal(Y, pvals[:, :Tk] @ v[:, head * D:(head + 1) * D])
