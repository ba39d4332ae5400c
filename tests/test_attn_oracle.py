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


# ------------------------------------------------------------------ streaming (flash) form


def test_dequant_mx_rows_matches_the_atom_layout_dequantizer():
    """Row-order MXFP4 dequantization equals the pinned dequantizer fed the same bytes in the
    128x4 atom layout."""
    rng = np.random.default_rng(11)
    R, K = 130, 512
    codes = rng.integers(0, 256, size=(R, K // 2), dtype=np.uint8)
    sf = rng.integers(100, 150, size=(R, K // 32), dtype=np.uint8)
    atoms = np.zeros(oracle.sf_bytes(R, K // 32), dtype=np.uint8)
    for i in range(R):
        for j in range(K // 32):
            atoms[oracle.sf_offset(i, j, K // 32)] = sf[i, j]
    np.testing.assert_array_equal(oracle.dequant_mx_rows(codes, sf), oracle.dequant_fp4(MX, codes, atoms, K))


def test_dequant_nv_rows_matches_the_atom_layout_dequantizer():
    """Row-order NVFP4 dequantization (E4M3 scales, a global) equals the pinned dequantizer
    fed the same bytes in the 128x4 atom layout."""
    rng = np.random.default_rng(15)
    R, K, g = 130, 256, 0.0123
    codes = rng.integers(0, 256, size=(R, K // 2), dtype=np.uint8)
    sf = rng.integers(0, 127, size=(R, K // 16), dtype=np.uint8)
    atoms = np.zeros(oracle.sf_bytes(R, K // 16), dtype=np.uint8)
    for i in range(R):
        for j in range(K // 16):
            atoms[oracle.sf_offset(i, j, K // 16)] = sf[i, j]
    np.testing.assert_array_equal(oracle.dequant_nv_rows(codes, sf, g), oracle.dequant_fp4(NV, codes, atoms, K, g))


def test_flash_maxima_and_sum_reduce_to_the_plain_softmax():
    """The last running maximum is the row maximum of s c, the maxima never fall, a block's
    maximum is reached inside it or before; with m_last the flash sum is the plain softmax
    oracle's l (which scipy pins)."""
    rng = np.random.default_rng(12)
    T_kv, scale = 1000, 0.0883883
    s = rng.normal(0.0, 4.0, size=(5, 1024)).astype(np.float32).astype(np.float64)
    m = oracle.flash_maxima(s, T_kv, scale)
    c = oracle.softmax_c(scale)
    assert m.shape == (5, 4)
    np.testing.assert_array_equal(m[:, -1], (s[:, :T_kv] * c).max(axis=1))
    assert (np.diff(m, axis=1) >= 0).all()
    np.testing.assert_array_equal(m[:, 0], (s[:, :256] * c).max(axis=1))
    bits = synth.f32_to_bf16_bits(s.astype(np.float32))
    sb = oracle.synth_bits_to_f64(bits)
    _, l_plain, _ = oracle.softmax_weights(bits, T_kv, scale)
    l_flash = oracle.flash_sum(sb, T_kv, scale, oracle.flash_maxima(sb, T_kv, scale)[:, -1])
    np.testing.assert_allclose(l_flash, l_plain, rtol=1e-13)


def test_flash_combine_is_softmax_attention_without_quantization():
    """Unquantized streaming weights combined by flash_combine and divided by flash_sum equal
    softmax(s scale) V computed by scipy, for a key count with a ragged last block."""
    from scipy.special import softmax

    rng = np.random.default_rng(13)
    T_kv, scale, R = 700, 0.125, 6
    s = rng.normal(0.0, 6.0, size=(R, T_kv))
    # a late key with a much larger score forces the maxima to grow block by block
    s[:, 650] += 30.0
    v = rng.normal(size=(T_kv, 128))
    m = oracle.flash_maxima(s, T_kv, scale)
    p = oracle.flash_weights(s, T_kv, scale, m)
    Y, _ = oracle.flash_combine(p, m, v.T)
    l = oracle.flash_sum(s, T_kv, scale, m[:, -1])
    c = oracle.softmax_c(scale)
    ref = softmax(s * c * np.log(2.0), axis=1) @ v
    np.testing.assert_allclose(Y / l[:, None], ref, rtol=1e-10, atol=1e-12)


def test_flash_combine_worked_two_blocks():
    """Block 0 of ones against m_0 = m_1 - 1, block 1 of halves, V of ones: each output is
    2^-1 * 256 + 0.5 * 256 = 256 (a reversed factor 2^(m_last - m_j) would give 640)."""
    p = np.concatenate([np.ones((2, 256)), np.full((2, 256), 0.5)], axis=1)
    m = np.array([[3.0, 4.0], [-7.5, -6.5]])
    Y, S = oracle.flash_combine(p, m, np.ones((128, 512)))
    np.testing.assert_array_equal(Y, np.full((2, 128), 256.0))
    np.testing.assert_array_equal(S, Y)


def test_flash_weight_interval_holds_an_fp32_evaluation():
    """For fp32 scores s' within es of s and m_j the fp32 running maxima of fl(s' c) (what a
    kernel computes), the fp32 weights exp2(fl(fl(s' c) - m_j)) lie in the interval built on
    the exact s (numpy's exp2 in fp64 rounded to fp32 stands in for a 2-ulp exp2f)."""
    rng = np.random.default_rng(14)
    T_kv, scale, R = 600, 0.0883883, 4
    s = rng.normal(0.0, 8.0, size=(R, 768))
    es = np.abs(s) * 1e-5 + 1e-3
    c = np.float32(oracle.softmax_c(scale))
    for pert in (-es, es, es * rng.uniform(-1, 1, size=s.shape), 0.0 * es):
        s32 = (s + pert).astype(np.float32)
        u = (s32[:, :T_kv] * c).astype(np.float32)
        full = np.full((R, 768), -np.inf, dtype=np.float32)
        full[:, :T_kv] = u
        mj = np.maximum.accumulate(full.reshape(R, 3, 256).max(axis=2), axis=1)
        lo, hi = oracle.flash_weight_interval(s, es, T_kv, scale, mj.astype(np.float64))
        t = (u - np.repeat(mj, 256, axis=1)[:, :T_kv]).astype(np.float32)
        w = np.exp2(t.astype(np.float64)).astype(np.float32).astype(np.float64)
        assert (w >= lo[:, :T_kv]).all() and (w <= hi[:, :T_kv]).all()
        assert (lo[:, T_kv:] == 0).all() and (hi[:, T_kv:] == 0).all()
    # an interval without the score error misses some of the perturbed weights
    s32 = (s + es).astype(np.float32)
    u = (s32[:, :T_kv] * c).astype(np.float32)
    full = np.full((R, 768), -np.inf, dtype=np.float32)
    full[:, :T_kv] = u
    mj = np.maximum.accumulate(full.reshape(R, 3, 256).max(axis=2), axis=1)
    lo, hi = oracle.flash_weight_interval(s, 0.0 * es, T_kv, scale, mj.astype(np.float64))
    t = (u - np.repeat(mj, 256, axis=1)[:, :T_kv]).astype(np.float32)
    w = np.exp2(t.astype(np.float64)).astype(np.float32).astype(np.float64)
    assert not ((w >= lo[:, :T_kv]).all() and (w <= hi[:, :T_kv]).all())
