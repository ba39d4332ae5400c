"""GPU parity of the fused FP4 attention kernel (fp4_attn_fused, MXFP4 and NVFP4), the streaming form of one
head's FP4 attention (Wan2.2-Animate-14B MXFP4 card, "Results": FP4 attention with
microscaling on Blackwell; no page gives its algorithm).

The kernel keeps S in fp32 and takes the keys in blocks of 256, so it is checked stage by
stage on whole query tiles through its trace outputs, each stage against the oracle fed the
exact scores of the oracle's own quantized Q and K:
  - every block's running maximum m_j within the scores' fp32 tolerance of the exact one;
  - every P~_j code and scale byte admissible for the exact weights 2^(s c - m_j) over the
    interval the score error, the two fp32 roundings and exp2f allow;
  - l within its stated bound of the exact sum of 2^(s c - m_last), stats' m equal to the
    last traced m_j;
  - O against sum_j 2^(m_j - m_last) deq(P~_j) deq(V_j) / l computed by the oracle from the
    traced codes, within the accumulation tolerance plus the rescaling factors' error.
Sizes span one 128-row tile up to the Wan2.2 sequence length (75600 tokens, 40 heads), with
ragged query tiles and key blocks, the last head (whose final key block runs past the
buffer) and a head whose final block reads the next head's rows (masked)."""
import math

import numpy as np
import pytest

import oracle
import synth
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
MX, NV = oracle.MX, oracle.NV
D = 128
SCALE = 1.0 / math.sqrt(D)
ACC_TOL = 1e-5  # fp32 accumulation of a block-scaled product (the GEMM tolerance)


@pytest.fixture(scope="module")
def fb():
    import fp4_block_scaled_act_b200 as fb

    fb.build()
    return fb


@pytest.fixture(scope="module")
def orc():
    oracle.build()
    return oracle


def _normal_bits(seed, T, K, sigma=1.0):
    rng = np.random.default_rng(seed)
    return synth.f32_to_bf16_bits(rng.normal(0.0, sigma, size=(T, K)).astype(np.float32))


def _check_tile(orc, what, t, Tq, Tk, head, q_head, k_head, vt_ref, o, stats, trace, fmt=MX, g=None):
    """One traced query tile against the oracle (q_head, k_head: the oracle's head-major
    buffers of this head alone, vt_ref its V^T; g: NVFP4's globals q, k, v, p as fp32 values)."""
    tm, tc, ts = (a.cpu().numpy() for a in trace)
    nb = tm.shape[0]
    G = orc.group_size(fmt)
    tk_pad = (Tk + 127) // 128 * 128
    r0, r1 = t * 128, min(Tq, t * 128 + 128)
    rows = np.arange(r0, r1)
    lr = rows - r0
    gq, gk, gv, gp = (g["q"], g["k"], g["v"], g["p"]) if fmt == NV else (None, None, None, None)
    Y, S = orc.attn_scores_rows(fmt, q_head, k_head, 0, rows, gq, gk)
    es = ACC_TOL * S
    c = orc.softmax_c(SCALE)
    # NVFP4 folds the scores' globals into the exponent multiplier: two more roundings
    rel = 2.0 ** -22 if fmt == NV else 2.0 ** -23
    m_gpu = tm[:, lr].T.astype(np.float64)                          # [R, nb]
    # running maxima: within the scores' error and the roundings of s c
    m_ref = orc.flash_maxima(Y, Tk, SCALE)
    u = np.abs(Y[:, :Tk]) * c
    dm = (c * es[:, :Tk] + rel * u).max(axis=1)
    bad = np.abs(m_gpu - m_ref) > dm[:, None]
    assert not bad.any(), f"{what} tile {t}: running maxima off, first at {np.argwhere(bad)[0]}"
    assert (np.diff(m_gpu, axis=1) >= 0).all(), f"{what}: running maxima fall"
    # the weights' codes and scales
    codes = tc[:, lr, :].transpose(1, 0, 2).reshape(len(rows), nb * 128)
    sf = ts[:, lr, :].transpose(1, 0, 2).reshape(len(rows), nb * 256 // G)
    lo, hi = orc.flash_weight_interval(Y, es, Tk, SCALE, m_gpu, rel=rel)
    H.check_quant_of_interval(fmt, codes, sf, lo, hi, np.float32(gp) if fmt == NV else None,
                              f"{what} tile {t} P~", row_ids=rows)
    # stats: m is the last running maximum; l within its bound
    st = stats[r0:r1].cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(st[:, 0], m_gpu[:, -1])
    l_gpu = st[:, 1]
    l_ref = orc.flash_sum(Y, Tk, SCALE, m_gpu[:, -1])
    d = c * es[:, :Tk] + rel * (u + np.abs(m_gpu[:, -1:]))
    e_w = np.log(2.0) * d.max(axis=1) * 1.01 + 2.0 ** -21
    e_f = nb * (2.0 ** -22 + 2.0 ** -24) + np.log(2.0) * 2.0 ** -24 * (m_gpu[:, -1] - m_gpu[:, 0])
    e_l = 2.0 * (e_w + (16 + 2 * nb) * 2.0 ** -24 + e_f)
    bad = np.abs(l_gpu - l_ref) > e_l * l_ref
    assert not bad.any(), f"{what} tile {t}: l off, first row {rows[np.argwhere(bad)[0][0]]}"
    # O = sum_j 2^(m_j - m_last) deq(P~_j) deq(V_j) / l
    Yo, So = orc.flash_pv_rows(codes, sf, m_gpu, vt_ref, 0, tk_pad, fmt=fmt, g_p=gp, g_v=gv)
    # NVFP4: fl(g_p g_v) and its product with fl(1 / l), two more roundings
    e_acc = (4 * nb + 8) * 2.0 ** -24 + e_f + 2.0 ** -22 + (2.0 ** -22 if fmt == NV else 0.0)
    Sn = So * (1.0 + e_acc[:, None] / ACC_TOL) / l_gpu[:, None]
    H.check_linear(o, Yo / l_gpu[:, None], Sn, rows, f"{what} tile {t} O")


def _globals(orc, fmt, tensors):
    """NVFP4: each tensor's global from its own amax, and P~'s constant (fp32 values and device
    scalars); MXFP4: none."""
    if fmt == MX:
        return None, {"q": None, "k": None, "v": None, "p": None}
    g = {n: orc.nv_global(orc.tensor_amax(x)) for n, x in tensors.items()}
    g["p"] = float(np.float32(orc.P_GLOBAL_NVFP4))
    return g, {n: H.dev_f32([x]) for n, x in g.items()}


def _fused(fb, fmt, qh, kh, vt, Tq, Tk, head, gd, **kw):
    return fb.attn_fused(qh, kh, vt, Tq, Tk, head, SCALE, "mxfp4" if fmt == MX else "nvfp4", gd["q"], gd["k"],
                         gd["v"], gd["p"], **kw)


def _run_case(fb, orc, Tq, Tk, Hn, head, seed, tiles=None, v_dist="lognormal", fmt=MX):
    import torch

    q = _normal_bits(seed, Tq, Hn * D)
    k = _normal_bits(seed + 1, Tk, Hn * D)
    v = synth.activation(seed + 2, Tk, Hn * D, v_dist)
    g, gd = _globals(orc, fmt, {"q": q, "k": k, "v": v})
    name = "mxfp4" if fmt == MX else "nvfp4"
    qh = fb.quantize_heads(H.dev_bf16(q), Hn, name, gd["q"])
    kh = fb.quantize_heads(H.dev_bf16(k), Hn, name, gd["k"])
    vt = fb.quantize_heads_vt(H.dev_bf16(v), Hn, name, gd["v"])
    cols = slice(head * D, (head + 1) * D)
    gq, gk, gv = (g["q"], g["k"], g["v"]) if fmt == NV else (None, None, None)
    q_head = orc.quantize_heads(fmt, np.ascontiguousarray(q[:, cols]), 1, gq)
    k_head = orc.quantize_heads(fmt, np.ascontiguousarray(k[:, cols]), 1, gk)
    vt_ref = orc.quantize_heads_vt(np.ascontiguousarray(v[:, cols]), 1, fmt, gv)
    np.testing.assert_array_equal(H.host_u8(vt[0][head]), vt_ref[0][0])
    np.testing.assert_array_equal(H.host_u8(vt[1][head]), vt_ref[1][0])
    n_tiles = (Tq + 127) // 128
    tiles = range(n_tiles) if tiles is None else tiles
    o_plain = _fused(fb, fmt, qh, kh, vt, Tq, Tk, head, gd)
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    for t in tiles:
        stats = torch.empty((Tq, 2), dtype=torch.float32, device="cuda")
        o, trace = _fused(fb, fmt, qh, kh, vt, Tq, Tk, head, gd, stats=stats, trace_tile=t)
        st = fb.fp4_sync_status()
        assert st == 0, fb.fp4_status_string(st)
        torch.cuda.synchronize()
        # tracing changes nothing in the output
        assert torch.equal(o.view(torch.int16), o_plain.view(torch.int16))
        _check_tile(orc, f"fused fmt={fmt} Tq={Tq} Tk={Tk} H={Hn} head={head}", t, Tq, Tk, head, q_head, k_head,
                    vt_ref, o, stats, trace, fmt, g)
    assert torch.isfinite(o_plain.float()).all()
    return o_plain


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("Tq,Tk,Hn,head", [(1, 1, 1, 0), (130, 200, 3, 2), (300, 257, 2, 0), (128, 256, 1, 0),
                                           (200, 4096, 40, 39), (129, 1000, 2, 1)])
def test_attn_fused_every_tile(fb, orc, fmt, Tq, Tk, Hn, head):
    _run_case(fb, orc, Tq, Tk, Hn, head, seed=5000 + Tq + Tk + head, fmt=fmt)


@pytest.mark.parametrize("fmt", [MX, NV])
def test_attn_fused_growing_maximum(fb, orc, fmt):
    """Scores that grow along the keys, so the running maximum rises in nearly every block and
    O and l are rescaled each time (q . k increases with the key index)."""
    import torch

    Tq, Tk, Hn, head = 200, 3000, 1, 0
    rng = np.random.default_rng(5100)
    q = np.abs(rng.normal(size=(Tq, D))).astype(np.float32)
    k = (np.abs(rng.normal(size=(Tk, D))) * np.linspace(0.2, 1.5, Tk)[:, None]).astype(np.float32)
    qb, kb = synth.f32_to_bf16_bits(q), synth.f32_to_bf16_bits(k)
    v = synth.activation(5101, Tk, D, "lognormal")
    g, gd = _globals(orc, fmt, {"q": qb, "k": kb, "v": v})
    name = "mxfp4" if fmt == MX else "nvfp4"
    qh = fb.quantize_heads(H.dev_bf16(qb), Hn, name, gd["q"])
    kh = fb.quantize_heads(H.dev_bf16(kb), Hn, name, gd["k"])
    vt = fb.quantize_heads_vt(H.dev_bf16(v), Hn, name, gd["v"])
    gq, gk, gv = (g["q"], g["k"], g["v"]) if fmt == NV else (None, None, None)
    q_head = orc.quantize_heads(fmt, qb, 1, gq)
    k_head = orc.quantize_heads(fmt, kb, 1, gk)
    vt_ref = orc.quantize_heads_vt(v, 1, fmt, gv)
    for t in range(2):
        stats = torch.empty((Tq, 2), dtype=torch.float32, device="cuda")
        o, trace = _fused(fb, fmt, qh, kh, vt, Tq, Tk, head, gd, stats=stats, trace_tile=t)
        st = fb.fp4_sync_status()
        assert st == 0, fb.fp4_status_string(st)
        torch.cuda.synchronize()
        m = trace[0].cpu().numpy()[:, :min(128, Tq - 128 * t)]
        assert (np.diff(m, axis=0) > 0).mean() > 0.6, "the maximum should grow in most blocks"
        _check_tile(orc, f"fused growing fmt={fmt}", t, Tq, Tk, head, q_head, k_head, vt_ref, o, stats, trace, fmt, g)


@pytest.mark.parametrize("fmt", [MX, NV])
def test_attn_fused_full_size_traced_tiles(fb, orc, fmt):
    """The Wan2.2 sequence length, 75600 tokens of 40 heads, head 17: the first query tile and
    the ragged last one (80 rows) checked stage by stage over all 296 key blocks."""
    T, Hn, head = 75600, 40, 17
    _run_case(fb, orc, T, T, Hn, head, seed=5200, tiles=[0, (T + 127) // 128 - 1], fmt=fmt)


def test_attn_fused_close_to_the_separate_chain_and_exact_attention(fb, orc):
    """Sanity of the wiring, not a parity claim: on q, k ~ N(0, 1) the fused head's output
    has row cosines against fp64 attention on the unquantized inputs like the separate-kernel
    chain's (median > 0.95, minimum > 0.7), and against that chain's output above 0.9."""
    import torch

    T, Hn, head = 1000, 2, 1
    q = _normal_bits(4200, T, Hn * D)
    k = _normal_bits(4201, T, Hn * D)
    v = synth.activation(4202, T, Hn * D, "lognormal")
    qh = fb.quantize_heads(H.dev_bf16(q), Hn)
    kh = fb.quantize_heads(H.dev_bf16(k), Hn)
    vt = fb.quantize_heads_vt(H.dev_bf16(v), Hn)
    o = fb.attn_fused(qh, kh, vt, T, T, head, SCALE)
    s = fb.attn_scores(qh, kh, T, T, head)
    pc, ps, stats = fb.attn_softmax_quant(s, T, T, SCALE)
    o_sep = fb.attn_pv((pc, ps, stats), vt, T, T, head)
    torch.cuda.synchronize()
    of, osep = H.host_bf16_as_f64(o), H.host_bf16_as_f64(o_sep)
    qf, kf, vf = (orc.synth_bits_to_f64(a)[:, head * D:(head + 1) * D] for a in (q, k, v))
    sc = qf @ kf.T * SCALE
    pr = np.exp(sc - sc.max(axis=1, keepdims=True))
    pr /= pr.sum(axis=1, keepdims=True)
    ref = pr @ vf

    def cos(a, b):
        return (a * b).sum(1) / np.linalg.norm(a, axis=1) / np.linalg.norm(b, axis=1)

    c_ref = cos(of, ref)
    assert np.median(c_ref) > 0.95 and c_ref.min() > 0.7, (np.median(c_ref), c_ref.min())
    assert cos(of, osep).min() > 0.9


def test_attn_fused_is_deterministic_and_replays_in_a_cuda_graph(fb, orc):
    """Two eager runs give the same bits; the call captured in a CUDA graph and replayed on new
    inputs copied into the same buffers gives the eager result bit for bit."""
    import torch

    T, Hn, head = 700, 2, 1
    bufs = {n: torch.empty((T, Hn * D), dtype=torch.bfloat16, device="cuda") for n in "qkv"}
    qh = fb.quantize_heads(bufs["q"], Hn)
    kh = fb.quantize_heads(bufs["k"], Hn)
    vt = fb.quantize_heads_vt(bufs["v"], Hn)
    o = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    stats = torch.empty((T, 2), dtype=torch.float32, device="cuda")

    def head_call():
        fb.fp4_quantize_heads(MX, bufs["q"], T, Hn, D, None, qh[0], qh[1])
        fb.fp4_quantize_heads(MX, bufs["k"], T, Hn, D, None, kh[0], kh[1])
        fb.fp4_quantize_heads_vt(MX, bufs["v"], T, Hn, D, None, vt[0], vt[1])
        fb.attn_fused(qh, kh, vt, T, T, head, SCALE, o=o, stats=stats)

    def load(seed):
        for i, n in enumerate("qkv"):
            bufs[n].copy_(H.dev_bf16(synth.activation(seed + i, T, Hn * D, "lognormal")))

    load(5300)
    head_call()
    torch.cuda.synchronize()
    first = o.clone()
    head_call()
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), o.view(torch.int16)), "two eager runs differ"
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        head_call()
        side.synchronize()
        with torch.cuda.graph(graph, stream=side):
            head_call()
    for seed in (5400, 5500):
        load(seed)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        replay = o.clone()
        head_call()
        torch.cuda.synchronize()
        assert torch.equal(replay.view(torch.int16), o.view(torch.int16)), f"graph replay differs (seed {seed})"
    assert fb.fp4_sync_status() == 0
    del graph
