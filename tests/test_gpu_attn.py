"""GPU parity of the FP4 attention operands: the head-major Q / K quantizer (bit-exact
against the oracle, every code and scale byte, padding included) and one head's score
GEMM S = deq(Q_h) deq(K_h)^T (every element at small sizes; at the Wan2.2 sequence
length of 75600 tokens and 40 heads of 128, sampled query rows -- every row of the ragged
last tile included -- against all 75648 key columns) within the GEMM tolerance."""
import numpy as np
import pytest

import oracle
import synth
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
MX, NV = oracle.MX, oracle.NV
D = 128


@pytest.fixture(scope="module")
def fb():
    import fp4_block_scaled_act_b200 as fb

    fb.build()
    return fb


@pytest.fixture(scope="module")
def orc():
    oracle.build()
    return oracle


def _inputs(orc, fmt, seed, T, Hn):
    x = synth.activation(seed, T, Hn * D, "lognormal", gain_seed=seed + 1)
    g = orc.nv_global(orc.tensor_amax(x)) if fmt == NV else None
    return x, g


def _gpu_heads(fb, fmt, x, Hn, g):
    import torch

    gd = H.dev_f32([g]) if fmt == NV else None
    codes, sf = fb.quantize_heads(H.dev_bf16(x), Hn, "mxfp4" if fmt == MX else "nvfp4", gd)
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    torch.cuda.synchronize()
    return codes, sf, gd


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("T,Hn", [(1, 1), (130, 3), (300, 40), (75600, 40)])
def test_quantize_heads_bit_exact(fb, orc, fmt, T, Hn):
    x, g = _inputs(orc, fmt, 3100 + T + Hn, T, Hn)
    c_ref, s_ref = orc.quantize_heads(fmt, x, Hn, g)
    codes, sf, _ = _gpu_heads(fb, fmt, x, Hn, g)
    assert tuple(codes.shape) == c_ref.shape and tuple(sf.shape) == s_ref.shape
    np.testing.assert_array_equal(H.host_u8(codes), c_ref)
    np.testing.assert_array_equal(H.host_u8(sf), s_ref)


def _scores_case(fb, orc, fmt, Tq, Tk, Hn, head, seed, rows=None):
    import torch

    q, g_q = _inputs(orc, fmt, seed, Tq, Hn)
    k, g_k = _inputs(orc, fmt, seed + 7, Tk, Hn)
    qc, qs, gq = _gpu_heads(fb, fmt, q, Hn, g_q)
    kc, ks, gk = _gpu_heads(fb, fmt, k, Hn, g_k)
    s = fb.attn_scores((qc, qs), (kc, ks), Tq, Tk, head, "mxfp4" if fmt == MX else "nvfp4", gq, gk)
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    rows = np.arange(Tq) if rows is None else rows
    y = s[torch.as_tensor(rows, device="cuda")]
    qh = orc.quantize_heads(fmt, q, Hn, g_q)
    kh = orc.quantize_heads(fmt, k, Hn, g_k)
    Y, S = orc.attn_scores_rows(fmt, qh, kh, head, rows, g_q, g_k)
    assert tuple(s.shape) == (Tq, (Tk + 127) // 128 * 128)
    H.check_linear(y, Y, S, np.arange(rows.size), f"scores fmt={fmt} Tq={Tq} Tk={Tk} H={Hn} head={head}")
    # the padding key columns hold exact zeros
    assert not y[:, Tk:].float().abs().sum().item()


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("Tq,Tk,Hn,head", [(1, 1, 1, 0), (130, 200, 3, 2), (300, 257, 2, 1), (600, 1000, 40, 39)])
def test_attn_scores_all_elements(fb, orc, fmt, Tq, Tk, Hn, head):
    _scores_case(fb, orc, fmt, Tq, Tk, Hn, head, seed=3300 + Tq + Tk)


@pytest.mark.parametrize("fmt", [MX, NV])
def test_attn_scores_full_size_sampled(fb, orc, fmt):
    """75600 query and key tokens, 40 heads: head 17's 75600 x 75648 scores (11.4 GB), on
    sampled query rows against every key column."""
    T = 75600
    rows = H.sample_rows(T, n_random=16, seed=17 + fmt)
    _scores_case(fb, orc, fmt, T, T, 40, 17, seed=3500 + fmt, rows=rows)


# ------------------------------------------------------------------ V^T, softmax + P quantize, P V
SCALE = 1.0 / np.sqrt(128.0)


def _fmt_name(fmt):
    return "mxfp4" if fmt == MX else "nvfp4"


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("T,Hn", [(1, 1), (130, 3), (300, 40), (75600, 40)])
def test_quantize_heads_vt_bit_exact(fb, orc, fmt, T, Hn):
    import torch

    v = synth.activation(3700 + T + Hn, T, Hn * D, "lognormal", gain_seed=3701)
    g = orc.nv_global(orc.tensor_amax(v)) if fmt == NV else None
    c_ref, s_ref = orc.quantize_heads_vt(v, Hn, fmt, g)
    codes, sf = fb.quantize_heads_vt(H.dev_bf16(v), Hn, _fmt_name(fmt), H.dev_f32([g]) if fmt == NV else None)
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(H.host_u8(codes), c_ref)
    np.testing.assert_array_equal(H.host_u8(sf), s_ref)


def _scores_bits(seed, Tq, kpad, T_kv, sigma=4.0):
    """Seeded bf16 scores [Tq, kpad]; the padding keys hold large values the softmax must ignore."""
    rng = np.random.default_rng(seed)
    s = rng.normal(0.0, sigma, size=(Tq, kpad)).astype(np.float32)
    s[:, T_kv:] = 1.0e4
    return synth.f32_to_bf16_bits(s)


def _check_p(orc, s_bits, T_kv, p_codes_h, p_sf_h, stats_h, rows, what, fmt=MX):
    """P~ codes / scales admissible for the fp64 weights 2^(s c - max) within the library's
    bound; stats' m exact (the fp32 maximum of fl(s c)), l within its bound of the exact sum."""
    p, l, tmax = orc.softmax_weights(s_bits, T_kv, SCALE)
    ew = orc.softmax_weight_bound(tmax)[:, None]
    tiny = 2.0 ** -125
    lo = np.maximum(p * (1 - ew) - tiny, 0.0)
    hi = p * (1 + ew) + tiny
    lo[:, T_kv:] = 0.0
    hi[:, T_kv:] = 0.0
    H.check_quant_of_interval(fmt, p_codes_h, p_sf_h, lo, hi, np.float32(orc.P_GLOBAL_NVFP4), what, row_ids=rows)
    c = np.float32(orc.softmax_c(SCALE))
    u = (orc.synth_bits_to_f64(s_bits)[:, :T_kv].astype(np.float32) * c).astype(np.float32)
    np.testing.assert_array_equal(stats_h[:, 0], u.max(axis=1))
    el = orc.softmax_sum_bound(s_bits.shape[1], tmax)
    assert (np.abs(stats_h[:, 1] - l) <= el * l).all(), what


def _row_scaled(o_raw_bits, l32):
    """bf16_rn(o * fl(1 / l)) row by row, as the library's row-scale step states it."""
    o = synth.bf16_bits_to_f32(o_raw_bits)
    inv = (np.float32(1.0) / l32.astype(np.float32)).astype(np.float32)
    return synth.f32_to_bf16_bits((o * inv[:, None]).astype(np.float32))


def _p_global(orc, fmt):
    return H.dev_f32([orc.P_GLOBAL_NVFP4]) if fmt == NV else None


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("Tq,T_kv", [(1, 1), (130, 200), (300, 257), (64, 75600), (8, 102500)])
def test_softmax_quant_admissible(fb, orc, fmt, Tq, T_kv):
    import torch

    from oracle import oracle_np as onp

    kpad = (T_kv + 127) // 128 * 128
    s_bits = _scores_bits(3800 + Tq + T_kv, Tq, kpad, T_kv)
    pc, ps, stats = fb.attn_softmax_quant(H.dev_bf16(s_bits), Tq, T_kv, SCALE, _fmt_name(fmt), _p_global(orc, fmt))
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    torch.cuda.synchronize()
    qpad = (Tq + 127) // 128 * 128
    sf_all = onp.unswizzle_sf(H.host_u8(ps), qpad, kpad // orc.group_size(fmt))
    assert not sf_all[Tq:].any(), "padding query rows hold zero scale bytes"
    _check_p(orc, s_bits, T_kv, H.host_u8(pc), sf_all[:Tq], stats.cpu().numpy(), np.arange(Tq),
             f"softmax fmt={fmt} Tq={Tq} T_kv={T_kv}", fmt)


def _resquare(orc, sf_rows, Kg):
    """Unswizzled scale bytes of R rows -> the atom layout of an [R, Kg * G] operand."""
    out = np.zeros(orc.sf_bytes(sf_rows.shape[0], Kg), dtype=np.uint8)
    for i in range(sf_rows.shape[0]):
        for j in range(Kg):
            out[orc.sf_offset(i, j, Kg)] = sf_rows[i, j]
    return out


def _pv_case(fb, orc, fmt, Tq, T_kv, Hn, head, seed, rows=None):
    import torch

    from oracle import oracle_np as onp

    kpad = (T_kv + 127) // 128 * 128
    G = orc.group_size(fmt)
    s_bits = _scores_bits(seed, Tq, kpad, T_kv, sigma=2.0)
    v = synth.activation(seed + 1, T_kv, Hn * D, "lognormal", gain_seed=seed + 2)
    g_v = orc.nv_global(orc.tensor_amax(v)) if fmt == NV else None
    gvd = H.dev_f32([g_v]) if fmt == NV else None
    gpd = _p_global(orc, fmt)
    pc, ps, stats = fb.attn_softmax_quant(H.dev_bf16(s_bits), Tq, T_kv, SCALE, _fmt_name(fmt), gpd)
    vt = fb.quantize_heads_vt(H.dev_bf16(v), Hn, _fmt_name(fmt), gvd)
    o = fb.attn_pv((pc, ps, stats), vt, Tq, T_kv, head, _fmt_name(fmt), gpd, gvd, normalize=False)
    o_n = fb.attn_pv((pc, ps, stats), vt, Tq, T_kv, head, _fmt_name(fmt), gpd, gvd)
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    torch.cuda.synchronize()
    rows = np.arange(Tq) if rows is None else rows
    vt_ref = orc.quantize_heads_vt(v, Hn, fmt, g_v)
    np.testing.assert_array_equal(H.host_u8(vt[0][head]), vt_ref[0][head])
    np.testing.assert_array_equal(H.host_u8(vt[1][head]), vt_ref[1][head])
    pc_h = H.host_u8(pc)[rows]
    qpad = (Tq + 127) // 128 * 128
    ps_rows = onp.unswizzle_sf(H.host_u8(ps), qpad, kpad // G)[rows]
    # the sampled rows' scales as a small [len(rows), kpad] operand for the oracle
    Y, S = orc.pv_rows(pc_h, _resquare(orc, ps_rows, kpad // G), vt_ref, head, kpad, np.arange(len(rows)), fmt,
                       float(np.float32(orc.P_GLOBAL_NVFP4)), g_v)
    H.check_linear(o[torch.as_tensor(rows, device="cuda")], Y, S, np.arange(len(rows)),
                   f"P V fmt={fmt} Tq={Tq} T_kv={T_kv} H={Hn} head={head}")
    # the normalized output is the unnormalized one scaled row by row, bit for bit
    o_bits = o.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    on_bits = o_n.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(on_bits, _row_scaled(o_bits, stats[:, 1].cpu().numpy()))
    return o


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("Tq,T_kv,Hn,head", [(1, 1, 1, 0), (130, 200, 3, 2), (300, 257, 2, 1), (200, 4096, 40, 39)])
def test_attn_pv_all_elements(fb, orc, fmt, Tq, T_kv, Hn, head):
    _pv_case(fb, orc, fmt, Tq, T_kv, Hn, head, seed=3900 + Tq + T_kv)


@pytest.mark.parametrize("fmt", [MX, NV])
def test_attn_chain_full_size_sampled(fb, orc, fmt):
    """The whole head at 75600 tokens, 40 heads, head 17: scores -> softmax + P quantize ->
    P V, each stage checked on sampled query rows against the oracle fed that stage's GPU input."""
    import torch

    from oracle import oracle_np as onp

    T, Hn, head = 75600, 40, 17
    kpad = 75648
    G = orc.group_size(fmt)
    name = _fmt_name(fmt)
    rows = H.sample_rows(T, n_random=12, seed=21)
    q = synth.activation(4100, T, Hn * D, "lognormal", gain_seed=4101)
    k = synth.activation(4102, T, Hn * D, "lognormal", gain_seed=4103)
    v = synth.activation(4104, T, Hn * D, "lognormal", gain_seed=4105)
    g = {n: (orc.nv_global(orc.tensor_amax(a)) if fmt == NV else None) for n, a in (("q", q), ("k", k), ("v", v))}
    gd = {n: (H.dev_f32([x]) if x is not None else None) for n, x in g.items()}
    gpd = _p_global(orc, fmt)
    qh = fb.quantize_heads(H.dev_bf16(q), Hn, name, gd["q"])
    kh = fb.quantize_heads(H.dev_bf16(k), Hn, name, gd["k"])
    s = fb.attn_scores(qh, kh, T, T, head, name, gd["q"], gd["k"])
    pc, ps, stats = fb.attn_softmax_quant(s, T, T, SCALE, name, gpd)
    vt = fb.quantize_heads_vt(H.dev_bf16(v), Hn, name, gd["v"])
    o = fb.attn_pv((pc, ps, stats), vt, T, T, head, name, gpd, gd["v"], normalize=False)
    o_n = fb.attn_pv((pc, ps, stats), vt, T, T, head, name, gpd, gd["v"])
    st = fb.fp4_sync_status()
    assert st == 0, fb.fp4_status_string(st)
    torch.cuda.synchronize()
    idx = torch.as_tensor(rows, device="cuda")
    s_bits = s[idx].contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    sf_all = onp.unswizzle_sf(H.host_u8(ps), kpad, kpad // G)
    _check_p(orc, s_bits, T, H.host_u8(pc[idx]), sf_all[rows], stats[idx].cpu().numpy(), rows,
             f"softmax full size fmt={fmt}", fmt)
    vt_ref = orc.quantize_heads_vt(v, Hn, fmt, g["v"])
    np.testing.assert_array_equal(H.host_u8(vt[0][head]), vt_ref[0][head])
    np.testing.assert_array_equal(H.host_u8(vt[1][head]), vt_ref[1][head])
    Y, S = orc.pv_rows(H.host_u8(pc[idx]), _resquare(orc, sf_all[rows], kpad // G), vt_ref, head, kpad,
                       np.arange(len(rows)), fmt, float(np.float32(orc.P_GLOBAL_NVFP4)), g["v"])
    H.check_linear(o[idx], Y, S, np.arange(len(rows)), f"P V full size fmt={fmt}")
    o_bits = o.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    on_bits = o_n.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(on_bits, _row_scaled(o_bits, stats[:, 1].cpu().numpy()))


def test_attn_chain_close_to_unquantized_attention(fb, orc):
    """Sanity of the wiring, not a parity claim: the FP4 chain's O against fp64 attention on
    the unquantized bf16 inputs (q, k ~ N(0, 1), so the softmax is not one-hot and FP4 noise
    in S cannot move its argmax).  The same chain emulated with the oracle (P rounded to
    bf16 before its quantization) gives row cosines of median 0.97, minimum 0.84 here;
    FP4 attention is coarse, as the card says of SageAttention v3."""
    import torch

    T, Hn, head = 1000, 2, 1
    rng = np.random.default_rng(4200)
    q = synth.f32_to_bf16_bits(rng.normal(size=(T, Hn * D)).astype(np.float32))
    k = synth.f32_to_bf16_bits(rng.normal(size=(T, Hn * D)).astype(np.float32))
    v = synth.activation(4202, T, Hn * D, "lognormal")
    qh = fb.quantize_heads(H.dev_bf16(q), Hn)
    kh = fb.quantize_heads(H.dev_bf16(k), Hn)
    s = fb.attn_scores(qh, kh, T, T, head)
    pc, ps, stats = fb.attn_softmax_quant(s, T, T, SCALE)
    o = fb.attn_pv((pc, ps, stats), fb.quantize_heads_vt(H.dev_bf16(v), Hn), T, T, head)
    torch.cuda.synchronize()
    of = H.host_bf16_as_f64(o)
    qf, kf, vf = (orc.synth_bits_to_f64(a)[:, head * D:(head + 1) * D] for a in (q, k, v))
    sc = qf @ kf.T * SCALE
    pr = np.exp(sc - sc.max(axis=1, keepdims=True))
    pr /= pr.sum(axis=1, keepdims=True)
    ref = pr @ vf
    cos = (of * ref).sum(1) / np.linalg.norm(of, axis=1) / np.linalg.norm(ref, axis=1)
    assert np.median(cos) > 0.95 and cos.min() > 0.7, (np.median(cos), cos.min())


def test_attn_chain_is_deterministic_and_replays_in_a_cuda_graph(fb, orc):
    """The head's kernels (quantizers, scores, softmax, P V, row scaling) allocate nothing
    and never synchronize: captured once in a CUDA graph and replayed on new inputs copied
    into the same buffers, they give bit for bit the eager results, which are themselves
    identical from run to run (every sum in a fixed order)."""
    import torch

    T, Hn, head = 700, 2, 1
    bufs = {n: torch.empty((T, Hn * D), dtype=torch.bfloat16, device="cuda") for n in "qkv"}
    qh = fb.quantize_heads(bufs["q"], Hn)
    kh = fb.quantize_heads(bufs["k"], Hn)
    vt = fb.quantize_heads_vt(bufs["v"], Hn)
    s = fb.attn_scores(qh, kh, T, T, head)
    p = fb.attn_softmax_quant(s, T, T, SCALE)
    o = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")

    def chain():
        fb.fp4_quantize_heads(MX, bufs["q"], T, Hn, D, None, qh[0], qh[1])
        fb.fp4_quantize_heads(MX, bufs["k"], T, Hn, D, None, kh[0], kh[1])
        fb.fp4_quantize_heads_vt(MX, bufs["v"], T, Hn, D, None, vt[0], vt[1])
        fb.attn_scores(qh, kh, T, T, head, s=s)
        fb.fp4_attn_softmax_quant(MX, s, T, T, SCALE, None, p[2], p[0], p[1])
        fb.attn_pv(p, vt, T, T, head, o=o)

    def load(seed):
        for i, n in enumerate("qkv"):
            bufs[n].copy_(H.dev_bf16(synth.activation(seed + i, T, Hn * D, "lognormal")))

    load(4300)
    chain()
    torch.cuda.synchronize()
    first = o.clone()
    chain()
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), o.view(torch.int16)), "two eager runs differ"
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        chain()
        side.synchronize()
        with torch.cuda.graph(graph, stream=side):
            chain()
    for seed in (4400, 4500):
        load(seed)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        replay = o.clone()
        chain()
        torch.cuda.synchronize()
        assert torch.equal(replay.view(torch.int16), o.view(torch.int16)), f"graph replay differs (seed {seed})"
    assert fb.fp4_sync_status() == 0
    del graph
