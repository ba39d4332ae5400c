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
