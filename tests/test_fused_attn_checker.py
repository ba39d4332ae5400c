"""CPU check of the stage-by-stage test used for the fused attention head
(tests/test_gpu_attn_fused._check_tile): a NumPy restatement of the kernel's stated steps
(per 256-key block: fp32 scores, the running maximum, the weights against it quantized by
the format's rule, O and the quarter sums rescaled when the maximum grows, O / l at the end)
passes it in both formats, and planted mistakes in that restatement are caught: O or l not
rescaled, the factor inverted, the block's own maximum used instead of the running one, one
code changed."""
import numpy as np
import pytest

import oracle
import synth
from oracle import oracle_np as onp
from tests import test_gpu_attn_fused as F

f32 = np.float32


def _restate(fmt, Tq, Tk, Hn, head, seed, plant=None):
    """The kernel's steps for the first query tile, in NumPy fp32 where the kernel is fp32;
    returns _check_tile's arguments."""
    import torch

    D = 128
    q = F._normal_bits(seed, Tq, Hn * D)
    k = F._normal_bits(seed + 1, Tk, Hn * D)
    v = synth.activation(seed + 2, Tk, Hn * D, "lognormal")
    nv = fmt == oracle.NV
    g = None
    if nv:
        g = {n: oracle.nv_global(oracle.tensor_amax(x)) for n, x in (("q", q), ("k", k), ("v", v))}
        g["p"] = float(f32(oracle.P_GLOBAL_NVFP4))
    gq, gk, gv, gp = (g["q"], g["k"], g["v"], g["p"]) if nv else (None, None, None, None)
    cols = slice(head * D, (head + 1) * D)
    qh = oracle.quantize_heads(fmt, np.ascontiguousarray(q[:, cols]), 1, gq)
    kh = oracle.quantize_heads(fmt, np.ascontiguousarray(k[:, cols]), 1, gk)
    vt = oracle.quantize_heads_vt(np.ascontiguousarray(v[:, cols]), 1, fmt, gv)
    tk_pad = (Tk + 127) // 128 * 128
    nb = (tk_pad + 255) // 256
    G = 16 if nv else 32
    ng = 256 // G
    rows = np.arange(min(Tq, 128))
    R = len(rows)
    Y, _ = oracle.attn_scores_rows(fmt, qh, kh, 0, rows, gq, gk)
    c = f32(oracle.softmax_c(F.SCALE))
    if nv:
        acc = (Y / (gq * gk)).astype(f32)
        cc = f32(c * f32(f32(gq) * f32(gk)))
    else:
        acc = Y.astype(f32)
        cc = c
    m_run = np.full(R, -np.inf, f32)
    lq = np.zeros((4, R), f32)
    O = np.zeros((R, D))
    tm = np.zeros((nb, 128), f32)
    tc = np.zeros((nb, 128, 128), np.uint8)
    ts = np.zeros((nb, 128, ng), np.uint8)
    w = oracle.dequant_fp4(fmt, vt[0][0], vt[1][0], tk_pad, 1.0)  # without V's global
    wf = np.zeros((D, nb * 256))
    wf[:, :tk_pad] = w
    for j in range(nb):
        valid = np.arange(j * 256, (j + 1) * 256) < Tk
        sb = np.zeros((R, 256), f32)
        n = min(256, tk_pad - j * 256)
        sb[:, :n] = acc[:, j * 256:j * 256 + n]
        mb = f32(np.where(valid[None, :], sb, -np.inf).max(1).astype(f32) * cc)
        mn = mb if plant == "block_max" else np.maximum(m_run, mb).astype(f32)
        if j > 0:
            f = np.exp2((m_run - mn).astype(f32).astype(np.float64)).astype(f32)
            if plant == "inverse_factor":
                f = (f32(1) / f).astype(f32)
            if plant != "no_l_rescale":
                lq = (lq * f[None, :]).astype(f32)
            if plant != "no_o_rescale":
                O = O * f[:, None]
        t = ((sb * cc).astype(f32) - mn[:, None]).astype(f32)
        p = np.where(valid[None, :], np.exp2(t.astype(np.float64)).astype(f32), f32(0)).astype(f32)
        for qq in range(4):
            lq[qq] = (lq[qq] + p[:, 64 * qq:64 * qq + 64].astype(np.float64).sum(1)).astype(f32)
        amax = p.reshape(R, ng, G).max(-1)
        if nv:
            six_g = f32(6.0 * f32(gp))
            sfb = onp.e4m3_encode((amax.astype(f32) / six_g).astype(f32)).astype(np.int64)
            d = (onp.e4m3_decode(sfb).astype(f32) * f32(gp)).astype(f32)
            rr = np.where(d != 0, f32(1.0) / np.where(d != 0, d, f32(1.0)), f32(0)).astype(f32)
            sc = (p.reshape(R, ng, G) * rr[..., None]).reshape(R, 256).astype(f32)
        else:
            eb = (amax.view(np.uint32) >> 23).astype(np.int64)
            sfb = np.maximum(eb - 2, 0)
            sc = (p.reshape(R, ng, G) * np.ldexp(1.0, 127 - sfb)[..., None]).reshape(R, 256).astype(f32)
        codes = onp.e2m1_encode(sc)
        if plant == "code" and j == nb - 1:
            codes[0, 0] = (codes[0, 0] + 3) % 8  # a different magnitude, same sign
        packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
        tm[j, :R], tc[j, :R], ts[j, :R] = mn, packed, sfb
        deq = oracle.dequant_nv_rows(packed, sfb, 1.0) if nv else oracle.dequant_mx_rows(packed, sfb)
        O = O + deq @ wf[:, j * 256:(j + 1) * 256].T
        m_run = mn
    lt = f32(f32(lq[0] + lq[1]) + f32(lq[2] + lq[3]))
    inv = (f32(1) / lt).astype(f32)
    if nv:
        inv = (f32(f32(gp) * f32(gv)) * inv).astype(f32)
    ob = synth.f32_to_bf16_bits((O * inv.astype(np.float64)[:, None]).astype(f32))
    o = torch.zeros((Tq, D), dtype=torch.bfloat16)
    o[:R] = torch.from_numpy(ob.view(np.int16)).view(torch.bfloat16)
    stats = torch.zeros((Tq, 2))
    stats[:R, 0] = torch.from_numpy(m_run)
    stats[:R, 1] = torch.from_numpy(lt)
    trace = (torch.from_numpy(tm), torch.from_numpy(tc), torch.from_numpy(ts))
    return (oracle, f"restated fmt={fmt}", 0, Tq, Tk, head, qh, kh, vt, o, stats, trace, fmt, g)


@pytest.mark.parametrize("fmt", [oracle.MX, oracle.NV])
@pytest.mark.parametrize("Tq,Tk,Hn,head", [(130, 700, 2, 1), (1, 1, 1, 0), (128, 300, 3, 2)])
def test_checker_accepts_the_stated_steps(fmt, Tq, Tk, Hn, head):
    oracle.build()
    F._check_tile(*_restate(fmt, Tq, Tk, Hn, head, seed=77 + Tk))


@pytest.mark.parametrize("fmt", [oracle.MX, oracle.NV])
@pytest.mark.parametrize("plant", ["no_o_rescale", "no_l_rescale", "inverse_factor", "block_max", "code"])
def test_checker_catches_planted_mistakes(fmt, plant):
    oracle.build()
    with pytest.raises(AssertionError):
        F._check_tile(*_restate(fmt, 130, 700, 2, 1, seed=777, plant=plant))
