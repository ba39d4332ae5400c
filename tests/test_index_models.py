"""CPU models of the GPU kernels' index arithmetic (in place of a sanitizer, which this GPU
pool does not offer): each test restates one kernel's work assignment as written in
fp4_block_scaled_act_b200/csrc and checks, over many shapes, that every unit of work is
done exactly once, that positions computed incrementally equal the direct ones, and that
every load and store stays inside its buffer.  A change to a kernel's indexing must be
mirrored here."""
import itertools

import pytest

QUANT_THREADS, QUANT_UNROLL = 256, 6           # quant.cuh
LR_ROWS, LR_THREADS, LR_KC = 128, 256, 64       # quant.cuh (low-rank projection)
SMS, QUANT_OCC = 148, 4                         # B200; resident quantize CTAs per SM


def sf_word_offset(r, atom_k, apr):
    """quant.cuh: byte offset of the 32-bit scale word of row r, atom atom_k."""
    return ((r >> 7) * apr + atom_k) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4


def quant_blocks(M, K):
    """fp4bsa.cu: one resident wave, at most one CTA per span of units."""
    units = (M + 127) // 128 * 128 * (K // 128)
    span = (QUANT_THREADS // 16) * QUANT_UNROLL
    return max(1, min(-(-units // span), SMS * QUANT_OCC))


def quant_walk(M, K, G):
    """quant_kernel: yields (u, row, chunk) per unit a half-warp processes, checking loads."""
    grid = quant_blocks(M, K)
    UPB = QUANT_THREADS // 16
    upr = K >> 7
    Mpad = (M + 127) // 128 * 128
    total = Mpad * upr
    span = UPB * QUANT_UNROLL
    per_cta = (-(-total // grid) + span - 1) // span * span
    adv_rows, adv_chunk = UPB // upr, UPB % upr
    for b in range(grid):
        u_begin = b * per_cta
        u_end = min(total, u_begin + per_cta)
        for my in range(UPB):
            row, chunk = divmod(u_begin + my, upr)
            for ub in range(u_begin, u_end, span):
                seen = []
                for it in range(QUANT_UNROLL):
                    u = ub + it * UPB + my
                    seen.append((u, row, chunk))
                    chunk += adv_chunk
                    row += adv_rows
                    if chunk >= upr:
                        chunk -= upr
                        row += 1
                for u, r, c in seen:
                    if u >= u_end:
                        break
                    yield u, r, c


SHAPES = list(itertools.product([1, 7, 128, 129, 300, 4290], [128, 256, 384, 3072, 5120]))


@pytest.mark.parametrize("M,K", SHAPES)
def test_quant_kernel_covers_every_unit_once_in_bounds(M, K):
    upr = K >> 7
    Mpad = (M + 127) // 128 * 128
    code_words = M * K // 8                       # uint32 words of [M, K/2] codes
    for G in (32, 16):
        apr = upr if G == 32 else K >> 6          # atoms (4 groups) per 128-row block
        sf_size = Mpad * K // G
        units, words = set(), set()
        for u, r, c in quant_walk(M, K, G):
            assert (r, c) == divmod(u, upr)
            assert u not in units
            units.add(u)
            if r < M:                             # code store: 16 words per unit
                assert u * 16 + 15 < code_words
            # scale words: one per unit (MX), two (NV, groups of 8 lanes)
            for half in ((0,) if G == 32 else (0, 1)):
                off = sf_word_offset(r, c if G == 32 else c * 2 + half, apr)
                assert 0 <= off and off + 4 <= sf_size and off % 4 == 0
                assert off not in words
                words.add(off)
        assert units == set(range(Mpad * upr))
        assert len(words) * 4 == sf_size         # the whole scale buffer, padding rows included


def lr_split(M, K):
    """fp4bsa.cu: K split for few 128-row blocks."""
    blocks, nkc = (M + 127) // 128, K // 64
    if blocks >= 64:
        return 1
    for sp in (8, 4, 2):
        if nkc % sp == 0 and nkc // sp >= 2:
            return sp
    return 1


@pytest.mark.parametrize("M,K", SHAPES + [(8300, 384), (75600, 5120)])
def test_lowrank_pass_covers_every_chunk_once_in_bounds(M, K):
    """lowrank_down_kernel (split or not, with the fused MX quantize): each (row block, K
    chunk) is projected and quantized by exactly one block; X loads stay in [M, K] (rows past
    M are zero-filled, not read); code and scale stores stay in their buffers."""
    blocks = (M + LR_ROWS - 1) // LR_ROWS
    for partial in (False, True):
        sp = lr_split(M, K) if partial else 1
        nkc_all = K // LR_KC
        kps = nkc_all // sp if sp > 1 else nkc_all
        done = set()
        for bx in range(blocks if M < 2000 else min(blocks, 3)):
            m0 = bx * LR_ROWS
            for by in range(sp):
                kc0 = by * kps if sp > 1 else 0
                for kc in range(kps):
                    key = (bx, kc0 + kc)
                    assert key not in done
                    done.add(key)
                    for tid in range(LR_THREADS):             # X loads: 128 rows x 8 pieces
                        for i in range(4):
                            idx = tid + i * LR_THREADS
                            row, c = idx >> 3, idx & 7
                            if m0 + row < M:
                                off = (m0 + row) * K + (kc0 + kc) * LR_KC + c * 8
                                assert off + 8 <= M * K
                        row, c = tid >> 2, tid & 3            # L1 loads: 64 rows x 4 pieces
                        assert ((kc0 + kc) * LR_KC + row) * 32 + c * 8 + 8 <= K * 32
                        qr, qg = tid >> 1, tid & 1            # fused quantize: group qg of row qr
                        m, col = m0 + qr, (kc0 + kc) * LR_KC + qg * 32
                        if m < M:
                            assert m * K + col + 32 <= M * K              # MXFP8 codes
                            assert m * (K // 2) + col // 2 + 16 <= M * K // 2   # MXFP4 codes
                        j = col >> 5
                        off = sf_word_offset(m, j >> 2, K >> 7) + (j & 3)
                        assert off < (M + 127) // 128 * 128 * K // 32
        if M < 2000:
            assert done == {(b, k) for b in range(blocks) for k in range(nkc_all)}


# ------------------------------------------------------------------ stream-K schedule
def sk_kstart(p, total, P):
    """fp4bsa.cu / gemm.cuh Sched::kstart: first flattened K block of pair p's share."""
    return p * total // P


def sk_pair_of(k, total, P):
    """fp4bsa.cu sk_pair_of / gemm.cuh Sched::pair_of: the pair whose share holds block k."""
    q = k * P // total
    while q + 1 < P and sk_kstart(q + 1, total, P) <= k:
        q += 1
    while q > 0 and sk_kstart(q, total, P) > k:
        q -= 1
    return q


def sk_seg_max(tiles, num_kb, P):
    """fp4bsa.cu: the slab count per tile the workspace is sized for."""
    total = tiles * num_kb
    return max([1] + [sk_pair_of(t * num_kb + num_kb - 1, total, P) - sk_pair_of(t * num_kb, total, P) + 1
                      for t in range(tiles)])


@pytest.mark.parametrize("M,K,N", [(512, 5120, 5120), (512, 5120, 13824), (300, 384, 256), (1, 1024, 512),
                                   (256, 2048, 1024), (4096, 5120, 13824), (129, 640, 384)])
@pytest.mark.parametrize("P", [74, 70, 37])
def test_stream_k_schedule_covers_every_block_once_within_the_slabs(M, K, N, P):
    tiles = -(-M // 256) * -(-N // 256)
    num_kb = -(-K // 256)
    total = tiles * num_kb
    if total < P:            # the host runs whole tiles then (every share must be non-empty)
        return
    seg_max = sk_seg_max(tiles, num_kb, P)
    done = {}
    for pair in range(P):
        lo, hi = sk_kstart(pair, total, P), sk_kstart(pair + 1, total, P)
        assert hi > lo                                        # no empty share
        while lo < hi:                                        # Sched::get / step
            tile = lo // num_kb
            kb0 = lo - tile * num_kb
            kb1 = min(num_kb, kb0 + (hi - lo))
            pf = sk_pair_of(tile * num_kb, total, P)
            nseg = sk_pair_of(tile * num_kb + num_kb - 1, total, P) - pf + 1
            seg = pair - pf
            assert 0 <= seg < nseg <= seg_max                 # slab (tile, seg) inside the workspace
            for kb in range(kb0, kb1):
                assert (tile, kb) not in done
                done[(tile, kb)] = pair
                assert sk_pair_of(tile * num_kb + kb, total, P) == pair
            for rank in range(2):                             # arrival counters: 16 per tile
                for ew in range(8):
                    assert tile * 16 + rank * 8 + ew < tiles * 16
            lo += kb1 - kb0
    assert len(done) == total


# ------------------------------------------------------------------ fused GELU + quantize epilogue
@pytest.mark.parametrize("M,N", [(1, 256), (129, 384), (300, 512), (600, 1024), (257, 128)])
@pytest.mark.parametrize("G", [32, 16])
def test_fused_epilogue_writes_every_code_and_scale_byte_once(M, N, G):
    """gemm2_kernel with OUTQ != 0 (epilogue_gelu_quant): per 256 x 256 tile, CTA rank r,
    lane quarter q, lane and column half h, a thread owns row mb*256 + 128r + 32q + lane and
    two 64-column pairs from nb*256 + 128h.  Codes of rows < M, scale bytes of rows < Mpad
    (zeros in the padding), nothing past them."""
    Mpad = (M + 127) // 128 * 128
    apr = N // (G * 4)
    codes, sf = {}, {}
    for mb in range(-(-M // 256)):
        for nb in range(-(-N // 256)):
            for r, q, lane, h in itertools.product(range(2), range(4), range(32), range(2)):
                row = mb * 256 + 128 * r + 32 * q + lane
                for pair in range(2):
                    col0 = nb * 256 + 128 * h + 64 * pair
                    if row >= Mpad or col0 >= N:
                        continue
                    j0 = col0 // G
                    word = sf_word_offset(row, j0 >> 2, apr)
                    if row < M:
                        for c in range(2):                  # two 16-byte stores of 32 codes
                            base = row * (N // 2) + col0 // 2 + 16 * c
                            for b in range(base, base + 16):
                                assert b not in codes and b < M * N // 2
                                codes[b] = 1
                    span = range(word + (j0 & 3), word + (j0 & 3) + 2) if G == 32 else range(word, word + 4)
                    for b in span:                          # MX: half a word, NV: the whole word
                        assert b not in sf and b < Mpad * N // G
                        sf[b] = 1
    assert len(codes) == M * N // 2
    assert len(sf) == Mpad * N // G
