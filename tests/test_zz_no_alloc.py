"""fp4_linear_noalloc: the quantized linear for callers that cannot allocate device memory.

Such callers (a plugin whose host owns every device allocation, code running under
another framework's memory pool, a real-time loop that must not block in an allocator)
cannot hand fp4_linear a workspace.  fp4_linear_noalloc keeps the quantized activations
in the library's own fixed-size device array instead.

This test calls it through the C ABI:
  - twice in a row with different formats and shapes (so the second call finds the first
    call's contents in the shared array), checking every output element against the CPU
    oracle within the tolerance every GEMM test uses, and against the existing fp4_linear
    entry point (the same kernels, so bit for bit);
  - three times back to back on one stream with no host synchronization in between, each
    call reusing the array the previous call's GEMM may still be reading, then checks all
    three outputs;
  - at the largest MXFP4 problem the array holds at K = 5120 (6161 rows), and one row more,
    which is refused with FP4_ERR_WORKSPACE before anything is launched.
The file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _stream():
    import torch

    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _inputs(fb, fmt, M, K, N, seed):
    x_bits = synth.activation(seed, M, K, "lognormal")
    w_bits = synth.weight(seed + 1, N, K)
    b_bits = synth.bias(seed + 2, N)
    g_a = oracle.nv_global(oracle.tensor_amax(x_bits)) if fmt == oracle.NV else None
    dev = dict(x=H.dev_bf16(x_bits), pw=fb.pack_weight(H.dev_bf16(w_bits), fmt), bias=H.dev_f16(b_bits),
               ga=H.dev_f32([g_a]) if fmt == oracle.NV else None)
    return dict(fmt=fmt, M=M, K=K, N=N, x_bits=x_bits, w_bits=w_bits, b_bits=b_bits, g_a=g_a, **dev)


def _noalloc(L, c, y):
    pw, ga = c["pw"], c["ga"]
    return L.fp4_linear_noalloc(c["fmt"], c["x"].data_ptr(), c["M"], c["K"], c["N"], pw.codes.data_ptr(),
                                pw.sf.data_ptr(), None if pw.w_global is None else pw.w_global.data_ptr(),
                                None if ga is None else ga.data_ptr(), c["bias"].data_ptr(), y.data_ptr(),
                                _stream())


def _check(fb, c, y, rows=None):
    """y against the oracle (tolerance) and against fp4_linear (bit for bit)."""
    import torch

    fmt, M, K, N = c["fmt"], c["M"], c["K"], c["N"]
    rows = np.arange(M) if rows is None else rows
    Y, S = oracle.fp4_linear_rows(fmt, c["x_bits"], c["w_bits"], c["b_bits"], rows, g_a=c["g_a"])
    H.check_linear(y, Y, S, rows, f"noalloc vs oracle fmt={fmt} M={M} K={K} N={N}")
    y_ref = fb.linear(c["x"], c["pw"], c["bias"], c["ga"])       # the existing entry point
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), "noalloc differs from fp4_linear"


def test_noalloc_twice_back_to_back_and_at_the_size_limit():
    import torch

    import fp4_block_scaled_act_b200 as fb

    fb.build()
    L = fb.lib()
    oracle.build()
    torch.cuda.init()

    # two calls in a row; the first one on this device sets up the array's address
    for fmt, M, K, N, seed in ((oracle.MX, 300, 1024, 512, 811), (oracle.NV, 129, 2048, 384, 822)):
        c = _inputs(fb, fmt, M, K, N, seed)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = _noalloc(L, c, y)
        assert st == 0, fb.fp4_status_string(st)
        assert fb.fp4_sync_status() == 0
        _check(fb, c, y)

    # three calls queued on one stream without a host sync: each reuses the array that the
    # previous call's GEMM reads (short GEMMs, launched right after their quantize kernel)
    cases = [_inputs(fb, oracle.MX, 260, 512, 512, 831), _inputs(fb, oracle.NV, 384, 768, 256, 842),
             _inputs(fb, oracle.MX, 200, 1536, 384, 853)]
    torch.cuda.synchronize()
    ys = [torch.full((c["M"], c["N"]), float("nan"), dtype=torch.bfloat16, device="cuda") for c in cases]
    for c, y in zip(cases, ys):
        st = _noalloc(L, c, y)
        assert st == 0, fb.fp4_status_string(st)
    assert fb.fp4_sync_status() == 0
    for c, y in zip(cases, ys):
        _check(fb, c, y)

    # the size limit: MXFP4 at K = 5120 fits 6161 rows (16,775,680 of 16,777,216 bytes)
    K, N = 5120, 256
    assert fb.fp4_linear_workspace_bytes(oracle.MX, 6161, K, N) <= (16 << 20)
    assert fb.fp4_linear_workspace_bytes(oracle.MX, 6162, K, N) > (16 << 20)
    c = _inputs(fb, oracle.MX, 6161, K, N, 861)
    y = torch.empty((6161, N), dtype=torch.bfloat16, device="cuda")
    st = _noalloc(L, c, y)
    assert st == 0, fb.fp4_status_string(st)
    assert fb.fp4_sync_status() == 0
    _check(fb, c, y, rows=H.sample_rows(6161, n_random=64, seed=9))

    # one row more: refused with FP4_ERR_WORKSPACE, nothing launched
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    for M in (6162, 100_000):
        st = L.fp4_linear_noalloc(oracle.MX, x.data_ptr(), M, K, N, x.data_ptr(), x.data_ptr(), None, None,
                                  None, x.data_ptr(), _stream())
        assert fb.fp4_status_string(st) == "FP4_ERR_WORKSPACE", M
    assert fb.fp4_sync_status() == 0
