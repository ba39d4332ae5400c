"""fp4_linear_noalloc: the quantized linear for callers that cannot allocate device memory.

Such callers (a plugin whose host owns every device allocation, code running under
another framework's memory pool, a real-time loop that must not block in an allocator)
cannot hand fp4_linear a workspace.  fp4_linear_noalloc keeps the quantized activations
in the library's own fixed-size device array instead.  This test calls it through the C
ABI twice in a row (different formats and shapes, so the second call finds the first
call's contents in the shared array) and checks each output against the existing
fp4_linear entry point within the tolerance every GEMM test uses, then checks that a
problem too large for the array is refused before anything is launched.  The file name
makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _case(fb, L, fmt, M, K, N, seed):
    import torch

    x_bits = synth.activation(seed, M, K, "lognormal")
    w_bits = synth.weight(seed + 1, N, K)
    b_bits = synth.bias(seed + 2, N)
    g_a = oracle.nv_global(oracle.tensor_amax(x_bits)) if fmt == oracle.NV else None
    x = H.dev_bf16(x_bits)
    pw = fb.pack_weight(H.dev_bf16(w_bits), fmt)
    bias = H.dev_f16(b_bits)
    ga = H.dev_f32([g_a]) if fmt == oracle.NV else None

    y_ref = fb.linear(x, pw, bias, ga)                       # existing entry point, torch workspace
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = L.fp4_linear_noalloc(fmt, x.data_ptr(), M, K, N, pw.codes.data_ptr(), pw.sf.data_ptr(),
                              None if pw.w_global is None else pw.w_global.data_ptr(),
                              None if ga is None else ga.data_ptr(), bias.data_ptr(), y.data_ptr(),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, fb.fp4_status_string(st)
    assert fb.fp4_sync_status() == 0
    torch.cuda.synchronize()

    rows = np.arange(M)
    _, S = oracle.fp4_linear_rows(fmt, x_bits, w_bits, b_bits, rows, g_a=g_a)
    ref = H.host_bf16_as_f64(y_ref)
    H.check_linear(y, ref, S, rows, f"noalloc vs fp4_linear fmt={fmt} M={M} K={K} N={N}")


def test_noalloc_matches_fp4_linear_twice_and_rejects_oversize():
    import torch

    import fp4_block_scaled_act_b200 as fb

    fb.build()
    L = fb.lib()
    oracle.build()
    torch.cuda.init()

    _case(fb, L, oracle.MX, 300, 1024, 512, seed=811)       # first call sets up the array's address
    _case(fb, L, oracle.NV, 129, 2048, 384, seed=822)       # second call reuses the array

    # too large for the built-in array: refused with FP4_ERR_WORKSPACE, nothing launched
    M, K, N = 100_000, 5120, 512
    assert fb.fp4_linear_workspace_bytes(oracle.MX, M, K, N) > (16 << 20)
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    st = L.fp4_linear_noalloc(oracle.MX, x.data_ptr(), M, K, N, x.data_ptr(), x.data_ptr(), None, None,
                              None, x.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert fb.fp4_status_string(st) == "FP4_ERR_WORKSPACE"
    assert fb.fp4_sync_status() == 0
