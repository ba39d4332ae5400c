"""Python binding of libfp4bsa.so, the block-scaled FP4 quantized linear for B200.

Every function below has the name of the C entry point it calls (include/fp4bsa.h)
and only marshals arguments: tensors become device pointers, the current torch CUDA
stream becomes the stream argument, and a non-OK status raises FP4Error.  All
arithmetic runs in the library's CUDA kernels.  There is no fallback: if the
library is missing or the device is not sm_100, the calls raise.

The helpers at the end (pack_weight, calibrate_act_global, quantize_act, linear, w4a8_linear,
w4a4_linear, gelu_quantize_act, linear_gelu_quant, linear_host)
allocate outputs and workspaces with torch and call the same entry points.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

from ._build import LIB as _LIB_PATH
from ._build import build

MXFP4, NVFP4 = 0, 1
_FMT = {"mxfp4": MXFP4, "nvfp4": NVFP4, MXFP4: MXFP4, NVFP4: NVFP4}

STATUS = ["FP4_OK", "FP4_ERR_INVALID_ARG", "FP4_ERR_UNSUPPORTED_SHAPE", "FP4_ERR_MISALIGNED",
          "FP4_ERR_WORKSPACE", "FP4_ERR_ARCH", "FP4_ERR_CUDA", "FP4_ERR_TIMEOUT"]

# every symbol include/fp4bsa.h declares
EXPORTS = [
    "fp4_codes_bytes", "fp4_sf_bytes", "fp4_linear_workspace_bytes", "w4a8_workspace_bytes",
    "fp4_tensor_amax", "fp4_pack_weight", "fp4_quantize_act", "fp4_gemm", "fp4_linear",
    "w4a8_quantize_act", "w4a8_gemm", "w4a8_svd_linear", "fp4_sync_status", "fp4_status_string",
    "fp4_set_wait_timeout_ns", "fp4_linear_noalloc",
    "w4a4_workspace_bytes", "w4a4_quantize_act", "w4a4_gemm", "w4a4_svd_linear",
    "fp4_gelu_quantize_act", "fp4_gemm_gelu_quant", "fp4_linear_gelu_quant", "fp4_calibrate_act_global",
    "fp4_heads_codes_bytes", "fp4_heads_sf_bytes", "fp4_quantize_heads", "fp4_attn_scores",
    "fp4_heads_vt_codes_bytes", "fp4_heads_vt_sf_bytes", "fp4_quantize_heads_vt", "fp4_attn_softmax_quant",
    "fp4_attn_pv",
    "fp4_attn_fused",
    "fp4_attn_fused_trace",
]


class FP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = STATUS[status] if 0 <= status < len(STATUS) else f"status {status}"
        super().__init__(f"{where}: {name}")


_lib = None


def lib():
    """Load libfp4bsa.so (it must have been built; see build())."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: run fp4_block_scaled_act_b200.build() first")
        L = ctypes.CDLL(_LIB_PATH)
        P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sig = {
            "fp4_codes_bytes": (SZ, [I, I64, I64]),
            "fp4_sf_bytes": (SZ, [I, I64, I64]),
            "fp4_linear_workspace_bytes": (SZ, [I, I64, I64, I64]),
            "w4a8_workspace_bytes": (SZ, [I64, I64, I64, I]),
            "fp4_tensor_amax": (I, [P, I64, P, P]),
            "fp4_pack_weight": (I, [I, P, I64, I64, P, P, P, P]),
            "fp4_calibrate_act_global": (I, [P, I64, P, P, P]),
            "fp4_quantize_act": (I, [I, P, I64, I64, P, P, P, P]),
            "fp4_gemm": (I, [I, P, P, I64, I64, I64, P, P, P, P, P, P, P]),
            "fp4_linear": (I, [I, P, I64, I64, I64, P, P, P, P, P, P, P, SZ, P]),
            "fp4_linear_noalloc": (I, [I, P, I64, I64, I64, P, P, P, P, P, P, P]),
            "w4a8_quantize_act": (I, [P, I64, I64, P, I, P, P, P, P]),
            "w4a4_workspace_bytes": (SZ, [I64, I64, I64, I]),
            "fp4_gelu_quantize_act": (I, [I, P, I64, I64, P, P, P, P]),
            "fp4_gemm_gelu_quant": (I, [I, P, P, I64, I64, I64, P, P, P, P, P, P, P, P, P]),
            "fp4_linear_gelu_quant": (I, [I, P, I64, I64, I64, P, P, P, P, P, P, P, P, P, SZ, P]),
            "w4a4_quantize_act": (I, [P, I64, I64, P, I, P, P, P, P]),
            "w4a4_gemm": (I, [P, P, P, I64, I64, I64, P, P, P, I, P, P, P]),
            "w4a4_svd_linear": (I, [P, I64, I64, I64, P, P, P, P, I, P, P, P, SZ, P]),
            "w4a8_gemm": (I, [P, P, P, I64, I64, I64, P, P, P, I, P, P, P]),
            "w4a8_svd_linear": (I, [P, I64, I64, I64, P, P, P, P, I, P, P, P, SZ, P]),
            "fp4_heads_codes_bytes": (SZ, [I, I64, I64, I64]),
            "fp4_heads_sf_bytes": (SZ, [I, I64, I64, I64]),
            "fp4_quantize_heads": (I, [I, P, I64, I64, I64, P, P, P, P]),
            "fp4_attn_scores": (I, [I, P, P, I64, P, P, I64, I64, I64, I64, P, P, P, P]),
            "fp4_heads_vt_codes_bytes": (SZ, [I, I64, I64, I64]),
            "fp4_heads_vt_sf_bytes": (SZ, [I, I64, I64, I64]),
            "fp4_quantize_heads_vt": (I, [I, P, I64, I64, I64, P, P, P, P]),
            "fp4_attn_softmax_quant": (I, [I, P, I64, I64, ctypes.c_float, P, P, P, P, P]),
            "fp4_attn_pv": (I, [I, P, P, P, I64, I64, P, P, P, I64, I64, I64, P, P, P]),
            "fp4_attn_fused": (I, [I, P, P, I64, P, P, I64, P, P, I64, I64, I64, ctypes.c_float, P, P, P, P, P, P,
                                   P]),
            "fp4_attn_fused_trace": (I, [I, P, P, I64, P, P, I64, P, P, I64, I64, I64, ctypes.c_float, P, P, P, P, P,
                                         P, I64, P, P, P, P]),
            "fp4_sync_status": (I, [P]),
            "fp4_status_string": (ctypes.c_char_p, [I]),
            "fp4_set_wait_timeout_ns": (None, [ctypes.c_uint64]),
            "fp4bsa_test_skip_iteration": (None, [I]),
            "fp4bsa_set_gemm_ctas": (None, [I]),
            "fp4bsa_set_stream_k": (None, [I]),
            "fp4bsa_set_pdl": (None, [I]),
            "fp4bsa_test_gelu_f32": (I, [P, I64, P, P]),
            "fp4bsa_clock_probe": (I, [P, I, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ----------------------------------------------------------------------------- marshalling
def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream=None):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != 0:
        raise FP4Error(status, where)


def _fmt(fmt) -> int:
    return _FMT[fmt]


# ----------------------------------------------------------------------------- entry points
def fp4_codes_bytes(fmt, rows: int, K: int) -> int:
    return lib().fp4_codes_bytes(_fmt(fmt), rows, K)


def fp4_sf_bytes(fmt, rows: int, K: int) -> int:
    return lib().fp4_sf_bytes(_fmt(fmt), rows, K)


def fp4_linear_workspace_bytes(fmt, M: int, K: int, N: int) -> int:
    return lib().fp4_linear_workspace_bytes(_fmt(fmt), M, K, N)


def w4a8_workspace_bytes(M: int, K: int, N: int, rank: int = 32) -> int:
    return lib().w4a8_workspace_bytes(M, K, N, rank)


def fp4_tensor_amax(x, n: int, amax_out, stream=None):
    _check(lib().fp4_tensor_amax(_ptr(x), n, _ptr(amax_out), _stream(stream)), "fp4_tensor_amax")


def fp4_calibrate_act_global(x, n: int, amax_inout, g_out, stream=None):
    _check(lib().fp4_calibrate_act_global(_ptr(x), n, _ptr(amax_inout), _ptr(g_out), _stream(stream)),
           "fp4_calibrate_act_global")


def fp4_pack_weight(fmt, w, N: int, K: int, w_codes, w_sf, w_global=None, stream=None):
    _check(lib().fp4_pack_weight(_fmt(fmt), _ptr(w), N, K, _ptr(w_codes), _ptr(w_sf), _ptr(w_global),
                                 _stream(stream)), "fp4_pack_weight")


def fp4_quantize_act(fmt, x, M: int, K: int, a_global, x_codes, x_sf, stream=None):
    _check(lib().fp4_quantize_act(_fmt(fmt), _ptr(x), M, K, _ptr(a_global), _ptr(x_codes), _ptr(x_sf),
                                  _stream(stream)), "fp4_quantize_act")


def fp4_gemm(fmt, a_codes, a_sf, M: int, K: int, N: int, w_codes, w_sf, w_global, a_global, bias, y,
             stream=None):
    _check(lib().fp4_gemm(_fmt(fmt), _ptr(a_codes), _ptr(a_sf), M, K, N, _ptr(w_codes), _ptr(w_sf),
                          _ptr(w_global), _ptr(a_global), _ptr(bias), _ptr(y), _stream(stream)), "fp4_gemm")


def fp4_linear(fmt, x, M: int, K: int, N: int, w_codes, w_sf, w_global, a_global, bias, y, workspace,
               ws_bytes: int, stream=None):
    _check(lib().fp4_linear(_fmt(fmt), _ptr(x), M, K, N, _ptr(w_codes), _ptr(w_sf), _ptr(w_global),
                            _ptr(a_global), _ptr(bias), _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)),
           "fp4_linear")


def fp4_linear_noalloc(fmt, x, M: int, K: int, N: int, w_codes, w_sf, w_global, a_global, bias, y,
                       stream=None):
    """fp4_linear without a workspace argument, for callers that cannot allocate device
    memory: the quantized activations use the library's built-in 16 MiB device array."""
    _check(lib().fp4_linear_noalloc(_fmt(fmt), _ptr(x), M, K, N, _ptr(w_codes), _ptr(w_sf), _ptr(w_global),
                                    _ptr(a_global), _ptr(bias), _ptr(y), _stream(stream)), "fp4_linear_noalloc")


def fp4_gelu_quantize_act(fmt, z, M: int, K: int, a_global, x_codes, x_sf, stream=None):
    _check(lib().fp4_gelu_quantize_act(_fmt(fmt), _ptr(z), M, K, _ptr(a_global), _ptr(x_codes), _ptr(x_sf),
                                       _stream(stream)), "fp4_gelu_quantize_act")


def fp4_gemm_gelu_quant(fmt, a_codes, a_sf, M: int, K: int, N: int, w_codes, w_sf, w_global, a_global, bias,
                        h_global, h_codes, h_sf, stream=None):
    _check(lib().fp4_gemm_gelu_quant(_fmt(fmt), _ptr(a_codes), _ptr(a_sf), M, K, N, _ptr(w_codes), _ptr(w_sf),
                                     _ptr(w_global), _ptr(a_global), _ptr(bias), _ptr(h_global), _ptr(h_codes),
                                     _ptr(h_sf), _stream(stream)), "fp4_gemm_gelu_quant")


def fp4_linear_gelu_quant(fmt, x, M: int, K: int, N: int, w_codes, w_sf, w_global, a_global, bias, h_global,
                          h_codes, h_sf, workspace, ws_bytes: int, stream=None):
    _check(lib().fp4_linear_gelu_quant(_fmt(fmt), _ptr(x), M, K, N, _ptr(w_codes), _ptr(w_sf), _ptr(w_global),
                                       _ptr(a_global), _ptr(bias), _ptr(h_global), _ptr(h_codes), _ptr(h_sf),
                                       _ptr(workspace), ws_bytes, _stream(stream)), "fp4_linear_gelu_quant")


def w4a8_quantize_act(x, M: int, K: int, l1, rank: int, x_e4m3, x_sf, u_pair, stream=None):
    _check(lib().w4a8_quantize_act(_ptr(x), M, K, _ptr(l1), rank, _ptr(x_e4m3), _ptr(x_sf), _ptr(u_pair),
                                   _stream(stream)), "w4a8_quantize_act")


def w4a8_gemm(x_e4m3, x_sf, u_pair, M: int, K: int, N: int, r_codes, r_sf, l2, rank: int, bias, y,
              stream=None):
    _check(lib().w4a8_gemm(_ptr(x_e4m3), _ptr(x_sf), _ptr(u_pair), M, K, N, _ptr(r_codes), _ptr(r_sf),
                           _ptr(l2), rank, _ptr(bias), _ptr(y), _stream(stream)), "w4a8_gemm")


def w4a8_svd_linear(x, M: int, K: int, N: int, r_codes, r_sf, l1, l2, rank: int, bias, y, workspace,
                    ws_bytes: int, stream=None):
    _check(lib().w4a8_svd_linear(_ptr(x), M, K, N, _ptr(r_codes), _ptr(r_sf), _ptr(l1), _ptr(l2), rank,
                                 _ptr(bias), _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)),
           "w4a8_svd_linear")


def w4a4_workspace_bytes(M: int, K: int, N: int, rank: int = 32) -> int:
    return lib().w4a4_workspace_bytes(M, K, N, rank)


def w4a4_quantize_act(x, M: int, K: int, l1, rank: int, x_codes, x_sf, u_pair, stream=None):
    _check(lib().w4a4_quantize_act(_ptr(x), M, K, _ptr(l1), rank, _ptr(x_codes), _ptr(x_sf), _ptr(u_pair),
                                   _stream(stream)), "w4a4_quantize_act")


def w4a4_gemm(x_codes, x_sf, u_pair, M: int, K: int, N: int, r_codes, r_sf, l2, rank: int, bias, y,
              stream=None):
    _check(lib().w4a4_gemm(_ptr(x_codes), _ptr(x_sf), _ptr(u_pair), M, K, N, _ptr(r_codes), _ptr(r_sf),
                           _ptr(l2), rank, _ptr(bias), _ptr(y), _stream(stream)), "w4a4_gemm")


def w4a4_svd_linear(x, M: int, K: int, N: int, r_codes, r_sf, l1, l2, rank: int, bias, y, workspace,
                    ws_bytes: int, stream=None):
    _check(lib().w4a4_svd_linear(_ptr(x), M, K, N, _ptr(r_codes), _ptr(r_sf), _ptr(l1), _ptr(l2), rank,
                                 _ptr(bias), _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)),
           "w4a4_svd_linear")


def fp4_heads_codes_bytes(fmt, T: int, H: int, D: int = 128) -> int:
    return lib().fp4_heads_codes_bytes(_fmt(fmt), T, H, D)


def fp4_heads_sf_bytes(fmt, T: int, H: int, D: int = 128) -> int:
    return lib().fp4_heads_sf_bytes(_fmt(fmt), T, H, D)


def fp4_quantize_heads(fmt, x, T: int, H: int, D: int, g, codes, sf, stream=None):
    _check(lib().fp4_quantize_heads(_fmt(fmt), _ptr(x), T, H, D, _ptr(g), _ptr(codes), _ptr(sf), _stream(stream)),
           "fp4_quantize_heads")


def fp4_attn_scores(fmt, q_codes, q_sf, T_q: int, k_codes, k_sf, T_kv: int, H: int, D: int, head: int, g_q, g_k,
                    s, stream=None):
    _check(lib().fp4_attn_scores(_fmt(fmt), _ptr(q_codes), _ptr(q_sf), T_q, _ptr(k_codes), _ptr(k_sf), T_kv, H, D,
                                 head, _ptr(g_q), _ptr(g_k), _ptr(s), _stream(stream)), "fp4_attn_scores")


def fp4_heads_vt_codes_bytes(fmt, T: int, H: int, D: int = 128) -> int:
    return lib().fp4_heads_vt_codes_bytes(_fmt(fmt), T, H, D)


def fp4_heads_vt_sf_bytes(fmt, T: int, H: int, D: int = 128) -> int:
    return lib().fp4_heads_vt_sf_bytes(_fmt(fmt), T, H, D)


def fp4_quantize_heads_vt(fmt, v, T: int, H: int, D: int, g, codes, sf, stream=None):
    _check(lib().fp4_quantize_heads_vt(_fmt(fmt), _ptr(v), T, H, D, _ptr(g), _ptr(codes), _ptr(sf),
                                       _stream(stream)), "fp4_quantize_heads_vt")


def fp4_attn_softmax_quant(fmt, s, T_q: int, T_kv: int, scale: float, p_global, stats, p_codes, p_sf,
                           stream=None):
    _check(lib().fp4_attn_softmax_quant(_fmt(fmt), _ptr(s), T_q, T_kv, float(scale), _ptr(p_global), _ptr(stats),
                                        _ptr(p_codes), _ptr(p_sf), _stream(stream)), "fp4_attn_softmax_quant")


def fp4_attn_pv(fmt, p_codes, p_sf, p_global, T_q: int, T_kv: int, vt_codes, vt_sf, v_global, H: int, D: int,
                head: int, stats, o, stream=None):
    _check(lib().fp4_attn_pv(_fmt(fmt), _ptr(p_codes), _ptr(p_sf), _ptr(p_global), T_q, T_kv, _ptr(vt_codes),
                             _ptr(vt_sf), _ptr(v_global), H, D, head, _ptr(stats), _ptr(o), _stream(stream)),
           "fp4_attn_pv")


def fp4_attn_fused(fmt, q_codes, q_sf, T_q: int, k_codes, k_sf, T_kv: int, vt_codes, vt_sf, H: int, D: int,
                   head: int, scale: float, g_q, g_k, g_v, p_global, stats, o, stream=None):
    _check(lib().fp4_attn_fused(_fmt(fmt), _ptr(q_codes), _ptr(q_sf), T_q, _ptr(k_codes), _ptr(k_sf), T_kv,
                                _ptr(vt_codes), _ptr(vt_sf), H, D, head, scale, _ptr(g_q), _ptr(g_k), _ptr(g_v),
                                _ptr(p_global), _ptr(stats), _ptr(o), _stream(stream)), "fp4_attn_fused")


def fp4_attn_fused_trace(fmt, q_codes, q_sf, T_q: int, k_codes, k_sf, T_kv: int, vt_codes, vt_sf, H: int, D: int,
                         head: int, scale: float, g_q, g_k, g_v, p_global, stats, o, trace_tile: int, trace_m,
                         trace_codes, trace_sf, stream=None):
    _check(lib().fp4_attn_fused_trace(_fmt(fmt), _ptr(q_codes), _ptr(q_sf), T_q, _ptr(k_codes), _ptr(k_sf), T_kv,
                                      _ptr(vt_codes), _ptr(vt_sf), H, D, head, scale, _ptr(g_q), _ptr(g_k),
                                      _ptr(g_v), _ptr(p_global), _ptr(stats), _ptr(o), trace_tile, _ptr(trace_m),
                                      _ptr(trace_codes), _ptr(trace_sf), _stream(stream)), "fp4_attn_fused_trace")


def fp4_sync_status(stream=None) -> int:
    return lib().fp4_sync_status(_stream(stream))


def fp4_status_string(status: int) -> str:
    return lib().fp4_status_string(status).decode()


def fp4_set_wait_timeout_ns(ns: int):
    lib().fp4_set_wait_timeout_ns(ns)


def fp4bsa_clock_probe(out, blocks: int, stream=None):
    """Measurement hook: out (int64 [3 * blocks], device) = (SM id, SM cycle counter, global
    ns timer) per block, recorded by a tiny kernel on `stream`."""
    _check(lib().fp4bsa_clock_probe(_ptr(out), blocks, _stream(stream)), "fp4bsa_clock_probe")


def fp4bsa_test_gelu_f32(z, n: int, g, stream=None):
    """Test hook: g (fp32, device) = the library's fp32 GELU-tanh of each bf16 z (device),
    before the bf16 rounding the fused activation applies."""
    _check(lib().fp4bsa_test_gelu_f32(_ptr(z), n, _ptr(g), _stream(stream)), "fp4bsa_test_gelu_f32")


# ----------------------------------------------------------------------------- helpers
@dataclass
class PackedWeight:
    fmt: int
    N: int
    K: int
    codes: "object"          # torch.uint8 [N, K/2]
    sf: "object"             # torch.uint8 [sf bytes]
    w_global: "object" = None  # torch.float32 [1] (NVFP4)


def pack_weight(w, fmt="mxfp4", stream=None) -> PackedWeight:
    """bf16 [N, K] weight (CUDA) -> PackedWeight (codes, scales, NVFP4 global)."""
    import torch

    f = _fmt(fmt)
    N, K = w.shape
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    sf = torch.empty(fp4_sf_bytes(f, N, K), dtype=torch.uint8, device=w.device)
    g = torch.empty(1, dtype=torch.float32, device=w.device) if f == NVFP4 else None
    fp4_pack_weight(f, w, N, K, codes, sf, g, stream)
    return PackedWeight(f, N, K, codes, sf, g)


def calibrate_act_global(batches, stream=None):
    """NVFP4 static activation global from one or more bf16 calibration batches (CUDA):
    returns (g_a, amax) as one-element fp32 device tensors."""
    import torch

    batches = [batches] if hasattr(batches, "is_cuda") else list(batches)
    dev = batches[0].device
    amax = torch.zeros(1, dtype=torch.float32, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    for b in batches:
        fp4_calibrate_act_global(b, b.numel(), amax, g, stream)
    return g, amax


def quantize_act(x, fmt="mxfp4", a_global=None, stream=None):
    """bf16 [M, K] activations (CUDA) -> (codes [M, K/2], scale factors)."""
    import torch

    f = _fmt(fmt)
    M, K = x.shape
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    sf = torch.empty(fp4_sf_bytes(f, M, K), dtype=torch.uint8, device=x.device)
    fp4_quantize_act(f, x, M, K, a_global, codes, sf, stream)
    return codes, sf


def quantize_heads(x, H: int, fmt="mxfp4", g=None, stream=None):
    """bf16 [T, H * 128] (CUDA) -> head-major (codes [H, Tpad, 64], scales [H, sf bytes per head])."""
    import torch

    f = _fmt(fmt)
    T, HD = x.shape
    D = HD // H
    Tpad = (T + 127) // 128 * 128
    codes = torch.empty((H, Tpad, D // 2), dtype=torch.uint8, device=x.device)
    sf = torch.empty((H, fp4_heads_sf_bytes(f, T, H, D) // H), dtype=torch.uint8, device=x.device)
    fp4_quantize_heads(f, x, T, H, D, g, codes, sf, stream)
    return codes, sf


def attn_scores(q_heads, k_heads, T_q: int, T_kv: int, head: int, fmt="mxfp4", g_q=None, g_k=None, s=None,
                stream=None):
    """Scores of one head from quantize_heads outputs: bf16 [T_q, T_kv rounded up to 128]."""
    import torch

    f = _fmt(fmt)
    qc, qs = q_heads
    kc, ks = k_heads
    H, _, half_d = qc.shape
    if s is None:
        s = torch.empty((T_q, (T_kv + 127) // 128 * 128), dtype=torch.bfloat16, device=qc.device)
    fp4_attn_scores(f, qc, qs, T_q, kc, ks, T_kv, H, 2 * half_d, head, g_q, g_k, s, stream)
    return s


P_GLOBAL_NVFP4 = 1.0 / 2688.0   # P's NVFP4 global: p <= 1, so T / (6 * 448) with T = 1


def quantize_heads_vt(v, H: int, fmt="mxfp4", g=None, stream=None):
    """bf16 [T, H * 128] (CUDA) -> head-major V^T (codes [H, 128, Tpad/2], scales [H, bytes per head])."""
    import torch

    f = _fmt(fmt)
    T, HD = v.shape
    D = HD // H
    Tpad = (T + 127) // 128 * 128
    codes = torch.empty((H, D, Tpad // 2), dtype=torch.uint8, device=v.device)
    sf = torch.empty((H, fp4_heads_vt_sf_bytes(f, T, H, D) // H), dtype=torch.uint8, device=v.device)
    fp4_quantize_heads_vt(f, v, T, H, D, g, codes, sf, stream)
    return codes, sf


def attn_softmax_quant(s, T_q: int, T_kv: int, scale: float, fmt="mxfp4", p_global=None, stream=None):
    """Scores bf16 [T_q, T_kv_pad] (CUDA) -> (P codes [T_q, T_kv_pad/2], P scales, (m, l) stats [T_q, 2]).
    NVFP4 needs p_global (a one-element fp32 device tensor, P_GLOBAL_NVFP4)."""
    import torch

    f = _fmt(fmt)
    kpad = s.shape[1]
    p_codes = torch.empty((T_q, kpad // 2), dtype=torch.uint8, device=s.device)
    p_sf = torch.empty(fp4_sf_bytes(f, T_q, kpad), dtype=torch.uint8, device=s.device)
    stats = torch.empty((T_q, 2), dtype=torch.float32, device=s.device)
    fp4_attn_softmax_quant(f, s, T_q, T_kv, scale, p_global, stats, p_codes, p_sf, stream)
    return p_codes, p_sf, stats


def attn_pv(p, vt_heads, T_q: int, T_kv: int, head: int, fmt="mxfp4", p_global=None, v_global=None, o=None,
            normalize=True, stream=None):
    """O -> bf16 [T_q, 128] from attn_softmax_quant's (codes, scales, stats) and quantize_heads_vt's V^T:
    deq(P~) deq(V_head), each row divided by its softmax sum unless normalize is False."""
    import torch

    f = _fmt(fmt)
    p_codes, p_sf = p[0], p[1]
    stats = p[2] if (normalize and len(p) > 2) else None
    vc, vs = vt_heads
    H, D, _ = vc.shape
    if o is None:
        o = torch.empty((T_q, D), dtype=torch.bfloat16, device=p_codes.device)
    fp4_attn_pv(f, p_codes, p_sf, p_global, T_q, T_kv, vc, vs, v_global, H, D, head, stats, o, stream)
    return o


def attn_fused(q_heads, k_heads, vt_heads, T_q: int, T_kv: int, head: int, scale: float, fmt="mxfp4", g_q=None,
               g_k=None, g_v=None, p_global=None, o=None, stats=None, trace_tile=None, stream=None):
    """One head's FP4 attention in one kernel (streaming form) from quantize_heads' Q and K and
    quantize_heads_vt's V^T: bf16 [T_q, 128].  NVFP4: the device fp32 globals of Q, K, V and P~
    (P_GLOBAL_NVFP4).  stats: an fp32 [T_q, 2] tensor to receive (final running maximum, l), or
    None.  trace_tile: a query tile whose per-block running maxima, P~ codes and scale bytes are
    returned too, as (o, (m [nblk, 128], codes [nblk, 128, 128], sf [nblk, 128, 256 / G]))."""
    import torch

    qc, qs = q_heads
    kc, ks = k_heads
    vc, vs = vt_heads
    H, _, half_d = qc.shape
    D = 2 * half_d
    if o is None:
        o = torch.empty((T_q, D), dtype=torch.bfloat16, device=qc.device)
    if trace_tile is None:
        fp4_attn_fused(fmt, qc, qs, T_q, kc, ks, T_kv, vc, vs, H, D, head, scale, g_q, g_k, g_v, p_global, stats, o,
                       stream)
        return o
    nblk = ((T_kv + 127) // 128 * 128 + 255) // 256
    G = 32 if _fmt(fmt) == MXFP4 else 16
    tm = torch.empty((nblk, 128), dtype=torch.float32, device=qc.device)
    tc = torch.empty((nblk, 128, 128), dtype=torch.uint8, device=qc.device)
    ts = torch.empty((nblk, 128, 256 // G), dtype=torch.uint8, device=qc.device)
    fp4_attn_fused_trace(fmt, qc, qs, T_q, kc, ks, T_kv, vc, vs, H, D, head, scale, g_q, g_k, g_v, p_global, stats, o,
                         trace_tile, tm, tc, ts, stream)
    return o, (tm, tc, ts)


def linear(x, pw: PackedWeight, bias=None, a_global=None, y=None, workspace=None, stream=None):
    """W4A4 quantized linear: bf16 [M, K] -> bf16 [M, N]."""
    import torch

    M, K = x.shape
    assert K == pw.K
    if y is None:
        y = torch.empty((M, pw.N), dtype=torch.bfloat16, device=x.device)
    ws = fp4_linear_workspace_bytes(pw.fmt, M, K, pw.N)
    if workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=x.device)
    fp4_linear(pw.fmt, x, M, K, pw.N, pw.codes, pw.sf, pw.w_global, a_global, bias, y, workspace,
               workspace.numel(), stream)
    return y


def w4a8_linear(x, r: PackedWeight, l1, l2, bias=None, y=None, workspace=None, stream=None):
    """W4A8 SVDQuant linear: bf16 [M, K] -> bf16 [M, N] (MXFP4 residual r, rank-32 L1 [K, rank]
    and L2 [rank, N] as stored)."""
    import torch

    M, K = x.shape
    rank = l1.shape[1]
    if y is None:
        y = torch.empty((M, r.N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(w4a8_workspace_bytes(M, K, r.N, rank), dtype=torch.uint8, device=x.device)
    w4a8_svd_linear(x, M, K, r.N, r.codes, r.sf, l1, l2, rank, bias, y, workspace, workspace.numel(), stream)
    return y


def w4a4_linear(x, r: PackedWeight, l1, l2, bias=None, y=None, workspace=None, stream=None):
    """W4A4 SVDQuant linear: bf16 [M, K] -> bf16 [M, N] (MXFP4 activations and residual r,
    rank-32 L1 [K, rank] and L2 [rank, N] as stored)."""
    import torch

    M, K = x.shape
    rank = l1.shape[1]
    if y is None:
        y = torch.empty((M, r.N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(w4a4_workspace_bytes(M, K, r.N, rank), dtype=torch.uint8, device=x.device)
    w4a4_svd_linear(x, M, K, r.N, r.codes, r.sf, l1, l2, rank, bias, y, workspace, workspace.numel(), stream)
    return y


def gelu_quantize_act(z, fmt="mxfp4", a_global=None, stream=None):
    """bf16 up-projection output z [M, K] (CUDA) -> (codes, scale factors) of
    bf16(gelu_tanh(z)) in fmt, the down projection's quantized input."""
    import torch

    f = _fmt(fmt)
    M, K = z.shape
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=z.device)
    sf = torch.empty(fp4_sf_bytes(f, M, K), dtype=torch.uint8, device=z.device)
    fp4_gelu_quantize_act(f, z, M, K, a_global, codes, sf, stream)
    return codes, sf


def linear_gelu_quant(x, pw: PackedWeight, bias=None, a_global=None, h_global=None, workspace=None, stream=None):
    """Up projection + GELU-tanh + quantize in one GEMM: bf16 x [M, K] -> (codes [M, N/2],
    scale factors) of h = bf16(gelu_tanh(bf16(x W^T + bias))) in the weight's format."""
    import torch

    M, K = x.shape
    N = pw.N
    codes = torch.empty((M, N // 2), dtype=torch.uint8, device=x.device)
    sf = torch.empty(fp4_sf_bytes(pw.fmt, M, N), dtype=torch.uint8, device=x.device)
    if workspace is None:
        workspace = torch.empty(fp4_linear_workspace_bytes(pw.fmt, M, K, N), dtype=torch.uint8, device=x.device)
    fp4_linear_gelu_quant(pw.fmt, x, M, K, N, pw.codes, pw.sf, pw.w_global, a_global, bias, h_global, codes, sf,
                          workspace, workspace.numel(), stream)
    return codes, sf


class HostPipeline:
    """Reusable device buffers, streams and events for linear_host: two sets of per-chunk
    device buffers (x rows, y rows, quantize workspace) so that the host->device copy of
    chunk i + 1, the linear of chunk i and the device->host copy of chunk i - 1 run
    concurrently on three streams."""

    def __init__(self, fmt, chunk_rows: int, K: int, N: int, device="cuda"):
        import torch

        self.fmt = _fmt(fmt)
        self.chunk_rows, self.K, self.N = chunk_rows, K, N
        ws = fp4_linear_workspace_bytes(self.fmt, chunk_rows, K, N)
        self.x = [torch.empty((chunk_rows, K), dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.y = [torch.empty((chunk_rows, N), dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.ws = [torch.empty(ws, dtype=torch.uint8, device=device) for _ in range(2)]
        self.streams = [torch.cuda.Stream(device=device) for _ in range(3)]
        self.ev_x = [torch.cuda.Event() for _ in range(2)]   # chunk copied in
        self.ev_c = [torch.cuda.Event() for _ in range(2)]   # chunk computed (x read, y written)
        self.ev_y = [torch.cuda.Event() for _ in range(2)]   # chunk copied out


def linear_host(x_host, pw: PackedWeight, pipe: HostPipeline, bias=None, a_global=None, y_host=None):
    """Host-to-host W4A4 linear: pinned bf16 x [M, K] in host memory -> pinned bf16 y
    [M, N] in host memory, in row chunks of pipe.chunk_rows through fp4_linear, with the
    copies in both directions overlapped with the GEMMs (see HostPipeline).  The work is
    ordered after everything already on the current stream, and the current stream waits
    for the last copy, so an event recorded on it afterwards marks completion."""
    import torch

    M, K = x_host.shape
    assert K == pipe.K and pw.N == pipe.N and pw.fmt == pipe.fmt
    if y_host is None:
        y_host = torch.empty((M, pw.N), dtype=torch.bfloat16, pin_memory=True)
    cur = torch.cuda.current_stream()
    s_in, s_mm, s_out = pipe.streams
    for s in pipe.streams:
        s.wait_stream(cur)
    C = pipe.chunk_rows
    for i, r0 in enumerate(range(0, M, C)):
        r1 = min(M, r0 + C)
        rows, b = r1 - r0, i % 2
        xd, yd = pipe.x[b][:rows], pipe.y[b][:rows]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(pipe.ev_c[b])        # chunk i - 2 no longer reads x[b]
            xd.copy_(x_host[r0:r1], non_blocking=True)
            pipe.ev_x[b].record(s_in)
        with torch.cuda.stream(s_mm):
            s_mm.wait_event(pipe.ev_x[b])
            if i >= 2:
                s_mm.wait_event(pipe.ev_y[b])        # chunk i - 2 copied y[b] out
            fp4_linear(pipe.fmt, xd, rows, K, pipe.N, pw.codes, pw.sf, pw.w_global, a_global, bias, yd,
                       pipe.ws[b], pipe.ws[b].numel(), s_mm)
            pipe.ev_c[b].record(s_mm)
        with torch.cuda.stream(s_out):
            s_out.wait_event(pipe.ev_c[b])
            y_host[r0:r1].copy_(yd, non_blocking=True)
            pipe.ev_y[b].record(s_out)
    cur.wait_stream(s_out)
    return y_host
