#!/usr/bin/env python
"""Benchmark of the W4A4 block-scaled FP4 quantized linear on B200.

Workload: the Wan2.2-A14B FFN up-projection in MXFP4, M = 75600 tokens (a 21x45x80
latent grid), K = 5120, N = 13824; bf16 activations N(0,1) x per-channel lognormal
gains, bf16 weights N(0, 0.02) packed offline, fp16 bias, bf16 output.  One step is
one quantized linear: dynamic activation quantization + block-scaled GEMM with the
fused bias epilogue (the weight pre-pack is offline and untimed).  `--fmt nvfp4` runs
the same layer in NVFP4 (the T2V-A14B NVFP4 card's format), its static activation
global calibrated once, untimed, on a separate batch of the same layer.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--fmt nvfp4]

Prints one JSON line.  `value` is TFLOPS (2*M*K*N per step, all ranks together)
with inputs resident in HBM; `e2e` is the same metric through fp4_linear (linear_host) with the
input copied from pinned host memory and the output copied back every step.  With
N > 1 (torchrun) every rank runs its own batch (weak scaling, no collective on the
data path); time is the max over ranks.  `--impl reference` times the CPU oracle on
a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, K, N = 75600, 5120, 13824
FMT = "mxfp4"
WORKLOAD = "wan22_a14b_ffn_up_mxfp4"
METRIC = "FP4 W4A4 linear TFLOPS incl. act-quant (M=75600 K=5120 N=13824), % FP4 peak"
FLOP_PER_STEP = 2.0 * M * K * N
NOMINAL_FP4_TFLOPS = 9000.0
FP4_PER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor ratio on B200 (9 / 2.25 PFLOP/s)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads timed after the headline (NVFP4, fused FFN, W4A8, text tokens)")
    ap.add_argument("--gemm-ctas", type=int, default=0, choices=[0, 1, 2],
                    help="GEMM kernel: 0 auto (2-CTA 256x256 tile for M > 128), 1 force the 1-CTA 128x256 tile, 2 force 2-CTA")
    ap.add_argument("--fmt", default="mxfp4", choices=["mxfp4", "nvfp4"])
    ap.add_argument("--m", type=int, default=75600,
                    help="tokens; smaller values run a reduced case of the same kernels (profiling only)")
    ap.add_argument("--attn-tokens", type=int, default=0,
                    help="profiling only: run one head of FP4 attention (K quantizer over 40 heads of 128, head 17's "
                         "scores, softmax weights + quantize, P V, then the fused head) at this many "
                         "tokens for --steps iterations, print timings, exit")
    return ap.parse_args()


def attn_profile(args):
    """One head of FP4 attention alone (a case for ncu): Q, K, V quantized ([T, 40 x 128] bf16),
    then per step the K quantizer, head 17's scores, the softmax weights + quantize and P V."""
    import torch

    import fp4_block_scaled_act_b200 as fb

    fb.lib()
    T, Hn, fmt = args.attn_tokens, 40, args.fmt
    gen = torch.Generator(device="cuda")
    gen.manual_seed(20261203)
    q = torch.randn(T, Hn * 128, generator=gen, device="cuda").to(torch.bfloat16)
    k = torch.randn(T, Hn * 128, generator=gen, device="cuda").to(torch.bfloat16)
    gq = gk = None
    if fmt == "nvfp4":
        gq, _ = fb.calibrate_act_global(q)
        gk, _ = fb.calibrate_act_global(k)
    v = torch.randn(T, Hn * 128, generator=gen, device="cuda").to(torch.bfloat16)
    gv = fb.calibrate_act_global(v)[0] if fmt == "nvfp4" else None
    gp = torch.tensor([fb.P_GLOBAL_NVFP4], dtype=torch.float32, device="cuda") if fmt == "nvfp4" else None
    qh = fb.quantize_heads(q, Hn, fmt, gq)
    kh = fb.quantize_heads(k, Hn, fmt, gk)
    vt = fb.quantize_heads_vt(v, Hn, fmt, gv)
    s_buf = torch.empty((T, (T + 127) // 128 * 128), dtype=torch.bfloat16, device="cuda")
    p = fb.attn_softmax_quant(s_buf.zero_(), T, T, 128 ** -0.5, fmt, gp)
    o = torch.empty((T, 128), dtype=torch.bfloat16, device="cuda")
    f = fb.MXFP4 if fmt == "mxfp4" else fb.NVFP4
    e = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    t = [0.0] * 5
    for _ in range(args.steps):
        e[0].record()
        fb.fp4_quantize_heads(f, k, T, Hn, 128, gk, kh[0], kh[1])
        e[1].record()
        fb.attn_scores(qh, kh, T, T, 17, fmt, gq, gk, s_buf)
        e[2].record()
        fb.fp4_attn_softmax_quant(f, s_buf, T, T, 128 ** -0.5, gp, p[2], p[0], p[1])
        e[3].record()
        fb.attn_pv(p, vt, T, T, 17, fmt, gp, gv, o=o)
        e[4].record()
        fb.attn_fused(qh, kh, vt, T, T, 17, 128 ** -0.5, fmt, gq, gk, gv, gp, o=o)
        e[5].record()
        torch.cuda.synchronize()
        for i in range(5):
            t[i] += e[i].elapsed_time(e[i + 1])
    st = fb.fp4_sync_status()
    if st != 0:
        raise RuntimeError(f"device status: {fb.fp4_status_string(st)}")
    print(json.dumps({"attn_tokens": T, "heads": Hn, "fmt": fmt, "quantize_heads_ms": t[0] / args.steps,
                      "scores_ms": t[1] / args.steps, "softmax_quant_ms": t[2] / args.steps,
                      "pv_ms": t[3] / args.steps, "fused_ms": t[4] / args.steps, "s_bytes": s_buf.numel() * 2}),
          flush=True)
    return 0


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=2)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if ts < t0 - 0.05 or ts > t1 + 0.1:
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------- inputs
def make_inputs(rank: int, m: int | None = None, k: int | None = None, n: int | None = None):
    """Rank r's batch: its own activations (weak scaling: every rank a different batch of the
    same size), the shared weight and bias.  Sizes default to the workload's."""
    import synth

    m, k, n = (M if m is None else m), (K if k is None else k), (N if n is None else n)
    s = synth.seeds_for(4, layer=1)
    x = synth.activation(s["x"] + 7919 * rank, m, k, "lognormal", gain_seed=s["gain"])
    w = synth.weight(s["w"], n, k)
    b = synth.bias(s["bias"], n)
    return x, w, b


def nv_calibration_batch(k: int | None = None):
    """The layer's NVFP4 calibration batch: 4096 tokens from a separate seed, same gains."""
    import synth

    k = K if k is None else k
    s = synth.seeds_for(4, layer=1)
    return synth.activation(s["x"] + 104729, 4096, k, "lognormal", gain_seed=s["gain"])


def nv_static_global(fb, torch, k: int | None = None):
    """NVFP4 static activation global of the layer (device fp32 [1]), calibrated once,
    untimed, by the library's fp4_calibrate_act_global on the calibration batch."""
    cal = to_dev(nv_calibration_batch(k), torch, torch.bfloat16)
    g, _ = fb.calibrate_act_global(cal)
    torch.cuda.synchronize()
    return g


def oracle_static_global(k: int | None = None) -> float:
    """The same global by the CPU oracle (for the oracle-timing legs)."""
    import oracle

    return oracle.nv_global(oracle.tensor_amax(nv_calibration_batch(k)))


def max_over_ranks(x: float, dist=None, device="cuda") -> float:
    """The largest x over all ranks: a job's time is its slowest rank's."""
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_tflops(flop_per_rank_step: float, world: int, steps: int, slowest_ms: float) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's timed region."""
    return flop_per_rank_step * world * steps / (slowest_ms / 1e3) / 1e12


def config_dict(gpus: int) -> dict:
    """The workload's config, identical in both arms."""
    return {"workload": WORKLOAD, "M": M, "K": K, "N": N, "fmt": FMT, "tokens_per_gpu": M,
            "parallelism": f"dp{gpus} (independent batches)" if gpus > 1 else "single GPU",
            "l2": "inputs larger than L2 (X 774 MB, Y 2.09 GB), no flush"}


def probe_clocks(fb, torch, blocks: int = 1024):
    """Record (SM id, SM cycle counter, ns timer) from `blocks` tiny blocks on the current stream."""
    buf = torch.zeros(3 * blocks, dtype=torch.int64, device="cuda")
    fb.fp4bsa_clock_probe(buf, blocks)
    return buf


def probe_mhz(before, after):
    """Median over SMs of each SM's average clock between two probes (cycles / ns), in MHz."""
    b = before.view(-1, 3).cpu().numpy()
    a = after.view(-1, 3).cpu().numpy()
    first = {}
    for sm, c, t in b:
        first.setdefault(int(sm), (int(c), int(t)))
    last = {}
    for sm, c, t in a:
        last[int(sm)] = (int(c), int(t))
    f = [(last[sm][0] - c0) / (last[sm][1] - t0) * 1e3 for sm, (c0, t0) in first.items()
         if sm in last and last[sm][1] > t0]
    return (float(statistics.median(f)), len(f)) if f else (None, 0)


def to_dev(bits, torch, dt):
    return torch.from_numpy(bits.view(np.int16)).view(dt).cuda()


def gemm_traffic(pair: bool):
    """DRAM bytes per launch of the timed GEMM kernel from the committed ncu summary, or
    None when the kernel code changed since those counters were taken."""
    name = "gemm2_mxfp4_ffn_up_traffic.txt" if pair else "gemm_mxfp4_ffn_up_traffic.txt"
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    fields = dict(l.split(":", 1) for l in open(path) if ":" in l)
    if kernel_code_digest() != fields.get("code_sha1", "").strip():
        return None
    return float(fields["bytes_per_launch"])


def kernel_code_digest() -> str:
    """sha1 (12 hex digits) of the GEMM kernel sources with // comments and blank lines
    removed: an edit to the code invalidates recorded counters, an edit to a comment does not."""
    import hashlib

    h = hashlib.sha1()
    for f in ("gemm.cuh", "ptx.cuh"):
        for line in open(os.path.join(ROOT, "fp4_block_scaled_act_b200", "csrc", f), encoding="utf-8"):
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:12]


# ----------------------------------------------------------------------------- cpu baseline
def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), recorded beside the core count."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(x_bits, w_bits, b_bits, target_s: float = 15.0):
    """The oracle, as it stands, on a bounded row sample of the same workload."""
    import oracle

    f = oracle.MX if FMT == "mxfp4" else oracle.NV
    g_a = oracle_static_global() if f == oracle.NV else 1.0
    wc, ws, g_w = oracle.pack_weight(f, w_bits)                 # offline step, untimed
    w_deq = oracle.dequant_fp4(f, wc, ws, K, g_w or 1.0)        # once, untimed

    def run(rows):
        xs = np.ascontiguousarray(x_bits[rows])
        c, sf = oracle.quantize(f, xs, g_a)
        a = oracle.dequant_fp4(f, c, sf, K, g_a)
        oracle.linear_fp64(a, w_deq, b_bits)

    t = time.perf_counter()
    run(np.arange(2))
    per_row = max((time.perf_counter() - t) / 2, 1e-4)
    nrows = int(max(2, min(512, target_s / per_row)))
    rows = np.linspace(0, M - 1, nrows).astype(np.int64)
    t = time.perf_counter()
    run(rows)
    dt = time.perf_counter() - t
    # the activation quantizer alone over a row sample of its own, as a bandwidth
    qrows = np.arange(min(M, 8192))
    xq = np.ascontiguousarray(x_bits[qrows])
    t = time.perf_counter()
    oracle.quantize(f, xq, g_a)
    dq = time.perf_counter() - t
    q_bytes = qrows.size * K * 2 + qrows.size * K // 2 + oracle.sf_bytes(qrows.size, K // oracle.group_size(f))
    return {"value": 2.0 * nrows * K * N / dt / 1e12, "unit": "TFLOPS", "cores": oracle.num_threads(),
            "cpu": cpu_model(), "kind": "oracle",
            "quantize_gbs": q_bytes / dq / 1e9,
            "sample": f"{nrows} of {M} rows: {FMT.upper()} quantize + dequantize + fp64 GEMM over full K={K}, N={N} "
                      f"({dt:.1f} s); weight pack and dequantize excluded (offline); quantize_gbs: the quantizer "
                      f"alone on {qrows.size} rows ({dq:.2f} s)"}


# ----------------------------------------------------------------------------- reference arm
def reference_arm(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    import synth

    oracle.build()
    s = synth.seeds_for(4, layer=1)
    w = synth.weight(s["w"], N, K)
    b = synth.bias(s["bias"], N)
    f = oracle.MX if FMT == "mxfp4" else oracle.NV
    g_a = oracle_static_global() if f == oracle.NV else 1.0
    wc, ws, g_w = oracle.pack_weight(f, w)
    w_deq = oracle.dequant_fp4(f, wc, ws, K, g_w or 1.0)
    # one step = the quantized linear for a bounded row sample of the workload
    total_steps = args.steps + args.warmup
    probe = synth.activation(s["x"], 1, K, "lognormal", gain_seed=s["gain"])
    t = time.perf_counter()
    c, sf = oracle.quantize(f, probe, g_a)
    oracle.linear_fp64(oracle.dequant_fp4(f, c, sf, K, g_a), w_deq, b)
    per_row = time.perf_counter() - t
    budget = 150.0
    rows_per_step = int(max(1, min(64, budget / max(total_steps, 1) / max(per_row, 1e-4))))
    x = synth.activation(s["x"], rows_per_step * 8, K, "lognormal", gain_seed=s["gain"])

    def step(i):
        r0 = (i * rows_per_step) % (x.shape[0] - rows_per_step + 1)
        xs = np.ascontiguousarray(x[r0:r0 + rows_per_step])
        c, sf = oracle.quantize(f, xs, g_a)
        oracle.linear_fp64(oracle.dequant_fp4(f, c, sf, K, g_a), w_deq, b)

    for i in range(args.warmup):
        step(i)
    t = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t
    flops = 2.0 * rows_per_step * K * N * args.steps
    value = flops / dt / 1e12
    sample = (f"{rows_per_step} row(s) of the {M}x{K}x{N} workload per step: {FMT.upper()} quantize + "
              f"dequantize + fp64 GEMM (weight packed once, untimed)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": oracle.num_threads(), "cpu": cpu_model(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- other workloads
def extra_workloads(fb, torch, args, steps: int = 20, warmup: int = 3):
    """The other Wan2.2 / TI2V-5B configurations of the path, each timed on its own after the
    headline (CUDA events on the launching stream, inputs resident in HBM and larger than L2
    except the text-token and W4A8 shapes).  Inputs are seeded synthetic tensors drawn on the
    device with the workload's distributions: x ~ N(0,1) times a per-channel lognormal(0,1)
    gain, weights ~ N(0, 0.02), bias ~ N(0, 0.01); the fused FFN's z is the up projection's own
    output; the W4A8 factors are N(0, 0.02) residual and N(0, 0.05) low-rank factors (timing
    does not depend on how they were obtained)."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(20261202)
    stream = torch.cuda.current_stream()

    def act(m, k):
        gain = torch.exp(torch.randn(k, generator=gen, device="cuda"))
        return (torch.randn(m, k, generator=gen, device="cuda") * gain).to(torch.bfloat16)

    def wgt(n, k, sd=0.02):
        return (torch.randn(n, k, generator=gen, device="cuda") * sd).to(torch.bfloat16)

    def bias(n):
        return (torch.randn(n, generator=gen, device="cuda") * 0.01).to(torch.float16)

    def timed(fn, flop, n=steps):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0 = probe_clocks(fb, torch)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        p1 = probe_clocks(fb, torch)
        torch.cuda.synchronize()
        st = fb.fp4_sync_status()
        if st != 0:
            raise RuntimeError(f"device status: {fb.fp4_status_string(st)}")
        ms = e0.elapsed_time(e1) / n
        mhz, _ = probe_mhz(p0, p1)
        return {"ms": ms, "tflops": flop / (ms / 1e3) / 1e12,
                "pct_nominal": 100.0 * flop / (ms / 1e3) / 1e12 / (NOMINAL_FP4_TFLOPS if flop else 1),
                "sm_mhz_in_kernel": mhz}

    out = {}
    Mx, Kx, Nx = 75600, 5120, 13824
    x = act(Mx, Kx)
    b_up = bias(Nx)
    # NVFP4 ffn up projection (quantize + GEMM), static activation global from a separate batch
    ga, _ = fb.calibrate_act_global(act(4096, Kx))
    pw_nv = fb.pack_weight(wgt(Nx, Kx), "nvfp4")
    y = torch.empty((Mx, Nx), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(fb.fp4_linear_workspace_bytes("nvfp4", Mx, Kx, Nx), dtype=torch.uint8, device="cuda")
    out["nvfp4_ffn_up_75600x5120x13824"] = timed(
        lambda: fb.fp4_linear("nvfp4", x, Mx, Kx, Nx, pw_nv.codes, pw_nv.sf, pw_nv.w_global, ga, b_up, y, ws,
                              ws.numel()), 2.0 * Mx * Kx * Nx)
    # the fused FFN activation: up projection + GELU-tanh + the down projection's quantize
    for fmt in ("mxfp4", "nvfp4"):
        pw = pw_nv if fmt == "nvfp4" else fb.pack_weight(wgt(Nx, Kx), "mxfp4")
        hc = torch.empty((Mx, Nx // 2), dtype=torch.uint8, device="cuda")
        hs = torch.empty(fb.fp4_sf_bytes(fmt, Mx, Nx), dtype=torch.uint8, device="cuda")
        hg = torch.tensor([0.01], device="cuda") if fmt == "nvfp4" else None
        a_g = ga if fmt == "nvfp4" else None
        out[f"{fmt}_ffn_up_gelu_quant_75600x5120x13824"] = timed(
            lambda: fb.fp4_linear_gelu_quant(fmt, x, Mx, Kx, Nx, pw.codes, pw.sf, pw.w_global, a_g, b_up, hg, hc,
                                             hs, ws, ws.numel()), 2.0 * Mx * Kx * Nx)
        del hc, hs
    del y, pw_nv
    # MXFP4 attention projection (75600 x 5120 -> 5120) and the text-token k/v (512 rows)
    pw_a = fb.pack_weight(wgt(5120, 5120), "mxfp4")
    b_a = bias(5120)
    ya = torch.empty((Mx, 5120), dtype=torch.bfloat16, device="cuda")
    out["mxfp4_attn_75600x5120x5120"] = timed(
        lambda: fb.fp4_linear("mxfp4", x, Mx, 5120, 5120, pw_a.codes, pw_a.sf, None, None, b_a, ya, ws,
                              ws.numel()), 2.0 * Mx * 5120 * 5120)
    del ya, x
    # the rest of the Wan2.2 block's linears and the M sweep, in both formats (quantize +
    # GEMM through fp4_linear; NVFP4 activation globals calibrated once on a separate batch)
    def linear_case(fmt, M, K, N, kind="act"):
        if kind == "gelu":  # the down projection's input: GELU-tanh of an N(0,1) tensor
            z = torch.randn(M, K, generator=gen, device="cuda")
            xs = torch.nn.functional.gelu(z, approximate="tanh").to(torch.bfloat16)
            del z
        else:
            xs = act(M, K)
        pw_c = fb.pack_weight(wgt(N, K), fmt)
        g_c = fb.calibrate_act_global(act(4096, K))[0] if fmt == "nvfp4" else None
        y_c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws_c = torch.empty(fb.fp4_linear_workspace_bytes(fmt, M, K, N), dtype=torch.uint8, device="cuda")
        b_c = bias(N)
        r = timed(lambda: fb.fp4_linear(fmt, xs, M, K, N, pw_c.codes, pw_c.sf, pw_c.w_global, g_c, b_c, y_c, ws_c,
                                        ws_c.numel()), 2.0 * M * K * N)
        del xs, pw_c, y_c, ws_c
        return r

    for fmt in ("mxfp4", "nvfp4"):
        out[f"{fmt}_ffn_down_75600x13824x5120"] = linear_case(fmt, Mx, 13824, 5120, "gelu")
        if fmt == "nvfp4":
            out["nvfp4_attn_75600x5120x5120"] = linear_case(fmt, Mx, 5120, 5120)
            out["nvfp4_text_kv_512x5120x5120_eager"] = linear_case(fmt, 512, 5120, 5120)
        for Ms in (512, 4096, 16384):
            out[f"{fmt}_m_sweep_{Ms}x5120x13824"] = linear_case(fmt, Ms, 5120, 13824)
    xt = act(512, 5120)
    yt = torch.empty((512, 5120), dtype=torch.bfloat16, device="cuda")
    wst = torch.empty(fb.fp4_linear_workspace_bytes("mxfp4", 512, 5120, 5120), dtype=torch.uint8, device="cuda")
    call_t = lambda: fb.fp4_linear("mxfp4", xt, 512, 5120, 5120, pw_a.codes, pw_a.sf, None, None, b_a, yt, wst,
                                   wst.numel())
    out["mxfp4_text_kv_512x5120x5120_eager"] = timed(call_t, 2.0 * 512 * 5120 * 5120, n=200)
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        call_t()
    side.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        call_t()
    out["mxfp4_text_kv_512x5120x5120_graph"] = timed(graph.replay, 2.0 * 512 * 5120 * 5120, n=200)
    del graph
    # FP4 attention operands at the Wan2.2 sequence length: the head-major K quantizer
    # (40 heads of 128) and one head's 75600 x 75648 score GEMM (bound by writing S)
    Ta, Ha = 75600, 40
    for fmt in ("mxfp4", "nvfp4"):
        f = fb.MXFP4 if fmt == "mxfp4" else fb.NVFP4
        qa, ka = act(Ta, Ha * 128), act(Ta, Ha * 128)
        g_q = g_k = None
        if fmt == "nvfp4":
            g_q, _ = fb.calibrate_act_global(qa)
            g_k, _ = fb.calibrate_act_global(ka)
        qh = fb.quantize_heads(qa, Ha, fmt, g_q)
        kh = fb.quantize_heads(ka, Ha, fmt, g_k)
        qb = Ta * Ha * 128 * 2 + fb.fp4_heads_codes_bytes(f, Ta, Ha) + fb.fp4_heads_sf_bytes(f, Ta, Ha)
        kc_buf, ks_buf = kh
        r_q = timed(lambda: fb.fp4_quantize_heads(f, ka, Ta, Ha, 128, g_k, kc_buf, ks_buf), 0.0)
        r_q["gbs"] = qb / (r_q["ms"] / 1e3) / 1e9
        out[f"{fmt}_attn_quantize_heads_75600x40x128"] = r_q
        s_buf = torch.empty((Ta, (Ta + 127) // 128 * 128), dtype=torch.bfloat16, device="cuda")
        r_s = timed(lambda: fb.attn_scores(qh, kh, Ta, Ta, 17, fmt, g_q, g_k, s_buf), 2.0 * Ta * s_buf.shape[1] * 128,
                    n=10)
        r_s["s_write_gbs"] = s_buf.numel() * 2 / (r_s["ms"] / 1e3) / 1e9
        out[f"{fmt}_attn_scores_head_75600x75648x128"] = r_s
        # the rest of the head: V^T quantizer (all 40 heads), softmax + P quantize, and O = P V
        # (K = the 75648 padded keys); NVFP4 with V's global and P's constant 1/2688
        va = act(Ta, Ha * 128)
        g_v = fb.calibrate_act_global(va)[0] if fmt == "nvfp4" else None
        g_p = torch.tensor([fb.P_GLOBAL_NVFP4], dtype=torch.float32, device="cuda") if fmt == "nvfp4" else None
        vt = fb.quantize_heads_vt(va, Ha, fmt, g_v)
        kp = s_buf.shape[1]
        r_v = timed(lambda: fb.fp4_quantize_heads_vt(f, va, Ta, Ha, 128, g_v, vt[0], vt[1]), 0.0)
        r_v["gbs"] = (Ta * Ha * 128 * 2 + vt[0].numel() + vt[1].numel()) / (r_v["ms"] / 1e3) / 1e9
        out[f"{fmt}_attn_quantize_heads_vt_75600x40x128"] = r_v
        pc, ps, st = fb.attn_softmax_quant(s_buf, Ta, Ta, 128 ** -0.5, fmt, g_p)
        r_m = timed(lambda: fb.fp4_attn_softmax_quant(f, s_buf, Ta, Ta, 128 ** -0.5, g_p, st, pc, ps), 0.0, n=10)
        # S read twice (row max, then weights + sums + quantize), P codes and scales written
        r_m["gbs"] = (2 * s_buf.numel() * 2 + pc.numel() + ps.numel()) / (r_m["ms"] / 1e3) / 1e9
        out[f"{fmt}_attn_softmax_quant_head_75600x75648"] = r_m
        o_buf = fb.attn_pv((pc, ps, st), vt, Ta, Ta, 17, fmt, g_p, g_v)
        out[f"{fmt}_attn_pv_head_75600x128x75648"] = timed(
            lambda: fb.attn_pv((pc, ps, st), vt, Ta, Ta, 17, fmt, g_p, g_v, o=o_buf), 2.0 * Ta * kp * 128, n=10)
        # the same head in one kernel (streaming form): S and P~ never leave the SM
        st_f = torch.empty((Ta, 2), dtype=torch.float32, device="cuda")
        out[f"{fmt}_attn_fused_head_75600x75648x128"] = timed(
            lambda: fb.attn_fused(qh, kh, vt, Ta, Ta, 17, 128 ** -0.5, fmt, g_q, g_k, g_v, g_p, o=o_buf, stats=st_f),
            4.0 * Ta * kp * 128, n=10)
        del st_f
        del va, vt, pc, ps, st, o_buf
        del qa, ka, qh, kh, kc_buf, ks_buf, s_buf
    # W4A8 SVDQuant linear at the TI2V-5B shape (MXFP8 activations, rank 32)
    Mw, Kw, Nw, r = 4290, 3072, 14336, 32
    xw = act(Mw, Kw)
    rp = fb.pack_weight(wgt(Nw, Kw), "mxfp4")
    l1 = wgt(Kw, r, 0.05)
    l2 = wgt(r, Nw, 0.05)
    bw = bias(Nw)
    yw = torch.empty((Mw, Nw), dtype=torch.bfloat16, device="cuda")
    wsw = torch.empty(fb.w4a8_workspace_bytes(Mw, Kw, Nw, r), dtype=torch.uint8, device="cuda")
    flop_w = 2.0 * Mw * Kw * Nw + 2.0 * Mw * Kw * r + 2.0 * Mw * r * Nw
    out["w4a8_svd_linear_4290x3072x14336"] = timed(
        lambda: fb.w4a8_svd_linear(xw, Mw, Kw, Nw, rp.codes, rp.sf, l1, l2, r, bw, yw, wsw, wsw.numel()), flop_w,
        n=100)
    wsw4 = torch.empty(fb.w4a4_workspace_bytes(Mw, Kw, Nw, r), dtype=torch.uint8, device="cuda")
    out["w4a4_svd_linear_4290x3072x14336"] = timed(
        lambda: fb.w4a4_svd_linear(xw, Mw, Kw, Nw, rp.codes, rp.sf, l1, l2, r, bw, yw, wsw4, wsw4.numel()), flop_w,
        n=100)
    for k, v in out.items():
        v["note"] = "pct_nominal: of 9 PFLOP/s dense FP4" + (" (W4A8 runs at the FP8 rate, nominal 4.5)"
                                                             if k.startswith("w4a8") else "")
        if "quantize_heads" in k:
            v["note"] = "HBM-bound: gbs = bf16 read + codes and scales written, per second"
        elif "softmax_quant" in k:
            v["note"] = "HBM- and exp2-bound: gbs = S read twice + P codes and scales written, per second"
        elif "attn_pv" in k:
            v["note"] = "P V with N = 128 (half of each 256-wide pair MMA); pct_nominal of 9 PFLOP/s dense FP4"
        elif "attn_fused" in k:
            v["note"] = ("one head in one kernel: S = Q K^T and O = P~ V on the tensor cores, softmax + P~ quantize "
                         "on the SM; pct_nominal of 9 PFLOP/s dense FP4 over both products")
        elif "attn_scores" in k:
            v["note"] = "bound by writing S (bf16): s_write_gbs; pct_nominal of 9 PFLOP/s dense FP4"
    return out


# ----------------------------------------------------------------------------- native arm
def native_arm(args):
    import torch

    rank, world, local = dist_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    import fp4_block_scaled_act_b200 as fb

    fb.lib()  # fails loudly if the CUDA library is missing
    fb.lib().fp4bsa_set_gemm_ctas(args.gemm_ctas)
    pair = args.gemm_ctas != 1 and M > 128
    x_bits, w_bits, b_bits = make_inputs(rank)
    x = to_dev(x_bits, torch, torch.bfloat16)
    bias = to_dev(b_bits, torch, torch.float16)
    pw = fb.pack_weight(to_dev(w_bits, torch, torch.bfloat16), FMT)
    # NVFP4: the layer's static activation global (device scalar), calibrated untimed
    a_global = nv_static_global(fb, torch) if FMT == "nvfp4" else None
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws_bytes = fb.fp4_linear_workspace_bytes(FMT, M, K, N)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    codes = ws[: fb.fp4_codes_bytes(FMT, M, K)]
    sf_off = (codes.numel() + 255) // 256 * 256
    sf = ws[sf_off: sf_off + fb.fp4_sf_bytes(FMT, M, K)]
    stream = torch.cuda.current_stream()

    def step(ev=None):
        # fp4_linear is exactly these two launches; calling them separately lets the
        # events time each kernel on the launching stream
        if ev is not None:
            ev[0].record(stream)
        fb.fp4_quantize_act(FMT, x, M, K, a_global, codes, sf)
        if ev is not None:
            ev[1].record(stream)
        fb.fp4_gemm(FMT, codes, sf, M, K, N, pw.codes, pw.sf, pw.w_global, a_global, bias, y)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    st = fb.fp4_sync_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {fb.fp4_status_string(st)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    clocks = ClockSampler(vis.split(",")[local].strip() if vis else str(local))
    clocks.start()
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.time()
    pr0 = probe_clocks(fb, torch)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    pr1 = probe_clocks(fb, torch)
    torch.cuda.synchronize()
    w1 = time.time()
    if dist:
        dist.barrier()
    clk = clocks.stop(w0, w1)
    clk["sm_mhz_in_kernel"], clk["sm_probed"] = probe_mhz(pr0, pr1)
    st = fb.fp4_sync_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {fb.fp4_status_string(st)}")
    total_ms = t_start.elapsed_time(t_end)
    q_ms = [e[0].elapsed_time(e[1]) for e in evs]
    g_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms = max_over_ranks(total_ms, dist)
    ms_per_step = total_ms / args.steps
    value = job_tflops(FLOP_PER_STEP, world, args.steps, total_ms)

    # ---- end to end through the public API, host buffers (pinned), copies inside the timing
    # (fb.linear_host: row chunks through fp4_linear with both copy directions overlapped)
    x_host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    pipe = fb.HostPipeline(FMT, min(M, 8192), K, N)

    def e2e_step():
        fb.linear_host(x_host, pw, pipe, bias, a_global, y_host)

    for _ in range(2):
        e2e_step()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dist)
    e2e_value = job_tflops(FLOP_PER_STEP, world, args.e2e_steps, e2e_ms)

    # ---- roofline of the dominant kernel (the GEMM), live CUDA-event durations
    pk, pk_kind = peaks()
    g_avg = sum(g_ms) / len(g_ms)
    q_avg = sum(q_ms) / len(q_ms)
    gemm_tflops = FLOP_PER_STEP / (g_avg / 1e3) / 1e12
    # denominator: the FP4 peak derived from the measured bf16 GEMM rate (x4, the nominal
    # FP4 / BF16 ratio) -- its sustained figure only when this run's timed region itself
    # lasted seconds under the power cap, else the burst figure
    region_s = total_ms / 1e3
    sustained = region_s >= 2.0 and "sw_power_cap" in (clk.get("reasons") or [])
    bf16 = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    fp4_peak = bf16 * FP4_PER_BF16
    # the tensor pipe's own rate: 32768 FP4 FLOP per clock per SM (a 256x256x64 block-scaled
    # MMA every 128 cycles per SM pair), at the SM clock measured inside the timed region
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    mhz = clk.get("sm_mhz_in_kernel")
    pipe_frac = FLOP_PER_STEP / (g_avg / 1e3) / (mhz * 1e6 * 32768 * sms) if mhz else None
    q_bytes = 2 * M * K + M * K // 2 + ((M + 127) // 128 * 128) * (K // (32 if FMT == "mxfp4" else 16))
    q_gbs = q_bytes / (q_avg / 1e3) / 1e9
    traffic = gemm_traffic(pair) if FMT == "mxfp4" else None  # counters recorded for MXFP4

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp4", "data": "synthetic",
        "config": config_dict(args.gpus),
        "pct_nominal_fp4_peak": 100.0 * value / world / NOMINAL_FP4_TFLOPS,
        "roofline": {"bound": "tensor", "kernel": f"gemm2_kernel<{FMT.upper()}> (2-CTA 256x256)" if pair
                     else f"gemm_kernel<{FMT.upper()}> (1-CTA 128x256)", "achieved": gemm_tflops,
                     "peak": fp4_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                     "peak_source": f"{pk_kind} bf16 {'sustained' if sustained else 'burst'} {bf16} x "
                                    f"{FP4_PER_BF16:g} (nominal FP4/BF16); timed region {region_s:.3f} s, "
                                    f"power cap {'seen' if 'sw_power_cap' in (clk.get('reasons') or []) else 'not seen'}",
                     "frac_of_nominal_9pf": gemm_tflops / NOMINAL_FP4_TFLOPS,
                     "tensor_pipe_frac_at_measured_clock": pipe_frac,
                     "traffic": traffic,
                     "algorithmic_flop_per_launch": FLOP_PER_STEP, "avg_launch_ms": g_avg,
                     "quant": {"bound": "hbm", "kernel": f"quant_kernel<{FMT.upper()}>", "achieved": q_gbs,
                               "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": q_gbs / pk["hbm_gbs"],
                               "algorithmic_bytes_per_launch": q_bytes, "avg_launch_ms": q_avg}},
        "kernels": {"quant_ms": q_avg, "quant_gbs": q_gbs, "quant_hbm_frac": q_gbs / pk["hbm_gbs"], "gemm_ms": g_avg},
        "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": x_bits.nbytes,
                "d2h_bytes_per_step": M * N * 2, "steps": args.e2e_steps},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
    }
    if not args.no_extra and world == 1:
        del x, y, ws, codes, sf
        torch.cuda.empty_cache()
        line["extra"] = extra_workloads(fb, torch, args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(x_bits, w_bits, b_bits)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    global M, WORKLOAD, FLOP_PER_STEP, FMT
    args = parse()
    if args.fmt != FMT:
        FMT = args.fmt
        WORKLOAD = f"wan22_t2v_a14b_ffn_up_{FMT}"
    if args.m != M:
        M = args.m
        WORKLOAD = f"ffn_up_{FMT}_m{M}"
        FLOP_PER_STEP = 2.0 * M * K * N
    if args.attn_tokens:
        return attn_profile(args)
    if args.impl == "reference":
        return reference_arm(args)
    return native_arm(args)


if __name__ == "__main__":
    sys.exit(main())
