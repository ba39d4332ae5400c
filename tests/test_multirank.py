"""Host logic of bench.py on CPU: multi-rank timing with world-size-2 gloo ranks, the
NVFP4 calibration, and the reference arm's JSON line.

The data-parallel path shards by batch: every rank quantizes and multiplies its own
activations against the shared weight, with no collective on the data path.  The only
cross-rank steps are the barriers around the timed region and the maximum over ranks of
its duration; the job's throughput is the work of all ranks over that maximum.
"""
import argparse
import datetime
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_q):
    import torch.distributed as dist

    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        slowest = bench.max_over_ranks(times[rank], dist, "cpu")
        value = bench.job_tflops(1e12, world, 10, slowest)
        dist.barrier()
        out_q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_count_all_work():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [3.0, 5.0]  # ms of each rank's timed region
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(60)
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, slowest, value in res:
        assert slowest == 5.0
        # 1 TFLOP per rank-step, 2 ranks, 10 steps, over the slowest rank's 5 ms
        assert value == pytest.approx(4000.0)


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(2.5) == 2.5
    assert bench.job_tflops(2.0e12, 1, 4, 8.0) == pytest.approx(1000.0)


def test_each_rank_gets_its_own_batch_and_the_shared_weight():
    import bench

    x0, w0, b0 = bench.make_inputs(0, 8, 128, 16)
    x1, w1, b1 = bench.make_inputs(1, 8, 128, 16)
    x0_again, _, _ = bench.make_inputs(0, 8, 128, 16)
    assert x0.shape == (8, 128) and w0.shape == (16, 128) and b0.shape == (16,)
    assert not np.array_equal(x0, x1)
    assert np.array_equal(x0, x0_again)
    assert np.array_equal(w0, w1) and np.array_equal(b0, b1)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(gpus=2, steps=1, warmup=0, impl="reference")
    assert bench.reference_arm(args) == 0
    assert capsys.readouterr().out == ""


def test_nvfp4_bench_oracle_global_is_the_calibration_batch_global():
    """bench.py --fmt nvfp4: the oracle legs use the oracle's global of the same 4096-token
    calibration batch that the native arm hands to fp4_calibrate_act_global (the native side
    is checked bit for bit on the GPU in test_gpu_quant.py)."""
    import bench
    import oracle
    import synth

    k = 256
    s = synth.seeds_for(4, layer=1)
    cal = synth.activation(s["x"] + 104729, 4096, k, "lognormal", gain_seed=s["gain"])
    np.testing.assert_array_equal(bench.nv_calibration_batch(k), cal)
    assert bench.oracle_static_global(k) == oracle.nv_global(oracle.tensor_amax(cal))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_reference_arm_json_line(fmt):
    """bench.py --impl reference on rank 0: one JSON line, the native arm's metric, unit and
    workload, the oracle as its own cpu_baseline and e2e (no host-device copies)."""
    import json
    import subprocess

    import bench

    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0", "--fmt", fmt], capture_output=True, text=True, timeout=300,
                         env={**os.environ, "RANK": "0", "WORLD_SIZE": "1"})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOPS"
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 0
    assert d["config"]["fmt"] == fmt and (d["config"]["M"], d["config"]["K"], d["config"]["N"]) == (75600, 5120, 13824)
    assert d["value"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and isinstance(cb["cores"], int) and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def _shard_main(rank, world, port, out_q):
    """Rank r quantizes and multiplies its own 256-row shard; rank 0 gathers the shards."""
    import torch
    import torch.distributed as dist

    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import oracle
    import synth

    oracle.build()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        M, K, N = 512, 256, 128
        x = synth.activation(71, M, K, "lognormal", gain_seed=72)
        w = synth.weight(73, N, K)
        b = synth.bias(74, N)
        g_a = oracle.nv_global(oracle.tensor_amax(x))
        rows = np.arange(rank * M // world, (rank + 1) * M // world)
        res = []
        for fmt in (oracle.MX, oracle.NV):
            g = g_a if fmt == oracle.NV else None
            c, s = oracle.quantize(fmt, np.ascontiguousarray(x[rows]), g)
            y, _ = oracle.fp4_linear_rows(fmt, x, w, b, rows, g_a=g)
            for part in (torch.from_numpy(c.astype(np.int32)), torch.from_numpy(s.astype(np.int32)),
                         torch.from_numpy(y)):
                got = [torch.empty_like(part) for _ in range(world)]
                dist.all_gather(got, part)
                res.append([t.numpy() for t in got])
        if rank == 0:
            out_q.put(res)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_row_shards_concatenate_to_the_whole():
    """The path shards by rows with no collective on the data: two gloo ranks, 256 rows each
    (whole 128-row scale blocks), give exactly the codes and scale bytes of the unsharded
    512-row quantize, and the unsharded GEMM rows, in both formats."""
    import torch.multiprocessing as mp

    import oracle
    import synth

    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=180)
    for p in procs:
        p.join(60)
    assert [p.exitcode for p in procs] == [0, 0]
    M, K, N = 512, 256, 128
    x = synth.activation(71, M, K, "lognormal", gain_seed=72)
    w = synth.weight(73, N, K)
    b = synth.bias(74, N)
    g_a = oracle.nv_global(oracle.tensor_amax(x))
    for i, fmt in enumerate((oracle.MX, oracle.NV)):
        g = g_a if fmt == oracle.NV else None
        c, s = oracle.quantize(fmt, x, g)
        y, S = oracle.fp4_linear_rows(fmt, x, w, b, np.arange(M), g_a=g)
        cs, ss, ys = res[3 * i: 3 * i + 3]
        np.testing.assert_array_equal(np.concatenate(cs).astype(np.uint8), c)
        np.testing.assert_array_equal(np.concatenate(ss).astype(np.uint8), s)
        # the same rows in fp64; only the product's summation blocking may differ
        assert np.all(np.abs(np.concatenate(ys) - y) <= 1e-12 * S)
