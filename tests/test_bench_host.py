"""Host-side logic of bench.py without a GPU: whole-job aggregation over gloo ranks (max over
ranks, world-size scaling), workload byte / FLOP accounting, and the reference (oracle) arm."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank               # rank 1 is the slowest
        value, max_ms = bench.job_throughput(local_ms, 1e12, 4, world)
        bench.barrier(world)
        out[rank] = (value, max_ms)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_job_throughput_is_max_over_ranks(world):
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        value, max_ms = out[rank]
        assert max_ms == 15.0
        # two ranks x 4 steps x 1 TFLOP over the slowest rank's 15 ms
        assert abs(value - world * 4 * 1e12 / 15e-3 / 1e12) < 1e-9


def test_single_rank_needs_no_process_group():
    value, max_ms = bench.job_throughput(20.0, 2e12, 10, 1)
    assert max_ms == 20.0 and abs(value - 1000.0) < 1e-9


def test_algorithmic_bytes_and_flops():
    # config 0: M=1, K=N=4096, gs 128, zeros: 8 MiB weights + scales + zeros + A + C
    b = bench.shape_bytes("w4a16", 1, 4096, 4096, 1)
    assert b == 4096 * 4096 // 2 + 4096 * 32 * 2 * 2 + 2 * 4096 + 2 * 4096
    assert bench.shape_bytes("w8a8", 1, 16384, 16384, 0) == 16384 * 16384 + 16384 + 4 * 16384
    assert bench.shape_bytes("w2a8", 1, 16384, 16384, 0) == 16384 * 16384 // 4 + 16384 + 4 * 16384
    assert bench.shape_flops(16384, 16384, 16384) == 2.0 * 16384 ** 3


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--workload", "w4a16_llama"],
                       capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_int_workload_and_non_zero_ranks():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--workload", "w2a8_nk16384",
                        "--cpu-budget", "4"],
                       capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([ln for ln in r.stdout.splitlines() if ln.strip()][-1])
    assert d["unit"] == "TOP/s" and d["dtype"] == "f64" and d["config"]["op"] == "w2a8"
    # under torchrun only rank 0 times the oracle; the others exit 0 without output
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_every_workload_is_consistent():
    for name, wl in bench.WORKLOADS.items():
        assert wl["op"] in bench.METRICS and wl["op"] in bench.UNITS and wl["op"] in bench.DTYPES
        for M, K, N in wl["shapes"]:
            assert bench.shape_bytes(wl["op"], M, K, N, wl["has_zero"]) > 0
            assert bench.shape_flops(M, K, N) == 2.0 * M * N * K


def test_tile_samples_cover_every_tile_in_bounds():
    for M, N in [(1, 1), (1, 16384), (32, 300), (129, 257), (16384, 4096)]:
        ms, ns = bench.tile_samples(M, N, seed=3)
        assert ms.min() >= 0 and ns.min() >= 0 and ms.max() < M and ns.max() < N
        tiles = set(zip((ms // 128).tolist(), (ns // 128).tolist()))
        assert tiles == {(i, j) for i in range(-(-M // 128)) for j in range(-(-N // 128))}
        for corner in [(0, 0), (0, N - 1), (M - 1, 0), (M - 1, N - 1)]:
            assert corner in set(zip(ms.tolist(), ns.tolist()))


def test_parity_leg_accepts_the_oracle_and_catches_a_planted_error():
    """The bench's parity leg on CPU: the oracle's own result rounded to fp16 passes; the same
    result with one element pushed past the tolerance, or an integer result off by one, fails."""
    import numpy as np
    import torch
    import oracle
    from gemv_w4a16_w8a8_b200 import synth
    M, K, N = 3, 256, 200
    h = synth.w4a16_inputs(M, N, K, 128, True, seed=5)
    ref = oracle.w4a16(h["A"], oracle.pack_int4(h["codes"]), h["scales"], h["zeros"], K, 128)
    C = torch.from_numpy(ref.astype(np.float16))
    p = bench.parity_check("w4a16", dict(h), C, M, K, N, 1, seed=9)
    assert p["bad"] == 0 and p["checked"] == 2 * 1 + 4
    C2 = C.clone()
    C2[M - 1, N - 1] += 0.5 + 0.02 * abs(float(C2[M - 1, N - 1]))
    assert bench.parity_check("w4a16", dict(h), C2, M, K, N, 1, seed=9)["bad"] >= 1
    e = synth.w8a8_inputs(2, 130, 64, seed=1)
    Ci = torch.from_numpy(oracle.w8a8(e["A"], e["W"]).astype(np.int32))
    assert bench.parity_check("w8a8", e, Ci, 2, 64, 130, 0, seed=2)["bad"] == 0
    Ci[0, 0] += 1
    assert bench.parity_check("w8a8", e, Ci, 2, 64, 130, 0, seed=2)["bad"] == 1
