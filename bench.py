"""Benchmark of the low-bit matmul library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--no-extras]

A step is one pass of the hot path over one batch of seeded synthetic input: for every shape
of the workload one matmul call (argument checks, configuration lookup, split-K zeroing when
the configuration splits K, the kernel). The per-shape configuration search runs once before
the timed region, as a deployment would run it once per shape. Inputs sit in HBM before the
timed region; weight sets rotate so that no call finds its weights in L2.

After the timed region the device error word is checked (a kernel that gave up a bounded wait
fails the run) and the output of every timed shape, under the configuration that was timed, is
compared with the host oracle on sampled elements: one random element in every 128 x 128 tile
of C plus its corners ("parity" in the line). Integer outputs must match exactly, fp16 outputs
within |C - ref| <= 0.02 + 0.01 |ref| per element and 5e-3 relative Frobenius error over the
sample. A failed check still prints the line and exits with status 3.

The headline workload (--workload, default the N = K = 16384 W4A16 sweep over M) gives `value`.
Unless --no-extras, the other benchmark configurations are timed after it, shape by shape, into
"configs" of the same line: one-token W4A16 at K = N = 4096 with split_k 1 and 4, the LLaMA-style
shapes with and without zero points, W8A8 and W2A8 over M at N = K = 16384, W4A16 without zero
points and the dense fp16 baseline at M = 512 / 16384, the same W4A16 codes in the pre-shuffled
(interleaved) int4 layout, and a sweep of the tensor-core pipeline depth (stages 2..5) on the
large-M shapes.

Prints one JSON line (rank 0). Under torchrun every rank runs the same workload on its own GPU
(independent replicas, no collective on the data path); `value` is the whole-job throughput
(all ranks' FLOPs over the slowest rank's time).

--impl reference times the host oracle (plain C, fp64) on a bounded sample of the same
workload on this machine's cores and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
GS = 128

# ---- workloads -------------------------------------------------------------------------------
# Each shape: (M, K, N). W4A16: group_size 128, fp16 zeros fixed at 8 (has_zero=1) unless noted.
WORKLOADS = {
    # int4-weight GEMM sweep over M at N = K = 16384 (the BitBLAS Matmul benchmark shapes)
    "w4a16_nk16384": {"op": "w4a16", "has_zero": 1,
                      "shapes": [(1, 16384, 16384), (32, 16384, 16384), (128, 16384, 16384),
                                 (512, 16384, 16384), (16384, 16384, 16384)]},
    # one token at K = N = 4096 (hidet issue #364, k-parts 1 and 4 sweep)
    "w4a16_m1_k4096": {"op": "w4a16", "has_zero": 1, "shapes": [(1, 4096, 4096)]},
    # LLaMA-style layer shapes (hidet issue #364, k-parts=4 table), M = 1 and 128
    "w4a16_llama": {"op": "w4a16", "has_zero": 1,
                    "shapes": [(1, 4096, 11008), (1, 11008, 4096), (1, 4096, 4096),
                               (1, 4096, 32000), (128, 4096, 11008), (128, 11008, 4096),
                               (128, 4096, 4096), (128, 4096, 32000)]},
    "w4a16_llama_nozero": {"op": "w4a16", "has_zero": 0,
                           "shapes": [(1, 4096, 11008), (1, 11008, 4096), (1, 4096, 4096),
                                      (1, 4096, 32000), (128, 4096, 11008), (128, 11008, 4096),
                                      (128, 4096, 4096), (128, 4096, 32000)]},
    # the small-M part of the sweep alone
    "w4a16_nk16384_small_m": {"op": "w4a16", "has_zero": 1,
                              "shapes": [(1, 16384, 16384), (32, 16384, 16384),
                                         (128, 16384, 16384)]},
    # int8 x int8 -> int32 and int8 x int2 -> int32 over the BitBLAS M sweep at N = K = 16384
    "w8a8_nk16384": {"op": "w8a8", "has_zero": 0,
                     "shapes": [(1, 16384, 16384), (32, 16384, 16384), (128, 16384, 16384),
                                (512, 16384, 16384)]},
    "w2a8_nk16384": {"op": "w2a8", "has_zero": 0,
                     "shapes": [(1, 16384, 16384), (32, 16384, 16384), (128, 16384, 16384),
                                (512, 16384, 16384)]},
    # the compute-bound shapes: W4A16 without zero points, and the dense fp16 baseline
    "w4a16_nozero_large_m": {"op": "w4a16", "has_zero": 0,
                             "shapes": [(512, 16384, 16384), (16384, 16384, 16384)]},
    # the same codes in the pre-shuffled (interleaved) int4 layout, zero points as the headline
    "w4a16_interleaved": {"op": "w4a16", "has_zero": 1, "layout": "interleaved",
                          "shapes": [(1, 16384, 16384), (128, 16384, 16384), (512, 16384, 16384),
                                     (16384, 16384, 16384)]},
    "dense_large_m": {"op": "dense", "has_zero": 0,
                      "shapes": [(512, 16384, 16384), (16384, 16384, 16384)]},
}
METRICS = {
    "w4a16": "int4-weight GEMM TFLOP/s & effective HBM GB/s, M=1..16384, N=K=16384",
    "w8a8": "int8 x int8 -> int32 GEMM TOP/s & effective HBM GB/s, N=K=16384",
    "w2a8": "int8 x int2 -> int32 GEMM TOP/s & effective HBM GB/s, N=K=16384",
    "dense": "fp16 x fp16 -> fp16 GEMM TFLOP/s (in-library baseline), N=K=16384",
}
DTYPES = {"w4a16": "f16xu4->f32acc->f16", "w8a8": "s8xs8->s32", "w2a8": "s8xs2->s32",
          "dense": "f16xf16->f32acc->f16"}
UNITS = {"w4a16": "TFLOP/s", "w8a8": "TOP/s", "w2a8": "TOP/s", "dense": "TFLOP/s"}
DEFAULT_WORKLOAD = "w4a16_nk16384"

# The other benchmark configurations, timed after the headline: (name, workload, explicit
# split_k values timed on the planner's path before the search, stage sweep on the large shapes)
EXTRAS = [
    ("w4a16_m1_k4096_n4096", "w4a16_m1_k4096", (1, 4), False),
    ("w4a16_llama", "w4a16_llama", (), False),
    ("w4a16_llama_nozero", "w4a16_llama_nozero", (), False),
    ("w8a8_nk16384", "w8a8_nk16384", (1, 4), False),
    ("w2a8_nk16384", "w2a8_nk16384", (), False),
    ("w4a16_nozero_large_m", "w4a16_nozero_large_m", (), True),
    ("w4a16_interleaved", "w4a16_interleaved", (), False),
    ("dense_large_m", "dense_large_m", (), True),
]
SWEEP_STAGES = (2, 3, 4, 5)


# DRAM bytes per launch of the dominant kernel (dram__bytes_read.sum + dram__bytes_write.sum),
# by weight-major token tile: on M = 4096, N = K = 16384 the 256-token tile (3 stages) read
# 1271.105 MB and wrote 129.454 MB; the 512-token tile (4 half-tile stages, transposed 16-byte
# epilogue stores) read 817.545 MB and wrote 121.407 MB. An M = 16384 launch runs the same
# pattern (groups of 2048 tokens against all 128 weight tiles, weights read once per group) 4
# times as often, so its traffic is scaled by 4.
TRAFFIC_BYTES = {(16384, 16384, 16384, 256): 4 * (1271105000 + 129453568),
                 (16384, 16384, 16384, 512): 4 * (817544704 + 121406976)}
TRAFFIC_SOURCE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of the M = 4096 launch of the "
                  "same tile, scaled by 4 (its 2 groups of 2048 tokens against 8)")


def shape_bytes(op, M, K, N, has_zero, gs=GS):
    if op == "w4a16":
        return N * K // 2 + N * (K // gs) * 2 * (1 + has_zero) + 2 * M * K + 2 * M * N
    if op == "w8a8":
        return N * K + M * K + 4 * M * N
    if op == "w2a8":
        return N * K // 4 + M * K + 4 * M * N
    return 2 * N * K + 2 * M * K + 2 * M * N


def shape_flops(M, K, N):
    return 2.0 * M * N * K


# ---- helpers ------------------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def roofline_of(op, M, K, N, hz, ms, peaks, burst=True):
    """Which roof bounds the shape (arithmetic intensity against the ridge of the measured
    peaks) and the achieved fraction of it for a call of `ms` milliseconds. int8 contractions
    take the measured bf16 peak times the nominal dense int8 / bf16 ratio (2)."""
    fl = shape_flops(M, K, N)
    by = shape_bytes(op, M, K, N, hz)
    tscale = 2.0 if op in ("w8a8", "w2a8") else 1.0
    tpeak = tscale * (peaks["bf16_tflops"] if burst else peaks["bf16_tflops_sustained"])
    ridge = tpeak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if fl / by >= ridge:
        ach = fl / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": round(ach, 2), "peak": round(tpeak, 1),
                "unit": UNITS[op], "frac": round(ach / tpeak, 4)}
    ach = by / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4)}


class ClockSampler:
    """nvidia-smi clock / throttle sampling every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"qgemm_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def wait_first_sample(self, timeout=5.0):
        t = time.time()
        while self.proc is not None and time.time() - t < timeout:
            self.f.flush()
            if os.path.exists(self.path) and os.path.getsize(self.path) > 0:
                return
            time.sleep(0.05)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [s for s in sm if smax and s > 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(local_ms: float, flops_per_step: float, steps: int, world: int,
                   device=None) -> tuple[float, float]:
    """Whole-job TFLOP/s: every rank ran `steps` steps of `flops_per_step`; the job took as
    long as its slowest rank. Returns (value, max_ms)."""
    max_ms = max_over_ranks(local_ms, world, device)
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12, max_ms


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def tile_samples(M: int, N: int, seed: int, tm: int = 128, tn: int = 128):
    """(m, n) positions of C to check: one seeded random element inside every tm x tn tile
    (the ragged edge tiles included) plus the four corners of C."""
    rng = np.random.default_rng(seed)
    mt, nt = -(-M // tm), -(-N // tn)
    i = np.repeat(np.arange(mt, dtype=np.int64), nt)
    j = np.tile(np.arange(nt, dtype=np.int64), mt)
    hm = np.minimum(tm, M - i * tm)
    hn = np.minimum(tn, N - j * tn)
    ms = i * tm + (rng.random(i.size) * hm).astype(np.int64)
    ns = j * tn + (rng.random(j.size) * hn).astype(np.int64)
    ms = np.concatenate([ms, np.array([0, 0, M - 1, M - 1], dtype=np.int64)])
    ns = np.concatenate([ns, np.array([0, N - 1, 0, N - 1], dtype=np.int64)])
    return ms, ns


# ---- parity leg: the timed outputs against the host oracle --------------------------------------

def parity_check(op, h, C, M, K, N, hz, seed):
    """Compare sampled elements of the device result C (torch, [M, N]) with the host oracle on
    the same seeded host inputs `h`. Returns {"checked", "bad", ...}."""
    import torch
    import oracle
    ms, ns = tile_samples(M, N, seed)
    idx = torch.from_numpy(ms * N + ns).to(C.device)
    got = C.reshape(-1).index_select(0, idx).cpu().numpy()
    if op == "w4a16":
        if "Wq_oracle" not in h:
            h["Wq_oracle"] = oracle.pack_int4(h["codes"])
        ref = oracle.w4a16_at(h["A"], h["Wq_oracle"], h["scales"], h["zeros"], K, GS, ms, ns)
    elif op == "dense":
        ref = oracle.dense_f16_at(h["A"], h["W"], ms, ns)
    elif op == "w8a8":
        ref = oracle.w8a8_at(h["A"], h["W"], ms, ns)
    else:
        if "Wq_oracle" not in h:
            h["Wq_oracle"] = oracle.pack_int2(h["Wv"])
        ref = oracle.w2a8_at(h["A"], h["Wq_oracle"], ms, ns)
    if op in ("w8a8", "w2a8"):
        bad = int(np.count_nonzero(got.astype(np.int64) != ref))
        return {"checked": int(ms.size), "bad": bad, "rule": "bit-exact"}
    g = got.astype(np.float64)
    err = np.abs(g - ref)
    bad = int(np.count_nonzero(~(err <= oracle.ATOL + oracle.RTOL * np.abs(ref))))
    nr = float(np.linalg.norm(ref))
    frob = float(np.linalg.norm(g - ref)) / nr if nr > 0 else float(np.linalg.norm(g - ref))
    if frob > oracle.FROB:
        bad = max(bad, 1)
    return {"checked": int(ms.size), "bad": bad, "frob": float(f"{frob:.3e}"),
            "rule": "|d| <= 0.02 + 0.01|ref|, frob <= 5e-3"}


def merge_parity(items):
    out = {"checked": 0, "bad": 0}
    for p in items:
        if p is None:
            continue
        out["checked"] += p["checked"]
        out["bad"] += p["bad"]
    return out


# ---- our arm ----------------------------------------------------------------------------------------

def op_code(op, sp=None):
    import gemv_w4a16_w8a8_b200 as qg
    if op == "w4a16" and sp is not None and sp.get("ilv"):
        return qg.OP_W4A16_INTERLEAVED
    return {"w4a16": qg.OP_W4A16, "w8a8": qg.OP_W8A8, "w2a8": qg.OP_W2A8,
            "dense": qg.OP_DENSE_F16}[op]


def host_inputs(op, M, K, N, hz, seed):
    from gemv_w4a16_w8a8_b200 import synth
    if op == "w4a16":
        return synth.w4a16_inputs(M, N, K, GS, bool(hz), seed=seed)
    if op == "w8a8":
        return synth.w8a8_inputs(M, N, K, seed=seed)
    if op == "w2a8":
        return synth.w2a8_inputs(M, N, K, seed=seed)
    return synth.dense_inputs(M, N, K, seed=seed)


def prepare_shape(op, M, K, N, hz, seed, dev, pinned=True, ilv=False):
    """Seeded inputs of one shape in HBM (weights replicated into enough copies, >= 3x L2 in
    total, that consecutive calls never find theirs in L2), plus page-locked host copies of A
    and C for the end-to-end form. The host arrays stay in sp["h"] for the parity leg."""
    import torch
    import gemv_w4a16_w8a8_b200 as qg
    h = host_inputs(op, M, K, N, hz, seed)
    sp = {"M": M, "K": K, "N": N, "hz": hz, "seed": seed, "h": h, "ilv": ilv}
    if op == "w4a16":
        codes = torch.from_numpy(h["codes"]).to(dev)
        W0 = (qg.quant_pack_int4_interleaved if ilv else qg.quant_pack_int4)(codes)
        del codes
        sp["S"] = torch.from_numpy(h["scales"]).to(dev)
        sp["Z"] = torch.from_numpy(h["zeros"]).to(dev) if hz else None
        c_dtype, wbytes = torch.float16, N * K // 2
    elif op == "w8a8":
        W0 = torch.from_numpy(h["W"]).to(dev)
        c_dtype, wbytes = torch.int32, N * K
    elif op == "w2a8":
        W0 = qg.quant_pack_int2(torch.from_numpy(h["Wv"]).to(dev))
        c_dtype, wbytes = torch.int32, N * K // 4
    else:
        W0 = torch.from_numpy(h["W"]).to(dev)
        c_dtype, wbytes = torch.float16, 2 * N * K
    n_sets = max(1, min(64, math.ceil(3 * L2_BYTES / wbytes)))
    sp.update({"A": torch.from_numpy(h["A"]).to(dev),
               "W": [W0] + [W0.clone() for _ in range(n_sets - 1)],
               "C": torch.empty((M, N), dtype=c_dtype, device=dev), "n_sets": n_sets})
    if pinned:
        sp["A_host"] = torch.from_numpy(h["A"]).pin_memory()
        sp["C_host"] = torch.empty((M, N), dtype=c_dtype).pin_memory()
    return sp


def matmul(op, sp, W, split_k=0, A=None, C=None):
    """One call of the library's entry point for this op."""
    import gemv_w4a16_w8a8_b200 as qg
    A = sp["A"] if A is None else A
    C = sp["C"] if C is None else C
    if op == "w4a16":
        mm = qg.qgemm_w4a16_interleaved if sp.get("ilv") else qg.qgemm_w4a16
        mm(A, W, sp["S"], sp["Z"], C=C, group_size=GS, split_k=split_k)
    elif op == "w8a8":
        qg.qgemm_w8a8(A, W, C=C, split_k=split_k)
    elif op == "w2a8":
        qg.qgemm_w2a8(A, W, C=C, split_k=split_k)
    else:
        qg.qgemm_dense_f16(A, W, C=C, split_k=split_k)


def tune_shape(op, sp, hz, no_tune, reps):
    import gemv_w4a16_w8a8_b200 as qg
    M, K, N = sp["M"], sp["K"], sp["N"]
    g_op = GS if op == "w4a16" else -1
    if no_tune:
        return qg.qgemm_plan(op_code(op, sp), M, N, K, g_op, hz)
    return qg.qgemm_tune(op_code(op, sp), sp["A"], sp["W"][0], sp.get("S"), sp.get("Z"), sp["C"],
                         M, N, K, g_op, hz, reps=reps)


def time_shape(op, sp, split_k=0, reps=None):
    """Mean device time (ms) of one call from a CUDA graph of back-to-back calls, weight sets
    cycling. The graph is replayed once untimed first."""
    import torch
    n = sp["n_sets"]
    reps = reps or min(64, max(n, 20))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for r in range(reps):
            matmul(op, sp, sp["W"][r % n], split_k)
    g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / reps


CFG_KEYS = ("path", "rows", "bm", "bn", "bk", "stages", "split_k", "swap_ab")


def shape_row(op, sp, ms, cfg, peaks, parity, split_req="tuned"):
    M, K, N, hz = sp["M"], sp["K"], sp["N"], sp["hz"]
    by, fl = shape_bytes(op, M, K, N, hz), shape_flops(M, K, N)
    roof = roofline_of(op, M, K, N, hz, ms, peaks)
    return {"shape_mkn": [M, K, N], "has_zero": hz, "split_k_req": split_req,
            "cfg": {k: cfg[k] for k in CFG_KEYS}, "us": round(ms * 1e3, 2),
            "gbs": round(by / (ms * 1e-3) / 1e9, 1),
            ("tops" if op in ("w8a8", "w2a8") else "tflops"): round(fl / (ms * 1e-3) / 1e12, 2),
            "bound": roof["bound"], "frac": roof["frac"], "parity": parity}


def run_extras(args, dev, peaks, headline_sps, deadline):
    """The other benchmark configurations, shape by shape (see the module docstring)."""
    import torch
    import gemv_w4a16_w8a8_b200 as qg
    out, sweep, skipped = {}, [], []
    for name, wl_name, splits, do_sweep in EXTRAS:
        if time.time() > deadline:
            skipped.append(name)
            continue
        wl = WORKLOADS[wl_name]
        op, hz = wl["op"], wl["has_zero"]
        ilv = wl.get("layout") == "interleaved"
        rows = []
        for si, (M, K, N) in enumerate(wl["shapes"]):
            sp = prepare_shape(op, M, K, N, hz, 7000 + 100 * si + hz, dev, pinned=False, ilv=ilv)
            g_op = GS if op == "w4a16" else -1
            for s in splits:   # the planner's path at the stated split, before the search
                cfg = qg.qgemm_plan(op_code(op, sp), M, N, K, g_op, hz, s)
                ms = time_shape(op, sp, split_k=s)
                par = parity_check(op, sp["h"], sp["C"], M, K, N, hz, sp["seed"])
                rows.append(shape_row(op, sp, ms, cfg, peaks, par, split_req=s))
            cfg = tune_shape(op, sp, hz, args.no_tune, args.tune_reps)
            ms = time_shape(op, sp)
            par = parity_check(op, sp["h"], sp["C"], M, K, N, hz, sp["seed"])
            rows.append(shape_row(op, sp, ms, cfg, peaks, par))
            if do_sweep:
                sweep += stage_sweep(op, sp, cfg, peaks)
            qg.qgemm_sync_check()
            del sp
            torch.cuda.empty_cache()
        out[name] = {"op": op, "has_zero": hz, "per_shape": rows}
        if ilv:
            out[name]["layout"] = "interleaved"
    # the headline's own large-M W4A16 shapes (zero points) in the stage sweep
    for sp in headline_sps:
        if sp["M"] >= 512 and time.time() <= deadline:
            sweep += stage_sweep("w4a16", sp, sp["cfg"], peaks)
    return out, sweep, skipped


def stage_sweep(op, sp, tuned, peaks):
    """Pipeline depth 2..5 of the tensor-core kernel on this shape, the tuned tile and split
    kept; each depth timed and parity-checked, then the tuned configuration restored. When the
    tuned tile is the 512-token one (2 or 4 half-tile stages only), the 256-token tile with the
    same split is swept over 2..5 as well."""
    import gemv_w4a16_w8a8_b200 as qg
    M, K, N, hz = sp["M"], sp["K"], sp["N"], sp["hz"]
    g_op = GS if op == "w4a16" else -1
    rows = []
    if tuned["path"] != qg.PATH_TC:
        return rows
    tiles = [dict(tuned)]
    if tuned["bn"] == 512:
        tiles.append(dict(tuned, bn=256))
    for tile in tiles:
        for st in SWEEP_STAGES:
            cfg = dict(tile)
            cfg["stages"] = st
            try:
                qg.qgemm_set_config(op_code(op, sp), M, N, K, g_op, hz, cfg)
            except qg.QGemmError:
                note = ("the 512-token tile takes 2 or 4 half-tile stages" if cfg["bn"] == 512
                        else "does not fit shared memory")
                rows.append({"op": op, "shape_mkn": [M, K, N], "has_zero": hz, "stages": st,
                             "cfg": cfg, "us": None, "note": note})
                continue
            ms = time_shape(op, sp, reps=max(4, min(20, sp["n_sets"])))
            par = parity_check(op, sp["h"], sp["C"], M, K, N, hz, sp["seed"] + st)
            r = shape_row(op, sp, ms, cfg, peaks, par)
            r.update({"op": op, "stages": st})
            rows.append(r)
    qg.qgemm_set_config(op_code(op, sp), M, N, K, g_op, hz, tuned)
    return rows


def run_ours(args, world, rank, local):
    import torch
    import gemv_w4a16_w8a8_b200 as qg

    t_start = time.time()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    wl = WORKLOADS[args.workload]
    op, hz = wl["op"], wl["has_zero"]
    shapes = wl["shapes"]
    peaks = load_peaks()

    # inputs: one A per shape; weights: each shape's packed matrix replicated into enough
    # copies (>= 3x L2 in total) that consecutive calls of a shape never find theirs in L2
    per_shape = [prepare_shape(op, M, K, N, hz, 1000 * si, dev)
                 for si, (M, K, N) in enumerate(shapes)]
    torch.cuda.synchronize()

    # configuration search (once per shape, before timing)
    tuned = []
    for sp in per_shape:
        cfg = tune_shape(op, sp, hz, args.no_tune, args.tune_reps)
        sp["cfg"] = cfg
        tuned.append({"shape": [sp["M"], sp["K"], sp["N"]], **{k: cfg[k] for k in CFG_KEYS}})
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()

    def call(sp, i):
        matmul(op, sp, sp["W"][i % sp["n_sets"]])

    n_sets = max(sp["n_sets"] for sp in per_shape)

    # eager warm-up (first calls probe the device), then one CUDA graph per weight set holding
    # one whole step: the timed loop replays graphs, so host launch overhead stays out of it
    for i in range(3):
        for sp in per_shape:
            call(sp, i)
    torch.cuda.synchronize()
    graphs = []
    for w in range(n_sets):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for sp in per_shape:
                call(sp, w)
        graphs.append(g)
    # per-shape graphs (R back-to-back calls, weight sets cycling) for the per-call timings
    reps = min(max(n_sets, 20), 64)
    shape_graphs = []
    for sp in per_shape:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(reps):
                call(sp, r)
        shape_graphs.append(g)
    torch.cuda.synchronize()

    clk = ClockSampler(local)
    clk.__enter__()
    clk.wait_first_sample()
    warmup = max(3, args.warmup)
    t_w = time.perf_counter()
    i = 0
    while i < warmup or (time.perf_counter() - t_w < 0.5 and i < 100000):
        graphs[i % n_sets].replay()
        i += 1
        if i % 16 == 0:
            torch.cuda.synchronize()
    warm_steps = i
    torch.cuda.synchronize()

    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("qgemm_timed")     # profilers can restrict capture to this range
    t0.record(stream)
    for i in range(args.steps):
        graphs[(warm_steps + i) % n_sets].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    barrier(world, dev)
    local_ms = t0.elapsed_time(t1)

    # per-call device time of every shape, same launch configuration as the step
    shape_ms = []
    for g in shape_graphs:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        shape_ms.append(e0.elapsed_time(e1) / reps)
    clk.__exit__(None, None, None)
    del graphs, shape_graphs

    # no kernel of the timed region may have given up a bounded wait
    device_error = None
    try:
        qg.qgemm_sync_check()
    except qg.QGemmError as e:
        device_error = str(e)

    # parity of what was timed: every shape's output under its tuned configuration
    parity_rows = [parity_check(op, sp["h"], sp["C"], sp["M"], sp["K"], sp["N"], hz, sp["seed"])
                   for sp in per_shape]

    flops_step = sum(shape_flops(s["M"], s["K"], s["N"]) for s in per_shape)
    bytes_step = sum(shape_bytes(op, s["M"], s["K"], s["N"], hz) for s in per_shape)
    value, total_ms = job_throughput(local_ms, flops_step, args.steps, world, dev)
    ms_per_step = total_ms / args.steps

    # ---- end to end: host A in, host C out, through the same entry point ----
    e2e = run_e2e(args, op, per_shape, hz, stream, world, dev, flops_step)

    # ---- roofline of the dominant call ----
    j = int(np.argmax(shape_ms))
    sp = per_shape[j]
    M, K, N = sp["M"], sp["K"], sp["N"]
    timed_alone = total_ms < 1000.0
    roof = roofline_of(op, M, K, N, hz, shape_ms[j], peaks, burst=timed_alone)
    if args.traffic is not None:
        roof["traffic"] = args.traffic
    elif (M, K, N, sp["cfg"]["bn"]) in TRAFFIC_BYTES and sp["cfg"]["path"] == 2 and \
            sp["cfg"]["swap_ab"] == 1 and sp["cfg"]["bm"] in (0, 128) and sp["cfg"]["rows"] == 0:
        roof["traffic"] = TRAFFIC_BYTES[(M, K, N, sp["cfg"]["bn"])]
        roof["traffic_source"] = TRAFFIC_SOURCE
    else:
        roof["traffic"] = None
    roof["kernel_shape"] = [M, K, N]
    roof["peak_source"] = (f"{peaks['source']} "
                           f"({'burst' if timed_alone else 'sustained'} for tensor peaks"
                           + (", x2 for int8 (nominal dense int8 / bf16)"
                              if op in ("w8a8", "w2a8") else "") + ")")

    details = [shape_row(op, s, t, s["cfg"], peaks, p)
               for s, t, p in zip(per_shape, shape_ms, parity_rows)]

    l2_sets = [s["n_sets"] for s in per_shape]
    extras, sweep, skipped = {}, [], []
    if not args.no_extras and world == 1:
        deadline = time.time() + args.extras_budget
        # the headline's device buffers stay for the stage sweep of its large shapes; the rest go
        for s in per_shape:
            s.pop("A_host", None)
            s.pop("C_host", None)
        big = [s for s in per_shape if s["M"] >= 512]
        for s in per_shape:
            if s["M"] < 512:
                s.clear()
        torch.cuda.empty_cache()
        extras, sweep, skipped = run_extras(args, dev, peaks, big, deadline)
        try:
            qg.qgemm_sync_check()
        except qg.QGemmError as e:
            device_error = device_error or str(e)

    parity = merge_parity(parity_rows + ([e2e.get("parity")] if e2e.get("parity") else []))
    extra_parity = merge_parity([r["parity"] for c in extras.values() for r in c["per_shape"]] +
                                [r.get("parity") for r in sweep])

    out = {
        "metric": METRICS[op],
        "value": round(value, 3),
        "unit": UNITS[op],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPES[op],
        "data": "synthetic",
        "config": {"workload": args.workload, "op": op, "shapes_mkn": [list(s) for s in shapes],
                   "group_size": GS, "has_zero": hz, "parallelism": f"replicas{world}",
                   "l2": "rotating weight copies per shape, >= 3x L2 between reuses "
                         f"({l2_sets})",
                   "tuned": tuned},
        "hbm_gbs_effective": round(world * bytes_step * args.steps / (total_ms * 1e-3) / 1e9, 1),
        "per_shape": details,
        "parity": parity,
        "roofline": roof,
        "e2e": e2e,
        "clocks": clk.summary(),
        "timing": {"step": "CUDA graph of one step replayed back to back (events around the K "
                           "replays)", "per_shape": f"graph of {reps} back-to-back calls per shape",
                   "warmup_steps_run": warm_steps},
        "gpu_launches": args.steps * len(per_shape),
    }
    if extras or sweep:
        out["configs"] = extras
        out["stage_sweep"] = sweep
        out["configs_parity"] = extra_parity
        if skipped:
            out["configs_skipped"] = skipped
    if device_error:
        out["device_error"] = device_error
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_budget)
    out["wall_s"] = round(time.time() - t_start, 1)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return out


def run_e2e(args, op, per_shape, hz, stream, world, dev, flops_step):
    """The same step end to end: A from page-locked host memory in, C to page-locked host
    memory out, every shape every step. W4A16 goes through the host-buffer entry point, which
    streams chunks of tokens through a device workspace so that both copy directions overlap
    the matmul; the other ops copy A in, call, and copy C out on the stream."""
    import torch
    import gemv_w4a16_w8a8_b200 as qg
    steps = max(1, min(args.steps, 5))
    h2d = sum(sp["A_host"].numel() * sp["A_host"].element_size() for sp in per_shape)
    d2h = sum(sp["C_host"].numel() * sp["C_host"].element_size() for sp in per_shape)
    if op == "w4a16":
        ws_bytes = max(qg.qgemm_w4a16_host_workspace_bytes(sp["M"], sp["N"], sp["K"],
                                                           args.e2e_chunk)
                       for sp in per_shape)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def one(i):
        for sp in per_shape:
            W = sp["W"][i % len(sp["W"])]
            if op == "w4a16":
                qg.qgemm_w4a16_host(sp["A_host"], W, sp["S"], sp["Z"], sp["C_host"], ws,
                                    group_size=GS)
            else:
                sp["A"].copy_(sp["A_host"], non_blocking=True)
                matmul(op, sp, W)
                sp["C_host"].copy_(sp["C"], non_blocking=True)

    one(0)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(steps):
        one(i + 1)
    e1.record(stream)
    torch.cuda.synchronize()
    value, ms = job_throughput(e0.elapsed_time(e1), flops_step, steps, world, dev)
    # the host-side results of the last step, sampled against the oracle
    par = merge_parity([parity_check(op, sp["h"], sp["C_host"], sp["M"], sp["K"], sp["N"], hz,
                                     sp["seed"] + 1) for sp in per_shape])
    path = (f"qgemm_w4a16_host (pinned host A and C, chunks of up to "
            f"{args.e2e_chunk or 1024} tokens, copies in both directions overlapped with the "
            f"matmul)" if op == "w4a16" else
            "pinned host A copied in, the call, C copied out, on one stream")
    return {"value": round(value, 3), "unit": UNITS[op],
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 3), "path": path, "parity": par}


# ---- oracle arm ------------------------------------------------------------------------------------

_ORACLE_INPUTS: dict = {}


def oracle_sample_rates(workload: str, budget_s: float, seed: int = 0):
    """Time the oracle on a slice of every shape: all of A's rows (at most 256) against the first
    n_s weight rows, n_s grown until the slice takes about budget_s / shapes seconds. Returns
    per-shape (flops_done, seconds, description) of the last (largest) timing, and the thread
    count."""
    import oracle
    from gemv_w4a16_w8a8_b200 import synth
    wl = WORKLOADS[workload]
    hz = wl["has_zero"]
    threads = oracle.max_threads()
    per = budget_s / len(wl["shapes"])
    out = []
    op = wl["op"]
    for si, (M, K, N) in enumerate(wl["shapes"]):
        m_s = min(M, 256)
        n_all = min(N, 8192)
        key = (op, m_s, n_all, K, hz, seed + si)
        if key not in _ORACLE_INPUTS:
            if op == "w4a16":
                d = synth.w4a16_inputs(m_s, n_all, K, GS, bool(hz), seed=seed + si)
                d["Wq"] = oracle.pack_int4(d["codes"])
            elif op == "w8a8":
                d = synth.w8a8_inputs(m_s, n_all, K, seed=seed + si)
            elif op == "w2a8":
                d = synth.w2a8_inputs(m_s, n_all, K, seed=seed + si)
                d["Wq"] = oracle.pack_int2(d["Wv"])
            else:
                d = synth.dense_inputs(m_s, n_all, K, seed=seed + si)
            _ORACLE_INPUTS[key] = d
        d = _ORACLE_INPUTS[key]

        def run_slice(n):
            if op == "w4a16":
                oracle.w4a16(d["A"], d["Wq"][:n], d["scales"][:n],
                             None if d["zeros"] is None else d["zeros"][:n], K, GS, nthreads=threads)
            elif op == "w8a8":
                oracle.w8a8(d["A"], d["W"][:n], nthreads=threads)
            elif op == "w2a8":
                oracle.w2a8(d["A"], d["Wq"][:n], nthreads=threads)
            else:
                oracle.dense_f16(d["A"], d["W"][:n], nthreads=threads)

        n_s, dt = 8, 0.0
        for _ in range(8):
            n_s = min(n_s, n_all)
            t = time.perf_counter()
            run_slice(n_s)
            dt = time.perf_counter() - t
            if dt >= 0.5 * per or n_s >= n_all:
                break
            n_s = int(n_s * min(16.0, max(2.0, 0.9 * per / max(dt, 1e-6))))
        out.append((2.0 * m_s * n_s * K, dt, f"{m_s}x{n_s} of ({M},{K},{N})"))
    return out, threads


def cpu_baseline(workload: str, budget_s: float = 15.0):
    rates, threads = oracle_sample_rates(workload, budget_s)
    wl = WORKLOADS[workload]
    # time the oracle would take for the whole step, shape by shape at its sampled rate
    est_s = sum(shape_flops(M, K, N) / (f / t) for (M, K, N), (f, t, _) in zip(wl["shapes"], rates))
    total = sum(shape_flops(M, K, N) for M, K, N in wl["shapes"])
    return {"value": total / est_s / 1e12, "unit": UNITS[wl["op"]], "cores": threads, "kind": "oracle",
            "sample": "; ".join(desc for _, _, desc in rates) +
                      f" (fp64 oracle, {sum(t for _, t, _ in rates):.1f} s wall on {threads} threads; "
                      f"each shape's rate applied to its full FLOPs)",
            "extrapolated": True}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    wl = WORKLOADS[args.workload]
    total_flops = sum(shape_flops(M, K, N) for M, K, N in wl["shapes"])
    per_step_budget = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(max(0, args.warmup)):
        oracle_sample_rates(args.workload, per_step_budget / 4)
    est = []
    sampled = []
    threads = 1
    samples = ""
    for _ in range(args.steps):
        rates, threads = oracle_sample_rates(args.workload, per_step_budget)
        est.append(sum(shape_flops(M, K, N) / (f / t)
                       for (M, K, N), (f, t, _) in zip(wl["shapes"], rates)))
        sampled.append(sum(t for _, t, _ in rates))
        samples = "; ".join(d for _, _, d in rates)
    ms_per_step = 1e3 * statistics.mean(est)
    value = total_flops / (ms_per_step * 1e-3) / 1e12
    return {
        "impl": "reference",
        "metric": METRICS[wl["op"]],
        "value": value, "unit": UNITS[wl["op"]], "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "extrapolated": True,
        "sample_s_per_step": round(statistics.mean(sampled), 3),
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "op": wl["op"],
                   "shapes_mkn": [list(s) for s in wl["shapes"]], "group_size": GS,
                   "has_zero": wl["has_zero"], "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNITS[wl["op"]], "cores": threads, "kind": "oracle",
                         "sample": samples + " per step; each shape's sampled rate applied to "
                                             "its full FLOPs (ms_per_step is that extrapolation; "
                                             "sample_s_per_step is the measured wall time)",
                         "extrapolated": True},
        "e2e": {"value": value, "unit": UNITS[wl["op"]], "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-tune", action="store_true")
    ap.add_argument("--tune-reps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-extras", action="store_true",
                    help="time only the headline workload")
    ap.add_argument("--extras-budget", type=float, default=240.0,
                    help="seconds after which the remaining extra configurations are skipped")
    ap.add_argument("--e2e-chunk", type=int, default=0,
                    help="tokens per chunk of the host-buffer form (0: the library's default)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture")
    args = ap.parse_args(argv)
    world, rank, local = dist_setup()
    if args.impl == "reference":
        out = run_reference(args, world, rank)
    else:
        out = run_ours(args, world, rank, local)
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)
    if out is not None and out.get("impl") != "reference":
        failed = (out.get("device_error") or out["parity"]["bad"] or
                  out.get("configs_parity", {}).get("bad", 0))
        if failed:
            return 3
    return 0


if __name__ == "__main__":
    sys.exit(main())
