"""Run one matmul problem repeatedly on the current GPU (for timing and for profilers).

    python -m gemv_w4a16_w8a8_b200.run_case --op w4a16 --M 1 --N 16384 --K 16384 --iters 20

Inputs are the seeded synthetic ones. Weights rotate over enough copies that each call reads
its weights from HBM. Prints the mean device time per call (CUDA events) and the effective
GB/s and TFLOP/s. --split-k / --rows / --path / --bn / --bk / --bm / --stages pin a
configuration first.
"""
from __future__ import annotations

import argparse
import math
import sys

import numpy as np


def main(argv=None) -> int:
    import torch
    import gemv_w4a16_w8a8_b200 as qg
    from gemv_w4a16_w8a8_b200 import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--op", default="w4a16", choices=["w4a16", "w8a8", "w2a8", "dense"])
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--gs", type=int, default=128)
    ap.add_argument("--has-zero", type=int, default=1)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--split-k", type=int, default=0)
    ap.add_argument("--path", type=int, default=0)
    ap.add_argument("--rows", type=int, default=0)
    ap.add_argument("--bn", type=int, default=0)
    ap.add_argument("--stages", type=int, default=-1)
    ap.add_argument("--bk", type=int, default=0)
    ap.add_argument("--bm", type=int, default=0, help="TC: tile M; STREAM: warps per CTA")
    ap.add_argument("--swap-ab", type=int, default=-1,
                    help="TC: 1 = weights in the MMA's M side, 0 = token-major tile")
    ap.add_argument("--copies", type=int, default=0, help="weight copies (0: >= 3x L2)")
    ap.add_argument("--interleaved", action="store_true",
                    help="w4a16 / w2a8: weights in the interleaved (pre-shuffled) layout")
    a = ap.parse_args(argv)

    dev = torch.device("cuda", 0)
    M, N, K = a.M, a.N, a.K
    ks = [a.split_k]
    up = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    opc = {"w4a16": qg.OP_W4A16, "w8a8": qg.OP_W8A8, "w2a8": qg.OP_W2A8,
           "dense": qg.OP_DENSE_F16}[a.op]
    ilv = a.interleaved and a.op in ("w4a16", "w2a8")
    if ilv:
        opc = qg.OP_W4A16_INTERLEAVED if a.op == "w4a16" else qg.OP_W2A8_INTERLEAVED
    gs = a.gs if a.op == "w4a16" else -1
    hz = a.has_zero if a.op == "w4a16" else 0
    if a.op == "w4a16":
        d = synth.w4a16_inputs(M, N, K, gs, bool(hz), seed=0)
        pack = qg.quant_pack_int4_interleaved if ilv else qg.quant_pack_int4
        mm = qg.qgemm_w4a16_interleaved if ilv else qg.qgemm_w4a16
        A, W = up(d["A"]), pack(up(d["codes"]))
        S = up(d["scales"])
        Z = up(d["zeros"]) if hz else None
        wbytes = N * K // 2
        run = lambda w, C: mm(A, w, S, Z, C=C, group_size=gs, split_k=ks[0])
        C = torch.empty((M, N), dtype=torch.float16, device=dev)
        nbytes = wbytes + N * (K // (K if gs <= 0 else gs)) * 2 * (1 + hz) + 2 * M * K + 2 * M * N
    elif a.op == "w8a8":
        d = synth.w8a8_inputs(M, N, K, seed=0)
        A, W = up(d["A"]), up(d["W"])
        wbytes = N * K
        run = lambda w, C: qg.qgemm_w8a8(A, w, C=C, split_k=ks[0])
        C = torch.empty((M, N), dtype=torch.int32, device=dev)
        nbytes = wbytes + M * K + 4 * M * N
    elif a.op == "w2a8":
        d = synth.w2a8_inputs(M, N, K, seed=0)
        pack = qg.quant_pack_int2_interleaved if ilv else qg.quant_pack_int2
        mm = qg.qgemm_w2a8_interleaved if ilv else qg.qgemm_w2a8
        A, W = up(d["A"]), pack(up(d["Wv"]))
        wbytes = N * K // 4
        run = lambda w, C: mm(A, w, C=C, split_k=ks[0])
        C = torch.empty((M, N), dtype=torch.int32, device=dev)
        nbytes = wbytes + M * K + 4 * M * N
    else:
        d = synth.dense_inputs(M, N, K, seed=0)
        A, W = up(d["A"]), up(d["W"])
        wbytes = 2 * N * K
        run = lambda w, C: qg.qgemm_dense_f16(A, w, C=C, split_k=ks[0])
        C = torch.empty((M, N), dtype=torch.float16, device=dev)
        nbytes = wbytes + 2 * M * K + 2 * M * N

    # the call's own split_k: 0 (the plan) once a configuration is pinned below, so that the
    # pinned one runs as given (an explicit split would override its schedule)
    ks[0] = a.split_k
    if a.path or a.rows or a.bn or a.bk or a.bm or a.stages >= 0 or a.swap_ab >= 0:
        ks[0] = 0
        cfg = qg.qgemm_plan(opc, M, N, K, gs, hz)
        if a.path and a.path != cfg["path"]:
            cfg = {k: 0 for k in cfg}
            cfg["split_k"] = 1
        for key, val in (("path", a.path), ("rows", a.rows), ("bn", a.bn), ("bk", a.bk),
                         ("bm", a.bm), ("split_k", a.split_k)):
            if val:
                cfg[key] = val
        if a.stages >= 0:
            cfg["stages"] = a.stages
        if a.swap_ab >= 0:
            cfg["swap_ab"] = a.swap_ab
        qg.qgemm_set_config(opc, M, N, K, gs, hz, cfg)
    print("config", qg.qgemm_plan(opc, M, N, K, gs, hz, ks[0]))

    copies = a.copies or max(1, min(64, math.ceil(3 * 126 * 2 ** 20 / wbytes)))
    Ws = [W] + [W.clone() for _ in range(copies - 1)]
    for i in range(3):
        run(Ws[i % copies], C)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(a.iters):
            run(Ws[i % copies], C)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    qg.qgemm_sync_check()
    us = e0.elapsed_time(e1) * 1e3 / a.iters
    flops = 2.0 * M * N * K
    cfg_used = qg.qgemm_plan(opc, M, N, K, gs, hz, ks[0])
    print(f"{a.op} M={M} N={N} K={K}: {us:.2f} us/call  {nbytes / us / 1e3:.1f} GB/s  "
          f"{flops / us / 1e6:.2f} TFLOP/s  ({copies} weight copies)  cfg={cfg_used}")
    qg.qgemm_set_config(opc, M, N, K, gs, hz, None)
    return 0


if __name__ == "__main__":
    sys.exit(main())
