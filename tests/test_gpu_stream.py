"""The persistent stream-K W4A16 kernel (path STREAM) against the oracle, within the fp16 rule:
every stage shape (256 / 512 / 1024 K, 1 / 2 / 4 K warps a row block), one and two token tiles,
group sizes from 128 to K, ragged N, a partial last K stage, CTAs whose rows lie beyond N, both
nibble orders, and the full-size M = 1 and M = 16 problems on sampled outputs."""
import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import DEV, W4Case, assert_fp16_close, sample_pairs, to_dev

pytestmark = pytest.mark.gpu


def _smem(bk, stages, wr, wk, M):
    """The kernel's shared-memory plan: weights, activations and prepared operands a stage."""
    up = lambda x: (x + 1023) // 1024 * 1024
    nt = 1 if M <= 8 else 2
    stage = 16 * wr * bk // 2 + up(M * bk * 2) + up(bk // 128 * (256 * M + 64 * nt))
    return 1024 + stages * (stage + 24) + wr * wk * 16 * 8 * nt * 4 + 8 + 16


def _cfg(bk=512, stages=0, wr=4, wk=2, M=16):
    wr = min(wr, 14 // wk)   # at most 14 consumer warps
    if stages == 0:   # the deepest ring that fits at this M
        stages = 16
        while stages > 2 and _smem(bk, stages, wr, wk, M) > 227 * 1024:
            stages -= 1
    return {"path": qg.PATH_STREAM, "rows": 16, "bm": wr, "bn": wk, "bk": bk,
            "stages": stages, "split_k": 1, "swap_ab": 0}


def _pinned(case, cfg, op=qg.OP_W4A16):
    key = (op, case.M, case.N, case.K, case.gs, int(case.has_zero))
    qg.qgemm_set_config(*key, cfg)
    try:
        got = qg.qgemm_plan(*key)
        assert got == cfg, got
        return case.run()
    finally:
        qg.qgemm_set_config(*key, None)


UNIT_SHAPES = [(256, 1), (256, 2), (512, 1), (512, 2), (512, 4), (1024, 2), (1024, 4)]


@pytest.mark.parametrize("bk,wk", UNIT_SHAPES)
@pytest.mark.parametrize("M", [1, 5, 8, 9, 16])
def test_stream_unit_shapes(bk, wk, M):
    # N ragged against the row tile; K = 3072 is a whole number of every stage size
    case = W4Case(M, 200, 3072, 128, 1, seed=bk + wk + M)
    wr = 4 if _smem(bk, 2, 4, wk, M) <= 227 * 1024 else 1
    C = _pinned(case, _cfg(bk, 0, wr, wk, M=M))
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), f"bk={bk} wk={wk} M={M}")


@pytest.mark.parametrize("K", [256, 768, 1280, 11008])
@pytest.mark.parametrize("bk,wk", [(512, 4), (1024, 2), (1024, 4)])
def test_stream_partial_last_stage(K, bk, wk):
    # K not a multiple of the stage: the last unit of every row holds fewer sub-blocks, and
    # some K warps have none of them
    case = W4Case(3, 96, K, 128, 1, seed=K + bk + wk)
    C = _pinned(case, _cfg(bk, 0, wk=wk, M=3))
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), f"K={K} bk={bk}")


@pytest.mark.parametrize("gs,hz", [(256, 1), (512, 0), (-1, 1), (128, 0)])
def test_stream_group_sizes(gs, hz):
    # group sizes above 128 take the per-sub-block scale loads; 128 the per-stage vector loads
    case = W4Case(4, 130, 2048, gs, hz, seed=abs(gs) + hz)
    C = _pinned(case, _cfg(1024, 0, M=4))
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), f"gs={gs} hz={hz}")


def test_stream_unaligned_scales():
    case = W4Case(2, 64, 2048, 128, 1, seed=3)
    G = 2048 // 128
    # scales / zeros one element into a larger buffer: 2-byte aligned only
    sbuf = torch.empty(64 * G + 1, dtype=torch.float16, device=DEV)
    zbuf = torch.empty(64 * G + 1, dtype=torch.float16, device=DEV)
    sbuf[1:] = case.S.reshape(-1)
    zbuf[1:] = case.Z.reshape(-1)
    case.S = sbuf[1:].view(64, G)
    case.Z = zbuf[1:].view(64, G)
    C = _pinned(case, _cfg(512, 0, M=2))
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), "scales 2-byte aligned")


@pytest.mark.parametrize("bk,wr,wk,stages", [(512, 4, 2, 10), (512, 3, 4, 8), (1024, 1, 2, 2),
                                             (1024, 2, 4, 6), (256, 8, 1, 11), (256, 6, 2, 3)])
def test_stream_grid_shapes(bk, wr, wk, stages):
    case = W4Case(1, 1000, 4096, 128, 1, seed=wr * 10 + wk)
    C = _pinned(case, _cfg(bk, stages, wr, wk, M=1))
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), f"bk={bk} wr={wr} wk={wk} stages={stages}")


@pytest.mark.parametrize("bk,stages", [(512, 2), (1024, 3), (256, 5)])
def test_stream_ring_wraps_many_times(bk, stages):
    # one CTA's run spans dozens of units, so every stage of the ring is reused many times
    case = W4Case(2, 2048, 8192, 128, 1, seed=bk + stages)
    key = (qg.OP_W4A16, 2, 2048, 8192, 128, 1)
    qg.qgemm_set_config(*key, _cfg(bk, stages, 4, 2, M=2))
    try:
        C = case.run()
        torch.cuda.synchronize()
        qg.qgemm_sync_check()
    finally:
        qg.qgemm_set_config(*key, None)
    assert_fp16_close(C, case.ref_full(), f"bk={bk} stages={stages}")


def test_stream_fewer_units_than_warps():
    # one unit in all: a single CTA, most of whose rows lie beyond N
    case = W4Case(1, 16, 256, 128, 1, seed=11)
    C = _pinned(case, _cfg(1024, 0, M=1))
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), "one unit")
    case = W4Case(2, 5, 256, 128, 0, seed=12)
    C = _pinned(case, _cfg(512, 2, 8, 1, M=2))
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), "N=5")


def test_stream_is_the_default_from_nine_tokens():
    plan = qg.qgemm_plan(qg.OP_W4A16, 12, 4096, 4096, 128, 1)
    assert plan["path"] == qg.PATH_STREAM
    # an explicit split_k keeps to a path that splits K into that many parts
    plan = qg.qgemm_plan(qg.OP_W4A16, 12, 4096, 4096, 128, 1, split_k=4)
    assert plan["path"] == qg.PATH_GEMV and plan["split_k"] == 4
    case = W4Case(12, 4096, 4096, 128, 1, seed=0)
    C = case.run()
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), "default plan, 12 tokens")


def test_stream_overwrites_stale_output():
    case = W4Case(2, 300, 2048, 128, 1, seed=21)
    C = torch.full((2, 300), 777.0, dtype=torch.float16, device=DEV)
    C = _pinned_into(case, _cfg(512, 0, M=2), C)
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), "stale C")


def _pinned_into(case, cfg, C):
    key = (qg.OP_W4A16, case.M, case.N, case.K, case.gs, int(case.has_zero))
    qg.qgemm_set_config(*key, cfg)
    try:
        return case.run(C=C)
    finally:
        qg.qgemm_set_config(*key, None)


def test_stream_interleaved_layout():
    M, N, K, gs = 3, 136, 2048, 128
    d = synth.w4a16_inputs(M, N, K, gs, True, 5)
    A, S, Z = to_dev(d["A"]), to_dev(d["scales"]), to_dev(d["zeros"])
    Wi = qg.quant_pack_int4_interleaved(to_dev(d["codes"]))
    ref = oracle.w4a16(d["A"], oracle.pack_int4(d["codes"]), d["scales"], d["zeros"], K, gs)
    for bk, wk in UNIT_SHAPES:
        key = (qg.OP_W4A16_INTERLEAVED, M, N, K, gs, 1)
        qg.qgemm_set_config(*key, _cfg(bk, 0, wk=wk, M=M))
        try:
            C = qg.qgemm_w4a16_interleaved(A, Wi, S, Z, group_size=gs)
        finally:
            qg.qgemm_set_config(*key, None)
        torch.cuda.synchronize()
        assert_fp16_close(C, ref, f"interleaved bk={bk} wk={wk}")


@pytest.mark.parametrize("M", [1, 16])
def test_stream_full_size_sampled(M):
    """N = K = 16384 in the benchmark's launch configuration, checked on sampled outputs."""
    N = K = 16384
    case = W4Case(M, N, K, 128, 1, seed=0)
    C = case.run()
    torch.cuda.synchronize()
    plan = qg.qgemm_plan(qg.OP_W4A16, M, N, K, 128, 1)
    assert plan["path"] in (qg.PATH_STREAM, qg.PATH_GEMV, qg.PATH_TC)
    ms, ns = sample_pairs(M, N, 300, seed=M)
    ref = case.ref_at(ms, ns)
    got = C.float().cpu().numpy()[ms, ns]
    ok, msg = oracle.fp16_close(got, ref)
    assert ok, msg
