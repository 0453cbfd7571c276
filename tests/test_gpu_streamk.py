"""The stream-K schedule of the tensor-core tiles (rows = 1: every persistent CTA takes an equal
share of the flattened (tile, K) work, partial tiles added into the zeroed output) against the
oracle: every operand format, both orientations, the 256- and 512-token tiles, shapes whose
shares cross one or several tile boundaries, problems smaller than the grid, and the full-size
benchmark shapes on one element of every tile."""
import contextlib

import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import IntCase, W4Case, assert_fp16_close, guarded, guards_intact, sample_pairs, to_dev

pytestmark = pytest.mark.gpu

OPS = {"w4a16": qg.OP_W4A16, "w8a8": qg.OP_W8A8, "w2a8": qg.OP_W2A8, "dense": qg.OP_DENSE_F16,
       "w4a16i": qg.OP_W4A16_INTERLEAVED}


def sk_cfg(bn, stages, swap=1):
    return {"path": qg.PATH_TC, "rows": 1, "bm": 128, "bn": bn, "bk": 0, "stages": stages,
            "split_k": 1, "swap_ab": swap}


@contextlib.contextmanager
def pinned(op, M, N, K, gs, hz, cfg):
    key = (OPS[op], M, N, K, gs, hz)
    qg.qgemm_set_config(*key, cfg)
    try:
        plan = qg.qgemm_plan(*key)
        assert plan["path"] == qg.PATH_TC and plan["rows"] == 1
        yield
    finally:
        qg.qgemm_set_config(*key, None)


# (M, N, K): a few tiles (shares shorter than a tile, crossing one boundary), more tiles than
# CTAs (shares crossing several), ragged tokens and weight rows, K of whole and partial 4-slab
# runs (1088: single-slab packed copies)
SHAPES = [(40, 256, 1024), (300, 1000, 2048), (512, 2048, 4096), (700, 520, 1088),
          (1100, 4096, 1024)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("bn,stages", [(256, 3), (128, 4), (512, 4), (64, 8)])
def test_streamk_w4a16_weight_major(M, N, K, bn, stages):
    case = W4Case(M, N, K, 64, 1, seed=M + N + bn)
    with pinned("w4a16", M, N, K, 64, 1, sk_cfg(bn, stages)):
        C = case.run()
        qg.qgemm_sync_check()
    assert_fp16_close(C, case.ref_full(), f"stream-K w4a16 {M},{N},{K} bn={bn}")


@pytest.mark.parametrize("M,N,K", [(40, 256, 1024), (128, 1000, 2048), (200, 4096, 4096),
                                   (100, 520, 1280)])
@pytest.mark.parametrize("stages", [2, 3, 4])
def test_streamk_w4a16_token_major(M, N, K, stages):
    case = W4Case(M, N, K, 128, 1, seed=M + stages)
    with pinned("w4a16", M, N, K, 128, 1, sk_cfg(256, stages, swap=0)):
        C = case.run()
        qg.qgemm_sync_check()
    assert_fp16_close(C, case.ref_full(), f"stream-K token-major {M},{N},{K}")


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("M,N,K", [(40, 256, 1024), (300, 1000, 2048), (512, 2048, 4096)])
@pytest.mark.parametrize("bn,stages", [(256, 3), (64, 4)])
def test_streamk_int(op, M, N, K, bn, stages):
    case = IntCase(op, M, N, K, seed=M + N + bn)
    with pinned(op, M, N, K, -1, 0, sk_cfg(bn, stages)):
        got = case.run().cpu().numpy()
        qg.qgemm_sync_check()
    assert np.array_equal(got, case.ref_full())   # integer partial sums add exactly


@pytest.mark.parametrize("M,N,K", [(300, 1000, 2048), (512, 2048, 4096)])
def test_streamk_dense(M, N, K):
    h = synth.dense_inputs(M, N, K, seed=M)
    with pinned("dense", M, N, K, -1, 0, sk_cfg(256, 4)):
        C = qg.qgemm_dense_f16(to_dev(h["A"]), to_dev(h["W"]))
        qg.qgemm_sync_check()
    assert_fp16_close(C, oracle.dense_f16(h["A"], h["W"]), f"stream-K dense {M},{N},{K}")


def test_streamk_interleaved_and_guard_bands():
    M, N, K = 700, 1032, 2048
    d = synth.w4a16_inputs(M, N, K, 128, True, seed=29)
    Wi = qg.quant_pack_int4_interleaved(to_dev(d["codes"]))
    ref = oracle.w4a16(d["A"], oracle.pack_int4(d["codes"]), d["scales"], d["zeros"], K, 128)
    buf, C, pad = guarded((M, N), torch.float16)
    with pinned("w4a16i", M, N, K, 128, 1, sk_cfg(512, 4)):
        qg.qgemm_w4a16_interleaved(to_dev(d["A"]), Wi, to_dev(d["scales"]), to_dev(d["zeros"]),
                                   C=C, group_size=128)
        qg.qgemm_sync_check()
    torch.cuda.synchronize()
    assert guards_intact(buf, pad, M * N)
    assert_fp16_close(C, ref, "stream-K interleaved")


def test_streamk_overwrites_stale_output():
    """The output is zeroed before the partial tiles are added: a C full of garbage is replaced."""
    M, N, K = 512, 2048, 4096
    case = W4Case(M, N, K, 128, 1, seed=3)
    C = torch.full((M, N), 1000.0, dtype=torch.float16, device=case.A.device)
    with pinned("w4a16", M, N, K, 128, 1, sk_cfg(512, 4)):
        case.run(C=C)
        qg.qgemm_sync_check()
    assert_fp16_close(C, case.ref_full(), "stream-K stale output")


def test_explicit_split_leaves_stream_k():
    """An explicit split_k asks for K parts of that count: a stream-K plan gives way to it."""
    M, N, K = 512, 2048, 4096
    case = W4Case(M, N, K, 128, 1, seed=4)
    with pinned("w4a16", M, N, K, 128, 1, sk_cfg(256, 3)):
        C = qg.qgemm_w4a16(case.A, case.Wq, case.S, case.Z, group_size=128, split_k=2)
        qg.qgemm_sync_check()
    assert_fp16_close(C, case.ref_full(), "explicit split over stream-K")


@pytest.mark.parametrize("M,bn", [(512, 512), (128, 256), (16384, 512)])
def test_streamk_full_size_sampled(M, bn):
    N = K = 16384
    case = W4Case(M, N, K, 128, 1, seed=M + 9)
    swap = 0 if M <= 128 else 1
    with pinned("w4a16", M, N, K, 128, 1, sk_cfg(bn, 3 if swap == 0 else 4, swap)):
        C = case.run().float().cpu().numpy()
        qg.qgemm_sync_check()
    ms, ns = sample_pairs(M, N, 300, seed=M + 2)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), f"stream-K M={M}")
