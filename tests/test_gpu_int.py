"""W8A8 and W2A8 on the GPU: bit-exact against the oracle for every split, at small shapes with
ragged tails in full and at the N = K = 16384 benchmark shapes on sampled outputs."""
import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import IntCase, guarded, guards_intact, sample_pairs, to_dev

pytestmark = pytest.mark.gpu


def test_pack_int2_bit_exact():
    for N, K in [(1, 64), (5, 192), (1000, 4096)]:
        vals = synth.uniform_int((N, K), -2, 1, N + K, synth.TID_W, np.int8)
        got = qg.quant_pack_int2(to_dev(vals)).cpu().numpy().view(np.uint32)
        assert np.array_equal(got, oracle.pack_int2(vals)), (N, K)


SMALL = [(1, 256, 512), (1, 4099, 1024), (2, 33, 256), (3, 100, 2048), (4, 17, 64),
         (5, 64, 1024), (9, 130, 512), (32, 96, 256), (1, 1, 128)]


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("M,N,K", SMALL)
def test_int_small_shapes_all_splits_identical(op, M, N, K):
    case = IntCase(op, M, N, K, seed=M * 7 + N)
    ref = case.ref_full()
    assert np.abs(ref).max() < 2 ** 31
    for split in (1, 2, 3, 4, 8):
        got = case.run(split_k=split).cpu().numpy()
        assert np.array_equal(got, ref), (op, M, N, K, split)


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("rows", [1, 2, 4, 8])
def test_int_each_row_tile(op, rows):
    M, N, K = 3, 70, 1024
    case = IntCase(op, M, N, K, seed=rows)
    opc = qg.OP_W8A8 if op == "w8a8" else qg.OP_W2A8
    cfg = {"path": qg.PATH_GEMV, "rows": rows, "bm": 0, "bn": 0, "bk": 0, "stages": 0,
           "split_k": 2, "swap_ab": 0}
    qg.qgemm_set_config(opc, M, N, K, -1, 0, cfg)
    try:
        assert np.array_equal(case.run().cpu().numpy(), case.ref_full())
    finally:
        qg.qgemm_set_config(opc, M, N, K, -1, 0, None)


def test_w8a8_extreme_values():
    K = 16384
    A = np.full((2, K), -128, dtype=np.int8)
    W = np.full((3, K), -128, dtype=np.int8)
    W[1] = 127
    W[2, ::2] = 127
    C = qg.qgemm_w8a8(to_dev(A), to_dev(W), split_k=4).cpu().numpy()
    assert np.array_equal(C, oracle.w8a8(A, W))
    assert C[0, 0] == K * 16384


def test_w2a8_extreme_values():
    K = 4096
    A = np.full((1, K), -128, dtype=np.int8)
    for v in (-2, -1, 0, 1):
        Wv = np.full((2, K), v, dtype=np.int8)
        C = qg.qgemm_w2a8(to_dev(A), qg.quant_pack_int2(to_dev(Wv))).cpu().numpy()
        assert np.all(C == -128 * v * K), v


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("M", [1, 32, 128, 512])
def test_int_benchmark_shapes_sampled(op, M):
    N = K = 16384
    case = IntCase(op, M, N, K, seed=M)
    got = case.run().cpu().numpy()
    ms, ns = sample_pairs(M, N, 400, seed=M + 1)
    assert np.array_equal(got[ms, ns], case.ref_at(ms, ns))
    got4 = case.run(split_k=4).cpu().numpy()
    assert np.array_equal(got4, got)


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
def test_int_guard_bands(op):
    case = IntCase(op, 3, 130, 1024, seed=2)
    buf, C, pad = guarded((3, 130), torch.int32)
    case.run(split_k=4, C=C)
    torch.cuda.synchronize()
    assert guards_intact(buf, pad, 3 * 130)
    assert np.array_equal(C.cpu().numpy(), case.ref_full())


@pytest.mark.parametrize("rows", [16, 32, 64])
@pytest.mark.parametrize("stages", [2, 3, 4, 6])
@pytest.mark.parametrize("M", [1, 7, 16])
def test_w2a8_tma_kernel_configs(rows, stages, M):
    N, K = 200, 4096
    case = IntCase("w2a8", M, N, K, seed=rows + stages + M)
    for split in (1, 3):
        cfg = {"path": qg.PATH_GEMV, "rows": rows, "bm": 0, "bn": 0, "bk": 0, "stages": stages,
               "split_k": split, "swap_ab": 0}
        qg.qgemm_set_config(qg.OP_W2A8, M, N, K, -1, 0, cfg)
        try:
            assert np.array_equal(case.run().cpu().numpy(), case.ref_full()), (rows, stages, split)
        finally:
            qg.qgemm_set_config(qg.OP_W2A8, M, N, K, -1, 0, None)
