"""The tcgen05 tensor-core path against the oracle: dense fp16, W4A16, W8A8 and W2A8 over token
tiles, pipeline depths and K splits, with ragged M / N / K tails, exact special cases, and the
full-size N = K = 16384 shapes on sampled outputs."""
import contextlib

import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import DEV, IntCase, W4Case, assert_fp16_close, guarded, guards_intact, sample_pairs, to_dev

pytestmark = pytest.mark.gpu

OPS = {"w4a16": qg.OP_W4A16, "w8a8": qg.OP_W8A8, "w2a8": qg.OP_W2A8, "dense": qg.OP_DENSE_F16}


@contextlib.contextmanager
def tc_config(op, M, N, K, gs, hz, bn, stages, split_k):
    cfg = {"path": qg.PATH_TC, "rows": 0, "bm": 128, "bn": bn, "bk": 0, "stages": stages,
           "split_k": split_k, "swap_ab": 1}
    try:
        qg.qgemm_set_config(OPS[op], M, N, K, gs, hz, cfg)
    except qg.QGemmError:
        # the deepest rings fit shared memory only with grouped packed copies (K a multiple of
        # four slabs); elsewhere the library refuses them up front
        if stages >= 5:
            pytest.skip(f"bn={bn} stages={stages} does not fit K={K}")
        raise
    try:
        assert qg.qgemm_plan(OPS[op], M, N, K, gs, hz)["path"] == qg.PATH_TC
        yield
    finally:
        qg.qgemm_set_config(OPS[op], M, N, K, gs, hz, None)


@contextlib.contextmanager
def toka_config(M, N, K, gs, hz, stages, split_k):
    """Pin the token-major tensor-core tile (128 tokens x 256 weight rows, W4A16)."""
    cfg = {"path": qg.PATH_TC, "rows": 0, "bm": 128, "bn": 256, "bk": 0, "stages": stages,
           "split_k": split_k, "swap_ab": 0}
    qg.qgemm_set_config(qg.OP_W4A16, M, N, K, gs, hz, cfg)
    try:
        plan = qg.qgemm_plan(qg.OP_W4A16, M, N, K, gs, hz)
        assert plan["path"] == qg.PATH_TC and plan["swap_ab"] == 0
        yield
    finally:
        qg.qgemm_set_config(qg.OP_W4A16, M, N, K, gs, hz, None)


class DenseCase:
    def __init__(self, M, N, K, seed=0):
        self.M, self.N, self.K = M, N, K
        self.h = synth.dense_inputs(M, N, K, seed)
        self.A = to_dev(self.h["A"])
        self.W = to_dev(self.h["W"])

    def run(self, split_k=0, C=None):
        return qg.qgemm_dense_f16(self.A, self.W, C=C, split_k=split_k)

    def ref_full(self):
        return oracle.dense_f16(self.h["A"], self.h["W"])

    def ref_at(self, ms, ns):
        return oracle.dense_f16_at(self.h["A"], self.h["W"], ms, ns)


# ---- dense fp16 ---------------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (16, 128, 128), (33, 200, 512), (128, 256, 1024),
                                   (200, 130, 320), (257, 384, 2048), (64, 1000, 72)])
@pytest.mark.parametrize("bn,stages", [(16, 2), (64, 3), (128, 4), (256, 2)])
def test_dense_tiles(M, N, K, bn, stages):
    case = DenseCase(M, N, K, seed=M + N + K)
    with tc_config("dense", M, N, K, -1, 0, bn, stages, 1):
        assert_fp16_close(case.run(), case.ref_full(), f"dense {M},{N},{K} bn={bn} st={stages}")


@pytest.mark.parametrize("split_k", [2, 3, 8])
def test_dense_split_k(split_k):
    M, N, K = 100, 300, 2048
    case = DenseCase(M, N, K, seed=split_k)
    with tc_config("dense", M, N, K, -1, 0, 128, 4, split_k):
        assert_fp16_close(case.run(), case.ref_full(), f"split={split_k}")


def test_dense_integer_case_is_exact():
    M, N, K = 96, 160, 256
    A = synth.uniform_int((M, K), -2, 1, 1, synth.TID_A, np.int8).astype(np.float16)
    W = synth.uniform_int((N, K), -2, 1, 1, synth.TID_W, np.int8).astype(np.float16)
    ref = oracle.dense_f16(A, W)
    assert np.abs(ref).max() < 2048
    with tc_config("dense", M, N, K, -1, 0, 64, 3, 1):
        C = qg.qgemm_dense_f16(to_dev(A), to_dev(W)).cpu().numpy().astype(np.float64)
    assert np.array_equal(C, ref)


def test_dense_one_hot_rows():
    """A = e_k: C[k, n] = W[n, k] exactly, for every k (pins the K order of both tiles)."""
    N, K = 136, 192
    W = synth.dense_inputs(1, N, K, 5)["W"]
    A = np.eye(K, dtype=np.float16)
    with tc_config("dense", K, N, K, -1, 0, 64, 2, 1):
        C = qg.qgemm_dense_f16(to_dev(A), to_dev(W)).cpu().numpy()
    assert np.array_equal(C, W.T)


@pytest.mark.parametrize("M", [512, 16384])
def test_dense_full_size_sampled(M):
    N = K = 16384
    case = DenseCase(M, N, K, seed=M)
    C = case.run().float().cpu().numpy()
    ms, ns = sample_pairs(M, N, 300, seed=M)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), f"dense M={M}")


# ---- W4A16 ------------------------------------------------------------------------------------

W4_SHAPES = [(17, 128, 256, 128, 1), (32, 200, 512, 64, 0), (64, 256, 1024, 128, 1),
             (100, 130, 384, 32, 1), (128, 384, 2048, -1, 1), (129, 512, 512, 128, 0),
             (300, 136, 1024, 128, 1), (8, 256, 512, 128, 1)]


# (128, 8), (256, 4), (256, 5): deep activation rings that leave 2-3 upcast buffers, handed over
# one slab at a time
TC_TILES = [(16, 3), (64, 4), (128, 2), (128, 8), (256, 3), (256, 4), (256, 5)]


@pytest.mark.parametrize("M,N,K,gs,hz", W4_SHAPES)
@pytest.mark.parametrize("bn,stages", TC_TILES)
def test_w4a16_tc_tiles(M, N, K, gs, hz, bn, stages):
    case = W4Case(M, N, K, gs, hz, seed=M * 3 + N)
    with tc_config("w4a16", M, N, K, gs, hz, bn, stages, 1):
        assert_fp16_close(case.run(), case.ref_full(), f"w4 {M},{N},{K} gs={gs} bn={bn}")


@pytest.mark.parametrize("split_k", [2, 3, 4, 16])
def test_w4a16_tc_split_k(split_k):
    M, N, K = 64, 256, 4096
    case = W4Case(M, N, K, 128, 1, seed=split_k)
    with tc_config("w4a16", M, N, K, 128, 1, 64, 4, split_k):
        assert_fp16_close(case.run(), case.ref_full(), f"split={split_k}")


@pytest.mark.parametrize("bn,stages,split_k", [(128, 8, 1), (128, 8, 3), (256, 4, 1),
                                               (256, 4, 2), (256, 5, 1)])
def test_w4a16_tc_long_k_deep_rings(bn, stages, split_k):
    """Several token and weight tiles per CTA with long K: the upcast and activation rings wrap
    hundreds of times inside a unit and carry on across units (and splits)."""
    M, N, K = 300, 384, 8192
    case = W4Case(M, N, K, 128, 1, seed=bn + stages + split_k)
    with tc_config("w4a16", M, N, K, 128, 1, bn, stages, split_k):
        assert_fp16_close(case.run(), case.ref_full(), f"bn={bn} st={stages} split={split_k}")


# ---- W4A16, token-major tiles (tokens in the MMA's M, 256 weight rows in its N) ----------------

TOKA_SHAPES = [(1, 256, 256, 64, 1), (8, 384, 1024, 128, 0), (17, 136, 512, 128, 1),
               (100, 1000, 2048, 128, 1), (128, 256, 1024, -1, 1), (129, 520, 768, 64, 0),
               (200, 257, 1024, 128, 1), (64, 4104, 1152, 128, 1)]


@pytest.mark.parametrize("M,N,K,gs,hz", TOKA_SHAPES)
@pytest.mark.parametrize("stages,split_k", [(2, 1), (3, 1), (4, 1), (4, 3), (2, 16)])
def test_w4a16_toka_tiles(M, N, K, gs, hz, stages, split_k):
    """Ragged tokens (rows past M read as zero), ragged weight tiles (N % 256, N odd, N % 8),
    single-slab packed copies (K = 768, 1152) and K splits."""
    case = W4Case(M, N, K, gs, hz, seed=M * 5 + N + K)
    try:
        cm = toka_config(M, N, K, gs, hz, stages, split_k)
        cm.__enter__()
    except qg.QGemmError:
        pytest.skip(f"stages={stages} does not fit K={K}")
    try:
        assert_fp16_close(case.run(), case.ref_full(), f"toka {M},{N},{K} gs={gs} st={stages}")
    finally:
        cm.__exit__(None, None, None)


def test_w4a16_toka_guard_bands_and_stream():
    M, N, K = 77, 520, 1024
    case = W4Case(M, N, K, 128, 1, seed=21)
    buf, C, pad = guarded((M, N), torch.float16)
    s = torch.cuda.Stream()
    with toka_config(M, N, K, 128, 1, 4, 3), torch.cuda.stream(s):
        case.run(C=C)
    s.synchronize()
    assert guards_intact(buf, pad, M * N)
    assert_fp16_close(C, case.ref_full(), "toka guarded")


def test_w4a16_toka_one_hot_element_order():
    """A = e_k (token k reads weight column k): C[k, n] = fp16((q - z) s) for every k and n."""
    N, K, gs = 300, 128, 64
    G = K // gs
    codes = synth.uniform_int((N, K), 0, 15, 13, synth.TID_W, np.uint8)
    s = synth.uniform_f16((N, G), 0.001, 0.01, 13, synth.TID_SCALE)
    z = synth.uniform_int((N, G), 0, 15, 13, synth.TID_ZERO, np.uint8).astype(np.float16)
    A = np.eye(K, dtype=np.float16)
    with toka_config(K, N, K, gs, 1, 2, 1):
        C = qg.qgemm_w4a16(to_dev(A), qg.quant_pack_int4(to_dev(codes)), to_dev(s), to_dev(z),
                           group_size=gs).cpu().numpy()
    ref = oracle.w4a16(A, oracle.pack_int4(codes), s, z, K, gs)
    assert_fp16_close(torch.from_numpy(C.astype(np.float32)), ref, "toka one-hot")


@pytest.mark.parametrize("M", [1, 16, 32, 128])
def test_w4a16_toka_full_size_sampled(M):
    N = K = 16384
    case = W4Case(M, N, K, 128, 1, seed=M + 70)
    with toka_config(M, N, K, 128, 1, 4, 16):
        C = case.run().float().cpu().numpy()
    ms, ns = sample_pairs(M, N, 300, seed=M + 1)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), f"toka M={M}")


@pytest.fixture(scope="module")
def copy_tagged_weights():
    """N = K = 16384 weights whose codes name their position: every weight of 256-wide K
    block c (one packed copy of four slabs) has code c mod 16, with s = 1 and z = 0. A copy read
    from the wrong ring slot, or before its bytes landed, or after the next copy overwrote it,
    changes the result by a multiple of 64."""
    N = K = 16384
    code_k = ((np.arange(K) // 256) % 16).astype(np.uint8)
    codes = torch.from_numpy(code_k).to(DEV).expand(N, K).contiguous()
    Wq = qg.quant_pack_int4(codes)
    del codes
    S = torch.ones((N, K // 128), dtype=torch.float16, device=DEV)
    Z = torch.zeros((N, K // 128), dtype=torch.float16, device=DEV)
    row = oracle.pack_int4(code_k[None, :])
    return Wq, S, Z, row


# bn = 0: the token-major tile
@pytest.mark.parametrize("bn,stages,split_k", [(16, 16, 1), (32, 16, 1), (32, 16, 2), (32, 4, 2),
                                               (64, 8, 1), (128, 8, 2), (256, 4, 1), (0, 2, 1),
                                               (0, 4, 1), (0, 4, 16), (0, 3, 5)])
def test_w4a16_tc_packed_ring_positions(copy_tagged_weights, bn, stages, split_k):
    """Token m reads exactly one slab (slab 4m + m % 4: every packed copy once, at every position
    inside it), so each output is 64 x the code of the copy the MMA actually used; compared
    bit-exactly with the oracle, three runs each (the hazard this pins is timing-dependent)."""
    Wq, S, Z, row = copy_tagged_weights
    M, N, K = 64, 16384, 16384
    slab = 4 * np.arange(M) + np.arange(M) % 4
    A = (np.arange(K)[None, :] // 64 == slab[:, None]).astype(np.float16)
    ones, zeros = np.ones((1, K // 128), np.float16), np.zeros((1, K // 128), np.float16)
    ref = oracle.w4a16(A, row, ones, zeros, K, 128)                  # one weight row: [M, 1]
    assert np.array_equal(ref[:, 0], 64.0 * ((slab // 4) % 16))
    Ad = to_dev(A)
    cfg = toka_config(M, N, K, 128, 1, stages, split_k) if bn == 0 else \
        tc_config("w4a16", M, N, K, 128, 1, bn, stages, split_k)
    with cfg:
        for _ in range(3):
            C = qg.qgemm_w4a16(Ad, Wq, S, Z, group_size=128).cpu().numpy().astype(np.float64)
            bad = np.argwhere(C != ref)
            assert len(bad) == 0, f"{len(bad)} wrong, first (m, n) = {bad[:4].tolist()}"


def test_w4a16_tc_one_hot_element_order():
    N, K, gs = 160, 256, 64
    G = K // gs
    codes = synth.uniform_int((N, K), 0, 15, 8, synth.TID_W, np.uint8)
    s = synth.uniform_f16((N, G), 0.001, 0.01, 8, synth.TID_SCALE)
    A = np.eye(K, dtype=np.float16)
    with tc_config("w4a16", K, N, K, gs, 0, 128, 3, 1):
        C = qg.qgemm_w4a16(to_dev(A), qg.quant_pack_int4(to_dev(codes)), to_dev(s), None,
                           group_size=gs).cpu().numpy()
    g = np.arange(K) // gs
    want = (codes.T.astype(np.float64) * s.T[g].astype(np.float64)).astype(np.float16)
    assert np.array_equal(C, want)


def test_w4a16_tc_unit_scale_integer_case_is_exact():
    M, N, K, gs = 48, 136, 256, 64
    codes = synth.uniform_int((N, K), 0, 15, 9, synth.TID_W, np.uint8)
    A = synth.uniform_int((M, K), -1, 0, 9, synth.TID_A, np.int8).astype(np.float16)
    ones = np.ones((N, K // gs), dtype=np.float16)
    ref = oracle.w4a16(A, oracle.pack_int4(codes), ones, None, K, gs)
    assert np.abs(ref).max() < 2048
    with tc_config("w4a16", M, N, K, gs, 0, 64, 2, 1):
        C = qg.qgemm_w4a16(to_dev(A), qg.quant_pack_int4(to_dev(codes)), to_dev(ones), None,
                           group_size=gs).cpu().numpy().astype(np.float64)
    assert np.array_equal(C, ref)


def test_w4a16_tc_guard_bands():
    M, N, K = 40, 136, 512
    case = W4Case(M, N, K, 128, 1, seed=4)
    buf, C, pad = guarded((M, N), torch.float16)
    with tc_config("w4a16", M, N, K, 128, 1, 64, 3, 2):
        case.run(C=C)
    torch.cuda.synchronize()
    assert guards_intact(buf, pad, M * N)
    assert_fp16_close(C, case.ref_full(), "guarded")


@pytest.mark.parametrize("M", [32, 128, 512, 16384])
def test_w4a16_full_size_sampled(M):
    N = K = 16384
    case = W4Case(M, N, K, 128, 1, seed=M + 7)
    C = case.run().float().cpu().numpy()
    ms, ns = sample_pairs(M, N, 300, seed=M)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), f"w4a16 M={M}")


def test_w4a16_full_size_no_zero_sampled():
    M, N, K = 512, 16384, 16384
    case = W4Case(M, N, K, 128, 0, seed=3)
    C = case.run().float().cpu().numpy()
    ms, ns = sample_pairs(M, N, 300, seed=4)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), "w4a16 hz=0")


# ---- W8A8 / W2A8 ---------------------------------------------------------------------------------

INT_SHAPES = [(17, 128, 256), (32, 200, 512), (64, 256, 1024), (100, 130, 384), (129, 512, 512),
              (300, 136, 1024), (8, 256, 512), (256, 256, 128)]


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("M,N,K", INT_SHAPES)
@pytest.mark.parametrize("bn,stages", TC_TILES)
def test_int_tc_tiles(op, M, N, K, bn, stages):
    case = IntCase(op, M, N, K, seed=M + N)
    with tc_config(op, M, N, K, -1, 0, bn, stages, 1):
        assert np.array_equal(case.run().cpu().numpy(), case.ref_full())


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("split_k", [2, 3, 4])
def test_int_tc_split_k(op, split_k):
    M, N, K = 64, 256, 4096
    case = IntCase(op, M, N, K, seed=split_k)
    with tc_config(op, M, N, K, -1, 0, 64, 3, split_k):
        assert np.array_equal(case.run().cpu().numpy(), case.ref_full())


def test_w8a8_tc_extremes():
    M, N, K = 32, 128, 16384
    A = np.full((M, K), -128, dtype=np.int8)
    W = np.full((N, K), -128, dtype=np.int8)
    W[1::2] = 127
    with tc_config("w8a8", M, N, K, -1, 0, 32, 3, 2):
        C = qg.qgemm_w8a8(to_dev(A), to_dev(W)).cpu().numpy()
    assert np.array_equal(C, oracle.w8a8(A, W))
    assert C[0, 0] == K * 16384


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("M", [32, 128, 512])
def test_int_tc_full_size_sampled(op, M):
    N = K = 16384
    case = IntCase(op, M, N, K, seed=M + 11)
    got = case.run().cpu().numpy()
    ms, ns = sample_pairs(M, N, 400, seed=M)
    assert np.array_equal(got[ms, ns], case.ref_at(ms, ns))


def test_tc_error_word_clear_after_runs():
    case = W4Case(64, 256, 512, 128, 1)
    with tc_config("w4a16", 64, 256, 512, 128, 1, 64, 2, 1):
        case.run()
    qg.qgemm_sync_check()
