"""The interleaved int2 layout on the GPU: quant_pack_int2_interleaved bit-exact against the
oracle's packing, and qgemm_w2a8_interleaved bit-exact against the oracle (on the naturally
packed weights of the same values) on every kernel path: the dp4a GEMV, the TMA-fed warp-level
MMA GEMV and the tensor-core tile, with K splits, ragged rows and the full benchmark shapes."""
import numpy as np
import pytest

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import sample_pairs, to_dev

pytestmark = pytest.mark.gpu


class Case:
    def __init__(self, M, N, K, seed):
        d = synth.w2a8_inputs(M, N, K, seed)
        self.M, self.N, self.K = M, N, K
        self.h = d
        self.A = to_dev(d["A"])
        self.Wi = qg.quant_pack_int2_interleaved(to_dev(d["Wv"]))
        self.Wn_host = oracle.pack_int2(d["Wv"])   # the oracle reads the natural layout

    def run(self, split_k=0):
        return qg.qgemm_w2a8_interleaved(self.A, self.Wi, split_k=split_k).cpu().numpy()

    def ref(self):
        return oracle.w2a8(self.h["A"], self.Wn_host)


def pinned(M, N, K, cfg):
    key = (qg.OP_W2A8_INTERLEAVED, M, N, K, -1, 0)

    class _P:
        def __enter__(self):
            qg.qgemm_set_config(*key, cfg)

        def __exit__(self, *exc):
            qg.qgemm_set_config(*key, None)
    return _P()


def test_pack_int2_interleaved_bit_exact():
    for N, K in [(1, 64), (5, 192), (1000, 4096)]:
        vals = synth.uniform_int((N, K), -2, 1, N + K + 1, synth.TID_W, np.int8)
        got = qg.quant_pack_int2_interleaved(to_dev(vals)).cpu().numpy().view(np.uint32)
        assert np.array_equal(got, oracle.pack_int2_interleaved(vals)), (N, K)


def test_pack_int2_interleaved_masks_high_bits():
    vals = synth.uniform_int((8, 128), -128, 127, 3, synth.TID_W, np.int8)
    got = qg.quant_pack_int2_interleaved(to_dev(vals)).cpu().numpy().view(np.uint32)
    assert np.array_equal(got, oracle.pack_int2_interleaved(vals))


SMALL = [(1, 256, 512), (1, 4099, 1024), (2, 33, 256), (3, 100, 2048), (5, 64, 1024),
         (9, 130, 512), (32, 96, 256), (64, 256, 1024), (129, 200, 512), (300, 136, 1024)]


@pytest.mark.parametrize("M,N,K", SMALL)
def test_w2a8_interleaved_default_plan_all_splits(M, N, K):
    case = Case(M, N, K, seed=M + N)
    ref = case.ref()
    for split in (0, 1, 3):
        assert np.array_equal(case.run(split), ref), (M, N, K, split)


@pytest.mark.parametrize("rows", [1, 4, 8])
@pytest.mark.parametrize("M", [1, 3, 4])
def test_w2a8_interleaved_dp4a_gemv(rows, M):
    N, K = 70, 1024
    case = Case(M, N, K, seed=rows + M)
    cfg = {"path": qg.PATH_GEMV, "rows": rows, "bm": 0, "bn": 0, "bk": 0, "stages": 0,
           "split_k": 2, "swap_ab": 0}
    with pinned(M, N, K, cfg):
        assert np.array_equal(case.run(), case.ref())


@pytest.mark.parametrize("rows,stages", [(16, 2), (32, 4), (64, 5), (64, 6)])
@pytest.mark.parametrize("M", [1, 7, 16])
def test_w2a8_interleaved_tma_gemv(rows, stages, M):
    N, K = 200, 4096
    case = Case(M, N, K, seed=rows + stages + M)
    for split in (1, 3):
        cfg = {"path": qg.PATH_GEMV, "rows": rows, "bm": 0, "bn": 0, "bk": 0, "stages": stages,
               "split_k": split, "swap_ab": 0}
        with pinned(M, N, K, cfg):
            assert np.array_equal(case.run(), case.ref()), (rows, stages, split)


@pytest.mark.parametrize("bn,stages,split", [(16, 3, 1), (64, 4, 2), (128, 5, 1), (256, 3, 3),
                                             (256, 4, 1)])
@pytest.mark.parametrize("M,N,K", [(40, 256, 1024), (130, 200, 2048), (256, 384, 4096)])
def test_w2a8_interleaved_tensor_core_tile(bn, stages, split, M, N, K):
    case = Case(M, N, K, seed=bn + M)
    cfg = {"path": qg.PATH_TC, "rows": 0, "bm": 128, "bn": bn, "bk": 0, "stages": stages,
           "split_k": split, "swap_ab": 1}
    try:
        qg.qgemm_set_config(qg.OP_W2A8_INTERLEAVED, M, N, K, -1, 0, cfg)
    except qg.QGemmError:
        pytest.skip(f"bn={bn} stages={stages} does not fit K={K}")
    try:
        assert np.array_equal(case.run(), case.ref())
    finally:
        qg.qgemm_set_config(qg.OP_W2A8_INTERLEAVED, M, N, K, -1, 0, None)


def test_w2a8_interleaved_one_hot_columns():
    """A = e_k: C[m, n] = W[n, k] for every k of a word, across two words and a 256-wide k-block,
    on the tensor-core tile (pins that the byte-table upcast keeps K order)."""
    M, N, K = 128, 128, 512
    Wv = synth.uniform_int((N, K), -2, 1, 77, synth.TID_W, np.int8)
    Wi = qg.quant_pack_int2_interleaved(to_dev(Wv))
    A = np.zeros((M, K), np.int8)
    ks = np.arange(M) * 5 % K
    A[np.arange(M), ks] = 1
    cfg = {"path": qg.PATH_TC, "rows": 0, "bm": 128, "bn": 128, "bk": 0, "stages": 3,
           "split_k": 1, "swap_ab": 1}
    with pinned(M, N, K, cfg):
        C = qg.qgemm_w2a8_interleaved(to_dev(A), Wi).cpu().numpy()
    assert np.array_equal(C, Wv[:, ks].T.astype(np.int32))


@pytest.mark.parametrize("M", [1, 32, 128, 512])
def test_w2a8_interleaved_benchmark_shapes_sampled(M):
    N = K = 16384
    case = Case(M, N, K, seed=M + 3)
    got = case.run()
    ms, ns = sample_pairs(M, N, 400, seed=M)
    assert np.array_equal(got[ms, ns], oracle.w2a8_at(case.h["A"], case.Wn_host, ms, ns))
