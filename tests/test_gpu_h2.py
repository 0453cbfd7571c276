"""The W4A16 GEMV on the packed fp16 FMA pipe (path GEMV, bn = 2; one to eight tokens in tiles of
1, 2 or 4) against the oracle: every output within the fp16 rule, element order pinned by one-hot
activations, the zero-point algebra by fractional and absent zero points, both weight layouts,
ragged rows and K splits, and the benchmark's full-size shapes on one element of every tile."""
import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import DEV, W4Case, assert_fp16_close, guarded, guards_intact, sample_pairs, to_dev

pytestmark = pytest.mark.gpu


def h2_cfg(rows, stages, split_k):
    return {"path": qg.PATH_GEMV, "rows": rows, "bm": 0, "bn": 2, "bk": 0, "stages": stages,
            "split_k": split_k, "swap_ab": 0}


class pinned:
    def __init__(self, op, M, N, K, gs, hz, cfg):
        self.key = (op, M, N, K, gs, hz)
        self.cfg = cfg

    def __enter__(self):
        qg.qgemm_set_config(*self.key, self.cfg)
        assert qg.qgemm_plan(*self.key)["bn"] == 2

    def __exit__(self, *exc):
        qg.qgemm_set_config(*self.key, None)


# (M, N, K, gs, hz): ragged row tiles (N % 32, N % 64), odd N (single-element stores), one-group
# K (gs = -1), group sizes 128 .. 512, token counts that leave part of a token tile empty
SHAPES = [(1, 64, 128, 128, 1), (1, 200, 1024, 128, 0), (1, 4104, 4096, 256, 1),
          (1, 513, 2048, -1, 1), (2, 4095, 1152, 128, 1), (2, 130, 384, 384, 0),
          (3, 96, 512, 128, 1), (4, 1000, 4096, 128, 1), (5, 77, 1024, 512, 0),
          (8, 257, 2048, 128, 1), (6, 33, 256, -1, 1)]
TILES = [(32, 2, 1), (64, 4, 3), (64, 6, 16), (32, 3, 1), (64, 5, 64), (32, 4, 2)]


@pytest.mark.parametrize("M,N,K,gs,hz", SHAPES)
@pytest.mark.parametrize("rows,stages,split_k", TILES)
def test_h2_shapes(M, N, K, gs, hz, rows, stages, split_k):
    case = W4Case(M, N, K, gs, hz, seed=M + N + K + rows)
    ge = K if gs == -1 else gs
    with pinned(qg.OP_W4A16, M, N, K, ge, hz, h2_cfg(rows, stages, split_k)):
        assert_fp16_close(case.run(), case.ref_full(), f"h2 M={M} N={N} K={K} rows={rows}")


@pytest.mark.parametrize("M", [1, 2, 4])
def test_h2_one_hot_element_order_and_fractional_zero(M):
    """A = e_k (every token the same one-hot row): C[m, n] = (q[n,k] - z) s for k at every
    position of a word, of a 32-wide lane quarter and of two groups, with a fractional zero
    point, so that a code paired with the wrong activation or scale shows."""
    N, K, gs = 96, 256, 128
    case = W4Case(M, N, K, gs, 1, seed=31, zero_value=6.5)
    with pinned(qg.OP_W4A16, M, N, K, gs, 1, h2_cfg(32, 2, 1)):
        for k in (0, 1, 3, 4, 5, 7, 8, 31, 32, 100, 127, 128, 130, 200, 255):
            A = np.zeros((M, K), np.float16)
            A[:, k] = 1.0
            C = qg.qgemm_w4a16(to_dev(A), case.Wq, case.S, case.Z, group_size=gs)
            ref = oracle.w4a16(A, case.Wq_host, case.h["scales"], case.h["zeros"], K, gs)
            assert_fp16_close(C, ref, f"k={k}")


def test_h2_interleaved_layout():
    M, N, K, gs = 2, 300, 2048, 128
    d = synth.w4a16_inputs(M, N, K, gs, True, seed=12)
    Wi = qg.quant_pack_int4_interleaved(to_dev(d["codes"]))
    ref = oracle.w4a16(d["A"], oracle.pack_int4(d["codes"]), d["scales"], d["zeros"], K, gs)
    for rows, stages, split in [(32, 3, 1), (64, 4, 4)]:
        with pinned(qg.OP_W4A16_INTERLEAVED, M, N, K, gs, 1, h2_cfg(rows, stages, split)):
            C = qg.qgemm_w4a16_interleaved(to_dev(d["A"]), Wi, to_dev(d["scales"]),
                                           to_dev(d["zeros"]), group_size=gs)
            assert_fp16_close(C, ref, f"interleaved rows={rows}")


def test_h2_large_activations_inside_the_stated_range():
    """Activations scaled by 80 (|a| up to ~300): the fp16 runs stay finite and the result keeps
    its relative accuracy. Products are rounded to fp16, so the absolute error grows with |A|:
    the rule's absolute term is scaled by the same factor here (relative Frobenius unchanged)."""
    M, N, K, gs, f = 1, 256, 4096, 128, 80.0
    case = W4Case(M, N, K, gs, 1, seed=3)
    A = (case.h["A"].astype(np.float32) * f).astype(np.float16)
    assert np.abs(A).max() < 512
    with pinned(qg.OP_W4A16, M, N, K, gs, 1, h2_cfg(64, 4, 1)):
        C = qg.qgemm_w4a16(to_dev(A), case.Wq, case.S, case.Z, group_size=gs)
    got = C.float().cpu().numpy().astype(np.float64)
    ref = oracle.w4a16(A, case.Wq_host, case.h["scales"], case.h["zeros"], K, gs)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= f * oracle.ATOL + oracle.RTOL * np.abs(ref))
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= oracle.FROB


def test_h2_split_overwrites_stale_output_and_keeps_guards():
    M, N, K = 3, 200, 2048
    case = W4Case(M, N, K, 128, 1, seed=8)
    buf, C, pad = guarded((M, N), torch.float16, fill=0x3C)   # stale 1.0-ish values inside too
    with pinned(qg.OP_W4A16, M, N, K, 128, 1, h2_cfg(32, 3, 4)):
        case.run(C=C)
    torch.cuda.synchronize()
    assert guards_intact(buf, pad, M * N, fill=0x3C)
    assert_fp16_close(C, case.ref_full(), "stale output")


def test_h2_non_default_stream_and_repeat_bits():
    M, N, K = 1, 512, 4096
    case = W4Case(M, N, K, 128, 1, seed=4)
    s = torch.cuda.Stream()
    with pinned(qg.OP_W4A16, M, N, K, 128, 1, h2_cfg(64, 4, 1)):
        with torch.cuda.stream(s):
            C1 = case.run()
            C2 = case.run()
        s.synchronize()
    assert torch.equal(C1, C2)     # no K split: no atomics, the same bits every time
    assert_fp16_close(C1, case.ref_full(), "side stream")


@pytest.mark.parametrize("M", [1, 2, 4])
def test_h2_full_size_sampled(M):
    """N = K = 16384, the benchmark's shape, one element of every 128 x 128 tile checked; the
    relative Frobenius error of the sample is reported against the 5e-3 bound."""
    N = K = 16384
    case = W4Case(M, N, K, 128, 1, seed=M + 90)
    with pinned(qg.OP_W4A16, M, N, K, 128, 1, h2_cfg(64, 4, 2)):
        C = case.run().float().cpu().numpy()
    ms, ns = sample_pairs(M, N, 2000, seed=M)
    ref = case.ref_at(ms, ns)
    ok, msg = oracle.fp16_close(C[ms, ns], ref)
    print(f"h2 M={M} full size: {msg}")
    assert ok, msg


def test_h2_rejects_more_than_eight_tokens():
    with pytest.raises(qg.QGemmError):
        qg.qgemm_set_config(qg.OP_W4A16, 9, 256, 1024, 128, 1, h2_cfg(64, 4, 1))
    with pytest.raises(qg.QGemmError):   # group sizes below 128 are not served
        qg.qgemm_set_config(qg.OP_W4A16, 1, 256, 1024, 64, 1, h2_cfg(64, 4, 1))
