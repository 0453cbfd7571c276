"""The 512-token weight-major tensor-core tile (each upcast weight slab feeds two 256-token
accumulators that fill TMEM) against the oracle for the packed formats: ragged weight rows and
tokens (a second half with some, or no, tokens), K splits, both ring depths, group sizes, both
packed layouts, element order, the copy-tagged packed ring, and the full-size benchmark shapes on
one element of every tile."""
import contextlib

import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import DEV, IntCase, W4Case, assert_fp16_close, guarded, guards_intact, sample_pairs, to_dev

pytestmark = pytest.mark.gpu

OPS = {"w4a16": qg.OP_W4A16, "w2a8": qg.OP_W2A8, "w4a16i": qg.OP_W4A16_INTERLEAVED,
       "w2a8i": qg.OP_W2A8_INTERLEAVED}


def dual_cfg(stages, split_k):
    return {"path": qg.PATH_TC, "rows": 0, "bm": 128, "bn": 512, "bk": 0, "stages": stages,
            "split_k": split_k, "swap_ab": 1}


@contextlib.contextmanager
def pinned(op, M, N, K, gs, hz, cfg):
    key = (OPS[op], M, N, K, gs, hz)
    qg.qgemm_set_config(*key, cfg)
    try:
        plan = qg.qgemm_plan(*key)
        assert plan["path"] == qg.PATH_TC and plan["bn"] == 512
        yield
    finally:
        qg.qgemm_set_config(*key, None)


# (M, N, K): tokens inside the first half only, across both halves, exactly one tile, across
# tiles with a ragged last one; weight rows with a ragged last tile; K of whole and partial
# 4-slab runs (K = 1088: 17 slabs, single-slab packed copies)
SHAPES = [(40, 256, 1024), (300, 200, 2048), (512, 384, 1024), (700, 520, 4096),
          (1100, 1000, 2048), (256, 130, 1088)]
TILES = [(2, 1), (4, 1), (4, 2), (2, 3)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("stages,split_k", TILES)
def test_dual_w4a16(M, N, K, stages, split_k):
    case = W4Case(M, N, K, 64, 1, seed=M + N + stages)
    with pinned("w4a16", M, N, K, 64, 1, dual_cfg(stages, split_k)):
        assert_fp16_close(case.run(), case.ref_full(), f"dual w4a16 {M},{N},{K}")


@pytest.mark.parametrize("M,N,K", [(40, 256, 1024), (300, 200, 2048), (700, 520, 4096),
                                   (1100, 1000, 2048)])
@pytest.mark.parametrize("stages,split_k", [(2, 1), (4, 2)])
def test_dual_w2a8(M, N, K, stages, split_k):
    case = IntCase("w2a8", M, N, K, seed=M + N)
    with pinned("w2a8", M, N, K, -1, 0, dual_cfg(stages, split_k)):
        assert np.array_equal(case.run().cpu().numpy(), case.ref_full())


@pytest.mark.parametrize("gs,hz", [(32, 1), (128, 0), (256, 1), (-1, 1)])
def test_dual_w4a16_group_sizes(gs, hz):
    M, N, K = 600, 384, 2048
    case = W4Case(M, N, K, gs, hz, seed=9)
    ge = K if gs == -1 else gs
    with pinned("w4a16", M, N, K, ge, hz, dual_cfg(4, 1)):
        assert_fp16_close(case.run(), case.ref_full(), f"dual gs={gs} hz={hz}")


def test_dual_interleaved_layouts():
    M, N, K = 700, 520, 2048
    d = synth.w4a16_inputs(M, N, K, 128, True, seed=23)
    Wi = qg.quant_pack_int4_interleaved(to_dev(d["codes"]))
    ref = oracle.w4a16(d["A"], oracle.pack_int4(d["codes"]), d["scales"], d["zeros"], K, 128)
    with pinned("w4a16i", M, N, K, 128, 1, dual_cfg(4, 1)):
        C = qg.qgemm_w4a16_interleaved(to_dev(d["A"]), Wi, to_dev(d["scales"]),
                                       to_dev(d["zeros"]), group_size=128)
    assert_fp16_close(C, ref, "dual interleaved int4")
    e = synth.w2a8_inputs(M, N, K, seed=24)
    W2 = qg.quant_pack_int2_interleaved(to_dev(e["Wv"]))
    with pinned("w2a8i", M, N, K, -1, 0, dual_cfg(2, 2)):
        C2 = qg.qgemm_w2a8_interleaved(to_dev(e["A"]), W2).cpu().numpy()
    assert np.array_equal(C2, oracle.w2a8(e["A"], oracle.pack_int2(e["Wv"])))


def test_dual_one_hot_element_order():
    """A = e_k over 512 tokens: C[k, n] = fp16(q[n,k] s[n, k/gs]) for every k, so a weight row or
    a token of either accumulator half read from the wrong place shows exactly."""
    N, K, gs = 384, 512, 64
    G = K // gs
    codes = synth.uniform_int((N, K), 0, 15, 12, synth.TID_W, np.uint8)
    s = synth.uniform_f16((N, G), 0.001, 0.01, 12, synth.TID_SCALE)
    A = np.eye(K, dtype=np.float16)
    with pinned("w4a16", K, N, K, gs, 0, dual_cfg(4, 1)):
        C = qg.qgemm_w4a16(to_dev(A), qg.quant_pack_int4(to_dev(codes)), to_dev(s), None,
                           group_size=gs).cpu().numpy()
    g = np.arange(K) // gs
    want = (codes.T.astype(np.float64) * s.T[g].astype(np.float64)).astype(np.float16)
    assert np.array_equal(C, want)


def test_dual_guard_bands_and_repeat_bits():
    M, N, K = 700, 520, 1024
    case = W4Case(M, N, K, 128, 1, seed=5)
    buf, C, pad = guarded((M, N), torch.float16)
    with pinned("w4a16", M, N, K, 128, 1, dual_cfg(4, 1)):
        case.run(C=C)
        C2 = case.run()
    torch.cuda.synchronize()
    assert guards_intact(buf, pad, M * N)
    assert torch.equal(C, C2)          # no K split: the same bits every run
    assert_fp16_close(C, case.ref_full(), "dual guarded")


@pytest.mark.parametrize("stages", [2, 4])
def test_dual_packed_ring_positions(stages):
    """Weights whose codes name their 4-slab copy (s = 1, z = 0); token m reads one slab, so a
    copy or an activation half read from the wrong ring slot, too early or after it was
    overwritten changes C by a multiple of 64 (bit-exact comparison, three runs)."""
    N = K = 16384
    code_k = ((np.arange(K) // 256) % 16).astype(np.uint8)
    codes = torch.from_numpy(code_k).to(DEV).expand(N, K).contiguous()
    Wq = qg.quant_pack_int4(codes)
    del codes
    S = torch.ones((N, K // 128), dtype=torch.float16, device=DEV)
    Z = torch.zeros((N, K // 128), dtype=torch.float16, device=DEV)
    row = oracle.pack_int4(code_k[None, :])
    M = 1024
    slab = (4 * np.arange(M) + np.arange(M) % 4) % (K // 64)
    A = (np.arange(K)[None, :] // 64 == slab[:, None]).astype(np.float16)
    ref = oracle.w4a16(A, row, np.ones((1, K // 128), np.float16),
                       np.zeros((1, K // 128), np.float16), K, 128)
    Ad = to_dev(A)
    with pinned("w4a16", M, N, K, 128, 1, dual_cfg(stages, 1)):
        for _ in range(3):
            C = qg.qgemm_w4a16(Ad, Wq, S, Z, group_size=128).cpu().numpy().astype(np.float64)
            bad = np.argwhere(C != ref)
            assert len(bad) == 0, f"{len(bad)} wrong, first (m, n) = {bad[:4].tolist()}"


@pytest.mark.parametrize("M", [4096, 16384])
def test_dual_full_size_sampled(M):
    N = K = 16384
    case = W4Case(M, N, K, 128, 1, seed=M + 7)
    with pinned("w4a16", M, N, K, 128, 1, dual_cfg(4, 1)):
        C = case.run().float().cpu().numpy()
        qg.qgemm_sync_check()
    ms, ns = sample_pairs(M, N, 300, seed=M + 1)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), f"dual M={M}")


def test_dual_w2a8_full_size_sampled():
    M, N, K = 2048, 16384, 16384
    case = IntCase("w2a8", M, N, K, seed=13)
    with pinned("w2a8", M, N, K, -1, 0, dual_cfg(4, 1)):
        got = case.run().cpu().numpy()
    ms, ns = sample_pairs(M, N, 300, seed=5)
    assert np.array_equal(got[ms, ns], case.ref_at(ms, ns))
