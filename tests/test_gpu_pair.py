"""The weight-major tensor-core tile shared by a CTA pair (cta_group::2: one MMA spans two SMs,
256 weight rows x 128 or 256 tokens, each CTA holding half of the token rows) against the oracle
for every operand format: ragged weight rows and tokens (tails of the 256-row pair tile and of
each CTA's half), K splits, pipeline depths, both packed layouts, element order, the
copy-tagged packed ring, and the full-size benchmark shapes on one element of every tile."""
import contextlib

import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import DEV, IntCase, W4Case, assert_fp16_close, guarded, guards_intact, sample_pairs, to_dev

pytestmark = pytest.mark.gpu

OPS = {"w4a16": qg.OP_W4A16, "w8a8": qg.OP_W8A8, "w2a8": qg.OP_W2A8, "dense": qg.OP_DENSE_F16,
       "w4a16i": qg.OP_W4A16_INTERLEAVED, "w2a8i": qg.OP_W2A8_INTERLEAVED}


def pair_cfg(bn, stages, split_k):
    return {"path": qg.PATH_TC, "rows": 0, "bm": 256, "bn": bn, "bk": 0, "stages": stages,
            "split_k": split_k, "swap_ab": 1}


@contextlib.contextmanager
def pinned(op, M, N, K, gs, hz, cfg):
    key = (OPS[op], M, N, K, gs, hz)
    try:
        qg.qgemm_set_config(*key, cfg)
    except qg.QGemmError:
        pytest.skip(f"{cfg} does not fit this problem")
    try:
        plan = qg.qgemm_plan(*key)
        assert plan["path"] == qg.PATH_TC and plan["bm"] == 256
        yield
    finally:
        qg.qgemm_set_config(*key, None)


# (M, N, K): tokens below / across one tile and a CTA's half of it, weight rows that leave the
# second CTA of the last pair partly or wholly empty (N % 256 < 128), K of 4-slab multiples
SHAPES = [(40, 256, 1024), (130, 200, 2048), (256, 384, 1024), (300, 520, 4096),
          (512, 1000, 2048), (64, 130, 1024)]
TILES = [(256, 3, 1), (256, 4, 2), (256, 5, 1), (128, 4, 1), (128, 8, 3), (256, 8, 1)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("bn,stages,split_k", TILES)
def test_pair_w4a16(M, N, K, bn, stages, split_k):
    case = W4Case(M, N, K, 128, 1, seed=M + N + bn)
    with pinned("w4a16", M, N, K, 128, 1, pair_cfg(bn, stages, split_k)):
        assert_fp16_close(case.run(), case.ref_full(), f"pair w4a16 {M},{N},{K}")


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("bn,stages,split_k", [(256, 3, 1), (128, 4, 2), (256, 5, 3)])
def test_pair_int(op, M, N, K, bn, stages, split_k):
    case = IntCase(op, M, N, K, seed=M + N + bn)
    with pinned(op, M, N, K, -1, 0, pair_cfg(bn, stages, split_k)):
        assert np.array_equal(case.run().cpu().numpy(), case.ref_full())


@pytest.mark.parametrize("M,N,K", [(40, 256, 1024), (300, 520, 2048), (512, 384, 1024)])
@pytest.mark.parametrize("bn,stages,split_k", [(256, 3, 1), (128, 4, 2), (256, 4, 1)])
def test_pair_dense(M, N, K, bn, stages, split_k):
    h = synth.dense_inputs(M, N, K, seed=M + bn)
    with pinned("dense", M, N, K, -1, 0, pair_cfg(bn, stages, split_k)):
        C = qg.qgemm_dense_f16(to_dev(h["A"]), to_dev(h["W"]))
    assert_fp16_close(C, oracle.dense_f16(h["A"], h["W"]), f"pair dense {M},{N},{K}")


@pytest.mark.parametrize("gs,hz", [(64, 0), (256, 1), (-1, 1), (32, 1)])
def test_pair_w4a16_group_sizes(gs, hz):
    M, N, K = 256, 384, 2048
    case = W4Case(M, N, K, gs, hz, seed=7)
    ge = K if gs == -1 else gs
    with pinned("w4a16", M, N, K, ge, hz, pair_cfg(256, 4, 1)):
        assert_fp16_close(case.run(), case.ref_full(), f"pair gs={gs} hz={hz}")


def test_pair_interleaved_layouts():
    M, N, K = 300, 520, 2048
    d = synth.w4a16_inputs(M, N, K, 128, True, seed=21)
    Wi = qg.quant_pack_int4_interleaved(to_dev(d["codes"]))
    ref = oracle.w4a16(d["A"], oracle.pack_int4(d["codes"]), d["scales"], d["zeros"], K, 128)
    with pinned("w4a16i", M, N, K, 128, 1, pair_cfg(256, 4, 1)):
        C = qg.qgemm_w4a16_interleaved(to_dev(d["A"]), Wi, to_dev(d["scales"]),
                                       to_dev(d["zeros"]), group_size=128)
    assert_fp16_close(C, ref, "pair interleaved int4")
    e = synth.w2a8_inputs(M, N, K, seed=22)
    W2 = qg.quant_pack_int2_interleaved(to_dev(e["Wv"]))
    with pinned("w2a8i", M, N, K, -1, 0, pair_cfg(256, 3, 2)):
        C2 = qg.qgemm_w2a8_interleaved(to_dev(e["A"]), W2).cpu().numpy()
    assert np.array_equal(C2, oracle.w2a8(e["A"], oracle.pack_int2(e["Wv"])))


def test_pair_one_hot_element_order():
    """A = e_k: C[k, n] = fp16((q[n,k] - 0) s[n, k/gs]) for every k, so a weight row of either CTA
    or a token of either half read from the wrong place shows exactly."""
    N, K, gs = 512, 256, 64
    G = K // gs
    codes = synth.uniform_int((N, K), 0, 15, 8, synth.TID_W, np.uint8)
    s = synth.uniform_f16((N, G), 0.001, 0.01, 8, synth.TID_SCALE)
    A = np.eye(K, dtype=np.float16)
    with pinned("w4a16", K, N, K, gs, 0, pair_cfg(256, 3, 1)):
        C = qg.qgemm_w4a16(to_dev(A), qg.quant_pack_int4(to_dev(codes)), to_dev(s), None,
                           group_size=gs).cpu().numpy()
    g = np.arange(K) // gs
    want = (codes.T.astype(np.float64) * s.T[g].astype(np.float64)).astype(np.float16)
    assert np.array_equal(C, want)


def test_pair_guard_bands_and_repeat_bits():
    M, N, K = 300, 520, 1024
    case = W4Case(M, N, K, 128, 1, seed=4)
    buf, C, pad = guarded((M, N), torch.float16)
    with pinned("w4a16", M, N, K, 128, 1, pair_cfg(256, 4, 1)):
        case.run(C=C)
        C2 = case.run()
    torch.cuda.synchronize()
    assert guards_intact(buf, pad, M * N)
    assert torch.equal(C, C2)          # no K split: the same bits every run
    assert_fp16_close(C, case.ref_full(), "pair guarded")


@pytest.mark.parametrize("bn,stages", [(256, 3), (256, 5), (128, 8)])
def test_pair_packed_ring_positions(bn, stages):
    """Weights whose codes name their 4-slab copy (s = 1, z = 0); token m reads one slab, so a
    copy read from the wrong ring slot, too early or after it was overwritten changes C by a
    multiple of 64 (bit-exact comparison, three runs)."""
    N = K = 16384
    code_k = ((np.arange(K) // 256) % 16).astype(np.uint8)
    codes = torch.from_numpy(code_k).to(DEV).expand(N, K).contiguous()
    Wq = qg.quant_pack_int4(codes)
    del codes
    S = torch.ones((N, K // 128), dtype=torch.float16, device=DEV)
    Z = torch.zeros((N, K // 128), dtype=torch.float16, device=DEV)
    row = oracle.pack_int4(code_k[None, :])
    M = 256
    slab = (4 * np.arange(M) + np.arange(M) % 4) % (K // 64)
    A = (np.arange(K)[None, :] // 64 == slab[:, None]).astype(np.float16)
    ref = oracle.w4a16(A, row, np.ones((1, K // 128), np.float16),
                       np.zeros((1, K // 128), np.float16), K, 128)
    Ad = to_dev(A)
    with pinned("w4a16", M, N, K, 128, 1, pair_cfg(bn, stages, 1)):
        for _ in range(3):
            C = qg.qgemm_w4a16(Ad, Wq, S, Z, group_size=128).cpu().numpy().astype(np.float64)
            bad = np.argwhere(C != ref)
            assert len(bad) == 0, f"{len(bad)} wrong, first (m, n) = {bad[:4].tolist()}"


@pytest.mark.parametrize("M", [512, 16384])
def test_pair_full_size_sampled(M):
    N = K = 16384
    case = W4Case(M, N, K, 128, 1, seed=M + 5)
    with pinned("w4a16", M, N, K, 128, 1, pair_cfg(256, 4, 1 if M > 512 else 2)):
        C = case.run().float().cpu().numpy()
        qg.qgemm_sync_check()
    ms, ns = sample_pairs(M, N, 300, seed=M)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), f"pair M={M}")


def test_pair_int_full_size_sampled():
    M, N, K = 512, 16384, 16384
    for op in ("w8a8", "w2a8"):
        case = IntCase(op, M, N, K, seed=11)
        with pinned(op, M, N, K, -1, 0, pair_cfg(256, 4, 1)):
            got = case.run().cpu().numpy()
        ms, ns = sample_pairs(M, N, 300, seed=3)
        assert np.array_equal(got[ms, ns], case.ref_at(ms, ns)), op
