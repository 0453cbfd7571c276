"""W4A16 on the GPU against the oracle: packing bit-exact, every output within the fp16 rule
(|C - ref| <= 0.02 + 0.01 |ref| per element and relative Frobenius error <= 5e-3), plus exact
special cases that pin element order and the zero/scale algebra."""
import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import DEV, W4Case, assert_fp16_close, guarded, guards_intact, sample_pairs, to_dev

pytestmark = pytest.mark.gpu


def test_pack_int4_bit_exact():
    for N, K in [(1, 32), (7, 96), (300, 4096), (4096, 11008)]:
        codes = synth.uniform_int((N, K), 0, 15, N + K, synth.TID_W, np.uint8)
        got = qg.quant_pack_int4(to_dev(codes)).cpu().numpy().view(np.uint32)
        assert np.array_equal(got, oracle.pack_int4(codes)), (N, K)


def test_pack_int4_masks_high_bits():
    codes = synth.uniform_int((16, 64), 0, 255, 5, synth.TID_W, np.uint8)
    got = qg.quant_pack_int4(to_dev(codes)).cpu().numpy().view(np.uint32)
    assert np.array_equal(got, oracle.pack_int4(codes))


# config 0 (M=1, K=N=4096, gs=128, zeros 8) at split_k 1 and 4, then shapes with ragged tails
SMALL = [
    (1, 4096, 4096, 128, 1),
    (1, 256, 512, 128, 0),
    (2, 100, 256, 32, 1),
    (3, 33, 1024, 64, 1),
    (7, 130, 512, 128, 0),
    (8, 64, 256, -1, 1),
    (9, 96, 384, 128, 1),
    (16, 200, 512, 64, 1),
    (17, 72, 256, 128, 1),
    (40, 50, 128, 32, 0),
    (1, 513, 4096, -1, 0),
    (1, 4095, 128, 128, 1),
    (5, 1, 256, 128, 1),
]


@pytest.mark.parametrize("M,N,K,gs,hz", SMALL)
@pytest.mark.parametrize("split_k", [1, 4])
def test_w4a16_small_shapes(M, N, K, gs, hz, split_k):
    case = W4Case(M, N, K, gs, hz, seed=M * 131 + N)
    assert np.array_equal(case.Wq.cpu().numpy().view(np.uint32), case.Wq_host)
    C = case.run(split_k=split_k)
    torch.cuda.synchronize()
    assert_fp16_close(C, case.ref_full(), f"M={M} N={N} K={K} gs={gs} hz={hz} split={split_k}")


@pytest.mark.parametrize("split_k", [2, 3, 5, 8, 16, 64])
def test_w4a16_split_k_values(split_k):
    case = W4Case(3, 160, 2048, 128, 1, seed=split_k)
    assert_fp16_close(case.run(split_k=split_k), case.ref_full(), f"split={split_k}")


@pytest.mark.parametrize("rows", [16, 32, 64])
@pytest.mark.parametrize("M", [1, 12])
@pytest.mark.parametrize("stages", [0, 2, 3, 4, 6])
def test_w4a16_each_row_tile(rows, M, stages):
    case = W4Case(M, 200, 1024, 128, 1, seed=rows)
    cfg = {"path": qg.PATH_GEMV, "rows": rows, "bm": 0, "bn": 0, "bk": 0, "stages": stages,
           "split_k": 2, "swap_ab": 0}
    qg.qgemm_set_config(qg.OP_W4A16, M, 200, 1024, 128, 1, cfg)
    try:
        assert qg.qgemm_plan(qg.OP_W4A16, M, 200, 1024, 128, 1)["rows"] == rows
        assert_fp16_close(case.run(), case.ref_full(), f"rows={rows}")
    finally:
        qg.qgemm_set_config(qg.OP_W4A16, M, 200, 1024, 128, 1, None)


# ---- one token on the FMA pipe (TMA-fed GEMV, bn = 1) -------------------------------------------

def simt_cfg(rows, stages, split_k):
    return {"path": qg.PATH_GEMV, "rows": rows, "bm": 0, "bn": 1, "bk": 0, "stages": stages,
            "split_k": split_k, "swap_ab": 0}


SIMT_SHAPES = [(64, 128, 128, 1), (200, 1024, 128, 0), (4104, 4096, 256, 1), (513, 2048, -1, 1),
               (4095, 1152, 128, 1), (130, 384, 384, 0)]


@pytest.mark.parametrize("N,K,gs,hz", SIMT_SHAPES)
@pytest.mark.parametrize("rows,stages,split_k", [(32, 2, 1), (64, 4, 3), (128, 6, 16),
                                                 (128, 3, 1), (64, 2, 64)])
def test_w4a16_simt_one_token(N, K, gs, hz, rows, stages, split_k):
    """Ragged weight rows (N % rows), one-group K (gs = -1), group sizes 128 .. 384, K splits that
    leave empty parts, each with and without zero points."""
    case = W4Case(1, N, K, gs, hz, seed=N + K + rows)
    ge = K if gs == -1 else gs
    qg.qgemm_set_config(qg.OP_W4A16, 1, N, K, ge, hz, simt_cfg(rows, stages, split_k))
    try:
        assert qg.qgemm_plan(qg.OP_W4A16, 1, N, K, ge, hz)["bn"] == 1
        assert_fp16_close(case.run(), case.ref_full(), f"simt N={N} K={K} rows={rows}")
    finally:
        qg.qgemm_set_config(qg.OP_W4A16, 1, N, K, ge, hz, None)


def test_w4a16_simt_rejects_more_tokens():
    with pytest.raises(qg.QGemmError):
        qg.qgemm_set_config(qg.OP_W4A16, 2, 256, 1024, 128, 1, simt_cfg(64, 4, 1))


def test_w4a16_simt_one_hot_rows_and_fractional_zero():
    """A = e_k for one k at a time (one token): C[0, n] = (q[n,k] - z) s for every k of two
    groups, with a fractional zero point."""
    N, K, gs = 96, 256, 128
    case = W4Case(1, N, K, gs, 1, seed=31, zero_value=6.5)
    qg.qgemm_set_config(qg.OP_W4A16, 1, N, K, gs, 1, simt_cfg(32, 2, 1))
    try:
        for k in (0, 1, 4, 7, 8, 127, 128, 200, 255):
            A = np.zeros((1, K), np.float16)
            A[0, k] = 1.0
            C = qg.qgemm_w4a16(to_dev(A), case.Wq, case.S, case.Z, group_size=gs)
            ref = oracle.w4a16(A, case.Wq_host, case.h["scales"], case.h["zeros"], K, gs)
            assert_fp16_close(C, ref, f"k={k}")
    finally:
        qg.qgemm_set_config(qg.OP_W4A16, 1, N, K, gs, 1, None)


@pytest.mark.parametrize("rows,split_k", [(64, 2), (128, 1)])
def test_w4a16_simt_full_size_sampled(rows, split_k):
    N = K = 16384
    case = W4Case(1, N, K, 128, 1, seed=rows)
    qg.qgemm_set_config(qg.OP_W4A16, 1, N, K, 128, 1, simt_cfg(rows, 4, split_k))
    try:
        C = case.run().float().cpu().numpy()
    finally:
        qg.qgemm_set_config(qg.OP_W4A16, 1, N, K, 128, 1, None)
    ms, ns = sample_pairs(1, N, 2000, seed=rows)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), "simt full size")


def test_w4a16_one_hot_element_order():
    """A = e_k for every k of a 256-wide K: C[k, n] must be exactly fp16((q[n,k] - z) * s)."""
    N, K, gs = 48, 256, 64
    G = K // gs
    codes = synth.uniform_int((N, K), 0, 15, 7, synth.TID_W, np.uint8)
    s = synth.uniform_f16((N, G), 0.001, 0.01, 7, synth.TID_SCALE)
    z = synth.uniform_int((N, G), 0, 15, 7, synth.TID_ZERO, np.int8).astype(np.float16)
    A = np.eye(K, dtype=np.float16)
    for hz in (0, 1):
        # the streaming kernel applies s and z in fp32 per k-block, so the result is exact
        cfg = {"path": qg.PATH_GEMV, "rows": 32, "bm": 0, "bn": 0, "bk": 0, "stages": 0,
               "split_k": 1, "swap_ab": 0}
        qg.qgemm_set_config(qg.OP_W4A16, K, N, K, gs, hz, cfg)
        try:
            C = qg.qgemm_w4a16(to_dev(A), qg.quant_pack_int4(to_dev(codes)), to_dev(s),
                               to_dev(z) if hz else None, group_size=gs, split_k=1)
        finally:
            qg.qgemm_set_config(qg.OP_W4A16, K, N, K, gs, hz, None)
        g = np.arange(K) // gs
        want = ((codes.T.astype(np.float64) - (z.T[g].astype(np.float64) if hz else 0.0))
                * s.T[g].astype(np.float64)).astype(np.float16)
        assert np.array_equal(C.cpu().numpy(), want), hz


def test_w4a16_unit_scale_integer_case_is_exact():
    """s = 1, z = 0, integer activations: every partial sum is an integer below 2^11, so the
    fp16 result equals the oracle exactly, for every split."""
    M, N, K, gs = 5, 96, 256, 64
    codes = synth.uniform_int((N, K), 0, 15, 9, synth.TID_W, np.uint8)
    A = synth.uniform_int((M, K), -1, 0, 9, synth.TID_A, np.int8).astype(np.float16)  # -1..0
    ones = np.ones((N, K // gs), dtype=np.float16)
    ref = oracle.w4a16(A, oracle.pack_int4(codes), ones, None, K, gs)
    assert np.abs(ref).max() < 2048
    for split in (1, 2, 4):
        C = qg.qgemm_w4a16(to_dev(A), qg.quant_pack_int4(to_dev(codes)), to_dev(ones), None,
                           group_size=gs, split_k=split)
        assert np.array_equal(C.cpu().numpy().astype(np.float64), ref), split


def test_w4a16_fractional_zero_point():
    case = W4Case(2, 128, 512, 128, 1, seed=3, zero_value=7.25)
    assert_fp16_close(case.run(split_k=1), case.ref_full(), "z=7.25")


def test_w4a16_guard_bands_and_repeatability():
    case = W4Case(3, 130, 1024, 128, 1, seed=11)
    buf, C, pad = guarded((3, 130), torch.float16)
    case.run(split_k=4, C=C)
    torch.cuda.synchronize()
    assert guards_intact(buf, pad, 3 * 130)
    assert_fp16_close(C, case.ref_full(), "guarded")
    a = case.run(split_k=1).clone()
    b = case.run(split_k=1).clone()
    assert torch.equal(a, b)          # no atomics: bit-identical reruns


def test_w4a16_non_default_stream():
    case = W4Case(1, 1024, 4096, 128, 1, seed=13)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        C = case.run(split_k=4)
    s.synchronize()
    assert_fp16_close(C, case.ref_full(), "side stream")


@pytest.mark.parametrize("M,K,N", [(1, 4096, 11008), (1, 11008, 4096), (1, 4096, 4096),
                                   (1, 4096, 32000)])
@pytest.mark.parametrize("hz", [0, 1])
def test_w4a16_llama_shapes_m1_full(M, K, N, hz):
    case = W4Case(M, N, K, 128, hz, seed=K + N)
    for split in (1, 2, 4, 8):
        assert_fp16_close(case.run(split_k=split), case.ref_full(), f"split={split}")


@pytest.mark.parametrize("M,K,N", [(128, 4096, 11008), (128, 11008, 4096), (128, 4096, 4096),
                                   (128, 4096, 32000)])
def test_w4a16_llama_shapes_m128_sampled(M, K, N):
    case = W4Case(M, N, K, 128, 1, seed=K + N + 1)
    C = case.run().float().cpu().numpy()
    ms, ns = sample_pairs(M, N, 300, seed=N)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), "sampled")


def test_w4a16_errors_raise():
    case = W4Case(1, 64, 256, 128, 1)
    with pytest.raises(qg.QGemmError):
        qg.qgemm_w4a16(case.A, case.Wq, case.S, case.Z, group_size=96)
    with pytest.raises(TypeError):
        qg.qgemm_w4a16(case.A.float(), case.Wq, case.S, case.Z)


def test_w4a16_tune_pins_a_working_config():
    case = W4Case(1, 2048, 4096, 128, 1, seed=17)
    C = torch.empty((1, 2048), dtype=torch.float16, device=DEV)
    best = qg.qgemm_tune(qg.OP_W4A16, case.A, case.Wq, case.S, case.Z, C, 1, 2048, 4096, 128, 1,
                         reps=5)
    try:
        assert qg.qgemm_plan(qg.OP_W4A16, 1, 2048, 4096, 128, 1) == best
        assert_fp16_close(case.run(), case.ref_full(), f"tuned {best}")
    finally:
        qg.qgemm_set_config(qg.OP_W4A16, 1, 2048, 4096, 128, 1, None)
    qg.qgemm_sync_check()


@pytest.mark.parametrize("stages", [2, 6])
@pytest.mark.parametrize("split_k", [1, 3, 8])
def test_w4a16_tma_kernel_long_k(stages, split_k):
    """K = 16384 through the TMA-fed kernel: many ring wrap-arounds per warp."""
    M, N, K = 5, 192, 16384
    case = W4Case(M, N, K, 128, 1, seed=stages + split_k)
    cfg = {"path": qg.PATH_GEMV, "rows": 64, "bm": 0, "bn": 0, "bk": 0, "stages": stages,
           "split_k": split_k, "swap_ab": 0}
    qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, cfg)
    try:
        assert_fp16_close(case.run(), case.ref_full(), f"stages={stages} split={split_k}")
    finally:
        qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, None)


# ---- deterministic split-K through an fp32 workspace ------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (5, 200, 1024), (16, 130, 2048), (9, 64, 4096)])
@pytest.mark.parametrize("split_k", [1, 2, 3, 8])
def test_w4a16_splitk_f32_parity_and_determinism(M, N, K, split_k):
    case = W4Case(M, N, K, 128, 1, seed=M + split_k)
    need = qg.qgemm_w4a16_workspace_bytes(M, N, K, 128, split_k)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=DEV)      # contents must not matter
    a = qg.qgemm_w4a16_splitk_f32(case.A, case.Wq, case.S, case.Z, group_size=128,
                                  split_k=split_k, workspace=ws).clone()
    b = qg.qgemm_w4a16_splitk_f32(case.A, case.Wq, case.S, case.Z, group_size=128,
                                  split_k=split_k, workspace=ws).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)                     # part order is fixed: bit-identical reruns
    assert_fp16_close(a, case.ref_full(), f"splitk_f32 split={split_k}")


def test_w4a16_splitk_f32_no_zero_point_and_per_channel():
    case = W4Case(3, 256, 2048, -1, 0, seed=5)
    C = qg.qgemm_w4a16_splitk_f32(case.A, case.Wq, case.S, None, group_size=-1, split_k=4)
    assert_fp16_close(C, case.ref_full(), "per-channel, no zero")


def test_w4a16_splitk_f32_rejects_bad_workspace():
    case = W4Case(2, 128, 1024, 128, 1)
    need = qg.qgemm_w4a16_workspace_bytes(2, 128, 1024, 128, 4)
    small = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(qg.QGemmError):
        qg.qgemm_w4a16_splitk_f32(case.A, case.Wq, case.S, case.Z, split_k=4, workspace=small)
    big = torch.empty(need + 512, dtype=torch.uint8, device=DEV)
    with pytest.raises(qg.QGemmError):                   # 16-byte offset breaks 256-byte alignment
        qg.qgemm_w4a16_splitk_f32(case.A, case.Wq, case.S, case.Z, split_k=4, workspace=big[16:])
    with pytest.raises(qg.QGemmError):                   # group size 64: not this kernel's
        c64 = W4Case(2, 128, 1024, 64, 1)
        qg.qgemm_w4a16_splitk_f32(c64.A, c64.Wq, c64.S, c64.Z, group_size=64, split_k=2)
