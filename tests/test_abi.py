"""The C ABI without a GPU: the library loads, exports exactly what include/qgemm.h declares,
validates arguments before touching a device, and plans / pins configurations on the host."""
import ctypes
import os
import re

import pytest

import gemv_w4a16_w8a8_b200 as qg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgemm.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M))


def test_header_and_binding_agree():
    names = declared_functions()
    assert names == set(qg.EXPORTS), names ^ set(qg.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = qg.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert qg.qgemm_version() >= 100


def test_status_strings():
    for code in range(8):
        assert qg.status_string(code) not in ("", "unknown status")
    assert qg.status_string(99) == "unknown status"


# fake, suitably aligned device addresses: every call below must fail validation (or the
# device probe) before it could dereference them
A, W, S, Z, C = (ctypes.c_void_p(0x10000 * i) for i in range(1, 6))


def w4(M=1, N=64, K=256, gs=128, split=0, hz=1, a=A, w=W, s=S, z=Z, c=C):
    return qg.lib().qgemm_w4a16(a, w, s, z if hz else None, c, M, N, K, gs, split, hz, None)


@pytest.mark.parametrize("kw,status", [
    (dict(M=0), qg.QG_ERR_INVALID_ARG),
    (dict(N=-1), qg.QG_ERR_INVALID_ARG),
    (dict(K=0), qg.QG_ERR_INVALID_ARG),
    (dict(K=100, gs=-1), qg.QG_ERR_UNSUPPORTED_SHAPE),      # K % 32
    (dict(K=256, gs=48), qg.QG_ERR_UNSUPPORTED_SHAPE),      # gs % 32
    (dict(K=320, gs=128), qg.QG_ERR_UNSUPPORTED_SHAPE),     # K % gs
    (dict(gs=-5), qg.QG_ERR_INVALID_ARG),
    (dict(split=65), qg.QG_ERR_INVALID_ARG),
    (dict(hz=2), qg.QG_ERR_INVALID_ARG),
    (dict(a=None), qg.QG_ERR_INVALID_ARG),
    (dict(s=None), qg.QG_ERR_INVALID_ARG),
    (dict(a=ctypes.c_void_p(0x10008)), qg.QG_ERR_ALIGNMENT),
    (dict(c=ctypes.c_void_p(0x10004)), qg.QG_ERR_ALIGNMENT),
    (dict(s=ctypes.c_void_p(0x10001)), qg.QG_ERR_ALIGNMENT),
])
def test_w4a16_validation(kw, status):
    assert w4(**kw) == status


def test_zero_pointer_must_match_flag():
    L = qg.lib()
    assert L.qgemm_w4a16(A, W, S, None, C, 1, 64, 256, 128, 0, 1, None) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_w4a16(A, W, S, Z, C, 1, 64, 256, 128, 0, 0, None) == qg.QG_ERR_INVALID_ARG


def test_int_paths_validation():
    L = qg.lib()
    assert L.qgemm_w8a8(A, W, C, 1, 64, 100, -1, 0, 0, None) == qg.QG_ERR_UNSUPPORTED_SHAPE
    assert L.qgemm_w8a8(A, W, C, 1, 64, 128, 128, 0, 0, None) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_w8a8(A, W, C, 1, 64, 128, -1, 0, 1, None) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_w2a8(A, W, C, 1, 64, 96, -1, 0, 0, None) == qg.QG_ERR_UNSUPPORTED_SHAPE
    assert L.qgemm_dense_f16(A, W, C, 1, 64, 12, 0, None) == qg.QG_ERR_UNSUPPORTED_SHAPE
    assert L.quant_pack_int4(A, W, 0, 4, 48, -1, 1, 0, None) == qg.QG_ERR_UNSUPPORTED_SHAPE
    assert L.quant_pack_int2(A, W, 0, 4, 32, -1, 1, 0, None) == qg.QG_ERR_UNSUPPORTED_SHAPE
    assert L.quant_pack_int4(None, W, 0, 4, 64, -1, 1, 0, None) == qg.QG_ERR_INVALID_ARG


def test_valid_call_without_gpu_fails_loudly():
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("a GPU is present")
    except ImportError:
        pass
    # arguments are valid, so the call reaches the device probe, which must refuse
    assert w4() in (qg.QG_ERR_CUDA, qg.QG_ERR_NOT_SM100)
    assert qg.lib().qgemm_sync_check(None) in (qg.QG_ERR_CUDA, qg.QG_ERR_NOT_SM100)


# ---- planning and pinned configurations (host only) ----------------------------------------------

def test_plan_small_m_uses_streaming_kernels():
    c = qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 4096, 128, 1)
    assert c["path"] == qg.PATH_GEMV and c["rows"] in (16, 32, 64)
    c = qg.qgemm_plan(qg.OP_W4A16, 12, 4096, 4096, 128, 1)
    assert c["path"] == qg.PATH_STREAM and c["rows"] == 16 and c["bk"] in (256, 512, 1024)
    # K not a multiple of 256 leaves the persistent kernel for the split-K streaming kernels
    c = qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 4224, 128, 1)
    assert c["path"] == qg.PATH_GEMV and c["split_k"] >= 1 and c["rows"] in (16, 32, 64)
    c = qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 4096, 128, 1, split_k=2)
    assert c["path"] == qg.PATH_GEMV and c["split_k"] == 2
    c = qg.qgemm_plan(qg.OP_W8A8, 1, 16384, 16384)
    assert c["path"] == qg.PATH_GEMV and c["rows"] in (1, 2, 4, 8)
    c = qg.qgemm_plan(qg.OP_W2A8, 1, 16384, 16384)
    assert c["path"] == qg.PATH_GEMV


def test_plan_split_override():
    assert qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 4096, 128, 1, split_k=4)["split_k"] == 4
    with pytest.raises(qg.QGemmError):
        qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 4096, 100, 1)


def test_stream_config_rules():
    ok = {"path": qg.PATH_STREAM, "rows": 16, "bm": 4, "bn": 2, "bk": 512, "stages": 10,
          "split_k": 1, "swap_ab": 0}
    qg.qgemm_set_config(qg.OP_W4A16, 1, 4096, 4096, 128, 1, ok)
    try:
        assert qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 4096, 128, 1) == ok
    finally:
        qg.qgemm_set_config(qg.OP_W4A16, 1, 4096, 4096, 128, 1, None)
    bad = [dict(ok, rows=32), dict(ok, bk=2048), dict(ok, stages=16),   # 304 KB of ring
           dict(ok, bn=3), dict(ok, bn=8), dict(ok, bk=256, bn=4),    # 2 sub-blocks, 4 K warps
           dict(ok, bm=8), dict(ok, bm=0), dict(ok, stages=1), dict(ok, stages=17)]
    for cfg in bad:
        with pytest.raises(qg.QGemmError):
            qg.qgemm_set_config(qg.OP_W4A16, 1, 4096, 4096, 128, 1, cfg)
    # the activations' share of shared memory grows with M
    with pytest.raises(qg.QGemmError):
        qg.qgemm_set_config(qg.OP_W4A16, 16, 4096, 4096, 128, 1, ok)
    # the persistent kernel covers M <= 16 and K a multiple of 256 only
    with pytest.raises(qg.QGemmError):
        qg.qgemm_set_config(qg.OP_W4A16, 17, 4096, 4096, 128, 1, dict(ok, stages=4))
    with pytest.raises(qg.QGemmError):
        qg.qgemm_set_config(qg.OP_W4A16, 4, 4096, 4224, 128, 1, dict(ok, stages=4))
    # the default plan fits at every M the heuristic gives the path
    for M in range(9, 17):
        c = qg.qgemm_plan(qg.OP_W4A16, M, 16384, 16384, 128, 1)
        assert c["path"] == qg.PATH_STREAM, (M, c)


def test_set_save_load_roundtrip(tmp_path):
    qg.qgemm_clear_configs()
    cfg = {"path": qg.PATH_GEMV, "rows": 64, "bm": 0, "bn": 0, "bk": 0, "stages": 0,
           "split_k": 8, "swap_ab": 0}
    qg.qgemm_set_config(qg.OP_W4A16, 1, 4096, 11008, 128, 0, cfg)
    assert qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 11008, 128, 0) == cfg
    path = str(tmp_path / "cfg.txt")
    qg.qgemm_save_configs(path)
    qg.qgemm_clear_configs()
    assert qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 11008, 128, 0) != cfg
    qg.qgemm_load_configs(path)
    assert qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 11008, 128, 0) == cfg
    qg.qgemm_set_config(qg.OP_W4A16, 1, 4096, 11008, 128, 0, None)
    assert qg.qgemm_plan(qg.OP_W4A16, 1, 4096, 11008, 128, 0) != cfg
    qg.qgemm_clear_configs()


def test_set_config_rejects_configs_that_cannot_run():
    bad = {"path": qg.PATH_GEMV, "rows": 48, "bm": 0, "bn": 0, "bk": 0, "stages": 0,
           "split_k": 1, "swap_ab": 0}
    with pytest.raises(qg.QGemmError) as e:
        qg.qgemm_set_config(qg.OP_W4A16, 1, 256, 256, 128, 0, bad)
    assert e.value.status == qg.QG_ERR_BAD_CONFIG
    bad.update(rows=32, path=7)
    with pytest.raises(qg.QGemmError):
        qg.qgemm_set_config(qg.OP_W4A16, 1, 256, 256, 128, 0, bad)


def test_corrupt_cache_file_is_ignored(tmp_path):
    p = tmp_path / "bad.txt"
    p.write_text("# header\nnot a line\n0 1 2\n0 1 256 256 128 0 1 48 0 0 0 0 1 0\n")
    qg.qgemm_clear_configs()
    qg.qgemm_load_configs(str(p))     # parses, skips every entry
    assert qg.qgemm_plan(qg.OP_W4A16, 1, 256, 256, 128, 0)["rows"] != 48
    qg.qgemm_clear_configs()


# ---- tensor-core path planning (host only) ---------------------------------------------------------

def _tc(bn, stages, split=1):
    return {"path": qg.PATH_TC, "rows": 0, "bm": 128, "bn": bn, "bk": 0, "stages": stages,
            "split_k": split, "swap_ab": 1}


def test_plan_large_m_uses_tensor_cores():
    c = qg.qgemm_plan(qg.OP_W4A16, 16384, 16384, 16384, 128, 1)
    assert c["path"] == qg.PATH_TC and c["bn"] == 512 and c["stages"] == 4
    assert c["split_k"] == 1                     # 4096 tiles fill the GPU many times
    assert c["swap_ab"] == 1                     # weights in the MMA's M side
    c = qg.qgemm_plan(qg.OP_DENSE_F16, 16384, 16384, 16384)
    assert c["path"] == qg.PATH_TC and c["bn"] == 256 and 2 <= c["stages"] <= 5
    # up to one tile of tokens: the token-major tile (128 tokens x 256 weight rows), K split
    # until the units fill the GPU
    c = qg.qgemm_plan(qg.OP_W4A16, 32, 16384, 16384, 128, 1)
    assert c["path"] == qg.PATH_TC and c["swap_ab"] == 0 and (c["bm"], c["bn"]) == (128, 256)
    assert c["split_k"] >= 2 and 2 <= c["stages"] <= 4
    # group size 32 (not whole slabs) keeps the weight-major tile
    c = qg.qgemm_plan(qg.OP_W4A16, 32, 16384, 16384, 32, 1)
    assert c["path"] == qg.PATH_TC and c["swap_ab"] == 1 and c["bn"] == 32
    c = qg.qgemm_plan(qg.OP_DENSE_F16, 1, 256, 256)
    assert c["path"] == qg.PATH_TC and c["bn"] == 16
    for op in (qg.OP_W8A8, qg.OP_W2A8):
        assert qg.qgemm_plan(op, 512, 16384, 16384)["path"] == qg.PATH_TC


def test_tc_split_fills_the_gpu():
    c = qg.qgemm_plan(qg.OP_W4A16, 128, 4096, 4096, 128, 1)   # 32 tiles -> split
    assert c["path"] == qg.PATH_TC and c["split_k"] >= 4


def test_tc_config_limits():
    M, N = 256, 512
    # K = 1152 (18 slabs, single-slab packed copies) at a 256-token tile: 4 activation stages
    # (128 KB) + 12 packed slabs (48 KB) + 3 upcast buffers (48 KB) fit; a fifth stage does not
    K = 1152
    qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, _tc(256, 4))
    with pytest.raises(qg.QGemmError):
        qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, _tc(256, 5))
    # K = 1024 (four-slab copies): two grouped copies and two upcast buffers leave room for a
    # fifth activation stage; 8 stages are for token tiles up to 128, 16 up to 64
    K = 1024
    qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, _tc(256, 4))
    qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, _tc(256, 5))
    qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, _tc(128, 8))
    for bad in (_tc(256, 8), _tc(128, 16), _tc(48, 3), _tc(64, 1), _tc(64, 6), _tc(64, 3, 65)):
        with pytest.raises(qg.QGemmError):
            qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, bad)
    qg.qgemm_set_config(qg.OP_DENSE_F16, M, N, K, -1, 0, _tc(256, 4))
    with pytest.raises(qg.QGemmError):
        qg.qgemm_set_config(qg.OP_DENSE_F16, M, N, K, -1, 0, _tc(256, 5))
    qg.qgemm_clear_configs()


def test_workspace_bytes():
    # counters (one per 16-row x 8-token tile, 256-byte aligned) + split_k planes of M x N fp32
    assert qg.qgemm_w4a16_workspace_bytes(1, 4096, 4096, 128, 4) == 1024 + 4 * 4096 * 4
    assert qg.qgemm_w4a16_workspace_bytes(16, 100, 1024, 128, 3) == 256 + 3 * 16 * 100 * 4
    assert qg.qgemm_w4a16_workspace_bytes(1, 4096, 4096, 128, 0) == 0
    assert qg.qgemm_w4a16_workspace_bytes(1, 4096, 4000, 128, 2) == 0


def test_splitk_f32_validation_without_gpu():
    L = qg.lib()
    ws = ctypes.c_void_p(0x100000)
    need = qg.qgemm_w4a16_workspace_bytes(1, 64, 256, 128, 2)
    assert L.qgemm_w4a16_splitk_f32(A, W, S, Z, C, 1, 64, 256, 128, 0, 1, ws, need, None) == \
        qg.QG_ERR_INVALID_ARG                                         # split_k must be given
    assert L.qgemm_w4a16_splitk_f32(A, W, S, Z, C, 1, 64, 256, 64, 2, 1, ws, need, None) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE                                   # group size 64
    assert L.qgemm_w4a16_splitk_f32(A, W, S, Z, C, 1, 64, 256, 128, 2, 1, ws, need - 4, None) == \
        qg.QG_ERR_INVALID_ARG                                         # workspace too small
    assert L.qgemm_w4a16_splitk_f32(A, W, S, Z, C, 1, 64, 256, 128, 2, 1,
                                    ctypes.c_void_p(0x100010), need, None) == qg.QG_ERR_ALIGNMENT


def test_host_workspace_bytes():
    # two A chunks and two C chunks, each rounded up to 256 bytes
    assert qg.qgemm_w4a16_host_workspace_bytes(16384, 16384, 16384, 2048) == \
        2 * (2048 * 16384 * 2 + 2048 * 16384 * 2)
    assert qg.qgemm_w4a16_host_workspace_bytes(1, 100, 64, 0) == 2 * (256 + 256)
    # the default chunk is 1024 tokens (the copy-bound optimum measured on B200)
    assert qg.qgemm_w4a16_host_workspace_bytes(5000, 64, 64, 0) == \
        qg.qgemm_w4a16_host_workspace_bytes(5000, 64, 64, 1024)
    assert qg.qgemm_w4a16_host_workspace_bytes(0, 64, 64, 0) == 0


def test_host_form_validation_without_gpu():
    L = qg.lib()
    ws = ctypes.c_void_p(0x100000)
    need = qg.qgemm_w4a16_host_workspace_bytes(8, 64, 256, 0)
    assert L.qgemm_w4a16_host(None, W, S, Z, C, 8, 64, 256, 128, 0, 1, ws, need, None) == \
        qg.QG_ERR_INVALID_ARG
    assert L.qgemm_w4a16_host(A, W, S, Z, C, 8, 64, 256, 128, 0, 1, None, need, None) == \
        qg.QG_ERR_INVALID_ARG
    assert L.qgemm_w4a16_host(A, W, S, None, C, 8, 64, 256, 128, 0, 1, ws, need, None) == \
        qg.QG_ERR_INVALID_ARG                                         # zeros vs has_zero
    assert L.qgemm_w4a16_host(A, W, S, Z, C, 8, 64, 256, 128, 0, 1, ws, 100, None) == \
        qg.QG_ERR_INVALID_ARG                                         # no chunk fits
    assert L.qgemm_w4a16_host(A, W, S, Z, C, 8, 64, 256, 128, 0, 1, ctypes.c_void_p(0x100010),
                              need, None) == qg.QG_ERR_ALIGNMENT
    assert L.qgemm_w4a16_host(A, W, S, Z, C, 8, 64, 100, 128, 0, 1, ws, need, None) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE
    # a workspace for fewer than 256 tokens still gives a usable (smaller) chunk: the call gets
    # past validation to the device probe, which refuses without a GPU
    small = qg.qgemm_w4a16_host_workspace_bytes(1000, 64, 256, 100)
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except ImportError:
        has_gpu = False
    if not has_gpu:
        assert L.qgemm_w4a16_host(A, W, S, Z, C, 1000, 64, 256, 128, 0, 1, ws, small, None) in \
            (qg.QG_ERR_CUDA, qg.QG_ERR_NOT_SM100)


def test_selftest_limit_validated_before_the_device():
    L = qg.lib()
    assert L.qgemm_selftest_bounded_wait(0, None) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_selftest_bounded_wait(2000001, None) == qg.QG_ERR_INVALID_ARG


def test_half2_gemv_config_rules():
    """Path GEMV with bn = 2 (packed fp16 FMA pipe): 1..8 tokens, 32 or 64 rows, 2..6 stages,
    group sizes that are multiples of 128; the fp32-workspace split-K form ignores it."""
    ok = {"path": qg.PATH_GEMV, "rows": 64, "bm": 0, "bn": 2, "bk": 0, "stages": 4, "split_k": 2,
          "swap_ab": 0}
    for M in (1, 2, 3, 4, 8):
        qg.qgemm_set_config(qg.OP_W4A16, M, 4096, 4096, 128, 1, ok)
        assert qg.qgemm_plan(qg.OP_W4A16, M, 4096, 4096, 128, 1)["bn"] == 2
        qg.qgemm_set_config(qg.OP_W4A16, M, 4096, 4096, 128, 1, None)
    for bad in ({"rows": 16}, {"rows": 128}, {"stages": 1}, {"stages": 7}, {"split_k": 65}):
        with pytest.raises(qg.QGemmError):
            qg.qgemm_set_config(qg.OP_W4A16, 1, 4096, 4096, 128, 1, {**ok, **bad})
    for M, gs in ((9, 128), (1, 64), (1, 32)):
        with pytest.raises(qg.QGemmError):
            qg.qgemm_set_config(qg.OP_W4A16, M, 4096, 4096, gs, 1, ok)


def test_pair_tile_rules():
    """Tensor-core tiles shared by a CTA pair (bm = 256): 128 or 256 tokens, stages 3, 4, 5 or 8,
    weight-major only; the library refuses other shapes of the config up front."""
    ok = {"path": qg.PATH_TC, "rows": 0, "bm": 256, "bn": 256, "bk": 0, "stages": 4,
          "split_k": 1, "swap_ab": 1}
    for op, gs in ((qg.OP_W4A16, 128), (qg.OP_W8A8, -1), (qg.OP_W2A8, -1), (qg.OP_DENSE_F16, -1)):
        packed = op in (qg.OP_W4A16, qg.OP_W2A8)
        for bn, st in ((256, 3), (256, 4), (256, 5), (128, 8)) + (((256, 8),) if packed else ()):
            cfg = {**ok, "bn": bn, "stages": st}
            qg.qgemm_set_config(op, 512, 16384, 16384, gs, 0, cfg)
            assert qg.qgemm_plan(op, 512, 16384, 16384, gs, 0)["bm"] == 256
            qg.qgemm_set_config(op, 512, 16384, 16384, gs, 0, None)
    for bad in ({"bn": 64}, {"stages": 2}, {"stages": 16}, {"bm": 192}, {"swap_ab": 0}):
        with pytest.raises(qg.QGemmError):
            qg.qgemm_set_config(qg.OP_W4A16, 512, 16384, 16384, 128, 1, {**ok, **bad})
    # weights carried in the activation ring (fp16 / int8) leave no room for 8 stages of 256
    with pytest.raises(qg.QGemmError):
        qg.qgemm_set_config(qg.OP_DENSE_F16, 512, 16384, 16384, -1, 0, {**ok, "stages": 8})


def test_dual_tile_rules():
    """512-token weight-major tiles (two 256-token accumulators per upcast slab): packed weights
    only (W4A16, W2A8, either layout), one CTA, 2 or 4 half-tile activation stages."""
    ok = {"path": qg.PATH_TC, "rows": 0, "bm": 128, "bn": 512, "bk": 0, "stages": 4,
          "split_k": 1, "swap_ab": 1}
    for op, gs in ((qg.OP_W4A16, 128), (qg.OP_W2A8, -1), (qg.OP_W4A16_INTERLEAVED, 128),
                   (qg.OP_W2A8_INTERLEAVED, -1)):
        for st in (2, 4):
            for sk in (1, 3):
                cfg = {**ok, "stages": st, "split_k": sk}
                qg.qgemm_set_config(op, 4096, 16384, 16384, gs, 0, cfg)
                plan = qg.qgemm_plan(op, 4096, 16384, 16384, gs, 0)
                assert (plan["bn"], plan["stages"], plan["split_k"]) == (512, st, sk)
                qg.qgemm_set_config(op, 4096, 16384, 16384, gs, 0, None)
    for bad in ({"stages": 3}, {"stages": 5}, {"bm": 256}, {"swap_ab": 0}):
        with pytest.raises(qg.QGemmError):
            qg.qgemm_set_config(qg.OP_W4A16, 4096, 16384, 16384, 128, 1, {**ok, **bad})
    for op in (qg.OP_DENSE_F16, qg.OP_W8A8):
        with pytest.raises(qg.QGemmError):
            qg.qgemm_set_config(op, 4096, 16384, 16384, -1, 0, ok)


def test_dual_tile_default_plan():
    """The default plan takes the 512-token tile for int4 weights when its schedule of whole
    waves (a unit of 512 tokens costing 1.71 of 256) is the shorter one, else the 256-token tile."""
    qg.qgemm_clear_configs()
    for op in (qg.OP_W4A16, qg.OP_W4A16_INTERLEAVED):
        for M in (1024, 4096, 16384):
            c = qg.qgemm_plan(op, M, 16384, 16384, 128, 1)
            assert (c["path"], c["bn"], c["stages"], c["split_k"]) == (qg.PATH_TC, 512, 4, 1), (M, c)
    # 3 token tiles of 256 against 2 of 512 on 32 weight tiles: one wave either way
    c = qg.qgemm_plan(qg.OP_W4A16, 600, 4096, 4096, 128, 1)
    assert c["bn"] == 256, c
    # int2 and int8 weights keep the 256-token tile
    assert qg.qgemm_plan(qg.OP_W2A8, 16384, 16384, 16384, -1, 0)["bn"] == 256
    assert qg.qgemm_plan(qg.OP_W8A8, 16384, 16384, 16384, -1, 0)["bn"] == 256


def test_stream_k_schedule_rules():
    """rows = 1 on a tensor-core config selects the stream-K schedule: single-CTA tiles (either
    orientation, any token tile), split_k = 1; the CTA pair and other rows values are refused."""
    base = {"path": qg.PATH_TC, "rows": 1, "bm": 128, "bn": 256, "bk": 0, "stages": 3,
            "split_k": 1, "swap_ab": 1}
    cases = [(qg.OP_W4A16, 128, base), (qg.OP_W4A16, 128, {**base, "bn": 512, "stages": 4}),
             (qg.OP_W4A16, 128, {**base, "swap_ab": 0, "stages": 3}),
             (qg.OP_W2A8, -1, base), (qg.OP_W8A8, -1, base), (qg.OP_DENSE_F16, -1, {**base, "stages": 4})]
    for op, gs, cfg in cases:
        M = 128 if cfg["swap_ab"] == 0 else 512
        qg.qgemm_set_config(op, M, 16384, 16384, gs, 0, cfg)
        assert qg.qgemm_plan(op, M, 16384, 16384, gs, 0)["rows"] == 1
        qg.qgemm_set_config(op, M, 16384, 16384, gs, 0, None)
    for bad in ({"split_k": 2}, {"rows": 2}, {"bm": 256}):
        with pytest.raises(qg.QGemmError):
            qg.qgemm_set_config(qg.OP_W4A16, 512, 16384, 16384, 128, 1, {**base, **bad})
