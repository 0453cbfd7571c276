"""The interleaved (pre-shuffled) int4 weight layout: packing bit-exact against the oracle, and
qgemm_w4a16_interleaved on every kernel path against the oracle (and bit-identical to the
natural layout on the tensor-core path, where the upcast tile is the same)."""
import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import DEV, W4Case, assert_fp16_close, to_dev

pytestmark = pytest.mark.gpu


def test_pack_int4_interleaved_bit_exact():
    for N, K in [(1, 32), (9, 96), (300, 4096)]:
        codes = synth.uniform_int((N, K), 0, 15, N + K, synth.TID_W, np.uint8)
        got = qg.quant_pack_int4_interleaved(to_dev(codes)).cpu().numpy().view(np.uint32)
        assert np.array_equal(got, oracle.pack_int4_interleaved(codes)), (N, K)


def _cfg(path, rows=0, bn=0, stages=0, split=1, swap=None):
    if swap is None:
        swap = 1 if path == qg.PATH_TC else 0
    return {"path": path, "rows": rows, "bm": 128 if path == qg.PATH_TC else 0, "bn": bn,
            "bk": 0, "stages": stages, "split_k": split, "swap_ab": swap}


CONFIGS = [
    _cfg(qg.PATH_GEMV, rows=32, stages=0, split=1),      # register-prefetch streaming kernel
    _cfg(qg.PATH_GEMV, rows=32, stages=0, split=3),
    _cfg(qg.PATH_GEMV, rows=64, stages=4, split=1),      # TMA-fed streaming kernel
    _cfg(qg.PATH_GEMV, rows=16, stages=2, split=4),
    _cfg(qg.PATH_TC, bn=64, stages=3, split=1),           # tensor-core kernel
    _cfg(qg.PATH_TC, bn=256, stages=4, split=2),
    _cfg(qg.PATH_TC, bn=256, stages=4, split=1, swap=0),  # token-major tile
    _cfg(qg.PATH_TC, bn=256, stages=2, split=3, swap=0),
]


@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: f"p{c['path']}r{c['rows']}b{c['bn']}s{c['stages']}k{c['split_k']}w{c['swap_ab']}")
@pytest.mark.parametrize("M,N,K,gs,hz", [(1, 200, 1024, 128, 1), (7, 136, 2048, 128, 0),
                                         (40, 256, 512, 128, 1), (3, 96, 512, 64, 1)])
def test_w4a16_interleaved_paths(cfg, M, N, K, gs, hz):
    if cfg["stages"] and cfg["path"] == qg.PATH_GEMV and gs % 128:
        pytest.skip("the TMA-fed streaming kernel needs group_size % 128 == 0")
    case = W4Case(M, N, K, gs, hz, seed=M + N + K)
    Wi = qg.quant_pack_int4_interleaved(case.codes)
    qg.qgemm_set_config(qg.OP_W4A16_INTERLEAVED, M, N, K, gs, hz, cfg)
    try:
        C = qg.qgemm_w4a16_interleaved(case.A, Wi, case.S, case.Z, group_size=gs)
        assert_fp16_close(C, case.ref_full(), f"interleaved {cfg}")
        if cfg["path"] == qg.PATH_TC and cfg["split_k"] == 1:
            qg.qgemm_set_config(qg.OP_W4A16, M, N, K, gs, hz, cfg)
            try:
                Cn = case.run()
            finally:
                qg.qgemm_set_config(qg.OP_W4A16, M, N, K, gs, hz, None)
            assert torch.equal(C, Cn)
    finally:
        qg.qgemm_set_config(qg.OP_W4A16_INTERLEAVED, M, N, K, gs, hz, None)


def test_w4a16_interleaved_full_size_sampled():
    from gpu_cases import sample_pairs
    for M in (1, 16384):
        N = K = 16384
        case = W4Case(M, N, K, 128, 1, seed=M + 3)
        C = qg.qgemm_w4a16_interleaved(case.A, qg.quant_pack_int4_interleaved(case.codes),
                                       case.S, case.Z).float().cpu().numpy()
        ms, ns = sample_pairs(M, N, 200, seed=M)
        assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), f"M={M}")
