"""Race detection by repetition: results that do not depend on the order of atomic additions
must come out bit for bit the same on every run. Integer paths are exact in any order (split-K
included); W4A16 tensor-core tiles without a K split write each output once. A race in a ring
hand-over (a buffer reused before its reader finished) shows up as run-to-run differences."""
import numpy as np
import pytest
import torch

import gemv_w4a16_w8a8_b200 as qg
from gpu_cases import IntCase, W4Case, assert_fp16_close

pytestmark = pytest.mark.gpu

RUNS = 3


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("M,split_k", [(1, 0), (1, 4), (64, 0), (300, 0), (300, 3)])
def test_int_paths_repeat_exactly(op, M, split_k):
    N, K = 4104, 4096
    case = IntCase(op, M, N, K, seed=M + split_k)
    first = case.run(split_k=split_k).cpu().numpy()
    assert np.array_equal(first, case.ref_full())
    for _ in range(RUNS - 1):
        assert np.array_equal(case.run(split_k=split_k).cpu().numpy(), first)


@pytest.mark.parametrize("M,swap,bn,stages", [(200, 1, 256, 3), (300, 1, 128, 8),
                                              (100, 0, 256, 4), (128, 0, 256, 2)])
def test_w4a16_tensor_core_tiles_repeat_exactly(M, swap, bn, stages):
    N, K = 1000, 2048
    case = W4Case(M, N, K, 128, 1, seed=M + bn)
    cfg = {"path": qg.PATH_TC, "rows": 0, "bm": 128, "bn": bn, "bk": 0, "stages": stages,
           "split_k": 1, "swap_ab": swap}
    qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, cfg)
    try:
        first = case.run()
        assert_fp16_close(first, case.ref_full(), f"M={M} swap={swap} bn={bn}")
        for _ in range(RUNS - 1):
            assert torch.equal(case.run(), first)
    finally:
        qg.qgemm_set_config(qg.OP_W4A16, M, N, K, 128, 1, None)
