"""The benchmark's shapes under the configuration the search picks (the launch configuration
bench.py times), checked on one sampled element of every 128 x 128 tile of C against the oracle.
The search is run here exactly as the benchmark runs it before its timed region."""
import numpy as np
import pytest
import torch

import gemv_w4a16_w8a8_b200 as qg
from gpu_cases import IntCase, W4Case, assert_fp16_close, sample_pairs

pytestmark = pytest.mark.gpu

N = K = 16384


@pytest.mark.parametrize("M", [1, 32, 128, 512, 16384])
@pytest.mark.parametrize("hz", [1, 0])
def test_w4a16_tuned_configuration_full_size(M, hz):
    if M == 16384 and hz == 0:
        pytest.skip("one M = 16384 case is enough for the tile check (the search is long)")
    case = W4Case(M, N, K, 128, hz, seed=M + 31 * hz)
    key = (qg.OP_W4A16, M, N, K, 128, hz)
    try:
        cfg = qg.qgemm_tune(qg.OP_W4A16, case.A, case.Wq, case.S, case.Z,
                            torch.empty((M, N), dtype=torch.float16, device=case.A.device),
                            M, N, K, 128, hz, reps=3)
        C = case.run().float().cpu().numpy()
        qg.qgemm_sync_check()
    finally:
        qg.qgemm_set_config(*key, None)
    ms, ns = sample_pairs(M, N, 200, seed=M)
    assert_fp16_close(torch.from_numpy(C[ms, ns]), case.ref_at(ms, ns), f"tuned {cfg}")


@pytest.mark.parametrize("op", ["w8a8", "w2a8"])
@pytest.mark.parametrize("M", [1, 32, 128, 512])
def test_int_tuned_configuration_full_size(op, M):
    case = IntCase(op, M, N, K, seed=M + 5)
    code = qg.OP_W8A8 if op == "w8a8" else qg.OP_W2A8
    try:
        qg.qgemm_tune(code, case.A, case.W, None, None,
                      torch.empty((M, N), dtype=torch.int32, device=case.A.device),
                      M, N, K, -1, 0, reps=3)
        got = case.run().cpu().numpy()
        qg.qgemm_sync_check()
    finally:
        qg.qgemm_set_config(code, M, N, K, -1, 0, None)
    ms, ns = sample_pairs(M, N, 200, seed=M)
    assert np.array_equal(got[ms, ns], case.ref_at(ms, ns))
