"""Round-to-nearest int4 quantisation on the GPU against the oracle: codes, scales and zeros
bit-exact (both sides take every code decision in binary32), for every supported group size,
ragged and special groups (all zero, constant, one-signed, exact ties), and end to end: the
quantised operands fed to qgemm_w4a16 match the oracle's matmul of the oracle's quantisation."""
import os

import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import DEV, assert_fp16_close, to_dev

pytestmark = pytest.mark.gpu


def _weights(N, K, seed):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K)) * np.exp2(rng.integers(-8, 6, (N, 1)))
    W[0::7] = np.abs(W[0::7])                 # rows of one sign
    W[1::7] = -np.abs(W[1::7])
    W[2::11] = 0.0                            # all-zero rows
    W[3::13] = 0.37                           # constant rows
    return W.astype(np.float16)


def _compare(W, gs):
    Wq, S, Z = qg.quant_rtn_int4(to_dev(W), group_size=gs)
    torch.cuda.synchronize()
    codes, S_ref, Z_ref = oracle.rtn_int4(W, gs)
    K = W.shape[1]
    got_codes = oracle.unpack_int4(Wq.cpu().numpy().view(np.uint32), K)
    assert np.array_equal(S.cpu().numpy().view(np.uint16), S_ref.view(np.uint16)), "scales"
    assert np.array_equal(Z.cpu().numpy().view(np.uint16), Z_ref.view(np.uint16)), "zeros"
    bad = np.flatnonzero(got_codes != codes)
    assert bad.size == 0, f"{bad.size} codes differ, first at {bad[:3]}"
    return Wq, S, Z, codes, S_ref, Z_ref


@pytest.mark.parametrize("gs", [32, 64, 128, 256, 512, -1])
@pytest.mark.parametrize("N,K", [(37, 512), (300, 2048), (9, 4128)])
def test_rtn_bit_exact(N, K, gs):
    if K % (K if gs <= 0 else gs) or (K == 4128 and gs not in (32,)):
        pytest.skip("group size does not divide K, or K is not a multiple of 256 for wide groups")
    _compare(_weights(N, K, N + K + gs), gs)


def test_rtn_golden_rows():
    path = os.path.join(os.path.dirname(__file__), "golden", "rtn_int4.txt")
    rows, gs = [], 32
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line.startswith("w "):
                rows.append([float(v) for v in line.split()[1:]])
    W = np.array(rows, dtype=np.float16)   # two rows of K = 64: ties, one-signed, constant groups
    _compare(W, gs)


def test_rtn_wide_group_and_big_matrix():
    _compare(_weights(64, 11008, 9), -1)          # one group of 11008 = 43 chunks of 256
    _compare(_weights(4096, 4096, 10), 128)


def test_rtn_then_matmul_end_to_end():
    M, N, K, gs = 5, 256, 2048, 128
    W = _weights(N, K, 11)
    Wq, S, Z, codes, S_ref, Z_ref = _compare(W, gs)
    A = synth.normal_f16((M, K), 12, synth.TID_A, synth.TID_A_NORMAL_2)
    C = qg.qgemm_w4a16(to_dev(A), Wq, S, Z, group_size=gs)
    torch.cuda.synchronize()
    ref = oracle.w4a16(A, oracle.pack_int4(codes), S_ref, Z_ref, K, gs)
    assert_fp16_close(C, ref, "rtn -> w4a16")


def test_rtn_rejects_bad_arguments():
    W = to_dev(_weights(16, 512, 13))
    with pytest.raises(ValueError):
        qg.quant_rtn_int4(W, group_size=96)       # does not divide K
    Wq = torch.empty((16, 64), dtype=torch.int32, device=DEV)
    S = torch.empty((16, 4), dtype=torch.float16, device=DEV)
    L = qg.lib()
    ptr = lambda t: t.data_ptr()
    # has_zero = 0 (no zero point) and a group size of 160 are refused before any launch
    assert L.quant_rtn_int4(ptr(W), ptr(Wq), ptr(S), ptr(S), 16, 512, 128, 0, None) == qg.QG_ERR_INVALID_ARG
    assert L.quant_rtn_int4(ptr(W), ptr(Wq), ptr(S), ptr(S), 16, 640, 160, 1, None) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE
