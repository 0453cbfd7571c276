"""qgemm_w4a16_splitk_f32_noalloc (the entry point for callers that cannot allocate device memory)
called straight through the C ABI, checked against qgemm_w4a16_splitk_f32 with a caller-owned
workspace: within the fp16 rule the other tests use, and bit-identical since both run the same
kernel and configuration. Consecutive calls of different shapes share the library's one scratch
buffer, so a stale counter left by one call would corrupt the next.

The file name sorts last so that pytest collects it after every other test; it also passes alone
in a fresh process (the first call on a device does the buffer's one-time address look-up)."""
import ctypes

import pytest
import torch

import gemv_w4a16_w8a8_b200 as qg
from gpu_cases import W4Case, assert_fp16_close

pytestmark = pytest.mark.gpu


def _noalloc(case, split_k, C=None):
    if C is None:
        C = torch.full((case.M, case.N), float("nan"), dtype=torch.float16, device=case.A.device)
    stream = torch.cuda.current_stream()
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = qg.lib().qgemm_w4a16_splitk_f32_noalloc(
        vp(case.A), vp(case.Wq), vp(case.S), vp(case.Z), vp(C), case.M, case.N, case.K, case.gs,
        split_k, int(case.Z is not None), ctypes.c_void_p(stream.cuda_stream))
    return st, C


def _with_workspace(case, split_k):
    return qg.qgemm_w4a16_splitk_f32(case.A, case.Wq, case.S, case.Z, group_size=case.gs,
                                     split_k=split_k)


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    first = W4Case(3, 160, 2048, 128, 1, seed=71)
    second = W4Case(16, 4096, 4096, 128, 0, seed=72)
    calls = [(first, 4), (second, 8), (first, 4)]
    outs = []
    for case, split_k in calls:
        st, C = _noalloc(case, split_k)
        assert st == qg.QG_OK, qg.lib().qgemm_status_string(st).decode()
        outs.append(C)
    torch.cuda.synchronize()
    qg.qgemm_sync_check()                 # raises if a kernel flagged an error
    for (case, split_k), got in zip(calls, outs):
        want = _with_workspace(case, split_k)
        torch.cuda.synchronize()
        assert_fp16_close(got, want.float().cpu().numpy(),
                          f"noalloc M={case.M} N={case.N} K={case.K} split={split_k}")
        assert torch.equal(got, want)
    assert torch.equal(outs[0], outs[2])


def test_noalloc_rejects_problems_beyond_the_scratch_buffer():
    M, N, K, split_k = 16, 65536, 256, 4
    need = qg.qgemm_w4a16_workspace_bytes(M, N, K, 128, split_k)
    assert need > qg.QGEMM_NOALLOC_SCRATCH_BYTES
    case = W4Case(M, N, K, 128, 1, seed=73)
    sentinel = torch.full((M, N), 3.0, dtype=torch.float16, device=case.A.device)
    st, C = _noalloc(case, split_k, C=sentinel)
    assert st == qg.QG_ERR_SCRATCH_TOO_SMALL
    torch.cuda.synchronize()
    assert bool((C == 3.0).all())   # nothing was queued
    # the same problem at a split that fits runs
    assert qg.qgemm_w4a16_workspace_bytes(M, N, K, 128, 1) <= qg.QGEMM_NOALLOC_SCRATCH_BYTES
    st, C = _noalloc(case, 1)
    assert st == qg.QG_OK
    torch.cuda.synchronize()
    assert torch.equal(C, _with_workspace(case, 1))
