"""qgemm_w4a16_host: activations and results in page-locked host memory, streamed through a
device workspace in chunks of tokens. Each chunk is an ordinary W4A16 call, so the result meets
the same fp16 rule against the oracle; these tests pin the chunking (ragged last chunk, one
chunk, one token), the stream order and the workspace reuse."""
import numpy as np
import pytest
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth
from gpu_cases import DEV, assert_fp16_close, to_dev

pytestmark = pytest.mark.gpu


def host_case(M, N, K, gs, hz, seed):
    d = synth.w4a16_inputs(M, N, K, gs, hz, seed)
    A_host = torch.from_numpy(d["A"]).pin_memory()
    C_host = torch.full((M, N), float("nan"), dtype=torch.float16).pin_memory()
    Wq = qg.quant_pack_int4(to_dev(d["codes"]))
    S = to_dev(d["scales"])
    Z = to_dev(d["zeros"]) if hz else None
    ref = oracle.w4a16(d["A"], oracle.pack_int4(d["codes"]), d["scales"], d["zeros"] if hz else None,
                       K, gs)
    return A_host, C_host, Wq, S, Z, ref


@pytest.mark.parametrize("M,N,K,gs,hz,chunk", [(700, 384, 1024, 128, 1, 256),   # 256 + 256 + 188
                                               (700, 384, 1024, 128, 0, 0),     # one chunk
                                               (1, 4096, 4096, 128, 1, 0),
                                               (513, 136, 512, 64, 1, 256),
                                               (1024, 520, 2048, 128, 1, 256),
                                               # 256 + 1024 + 1024 + 440 + 256 (ramped ends)
                                               (3000, 264, 512, 128, 1, 1024)])
def test_host_form_matches_oracle(M, N, K, gs, hz, chunk):
    A_host, C_host, Wq, S, Z, ref = host_case(M, N, K, gs, bool(hz), seed=M + N)
    ws = torch.empty(qg.qgemm_w4a16_host_workspace_bytes(M, N, K, chunk), dtype=torch.uint8,
                     device=DEV)
    s = torch.cuda.Stream()
    qg.qgemm_w4a16_host(A_host, Wq, S, Z, C_host, ws, group_size=gs, stream=s)
    s.synchronize()                       # the call is ordered on its stream, nothing else
    assert not torch.isnan(C_host).any()
    assert_fp16_close(C_host, ref, f"host form M={M} N={N} K={K} chunk={chunk}")
    qg.qgemm_sync_check()


def test_host_form_two_calls_share_a_workspace():
    M, N, K = 600, 256, 1024
    a1 = host_case(M, N, K, 128, True, seed=1)
    a2 = host_case(M, N, K, 128, True, seed=2)
    ws = torch.empty(qg.qgemm_w4a16_host_workspace_bytes(M, N, K, 256), dtype=torch.uint8,
                     device=DEV)
    for A_host, C_host, Wq, S, Z, _ in (a1, a2):
        qg.qgemm_w4a16_host(A_host, Wq, S, Z, C_host, ws, group_size=128)
    torch.cuda.current_stream().synchronize()
    for _, C_host, _, _, _, ref in (a1, a2):
        assert_fp16_close(C_host, ref, "shared workspace")


def test_host_form_rejects_pageable_memory():
    M, N, K = 4, 64, 256
    A_host, C_host, Wq, S, Z, _ = host_case(M, N, K, 128, True, seed=3)
    ws = torch.empty(qg.qgemm_w4a16_host_workspace_bytes(M, N, K, 0), dtype=torch.uint8,
                     device=DEV)
    pageable = torch.zeros((M, K), dtype=torch.float16)
    st = qg.lib().qgemm_w4a16_host(pageable.data_ptr(), Wq.data_ptr(), S.data_ptr(), Z.data_ptr(),
                                   C_host.data_ptr(), M, N, K, 128, 0, 1, ws.data_ptr(), ws.numel(),
                                   None)
    assert st == qg.QG_ERR_INVALID_ARG
