"""Shared set-up for the GPU parity tests: seeded inputs on the host (synth), their device
copies, and the oracle's answer computed from the host copies only."""
import numpy as np
import torch

import oracle
import gemv_w4a16_w8a8_b200 as qg
from gemv_w4a16_w8a8_b200 import synth

DEV = "cuda:0"


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def sample_pairs(M, N, count, seed, K=None):
    """(m, n) positions: every tile corner and edge, one seeded random element inside every
    128 x 128 tile of C (so that a fault confined to some output tiles or persistent units is
    seen), plus `count` seeded random ones."""
    rng = np.random.default_rng(seed)
    ms = [0, M - 1, M // 2, min(M - 1, 15), min(M - 1, 16), min(M - 1, 127), min(M - 1, 128)]
    ns = [0, N - 1, N // 2, min(N - 1, 127), min(N - 1, 128), min(N - 1, 255), min(N - 1, 256)]
    pm = [m for m in ms for _ in ns]
    pn = [n for _ in ms for n in ns]
    mt, nt = -(-M // 128), -(-N // 128)
    ti = np.repeat(np.arange(mt, dtype=np.int64), nt)
    tj = np.tile(np.arange(nt, dtype=np.int64), mt)
    pm += list(ti * 128 + (rng.random(ti.size) * np.minimum(128, M - ti * 128)).astype(np.int64))
    pn += list(tj * 128 + (rng.random(tj.size) * np.minimum(128, N - tj * 128)).astype(np.int64))
    pm += list(rng.integers(0, M, count))
    pn += list(rng.integers(0, N, count))
    return np.array(pm, dtype=np.int64), np.array(pn, dtype=np.int64)


class W4Case:
    def __init__(self, M, N, K, gs, has_zero, seed=0, zero_value=8.0):
        self.M, self.N, self.K, self.gs, self.has_zero = M, N, K, gs, has_zero
        d = synth.w4a16_inputs(M, N, K, gs, has_zero, seed, zero_value)
        self.h = d
        self.Wq_host = oracle.pack_int4(d["codes"])          # oracle side packs on the host
        self.A = to_dev(d["A"])
        self.codes = to_dev(d["codes"])
        self.Wq = qg.quant_pack_int4(self.codes)              # CUDA side packs on the device
        self.S = to_dev(d["scales"])
        self.Z = to_dev(d["zeros"]) if has_zero else None

    def run(self, split_k=0, C=None):
        return qg.qgemm_w4a16(self.A, self.Wq, self.S, self.Z, C=C, group_size=self.gs,
                              split_k=split_k)

    def ref_full(self):
        d = self.h
        return oracle.w4a16(d["A"], self.Wq_host, d["scales"], d["zeros"], self.K, self.gs)

    def ref_at(self, ms, ns):
        d = self.h
        return oracle.w4a16_at(d["A"], self.Wq_host, d["scales"], d["zeros"], self.K, self.gs,
                               ms, ns)


class IntCase:
    def __init__(self, op, M, N, K, seed=0):
        self.op, self.M, self.N, self.K = op, M, N, K
        if op == "w8a8":
            d = synth.w8a8_inputs(M, N, K, seed)
            self.Wh = d["W"]
            self.W = to_dev(d["W"])
        else:
            d = synth.w2a8_inputs(M, N, K, seed)
            self.Wh = oracle.pack_int2(d["Wv"])
            self.W = qg.quant_pack_int2(to_dev(d["Wv"]))
        self.h = d
        self.A = to_dev(d["A"])

    def run(self, split_k=0, C=None):
        if self.op == "w8a8":
            return qg.qgemm_w8a8(self.A, self.W, C=C, split_k=split_k)
        return qg.qgemm_w2a8(self.A, self.W, C=C, split_k=split_k)

    def ref_full(self):
        f = oracle.w8a8 if self.op == "w8a8" else oracle.w2a8
        return f(self.h["A"], self.Wh)

    def ref_at(self, ms, ns):
        f = oracle.w8a8_at if self.op == "w8a8" else oracle.w2a8_at
        return f(self.h["A"], self.Wh, ms, ns)


def assert_fp16_close(got: torch.Tensor, ref: np.ndarray, what=""):
    ok, msg = oracle.fp16_close(got.float().cpu().numpy(), ref)
    assert ok, f"{what}: {msg}"


def guarded(shape, dtype, guard=4096, fill=0x5A):
    """A tensor view with guard bands on both sides, filled with a byte pattern."""
    n = int(np.prod(shape))
    esz = torch.empty((), dtype=dtype).element_size()
    pad = guard // esz
    buf = torch.empty(n + 2 * pad, dtype=dtype, device=DEV)
    buf.view(torch.uint8).fill_(fill)
    return buf, buf[pad:pad + n].view(shape), pad


def guards_intact(buf, pad, n, fill=0x5A):
    b = buf.view(torch.uint8)
    esz = buf.element_size()
    head = b[:pad * esz]
    tail = b[(pad + n) * esz:]
    return bool((head == fill).all()) and bool((tail == fill).all())
