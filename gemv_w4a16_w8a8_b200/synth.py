"""Seeded synthetic inputs for the low-bit matmul C[M,N] = A[M,K] . dequant(W[N,K])^T.

This module only draws random numbers and rounds them to their storage type. It holds none
of the method's arithmetic (no packing, no dequantisation, no products), so that the oracle
and the CUDA path can both be fed from it without sharing any of the computation.

Generator: counter-based splitmix64. Element i of stream (seed, tensor_id) is

    key    = mix(seed * 0x9E3779B97F4A7C15 + tensor_id)
    bits_i = mix(key + (i + 1) * 0x9E3779B97F4A7C15)

where mix is the splitmix64 finaliser (xor-shift 30/27/31 with the multipliers
0xBF58476D1CE4E5B9 and 0x94D049BB133111EB; Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014). Any element can be regenerated on its own,
which lets large tensors be made in parallel chunks.

Distributions follow the workloads of the BitBLAS "nt" Matmul benchmark (microsoft/BitBLAS
issue #252, benchmark configuration listing) and the hidet quantized-matmul LLaMA shapes
(hidet-org/hidet issue #364, k-parts=4 table):
  * fp16 activations ~ N(0, 1) (Box-Muller on two uniform streams), rounded to nearest fp16;
  * int4 weight codes uniform in {0..15};
  * scales uniform in [0.001, 0.01], rounded to fp16; zero points the constant 8.0 (fp16);
  * int8 values uniform in [-128, 127];
  * int2 values uniform in {-2, -1, 0, 1};
  * dense fp16 operands ~ N(0, 1) * 0.02.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

# tensor ids: one independent stream per tensor role
TID_A = 1
TID_W = 2
TID_SCALE = 3
TID_ZERO = 4
TID_A_NORMAL_2 = 5
TID_W_NORMAL_2 = 6


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.array([seed], dtype=np.uint64) * _GOLDEN + np.uint64(tensor_id)
        return _mix(s)[0]


def bits(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """uint64 words start..start+count-1 of stream (seed, tensor_id)."""
    key = _key(seed, tensor_id)
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        return _mix(key + idx * _GOLDEN)


def _workers() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _chunked(total: int, fill) -> None:
    """Run fill(start, count) over [0, total) in chunks on a thread pool (numpy drops the GIL)."""
    spans = [(s, min(_CHUNK, total - s)) for s in range(0, total, _CHUNK)]
    if len(spans) <= 1:
        for s, c in spans:
            fill(s, c)
        return
    with ThreadPoolExecutor(_workers()) as ex:
        list(ex.map(lambda sc: fill(*sc), spans))


def uniform01(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """Doubles in [0, 1) from the top 53 bits."""
    return (bits(seed, tensor_id, start, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal_f16(shape, seed: int, tid: int, tid2: int, sigma: float = 1.0) -> np.ndarray:
    """fp16 array ~ N(0, sigma^2): Box-Muller (cos branch) on streams tid and tid2, then RN to fp16."""
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.float16)

    def fill(s, c):
        u1 = 1.0 - uniform01(seed, tid, s, c)          # (0, 1]
        u2 = uniform01(seed, tid2, s, c)
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
        out[s:s + c] = (z * sigma).astype(np.float16)

    _chunked(total, fill)
    return out.reshape(shape)


def uniform_f16(shape, lo: float, hi: float, seed: int, tid: int) -> np.ndarray:
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.float16)

    def fill(s, c):
        out[s:s + c] = (lo + (hi - lo) * uniform01(seed, tid, s, c)).astype(np.float16)

    _chunked(total, fill)
    return out.reshape(shape)


def uniform_int(shape, lo: int, hi: int, seed: int, tid: int, dtype) -> np.ndarray:
    """Integers uniform in [lo, hi] (hi - lo + 1 a power of two) from the top bits."""
    span = hi - lo + 1
    nbits = span.bit_length() - 1
    assert 1 << nbits == span, "span must be a power of two"
    total = int(np.prod(shape))
    out = np.empty(total, dtype=dtype)

    def fill(s, c):
        top = bits(seed, tid, s, c) >> np.uint64(64 - nbits) if nbits else np.zeros(c, np.uint64)
        out[s:s + c] = (top.astype(np.int64) + lo).astype(dtype)

    _chunked(total, fill)
    return out.reshape(shape)


# ---------------------------------------------------------------------------------------------
# Workload recipes
# ---------------------------------------------------------------------------------------------

def groups_of(K: int, group_size: int) -> int:
    gs = K if group_size in (-1, 0) else group_size
    return K // gs


def w4a16_inputs(M: int, N: int, K: int, group_size: int = 128, has_zero: bool = True,
                 seed: int = 0, zero_value: float = 8.0) -> dict:
    """fp16 A ~ N(0,1) [M,K]; uint8 codes uniform 0..15 [N,K]; fp16 scales U[0.001,0.01]
    [N,G]; fp16 zeros = zero_value [N,G] when has_zero (else None)."""
    G = groups_of(K, group_size)
    A = normal_f16((M, K), seed, TID_A, TID_A_NORMAL_2)
    codes = uniform_int((N, K), 0, 15, seed, TID_W, np.uint8)
    scales = uniform_f16((N, G), 0.001, 0.01, seed, TID_SCALE)
    zeros = np.full((N, G), zero_value, dtype=np.float16) if has_zero else None
    return {"A": A, "codes": codes, "scales": scales, "zeros": zeros}


def w8a8_inputs(M: int, N: int, K: int, seed: int = 0) -> dict:
    """int8 A [M,K] and W [N,K], both uniform in [-128, 127]."""
    A = uniform_int((M, K), -128, 127, seed, TID_A, np.int8)
    W = uniform_int((N, K), -128, 127, seed, TID_W, np.int8)
    return {"A": A, "W": W}


def w2a8_inputs(M: int, N: int, K: int, seed: int = 0) -> dict:
    """int8 A [M,K] uniform in [-128,127]; int2 weight values [N,K] uniform in {-2,-1,0,1}
    (held one per int8)."""
    A = uniform_int((M, K), -128, 127, seed, TID_A, np.int8)
    Wv = uniform_int((N, K), -2, 1, seed, TID_W, np.int8)
    return {"A": A, "Wv": Wv}


def dense_inputs(M: int, N: int, K: int, seed: int = 0) -> dict:
    """fp16 A [M,K] and W [N,K], both ~ N(0,1) * 0.02."""
    A = normal_f16((M, K), seed, TID_A, TID_A_NORMAL_2, sigma=0.02)
    W = normal_f16((N, K), seed, TID_W, TID_W_NORMAL_2, sigma=0.02)
    return {"A": A, "W": W}
