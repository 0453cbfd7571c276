"""Python face of the host oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg are
the only callers. The CUDA library never imports this package and this package imports
nothing from the library. Every function takes and returns numpy arrays; fp16 tensors are
passed as their raw binary16 bits.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (-O2, OpenMP) into liboracle.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class Oracle:
    """ctypes binding of one compiled copy of oracle.c (the default build, or a test's mutant)."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        L.orc_half_to_double.restype = ctypes.c_double
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]
        for name in ("orc_pack_int4", "orc_unpack_int4", "orc_pack_int2", "orc_unpack_int2",
                     "orc_pack_int4_interleaved", "orc_unpack_int4_interleaved",
                     "orc_pack_int2_interleaved", "orc_unpack_int2_interleaved"):
            getattr(L, name).argtypes = [_ptr, _ptr, _i64, _i64]
            getattr(L, name).restype = ctypes.c_int
        L.orc_decode_half.argtypes = [_ptr, _ptr, _i64]
        L.orc_float_to_half.argtypes = [ctypes.c_float]
        L.orc_float_to_half.restype = ctypes.c_uint16
        L.orc_rtn_int4.argtypes = [_ptr, _i64, _i64, _i64, _ptr, _ptr, _ptr]
        L.orc_w8a8_requant.argtypes = [_ptr, _ptr, _ptr, _i64, _i64, _i64, _ptr, ctypes.c_int]
        L.orc_w4a16.argtypes = [_ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _i64, ctypes.c_int,
                                _ptr, ctypes.c_int]
        L.orc_w4a16_at.argtypes = [_ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _i64, ctypes.c_int,
                                   _ptr, _ptr, _i64, _ptr, ctypes.c_int]
        L.orc_dense_f16.argtypes = [_ptr, _ptr, _i64, _i64, _i64, _ptr, ctypes.c_int]
        L.orc_dense_f16_at.argtypes = [_ptr, _ptr, _i64, _i64, _i64, _ptr, _ptr, _i64, _ptr,
                                       ctypes.c_int]
        for name in ("orc_w8a8", "orc_w2a8"):
            getattr(L, name).argtypes = [_ptr, _ptr, _i64, _i64, _i64, _ptr, ctypes.c_int]
        for name in ("orc_w8a8_at", "orc_w2a8_at"):
            getattr(L, name).argtypes = [_ptr, _ptr, _i64, _i64, _i64, _ptr, _ptr, _i64, _ptr,
                                         ctypes.c_int]
        for name in ("orc_w4a16", "orc_w4a16_at", "orc_dense_f16", "orc_dense_f16_at",
                     "orc_w8a8", "orc_w8a8_at", "orc_w2a8", "orc_w2a8_at"):
            getattr(L, name).restype = ctypes.c_int
        L.orc_max_threads.restype = ctypes.c_int
        self.L = L

    def max_threads(self) -> int:
        return int(self.L.orc_max_threads())

    def _threads(self, nthreads):
        return self.max_threads() if nthreads is None else int(nthreads)

    # ---- scalar / packing ------------------------------------------------------------------

    def half_to_double(self, bits16: np.ndarray) -> np.ndarray:
        b = np.ascontiguousarray(bits16, dtype=np.uint16)
        out = np.empty(b.shape, dtype=np.float64)
        self.L.orc_decode_half(_p(b), _p(out), b.size)
        return out

    def float_to_half(self, x: np.ndarray) -> np.ndarray:
        """binary16 bits of each float32 value, round to nearest even."""
        x = np.ascontiguousarray(x, dtype=np.float32).ravel()
        out = np.empty(x.size, dtype=np.uint16)
        for i, v in enumerate(x):
            out[i] = self.L.orc_float_to_half(ctypes.c_float(float(v)))
        return out

    def rtn_int4(self, W, group_size: int):
        """Round-to-nearest int4 quantisation of fp16 W [N, K]: (codes u8 [N, K], scales fp16
        [N, G], zeros fp16 [N, G])."""
        Wb = _bits16(W)
        N, K = Wb.shape
        gs = K if group_size <= 0 else group_size
        codes = np.empty((N, K), dtype=np.uint8)
        S = np.empty((N, K // gs), dtype=np.uint16)
        Z = np.empty((N, K // gs), dtype=np.uint16)
        _check(self.L.orc_rtn_int4(_p(Wb), N, K, group_size, _p(codes), _p(S), _p(Z)), "rtn_int4")
        return codes, S.view(np.float16), Z.view(np.float16)

    def w8a8_requant(self, A, W, mult, nthreads=None):
        """int8 [M, N]: the int32 product of A and W times mult[n], rounded half to even and
        saturated (binary32 arithmetic)."""
        A = np.ascontiguousarray(A, dtype=np.int8)
        W = np.ascontiguousarray(W, dtype=np.int8)
        mult = np.ascontiguousarray(mult, dtype=np.float32)
        M, K = A.shape
        N = W.shape[0]
        assert W.shape == (N, K) and mult.shape == (N,)
        C8 = np.empty((M, N), dtype=np.int8)
        _check(self.L.orc_w8a8_requant(_p(A), _p(W), _p(mult), M, N, K, _p(C8),
                                       self._threads(nthreads)), "w8a8_requant")
        return C8

    def pack_int4(self, codes: np.ndarray) -> np.ndarray:
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        N, K = codes.shape
        out = np.empty((N, K // 8), dtype=np.uint32)
        _check(self.L.orc_pack_int4(_p(codes), _p(out), N, K), "pack_int4")
        return out

    def unpack_int4(self, packed: np.ndarray, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        N = packed.shape[0]
        out = np.empty((N, K), dtype=np.uint8)
        _check(self.L.orc_unpack_int4(_p(packed), _p(out), N, K), "unpack_int4")
        return out

    def pack_int4_interleaved(self, codes: np.ndarray) -> np.ndarray:
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        N, K = codes.shape
        out = np.empty((N, K // 8), dtype=np.uint32)
        _check(self.L.orc_pack_int4_interleaved(_p(codes), _p(out), N, K), "pack_int4_interleaved")
        return out

    def unpack_int4_interleaved(self, packed: np.ndarray, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        N = packed.shape[0]
        out = np.empty((N, K), dtype=np.uint8)
        _check(self.L.orc_unpack_int4_interleaved(_p(packed), _p(out), N, K),
               "unpack_int4_interleaved")
        return out

    def pack_int2(self, vals: np.ndarray) -> np.ndarray:
        vals = np.ascontiguousarray(vals, dtype=np.int8)
        N, K = vals.shape
        out = np.empty((N, K // 16), dtype=np.uint32)
        _check(self.L.orc_pack_int2(_p(vals), _p(out), N, K), "pack_int2")
        return out

    def unpack_int2(self, packed: np.ndarray, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        N = packed.shape[0]
        out = np.empty((N, K), dtype=np.int8)
        _check(self.L.orc_unpack_int2(_p(packed), _p(out), N, K), "unpack_int2")
        return out

    def pack_int2_interleaved(self, vals: np.ndarray) -> np.ndarray:
        vals = np.ascontiguousarray(vals, dtype=np.int8)
        N, K = vals.shape
        out = np.empty((N, K // 16), dtype=np.uint32)
        _check(self.L.orc_pack_int2_interleaved(_p(vals), _p(out), N, K), "pack_int2_interleaved")
        return out

    def unpack_int2_interleaved(self, packed: np.ndarray, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        N = packed.shape[0]
        out = np.empty((N, K), dtype=np.int8)
        _check(self.L.orc_unpack_int2_interleaved(_p(packed), _p(out), N, K),
               "unpack_int2_interleaved")
        return out

    # ---- matmuls ----------------------------------------------------------------------------

    def w4a16(self, A, Wq, scales, zeros, K: int, group_size: int, nthreads=None):
        """fp64 C[M,N] = A . ((q - z) * s)^T from packed Wq [N, K/8]."""
        A16 = _bits16(A)
        M = A16.shape[0]
        Wq = np.ascontiguousarray(Wq, dtype=np.uint32)
        N = Wq.shape[0]
        S = _bits16(scales)
        Z = None if zeros is None else _bits16(zeros)
        C = np.empty((M, N), dtype=np.float64)
        _check(self.L.orc_w4a16(_p(A16), _p(Wq), _p(S), _p(Z), M, N, K, group_size,
                                int(Z is not None), _p(C), self._threads(nthreads)), "w4a16")
        return C

    def w4a16_at(self, A, Wq, scales, zeros, K: int, group_size: int, ms, ns, nthreads=None):
        A16 = _bits16(A)
        Wq = np.ascontiguousarray(Wq, dtype=np.uint32)
        S = _bits16(scales)
        Z = None if zeros is None else _bits16(zeros)
        ms, ns = _pairs(ms, ns)
        out = np.empty(ms.shape, dtype=np.float64)
        _check(self.L.orc_w4a16_at(_p(A16), _p(Wq), _p(S), _p(Z), A16.shape[0], Wq.shape[0],
                                   K, group_size, int(Z is not None), _p(ms), _p(ns), ms.size,
                                   _p(out), self._threads(nthreads)), "w4a16_at")
        return out

    def dense_f16(self, A, W, nthreads=None):
        A16, W16 = _bits16(A), _bits16(W)
        M, K = A16.shape
        N = W16.shape[0]
        C = np.empty((M, N), dtype=np.float64)
        _check(self.L.orc_dense_f16(_p(A16), _p(W16), M, N, K, _p(C), self._threads(nthreads)),
               "dense")
        return C

    def dense_f16_at(self, A, W, ms, ns, nthreads=None):
        A16, W16 = _bits16(A), _bits16(W)
        ms, ns = _pairs(ms, ns)
        out = np.empty(ms.shape, dtype=np.float64)
        _check(self.L.orc_dense_f16_at(_p(A16), _p(W16), A16.shape[0], W16.shape[0],
                                       A16.shape[1], _p(ms), _p(ns), ms.size, _p(out),
                                       self._threads(nthreads)), "dense_at")
        return out

    def w8a8(self, A, W, nthreads=None):
        A = np.ascontiguousarray(A, dtype=np.int8)
        W = np.ascontiguousarray(W, dtype=np.int8)
        M, K = A.shape
        N = W.shape[0]
        C = np.empty((M, N), dtype=np.int64)
        _check(self.L.orc_w8a8(_p(A), _p(W), M, N, K, _p(C), self._threads(nthreads)), "w8a8")
        return C

    def w8a8_at(self, A, W, ms, ns, nthreads=None):
        A = np.ascontiguousarray(A, dtype=np.int8)
        W = np.ascontiguousarray(W, dtype=np.int8)
        ms, ns = _pairs(ms, ns)
        out = np.empty(ms.shape, dtype=np.int64)
        _check(self.L.orc_w8a8_at(_p(A), _p(W), A.shape[0], W.shape[0], A.shape[1], _p(ms),
                                  _p(ns), ms.size, _p(out), self._threads(nthreads)), "w8a8_at")
        return out

    def w2a8(self, A, Wq, nthreads=None):
        A = np.ascontiguousarray(A, dtype=np.int8)
        Wq = np.ascontiguousarray(Wq, dtype=np.uint32)
        M, K = A.shape
        N = Wq.shape[0]
        C = np.empty((M, N), dtype=np.int64)
        _check(self.L.orc_w2a8(_p(A), _p(Wq), M, N, K, _p(C), self._threads(nthreads)), "w2a8")
        return C

    def w2a8_at(self, A, Wq, ms, ns, nthreads=None):
        A = np.ascontiguousarray(A, dtype=np.int8)
        Wq = np.ascontiguousarray(Wq, dtype=np.uint32)
        ms, ns = _pairs(ms, ns)
        out = np.empty(ms.shape, dtype=np.int64)
        _check(self.L.orc_w2a8_at(_p(A), _p(Wq), A.shape[0], Wq.shape[0], A.shape[1], _p(ms),
                                  _p(ns), ms.size, _p(out), self._threads(nthreads)), "w2a8_at")
        return out


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype in (np.float16, np.uint16)
    return a.view(np.uint16)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: status {rc}")


def _pairs(ms, ns):
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    assert ms.shape == ns.shape and ms.ndim == 1
    return ms, ns


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from oracle.c (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def max_threads() -> int: return get().max_threads()
def half_to_double(b): return get().half_to_double(b)
def w8a8_requant(A, W, mult, nthreads=None): return get().w8a8_requant(A, W, mult, nthreads)
def float_to_half(x): return get().float_to_half(x)
def rtn_int4(W, group_size): return get().rtn_int4(W, group_size)
def pack_int4(c): return get().pack_int4(c)
def unpack_int4(p, K): return get().unpack_int4(p, K)
def pack_int4_interleaved(c): return get().pack_int4_interleaved(c)
def unpack_int4_interleaved(p, K): return get().unpack_int4_interleaved(p, K)
def pack_int2(v): return get().pack_int2(v)
def unpack_int2(p, K): return get().unpack_int2(p, K)
def pack_int2_interleaved(v): return get().pack_int2_interleaved(v)
def unpack_int2_interleaved(p, K): return get().unpack_int2_interleaved(p, K)
def w4a16(*a, **k): return get().w4a16(*a, **k)
def w4a16_at(*a, **k): return get().w4a16_at(*a, **k)
def dense_f16(*a, **k): return get().dense_f16(*a, **k)
def dense_f16_at(*a, **k): return get().dense_f16_at(*a, **k)
def w8a8(*a, **k): return get().w8a8(*a, **k)
def w8a8_at(*a, **k): return get().w8a8_at(*a, **k)
def w2a8(*a, **k): return get().w2a8(*a, **k)
def w2a8_at(*a, **k): return get().w2a8_at(*a, **k)


# ---- acceptance rule for fp16-output paths ------------------------------------------------------

ATOL = 0.02
RTOL = 0.01
FROB = 5e-3


def fp16_close(got: np.ndarray, ref: np.ndarray) -> tuple[bool, str]:
    """Per element |got - ref| <= 0.02 + 0.01 |ref| and ||got - ref||_F / ||ref||_F <= 5e-3."""
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    if g.shape != r.shape:
        return False, f"shape {g.shape} vs {r.shape}"
    if not np.all(np.isfinite(g)):
        return False, "non-finite output"
    err = np.abs(g - r)
    bound = ATOL + RTOL * np.abs(r)
    bad = int(np.count_nonzero(err > bound))
    nr = float(np.linalg.norm(r))
    frob = float(np.linalg.norm(g - r)) / nr if nr > 0 else float(np.linalg.norm(g - r))
    ok = bad == 0 and frob <= FROB
    worst = int(np.argmax(err - bound)) if err.size else 0
    msg = (f"bad={bad}/{err.size} frob={frob:.3e} max_err={err.max() if err.size else 0:.4g} "
           f"at flat {worst} (got {g.ravel()[worst] if err.size else 0}, "
           f"ref {r.ravel()[worst] if err.size else 0})")
    return ok, msg
