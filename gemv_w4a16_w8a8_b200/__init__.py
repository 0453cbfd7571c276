"""Python binding of libqgemm.so, the B200 low-bit matmul library (C ABI in include/qgemm.h).

Argument marshalling only: every function here checks tensor types, takes raw device pointers
and the current CUDA stream from PyTorch, and calls the C entry point of the same name. All
arithmetic runs in the library's CUDA kernels. There is no fallback: if the library is not
built, or the device is not a B200, calls raise.

    C = qgemm_w4a16(A, Wq, scales, zeros, group_size=128)        # A fp16 [M,K], Wq int32 [N,K/8]
    C = qgemm_w8a8(A, W)                                         # int8 x int8 -> int32
    C = qgemm_w2a8(A, Wq)                                        # int8 x packed int2 -> int32
    Wq = quant_pack_int4(codes)                                  # uint8 [N,K] -> int32 [N,K/8]
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libqgemm.so")

QG_OK = 0
QG_ERR_INVALID_ARG = 1
QG_ERR_ALIGNMENT = 2
QG_ERR_UNSUPPORTED_SHAPE = 3
QG_ERR_CUDA = 4
QG_ERR_DEVICE_TIMEOUT = 5
QG_ERR_NOT_SM100 = 6
QG_ERR_BAD_CONFIG = 7
QG_ERR_SCRATCH_TOO_SMALL = 8
# size of the library's fixed device scratch used by qgemm_w4a16_splitk_f32_noalloc
QGEMM_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024

OP_W4A16, OP_W8A8, OP_W2A8, OP_DENSE_F16, OP_W4A16_INTERLEAVED = 0, 1, 2, 3, 4
OP_W2A8_INTERLEAVED = 5
PATH_AUTO, PATH_GEMV, PATH_TC, PATH_STREAM = 0, 1, 2, 3

# every symbol include/qgemm.h declares
EXPORTS = (
    "qgemm_w4a16", "qgemm_w4a16_interleaved", "quant_pack_int4_interleaved", "qgemm_w4a16_splitk_f32", "qgemm_w4a16_workspace_bytes",
    "qgemm_w4a16_splitk_f32_noalloc", "qgemm_w4a16_host", "qgemm_w4a16_host_workspace_bytes",
    "qgemm_w8a8", "qgemm_w2a8", "qgemm_w2a8_interleaved", "qgemm_dense_f16", "quant_pack_int4",
    "quant_rtn_int4", "qgemm_w8a8_requant",
    "quant_pack_int2", "quant_pack_int2_interleaved", "qgemm_plan", "qgemm_set_config", "qgemm_tune", "qgemm_save_configs",
    "qgemm_load_configs", "qgemm_clear_configs", "qgemm_sync_check", "qgemm_selftest_bounded_wait",
    "qgemm_status_string",
    "qgemm_version",
)


class QGemmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class Config(ctypes.Structure):
    """qgemm_config_t"""
    _fields_ = [("path", ctypes.c_int32), ("rows", ctypes.c_int32), ("bm", ctypes.c_int32),
                ("bn", ctypes.c_int32), ("bk", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("split_k", ctypes.c_int32), ("swap_ab", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {name: int(getattr(self, name)) for name, _ in self._fields_}


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library. Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              f"`python -m gemv_w4a16_w8a8_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32 = ctypes.c_void_p, ctypes.c_int
        L.qgemm_w4a16.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.qgemm_w4a16_interleaved.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.quant_pack_int4_interleaved.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.qgemm_w4a16_splitk_f32.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp,
                                             ctypes.c_size_t, vp]
        L.qgemm_w4a16_splitk_f32_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                                     i32, vp]
        L.quant_rtn_int4.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.qgemm_w8a8_requant.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp]
        L.qgemm_w4a16_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.qgemm_w4a16_workspace_bytes.restype = ctypes.c_size_t
        L.qgemm_w4a16_host.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp,
                                       ctypes.c_size_t, vp]
        L.qgemm_w4a16_host_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.qgemm_w4a16_host_workspace_bytes.restype = ctypes.c_size_t
        L.qgemm_w8a8.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.qgemm_w2a8.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.qgemm_w2a8_interleaved.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.qgemm_dense_f16.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
        L.quant_pack_int4.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.quant_pack_int2.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.quant_pack_int2_interleaved.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.qgemm_plan.argtypes = [i32, i32, i32, i32, i32, i32, i32, ctypes.POINTER(Config)]
        L.qgemm_set_config.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(Config)]
        L.qgemm_tune.argtypes = [i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp,
                                 ctypes.POINTER(Config)]
        L.qgemm_save_configs.argtypes = [ctypes.c_char_p]
        L.qgemm_load_configs.argtypes = [ctypes.c_char_p]
        L.qgemm_clear_configs.argtypes = []
        L.qgemm_clear_configs.restype = None
        L.qgemm_sync_check.argtypes = [vp]
        L.qgemm_selftest_bounded_wait.argtypes = [i32, vp]
        L.qgemm_status_string.argtypes = [i32]
        L.qgemm_status_string.restype = ctypes.c_char_p
        L.qgemm_version.restype = i32
        for name in EXPORTS:
            if name not in ("qgemm_status_string", "qgemm_clear_configs", "qgemm_version",
                            "qgemm_w4a16_workspace_bytes", "qgemm_w4a16_host_workspace_bytes"):
                getattr(L, name).restype = i32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().qgemm_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != QG_OK:
        raise QGemmError(status, what)


# ---- torch marshalling ------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, ndim, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    allowed = dtype if isinstance(dtype, tuple) else (dtype,)
    if t.dtype not in allowed:
        raise TypeError(f"{name} must be {' or '.join(map(str, allowed))}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def qgemm_w4a16(A, Wq, scales, zeros=None, C=None, group_size: int = 128, split_k: int = 0,
                stream=None):
    """A fp16 [M,K]; Wq int32/uint32 [N,K/8]; scales (zeros) fp16 [N,G]. Returns C fp16 [M,N]."""
    torch = _torch()
    _need(A, torch.float16, 2, "A")
    _need(Wq, (torch.int32, torch.uint32), 2, "Wq")
    _need(scales, torch.float16, 2, "scales")
    if zeros is not None:
        _need(zeros, torch.float16, 2, "zeros")
    M, K = A.shape
    N = Wq.shape[0]
    if Wq.shape[1] * 8 != K:
        raise ValueError(f"Wq must be [N, K/8] = [{N}, {K // 8}], got {tuple(Wq.shape)}")
    if C is None:
        C = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _need(C, torch.float16, 2, "C")
    st = lib().qgemm_w4a16(_ptr(A), _ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(C), M, N, K,
                           group_size, split_k, int(zeros is not None), _stream(stream))
    _check(st, "qgemm_w4a16")
    return C


def qgemm_w4a16_interleaved(A, Wq, scales, zeros=None, C=None, group_size: int = 128,
                            split_k: int = 0, stream=None):
    """As qgemm_w4a16, with Wq from quant_pack_int4_interleaved."""
    torch = _torch()
    _need(A, torch.float16, 2, "A")
    _need(Wq, (torch.int32, torch.uint32), 2, "Wq")
    _need(scales, torch.float16, 2, "scales")
    if zeros is not None:
        _need(zeros, torch.float16, 2, "zeros")
    M, K = A.shape
    N = Wq.shape[0]
    if Wq.shape[1] * 8 != K:
        raise ValueError(f"Wq must be [N, K/8] = [{N}, {K // 8}], got {tuple(Wq.shape)}")
    if C is None:
        C = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _need(C, torch.float16, 2, "C")
    st = lib().qgemm_w4a16_interleaved(_ptr(A), _ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(C), M,
                                       N, K, group_size, split_k, int(zeros is not None),
                                       _stream(stream))
    _check(st, "qgemm_w4a16_interleaved")
    return C


def quant_pack_int4_interleaved(codes, out=None, stream=None):
    """codes uint8 [N,K] -> int32 [N,K/8] in the interleaved layout (nibbles 0..7 of each word
    hold codes 0,2,4,6,1,3,5,7 of its eight)."""
    torch = _torch()
    _need(codes, torch.uint8, 2, "codes")
    N, K = codes.shape
    if out is None:
        out = torch.empty((N, K // 8), dtype=torch.int32, device=codes.device)
    _check(lib().quant_pack_int4_interleaved(_ptr(codes), _ptr(out), 0, N, K, -1, 1, 0,
                                             _stream(stream)), "quant_pack_int4_interleaved")
    return out


def qgemm_w4a16_workspace_bytes(M: int, N: int, K: int, group_size: int, split_k: int) -> int:
    return int(lib().qgemm_w4a16_workspace_bytes(M, N, K, group_size, split_k))


def qgemm_w4a16_splitk_f32(A, Wq, scales, zeros=None, C=None, group_size: int = 128,
                           split_k: int = 4, workspace=None, stream=None):
    """Deterministic split-K W4A16 through an fp32 workspace (a uint8 CUDA tensor of at least
    qgemm_w4a16_workspace_bytes(...) bytes; allocated here when not given)."""
    torch = _torch()
    _need(A, torch.float16, 2, "A")
    _need(Wq, (torch.int32, torch.uint32), 2, "Wq")
    _need(scales, torch.float16, 2, "scales")
    if zeros is not None:
        _need(zeros, torch.float16, 2, "zeros")
    M, K = A.shape
    N = Wq.shape[0]
    if C is None:
        C = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _need(C, torch.float16, 2, "C")
    need = qgemm_w4a16_workspace_bytes(M, N, K, group_size, split_k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=A.device)
    _need(workspace, torch.uint8, 1, "workspace")
    st = lib().qgemm_w4a16_splitk_f32(_ptr(A), _ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(C), M, N,
                                      K, group_size, split_k, int(zeros is not None),
                                      _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "qgemm_w4a16_splitk_f32")
    return C


def qgemm_w4a16_host_workspace_bytes(M: int, N: int, K: int, chunk_tokens: int = 0) -> int:
    return int(lib().qgemm_w4a16_host_workspace_bytes(M, N, K, chunk_tokens))


def qgemm_w4a16_host(A_host, Wq, scales, zeros, C_host, workspace, group_size: int = 128,
                     split_k: int = 0, stream=None):
    """W4A16 with A_host fp16 [M,K] and C_host fp16 [M,N] in page-locked host memory (CPU tensors
    from pin_memory()); A streams in and C out in chunks through `workspace` (a uint8 CUDA tensor
    of qgemm_w4a16_host_workspace_bytes(...) bytes or more). Asynchronous on `stream`: wait on
    it before reading C_host."""
    torch = _torch()
    for name, t in (("A_host", A_host), ("C_host", C_host)):
        if t.dtype != torch.float16 or t.dim() != 2 or t.device.type != "cpu" or \
                not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 2-D float16 CPU tensor")
        if not t.is_pinned():
            raise ValueError(f"{name} must be in page-locked memory (pin_memory())")
    _need(Wq, (torch.int32, torch.uint32), 2, "Wq")
    _need(scales, torch.float16, 2, "scales")
    if zeros is not None:
        _need(zeros, torch.float16, 2, "zeros")
    _need(workspace, torch.uint8, 1, "workspace")
    M, K = A_host.shape
    N = Wq.shape[0]
    if tuple(C_host.shape) != (M, N):
        raise ValueError("C_host must be [M, N]")
    st = lib().qgemm_w4a16_host(A_host.data_ptr(), _ptr(Wq), _ptr(scales), _ptr(zeros),
                                C_host.data_ptr(), M, N, K, group_size, split_k,
                                int(zeros is not None), _ptr(workspace), workspace.numel(),
                                _stream(stream))
    _check(st, "qgemm_w4a16_host")
    return C_host


def qgemm_w8a8(A, W, C=None, split_k: int = 0, stream=None):
    """A int8 [M,K]; W int8 [N,K]. Returns C int32 [M,N]."""
    torch = _torch()
    _need(A, torch.int8, 2, "A")
    _need(W, torch.int8, 2, "W")
    M, K = A.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N, K]")
    if C is None:
        C = torch.empty((M, N), dtype=torch.int32, device=A.device)
    _need(C, torch.int32, 2, "C")
    _check(lib().qgemm_w8a8(_ptr(A), _ptr(W), _ptr(C), M, N, K, -1, split_k, 0, _stream(stream)),
           "qgemm_w8a8")
    return C


def qgemm_w8a8_requant(A, W, mult, C=None, stream=None):
    """int8 A [M,K] x int8 W [N,K] -> int8 C [M,N] = sat8(rint(acc * mult[n])), mult fp32 [N]."""
    torch = _torch()
    _need(A, torch.int8, 2, "A")
    _need(W, torch.int8, 2, "W")
    _need(mult, torch.float32, 1, "mult")
    M, K = A.shape
    N = W.shape[0]
    if W.shape[1] != K or mult.shape[0] != N:
        raise ValueError("shapes of A, W and mult do not agree")
    if C is None:
        C = torch.empty((M, N), dtype=torch.int8, device=A.device)
    _check(lib().qgemm_w8a8_requant(_ptr(A), _ptr(W), _ptr(mult), _ptr(C), M, N, K,
                                    _stream(stream)), "qgemm_w8a8_requant")
    return C


def qgemm_w2a8(A, Wq, C=None, split_k: int = 0, stream=None):
    """A int8 [M,K]; Wq int32/uint32 [N,K/16]. Returns C int32 [M,N]."""
    torch = _torch()
    _need(A, torch.int8, 2, "A")
    _need(Wq, (torch.int32, torch.uint32), 2, "Wq")
    M, K = A.shape
    N = Wq.shape[0]
    if Wq.shape[1] * 16 != K:
        raise ValueError("Wq must be [N, K/16]")
    if C is None:
        C = torch.empty((M, N), dtype=torch.int32, device=A.device)
    _need(C, torch.int32, 2, "C")
    _check(lib().qgemm_w2a8(_ptr(A), _ptr(Wq), _ptr(C), M, N, K, -1, split_k, 0, _stream(stream)),
           "qgemm_w2a8")
    return C


def qgemm_w2a8_interleaved(A, Wq, C=None, split_k: int = 0, stream=None):
    """As qgemm_w2a8, with Wq from quant_pack_int2_interleaved."""
    torch = _torch()
    _need(A, torch.int8, 2, "A")
    _need(Wq, (torch.int32, torch.uint32), 2, "Wq")
    M, K = A.shape
    N = Wq.shape[0]
    if Wq.shape[1] * 16 != K:
        raise ValueError("Wq must be [N, K/16]")
    if C is None:
        C = torch.empty((M, N), dtype=torch.int32, device=A.device)
    _need(C, torch.int32, 2, "C")
    _check(lib().qgemm_w2a8_interleaved(_ptr(A), _ptr(Wq), _ptr(C), M, N, K, -1, split_k, 0,
                                        _stream(stream)), "qgemm_w2a8_interleaved")
    return C


def qgemm_dense_f16(A, W, C=None, split_k: int = 0, stream=None):
    """A fp16 [M,K]; W fp16 [N,K]. Returns C fp16 [M,N]."""
    torch = _torch()
    _need(A, torch.float16, 2, "A")
    _need(W, torch.float16, 2, "W")
    M, K = A.shape
    N = W.shape[0]
    if C is None:
        C = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _need(C, torch.float16, 2, "C")
    _check(lib().qgemm_dense_f16(_ptr(A), _ptr(W), _ptr(C), M, N, K, split_k, _stream(stream)),
           "qgemm_dense_f16")
    return C


def quant_pack_int4(codes, out=None, stream=None):
    """codes uint8 [N,K] (0..15) -> int32 [N,K/8], code k at bits 4*(k%8) of word k/8."""
    torch = _torch()
    _need(codes, torch.uint8, 2, "codes")
    N, K = codes.shape
    if out is None:
        out = torch.empty((N, K // 8), dtype=torch.int32, device=codes.device)
    _check(lib().quant_pack_int4(_ptr(codes), _ptr(out), 0, N, K, -1, 1, 0, _stream(stream)),
           "quant_pack_int4")
    return out


def quant_rtn_int4(W, group_size: int = 128, stream=None):
    """Round-to-nearest int4 quantisation of fp16 W [N,K] (rule in include/qgemm.h):
    returns (packed int32 [N,K/8], scales fp16 [N,G], zeros fp16 [N,G])."""
    torch = _torch()
    _need(W, torch.float16, 2, "W")
    N, K = W.shape
    gs = K if group_size <= 0 else group_size
    if gs <= 0 or K % gs:
        raise ValueError(f"group_size {group_size} does not divide K = {K}")
    Wq = torch.empty((N, K // 8), dtype=torch.int32, device=W.device)
    S = torch.empty((N, K // gs), dtype=torch.float16, device=W.device)
    Z = torch.empty((N, K // gs), dtype=torch.float16, device=W.device)
    _check(lib().quant_rtn_int4(_ptr(W), _ptr(Wq), _ptr(S), _ptr(Z), N, K, group_size, 1,
                                _stream(stream)), "quant_rtn_int4")
    return Wq, S, Z


def quant_pack_int2(vals, out=None, stream=None):
    """vals int8 [N,K] (-2..1) -> int32 [N,K/16], value k at bits 2*(k%16) of word k/16."""
    torch = _torch()
    _need(vals, torch.int8, 2, "vals")
    N, K = vals.shape
    if out is None:
        out = torch.empty((N, K // 16), dtype=torch.int32, device=vals.device)
    _check(lib().quant_pack_int2(_ptr(vals), _ptr(out), 0, N, K, -1, 1, 0, _stream(stream)),
           "quant_pack_int2")
    return out


def quant_pack_int2_interleaved(vals, out=None, stream=None):
    """vals int8 [N,K] (-2..1) -> int32 [N,K/16] in the interleaved layout (2-bit fields 0..15
    of each word hold values 0,4,1,5,2,6,3,7, 8,12,9,13,10,14,11,15 of its sixteen)."""
    torch = _torch()
    _need(vals, torch.int8, 2, "vals")
    N, K = vals.shape
    if out is None:
        out = torch.empty((N, K // 16), dtype=torch.int32, device=vals.device)
    _check(lib().quant_pack_int2_interleaved(_ptr(vals), _ptr(out), 0, N, K, -1, 1, 0,
                                             _stream(stream)), "quant_pack_int2_interleaved")
    return out


# ---- configuration -------------------------------------------------------------------------------

def qgemm_plan(op: int, M: int, N: int, K: int, group_size: int = -1, has_zero: int = 0,
               split_k: int = 0) -> dict:
    cfg = Config()
    _check(lib().qgemm_plan(op, M, N, K, group_size, has_zero, split_k, ctypes.byref(cfg)),
           "qgemm_plan")
    return cfg.as_dict()


def qgemm_set_config(op: int, M: int, N: int, K: int, group_size: int, has_zero: int,
                     cfg: dict | None):
    c = None
    if cfg is not None:
        c = Config(**{k: int(v) for k, v in cfg.items()})
    _check(lib().qgemm_set_config(op, M, N, K, group_size, has_zero,
                                  ctypes.byref(c) if c is not None else None),
           "qgemm_set_config")


def qgemm_tune(op: int, A, W, scales, zeros, C, M: int, N: int, K: int, group_size: int = -1,
               has_zero: int = 0, reps: int = 20, stream=None) -> dict:
    best = Config()
    _check(lib().qgemm_tune(op, _ptr(A), _ptr(W), _ptr(scales), _ptr(zeros), _ptr(C), M, N, K,
                            group_size, has_zero, reps, _stream(stream), ctypes.byref(best)),
           "qgemm_tune")
    return best.as_dict()


def qgemm_save_configs(path: str):
    _check(lib().qgemm_save_configs(path.encode()), "qgemm_save_configs")


def qgemm_load_configs(path: str):
    _check(lib().qgemm_load_configs(path.encode()), "qgemm_load_configs")


def qgemm_clear_configs():
    lib().qgemm_clear_configs()


def qgemm_sync_check(stream=None):
    _check(lib().qgemm_sync_check(_stream(stream)), "qgemm_sync_check")


def qgemm_selftest_bounded_wait(limit_us: int = 20000, stream=None):
    """Queue a kernel whose bounded wait runs out after limit_us; the next qgemm_sync_check raises
    QG_ERR_DEVICE_TIMEOUT."""
    _check(lib().qgemm_selftest_bounded_wait(limit_us, _stream(stream)),
           "qgemm_selftest_bounded_wait")


def qgemm_version() -> int:
    return int(lib().qgemm_version())
