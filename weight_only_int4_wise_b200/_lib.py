"""ctypes binding of libw4a16.so (include/w4a16.h). Argument marshalling only.

Functions named like the C entry points (`w4a16_gemm`, ...) take torch tensors
or raw integer addresses and return the C status code. The short names
(`gemm`, `pack`, ...) allocate outputs with torch, pass
`torch.cuda.current_stream()`, and raise `W4A16Error` on any non-zero status.
Every byte of the product is computed by the CUDA library; nothing here falls
back to another implementation, and a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libw4a16.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_MISALIGNED = 2
ERR_UNSUPPORTED = 3
ERR_CUDA = 4
ERR_TIMEOUT = 5
ERR_BAD_OFFSETS = 6
MAX_EXPERTS = 64

EXPORTED = [
    "w4a16_status_string", "w4a16_pack", "w4a16_unpack", "w4a16_tiled_bytes", "w4a16_repack",
    "w4a16_gemm", "w4a16_grouped_gemm", "w4a16_gemm_launch_info", "w4a16_grouped_launch_info",
    "w4a16_device_status", "w4a16_set_static_weights", "w4a16_quantize", "w4a16_set_fault_injection",
]


class W4A16Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class LaunchInfo(ctypes.Structure):
    _fields_ = [("token_tile", ctypes.c_int32), ("k_splits", ctypes.c_int32), ("grid_x", ctypes.c_int32),
                ("grid_y", ctypes.c_int32), ("grid_z", ctypes.c_int32), ("threads_per_cta", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("ctas_per_sm", ctypes.c_int32)]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


_lib = None
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


def load() -> ctypes.CDLL:
    """The CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run `python -m weight_only_int4_wise_b200.build`)")
        lib = ctypes.CDLL(LIB_PATH)
        lib.w4a16_status_string.argtypes = [ctypes.c_int]
        lib.w4a16_status_string.restype = ctypes.c_char_p
        for name in ("w4a16_pack", "w4a16_unpack", "w4a16_repack"):
            f = getattr(lib, name)
            f.argtypes = [_vp, _vp, _i64, _i64, _vp]
            f.restype = ctypes.c_int
        lib.w4a16_quantize.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _vp]
        lib.w4a16_quantize.restype = ctypes.c_int
        lib.w4a16_tiled_bytes.argtypes = [_i64, _i64]
        lib.w4a16_tiled_bytes.restype = _i64
        lib.w4a16_gemm.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp]
        lib.w4a16_gemm.restype = ctypes.c_int
        lib.w4a16_grouped_gemm.argtypes = [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp, _vp, _i64, _i64,
                                           _i64, _i64, _i64, _vp]
        lib.w4a16_grouped_gemm.restype = ctypes.c_int
        lib.w4a16_gemm_launch_info.argtypes = [_i64, _i64, _i64, _i64, ctypes.POINTER(LaunchInfo)]
        lib.w4a16_gemm_launch_info.restype = ctypes.c_int
        lib.w4a16_grouped_launch_info.argtypes = [_i64, _i64, _i64, _i64, _i64, ctypes.POINTER(LaunchInfo)]
        lib.w4a16_grouped_launch_info.restype = ctypes.c_int
        lib.w4a16_device_status.argtypes = [ctypes.c_int]
        lib.w4a16_device_status.restype = ctypes.c_int
        lib.w4a16_set_static_weights.argtypes = [ctypes.c_int]
        lib.w4a16_set_static_weights.restype = ctypes.c_int
        lib.w4a16_set_fault_injection.argtypes = [_i64, _i64]
        lib.w4a16_set_fault_injection.restype = ctypes.c_int
        _lib = lib
    return _lib


def _addr(x) -> Optional[int]:
    """Device/host address of a tensor, or an int passed through (None -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _current_stream(device_index: Optional[int] = None) -> int:
    """Raw handle of torch's current stream (the cheap accessor when torch has it)."""
    import torch
    if device_index is None:
        device_index = torch.cuda.current_device()
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    if raw is not None:
        return raw(device_index)
    return torch.cuda.current_stream(device_index).cuda_stream


def _stream(stream) -> Optional[int]:
    if stream is None:
        return _current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def status_string(status: int) -> str:
    return load().w4a16_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise W4A16Error(status, where)


# ------------------------------------------------------------- C-ABI mirrors

def w4a16_pack(q, wp, K: int, N: int, stream=None) -> int:
    return load().w4a16_pack(_addr(q), _addr(wp), K, N, _stream(stream))


def w4a16_quantize(W, wp, S, K: int, N: int, G: int, stream=None) -> int:
    return load().w4a16_quantize(_addr(W), _addr(wp), _addr(S), K, N, G, _stream(stream))


def w4a16_unpack(wp, q, K: int, N: int, stream=None) -> int:
    return load().w4a16_unpack(_addr(wp), _addr(q), K, N, _stream(stream))


def w4a16_tiled_bytes(K: int, N: int) -> int:
    return int(load().w4a16_tiled_bytes(K, N))


def w4a16_repack(wp, wt, K: int, N: int, stream=None) -> int:
    return load().w4a16_repack(_addr(wp), _addr(wt), K, N, _stream(stream))


def w4a16_gemm(A, Wt, S, C, M: int, N: int, K: int, G: int, stream=None) -> int:
    return load().w4a16_gemm(_addr(A), _addr(Wt), _addr(S), _addr(C), M, N, K, G, _stream(stream))


def w4a16_grouped_gemm(A, Wt: Sequence, S: Sequence, offsets, C, E: int, total_rows: int, N: int, K: int,
                       G: int, stream=None) -> int:
    wt_arr = (_vp * max(1, len(Wt)))(*[_addr(w) for w in Wt])
    s_arr = (_vp * max(1, len(S)))(*[_addr(s) for s in S])
    return load().w4a16_grouped_gemm(_addr(A), wt_arr, s_arr, _addr(offsets), _addr(C), E, total_rows, N, K, G,
                                     _stream(stream))


def w4a16_gemm_launch_info(M: int, N: int, K: int, G: int):
    info = LaunchInfo()
    rc = load().w4a16_gemm_launch_info(M, N, K, G, ctypes.byref(info))
    return rc, info


def w4a16_grouped_launch_info(E: int, total_rows: int, N: int, K: int, G: int):
    info = LaunchInfo()
    rc = load().w4a16_grouped_launch_info(E, total_rows, N, K, G, ctypes.byref(info))
    return rc, info


def w4a16_device_status(clear: bool = True) -> int:
    return int(load().w4a16_device_status(1 if clear else 0))


def w4a16_set_static_weights(enable: bool) -> int:
    """Declare weights and scales static (see include/w4a16.h); returns the previous setting."""
    return int(load().w4a16_set_static_weights(1 if enable else 0))


def w4a16_set_fault_injection(stall_stage: int, wait_limit_cycles: int) -> int:
    """Test aid: stall one K stage and bound every device wait (see include/w4a16.h)."""
    return int(load().w4a16_set_fault_injection(int(stall_stage), int(wait_limit_cycles)))


# ------------------------------------------------------------- torch helpers

def _require_cuda(*tensors):
    for t in tensors:
        if not t.is_cuda:
            raise ValueError("all tensors must live on a CUDA device")


def pack(q, stream=None):
    """int8 codes [K, N] (device) -> canonical packed [ceil(K/2), N] uint8."""
    import torch
    _require_cuda(q)
    K, N = q.shape
    wp = torch.empty(((K + 1) // 2, N), dtype=torch.uint8, device=q.device)
    _check(w4a16_pack(q.contiguous(), wp, K, N, stream), "w4a16_pack")
    return wp


def quantize(W, G: int, stream=None):
    """fp16 weights [K, N] (device) -> (canonical packed codes [ceil(K/2), N] uint8,
    fp16 scales [ceil(K/G), N]): group-wise symmetric int4 quantisation."""
    import torch
    _require_cuda(W)
    if W.dtype != torch.float16:
        raise TypeError("W must be float16")
    K, N = W.shape
    wp = torch.empty(((K + 1) // 2, N), dtype=torch.uint8, device=W.device)
    S = torch.empty(((K + G - 1) // G, N), dtype=torch.float16, device=W.device)
    _check(w4a16_quantize(W.contiguous(), wp, S, K, N, G, stream), "w4a16_quantize")
    return wp, S


def unpack(wp, K: int, stream=None):
    import torch
    _require_cuda(wp)
    N = wp.shape[1]
    q = torch.empty((K, N), dtype=torch.int8, device=wp.device)
    _check(w4a16_unpack(wp.contiguous(), q, K, N, stream), "w4a16_unpack")
    return q


def repack(wp, K: int, stream=None):
    """canonical packed [ceil(K/2), N] -> tiled layout (flat uint8)."""
    import torch
    _require_cuda(wp)
    N = wp.shape[1]
    wt = torch.empty(w4a16_tiled_bytes(K, N), dtype=torch.uint8, device=wp.device)
    _check(w4a16_repack(wp.contiguous(), wt, K, N, stream), "w4a16_repack")
    return wt


def prepare_weights(q, stream=None):
    """int8 codes [K, N] -> (canonical packed, tiled) on the device."""
    wp = pack(q, stream)
    return wp, repack(wp, q.shape[0], stream)


def gemm(A, wt, S, N: int, G: int, out=None, stream=None):
    """C [M, N] fp16 = A [M, K] fp16 x dequant(tiled weights, scales S [ceil(K/G), N])."""
    import torch
    if not (A.is_cuda and wt.is_cuda and S.is_cuda):
        raise ValueError("all tensors must live on a CUDA device")
    if A.dtype != torch.float16 or S.dtype != torch.float16:
        raise TypeError("A and S must be float16")
    M, K = A.shape
    if not A.is_contiguous():
        A = A.contiguous()
    if not S.is_contiguous():
        S = S.contiguous()
    C = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=A.device)
    st = _current_stream(A.device.index) if stream is None else _stream(stream)
    rc = (_lib or load()).w4a16_gemm(A.data_ptr(), wt.data_ptr(), S.data_ptr(), C.data_ptr(), M, N, K, G, st)
    if rc != OK:
        raise W4A16Error(rc, "w4a16_gemm")
    return C


def grouped_gemm(A, wts: Sequence, Ss: Sequence, offsets, N: int, G: int, out=None, stream=None):
    """Grouped-expert product over gathered rows A [rows, K] with int32 offsets [E+1] on the device."""
    import torch
    _require_cuda(A, offsets)
    rows, K = A.shape
    C = out if out is not None else torch.empty((rows, N), dtype=torch.float16, device=A.device)
    _check(w4a16_grouped_gemm(A.contiguous(), list(wts), [s.contiguous() for s in Ss], offsets, C, len(wts),
                              rows, N, K, G, stream), "w4a16_grouped_gemm")
    return C


def device_status(clear: bool = True) -> int:
    return w4a16_device_status(clear)
