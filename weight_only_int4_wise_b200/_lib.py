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
ERR_BAD_ROUTING = 7
ERR_SCRATCH_TOO_SMALL = 8
MAX_EXPERTS = 64
MAX_TOPK = 8
FLAG_STATIC_WEIGHTS = 1
ACT_IDENTITY = 0
ACT_RELU = 1
ACT_GELU_ERF = 2
ACT_GELU_TANH = 3

EXPORTED = [
    "w4a16_status_string", "w4a16_pack", "w4a16_unpack", "w4a16_tiled_bytes", "w4a16_repack",
    "w4a16_gemm", "w4a16_grouped_gemm", "w4a16_gemm_launch_info", "w4a16_grouped_launch_info",
    "w4a16_device_status", "w4a16_set_static_weights", "w4a16_quantize", "w4a16_set_fault_injection",
    "w4a16_grouped_gemm_act", "w4a16_moe_route", "w4a16_moe_dispatch", "w4a16_moe_gather", "w4a16_moe_combine",
    "w4a16_moe_workspace_size", "w4a16_moe_layer", "w4a16_get_valid_tactics", "w4a16_tactic_launch_info",
    "w4a16_set_tactic", "w4a16_get_tactic", "w4a16_clear_tactics", "w4a16_autotune",
    "w8a16_tiled_bytes", "w8a16_repack", "w8a16_gemm", "w8a16_gemm_launch_info",
    "w4a16_moe_layer_static", "w4a16_moe_static_scratch_bytes", "w4a16_gemm_ex", "w8a16_quantize",
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
        lib.w4a16_gemm_ex.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.c_uint32, _vp]
        lib.w4a16_gemm_ex.restype = ctypes.c_int
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
        lib.w4a16_grouped_gemm_act.argtypes = [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp, _vp, _i64,
                                               _i64, _i64, _i64, _i64, ctypes.c_int, _vp]
        lib.w4a16_grouped_gemm_act.restype = ctypes.c_int
        lib.w4a16_moe_route.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _vp]
        lib.w4a16_moe_route.restype = ctypes.c_int
        lib.w4a16_moe_dispatch.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]
        lib.w4a16_moe_dispatch.restype = ctypes.c_int
        lib.w4a16_moe_gather.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _vp]
        lib.w4a16_moe_gather.restype = ctypes.c_int
        lib.w4a16_moe_combine.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]
        lib.w4a16_moe_combine.restype = ctypes.c_int
        lib.w4a16_moe_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i64]
        lib.w4a16_moe_workspace_size.restype = _i64
        lib.w4a16_moe_layer.argtypes = [_vp, _vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                        ctypes.POINTER(_vp), _vp, _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_int,
                                        _vp, _i64, _vp]
        lib.w4a16_moe_layer.restype = ctypes.c_int
        lib.w4a16_moe_layer_static.argtypes = [_vp, _vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                               ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp, _i64, _i64, _i64,
                                               _i64, _i64, _i64, ctypes.c_int, _vp]
        lib.w4a16_moe_layer_static.restype = ctypes.c_int
        lib.w4a16_moe_static_scratch_bytes.argtypes = []
        lib.w4a16_moe_static_scratch_bytes.restype = _i64
        lib.w8a16_quantize.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _vp]
        lib.w8a16_quantize.restype = ctypes.c_int
        lib.w8a16_tiled_bytes.argtypes = [_i64, _i64]
        lib.w8a16_tiled_bytes.restype = _i64
        lib.w8a16_repack.argtypes = [_vp, _vp, _i64, _i64, _vp]
        lib.w8a16_repack.restype = ctypes.c_int
        lib.w8a16_gemm.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp]
        lib.w8a16_gemm.restype = ctypes.c_int
        lib.w8a16_gemm_launch_info.argtypes = [_i64, _i64, _i64, _i64, ctypes.POINTER(LaunchInfo)]
        lib.w8a16_gemm_launch_info.restype = ctypes.c_int
        _i32p = ctypes.POINTER(ctypes.c_int32)
        lib.w4a16_get_valid_tactics.argtypes = [_i64, _i64, _i64, _i64, _i32p, ctypes.c_int32, _i32p]
        lib.w4a16_get_valid_tactics.restype = ctypes.c_int
        lib.w4a16_tactic_launch_info.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int32, ctypes.POINTER(LaunchInfo)]
        lib.w4a16_tactic_launch_info.restype = ctypes.c_int
        lib.w4a16_set_tactic.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int32]
        lib.w4a16_set_tactic.restype = ctypes.c_int
        lib.w4a16_get_tactic.argtypes = [_i64, _i64, _i64, _i64, _i32p]
        lib.w4a16_get_tactic.restype = ctypes.c_int
        lib.w4a16_clear_tactics.argtypes = []
        lib.w4a16_clear_tactics.restype = ctypes.c_int
        lib.w4a16_autotune.argtypes = [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.c_int32, _vp, _i64, _i64,
                                       _i64, _i64, ctypes.c_int32, _i32p, ctypes.POINTER(ctypes.c_float),
                                       ctypes.POINTER(ctypes.c_float), ctypes.c_int32, _vp]
        lib.w4a16_autotune.restype = ctypes.c_int
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


def w4a16_gemm_ex(A, Wt, S, C, M: int, N: int, K: int, G: int, flags: int, stream=None) -> int:
    return load().w4a16_gemm_ex(_addr(A), _addr(Wt), _addr(S), _addr(C), M, N, K, G, flags, _stream(stream))


def w4a16_grouped_gemm(A, Wt: Sequence, S: Sequence, offsets, C, E: int, total_rows: int, N: int, K: int,
                       G: int, stream=None) -> int:
    wt_arr = (_vp * max(1, len(Wt)))(*[_addr(w) for w in Wt])
    s_arr = (_vp * max(1, len(S)))(*[_addr(s) for s in S])
    return load().w4a16_grouped_gemm(_addr(A), wt_arr, s_arr, _addr(offsets), _addr(C), E, total_rows, N, K, G,
                                     _stream(stream))


def _ptr_array(xs: Sequence):
    return (_vp * max(1, len(xs)))(*[_addr(x) for x in xs])


def w4a16_grouped_gemm_act(A, Wt: Sequence, S: Sequence, offsets, C, E: int, total_rows: int, N: int, K: int,
                           G: int, act: int, stream=None) -> int:
    return load().w4a16_grouped_gemm_act(_addr(A), _ptr_array(Wt), _ptr_array(S), _addr(offsets), _addr(C), E,
                                         total_rows, N, K, G, act, _stream(stream))


def w4a16_moe_route(logits, ids, weights, T: int, E: int, top_k: int, stream=None) -> int:
    return load().w4a16_moe_route(_addr(logits), _addr(ids), _addr(weights), T, E, top_k, _stream(stream))


def w4a16_moe_dispatch(ids, offsets, pos, src_row, T: int, E: int, top_k: int, stream=None) -> int:
    return load().w4a16_moe_dispatch(_addr(ids), _addr(offsets), _addr(pos), _addr(src_row), T, E, top_k,
                                     _stream(stream))


def w4a16_moe_gather(X, src_row, Xg, T: int, rows: int, H: int, stream=None) -> int:
    return load().w4a16_moe_gather(_addr(X), _addr(src_row), _addr(Xg), T, rows, H, _stream(stream))


def w4a16_moe_combine(Y, weights, pos, out, T: int, top_k: int, H: int, stream=None) -> int:
    return load().w4a16_moe_combine(_addr(Y), _addr(weights), _addr(pos), _addr(out), T, top_k, H,
                                    _stream(stream))


def w4a16_moe_workspace_size(T: int, E: int, top_k: int, H: int, I: int) -> int:
    return int(load().w4a16_moe_workspace_size(T, E, top_k, H, I))


def w4a16_moe_layer(X, logits, Wt_up: Sequence, S_up: Sequence, Wt_down: Sequence, S_down: Sequence, out,
                    T: int, E: int, top_k: int, H: int, I: int, G: int, act: int, workspace, workspace_bytes: int,
                    stream=None) -> int:
    return load().w4a16_moe_layer(_addr(X), _addr(logits), _ptr_array(Wt_up), _ptr_array(S_up),
                                  _ptr_array(Wt_down), _ptr_array(S_down), _addr(out), T, E, top_k, H, I, G, act,
                                  _addr(workspace), workspace_bytes, _stream(stream))


def w4a16_get_valid_tactics(M: int, N: int, K: int, G: int):
    """(status, [tactic ids]) for a shape."""
    count = ctypes.c_int32(0)
    arr = (ctypes.c_int32 * 96)()
    rc = load().w4a16_get_valid_tactics(M, N, K, G, arr, 96, ctypes.byref(count))
    return rc, [arr[i] for i in range(min(count.value, 96))]


def w4a16_tactic_launch_info(M: int, N: int, K: int, G: int, tactic: int):
    info = LaunchInfo()
    rc = load().w4a16_tactic_launch_info(M, N, K, G, tactic, ctypes.byref(info))
    return rc, info


def w4a16_set_tactic(M: int, N: int, K: int, G: int, tactic: int) -> int:
    return load().w4a16_set_tactic(M, N, K, G, tactic)


def w4a16_get_tactic(M: int, N: int, K: int, G: int) -> int:
    t = ctypes.c_int32(-1)
    rc = load().w4a16_get_tactic(M, N, K, G, ctypes.byref(t))
    _check(rc, "w4a16_get_tactic")
    return t.value


def w4a16_clear_tactics() -> int:
    return load().w4a16_clear_tactics()


def w4a16_autotune(A, Wts: Sequence, Ss: Sequence, C, M: int, N: int, K: int, G: int, reps: int = 20,
                   stream=None, with_times: bool = False):
    """Times every tactic over the weight copies Wts / Ss (rotating); (status, best tactic id,
    its microseconds per launch[, microseconds of every tactic])."""
    best = ctypes.c_int32(0)
    us = ctypes.c_float(0.0)
    times = (ctypes.c_float * 96)()
    rc = load().w4a16_autotune(_addr(A), _ptr_array(Wts), _ptr_array(Ss), len(Wts), _addr(C), M, N, K, G, reps,
                               ctypes.byref(best), ctypes.byref(us), times, 96, _stream(stream))
    if with_times:
        n = len(w4a16_get_valid_tactics(M, N, K, G)[1])
        return rc, best.value, us.value, [times[i] for i in range(min(n, 96))]
    return rc, best.value, us.value


def w8a16_quantize(W, q8, S, K: int, N: int, G: int, stream=None) -> int:
    return load().w8a16_quantize(_addr(W), _addr(q8), _addr(S), K, N, G, _stream(stream))


def w8a16_tiled_bytes(K: int, N: int) -> int:
    return int(load().w8a16_tiled_bytes(K, N))


def w8a16_repack(q, wt, K: int, N: int, stream=None) -> int:
    return load().w8a16_repack(_addr(q), _addr(wt), K, N, _stream(stream))


def w8a16_gemm(A, Wt8, S, C, M: int, N: int, K: int, G: int, stream=None) -> int:
    return load().w8a16_gemm(_addr(A), _addr(Wt8), _addr(S), _addr(C), M, N, K, G, _stream(stream))


def w8a16_gemm_launch_info(M: int, N: int, K: int, G: int):
    info = LaunchInfo()
    rc = load().w8a16_gemm_launch_info(M, N, K, G, ctypes.byref(info))
    return rc, info


def w4a16_moe_layer_static(X, logits, Wt_up: Sequence, S_up: Sequence, Wt_down: Sequence, S_down: Sequence, out,
                           T: int, E: int, top_k: int, H: int, I: int, G: int, act: int, stream=None) -> int:
    """The expert layer without a workspace argument: its intermediates live in the library's
    static per-device scratch (see include/w4a16.h for the limits and the race between
    overlapping calls)."""
    return load().w4a16_moe_layer_static(_addr(X), _addr(logits), _ptr_array(Wt_up), _ptr_array(S_up),
                                         _ptr_array(Wt_down), _ptr_array(S_down), _addr(out), T, E, top_k, H, I,
                                         G, act, _stream(stream))


def w4a16_moe_static_scratch_bytes() -> int:
    return int(load().w4a16_moe_static_scratch_bytes())


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


def moe_layer(X, logits, wts_up: Sequence, Ss_up: Sequence, wts_down: Sequence, Ss_down: Sequence, top_k: int,
              I: int, G: int, act: int, workspace=None, out=None, stream=None):
    """The INT4 mixture-of-experts layer: out [T, H] from hidden states X [T, H] fp16 and router logits
    [T, E] fp16 with per-expert tiled weights and scales (up: H -> I, down: I -> H). The workspace
    (uint8, at least w4a16_moe_workspace_size bytes) is allocated here when not given."""
    import torch
    _require_cuda(X, logits)
    T, H = X.shape
    E = logits.shape[1]
    need = w4a16_moe_workspace_size(T, E, top_k, H, I)
    if need < 0:
        raise W4A16Error(ERR_INVALID_ARG, "w4a16_moe_workspace_size")
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=X.device)
    C = out if out is not None else torch.empty((T, H), dtype=torch.float16, device=X.device)
    _check(w4a16_moe_layer(X.contiguous(), logits.contiguous(), list(wts_up), [s.contiguous() for s in Ss_up],
                           list(wts_down), [s.contiguous() for s in Ss_down], C, T, E, top_k, H, I, G, act,
                           workspace, workspace.numel(), stream), "w4a16_moe_layer")
    return C


def quantize_w8(W, G: int, stream=None):
    """fp16 weights [K, N] (device) -> (int8 codes [K, N], fp16 scales [ceil(K/G), N]): group-wise
    symmetric 8-bit quantisation."""
    import torch
    _require_cuda(W)
    if W.dtype != torch.float16:
        raise TypeError("W must be float16")
    K, N = W.shape
    q8 = torch.empty((K, N), dtype=torch.int8, device=W.device)
    S = torch.empty(((K + G - 1) // G, N), dtype=torch.float16, device=W.device)
    _check(w8a16_quantize(W.contiguous(), q8, S, K, N, G, stream), "w8a16_quantize")
    return q8, S


def repack_w8(q, stream=None):
    """int8 codes [K, N] (device) -> the 8-bit tiled layout (flat uint8)."""
    import torch
    _require_cuda(q)
    K, N = q.shape
    wt = torch.empty(w8a16_tiled_bytes(K, N), dtype=torch.uint8, device=q.device)
    _check(w8a16_repack(q.contiguous(), wt, K, N, stream), "w8a16_repack")
    return wt


def gemm_w8(A, wt8, S, N: int, G: int, out=None, stream=None):
    """C [M, N] fp16 = A [M, K] fp16 x (8-bit codes in the tiled layout) * scales S."""
    import torch
    _require_cuda(A, wt8, S)
    M, K = A.shape
    C = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(w8a16_gemm(A.contiguous(), wt8, S.contiguous(), C, M, N, K, G, stream), "w8a16_gemm")
    return C


def device_status(clear: bool = True) -> int:
    return w4a16_device_status(clear)
