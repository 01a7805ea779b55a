"""CPU oracle for the W4A16 group-wise GEMM — TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s CPU-baseline leg may
import this package. The CUDA library never calls it, and it never calls the
CUDA library: the two share nothing but the seeded input generators in
`workloads`.

`w4a16_oracle.c` holds the arithmetic (fp64 accumulation, one direct
round-to-nearest-even to fp16); this module compiles it with gcc into
`_liboracle.so` next to the source and marshals numpy arrays through ctypes.
`exact.py` is an independent brute force in exact integer arithmetic that pins
it on small shapes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile
from typing import Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "w4a16_oracle.c")
LIB = os.path.join(HERE, "_liboracle.so")

_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i8p = ctypes.POINTER(ctypes.c_int8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def compile_oracle(out: str = LIB, mutant: int = 0) -> str:
    """Compile the C oracle (optionally one planted-mistake mutant) to `out`."""
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", f"-DORACLE_MUTANT={int(mutant)}", SRC, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    os.replace(out + ".tmp", out)
    return out


def _needs_build(path: str) -> bool:
    return not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(SRC)


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _bits(a: np.ndarray) -> np.ndarray:
    """float16 array -> its uint16 bit patterns (a view, C-contiguous)."""
    a = np.ascontiguousarray(a, dtype=np.float16)
    return a.view(np.uint16)


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_double_to_half.argtypes = [ctypes.c_double]
        lib.oracle_double_to_half.restype = ctypes.c_uint16
        lib.oracle_pack.argtypes = [_i8p, _i64, _i64, _u8p]
        lib.oracle_unpack.argtypes = [_u8p, _i64, _i64, _i8p]
        lib.oracle_tiled_bytes.argtypes = [_i64, _i64]
        lib.oracle_tiled_bytes.restype = _i64
        lib.oracle_tile.argtypes = [_i8p, _i64, _i64, _u8p]
        lib.oracle_gemm.argtypes = [_u16p, _u8p, _u16p, _i64, _i64, _i64, _i64, _u16p, ctypes.c_int]
        lib.oracle_gemm.restype = ctypes.c_int
        lib.oracle_gemm_sample.argtypes = [_u16p, _u8p, _u16p, _i64, _i64, _i64, _i64,
                                           _i64p, _i64p, _i64, _u16p]
        lib.oracle_gemm_sample.restype = ctypes.c_int
        lib.oracle_grouped_gemm.argtypes = [_u16p, ctypes.POINTER(_u8p), ctypes.POINTER(_u16p),
                                            _i32p, _i64, _i64, _i64, _i64, _i64, _u16p, ctypes.c_int]
        lib.oracle_grouped_gemm.restype = ctypes.c_int
        lib.oracle_quantize.argtypes = [_u16p, _i64, _i64, _i64, _u8p, _u16p]
        lib.oracle_quantize.restype = None
        lib.oracle_tiled_bytes_w8.argtypes = [_i64, _i64]
        lib.oracle_tiled_bytes_w8.restype = _i64
        lib.oracle_tile_w8.argtypes = [_i8p, _i64, _i64, _u8p]
        lib.oracle_tile_w8.restype = None
        lib.oracle_gemm_w8.argtypes = [_u16p, _i8p, _u16p, _i64, _i64, _i64, _i64, _u16p, ctypes.c_int]
        lib.oracle_gemm_w8.restype = ctypes.c_int
        lib.oracle_quantize_w8.argtypes = [_u16p, _i64, _i64, _i64, _i8p, _u16p]
        lib.oracle_quantize_w8.restype = None
        lib.oracle_threads.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    # -- binary16 ---------------------------------------------------------
    def half_to_double(self, bits: int) -> float:
        return self.lib.oracle_half_to_double(int(bits))

    def double_to_half(self, x: float) -> int:
        return int(self.lib.oracle_double_to_half(float(x)))

    def threads(self) -> int:
        return int(self.lib.oracle_threads())

    # -- encodings --------------------------------------------------------
    def pack(self, q: np.ndarray) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.int8)
        K, N = q.shape
        wp = np.empty(((K + 1) // 2, N), dtype=np.uint8)
        self.lib.oracle_pack(_ptr(q, _i8p), K, N, _ptr(wp, _u8p))
        return wp

    def unpack(self, wp: np.ndarray, K: int) -> np.ndarray:
        wp = np.ascontiguousarray(wp, dtype=np.uint8)
        N = wp.shape[1]
        q = np.empty((K, N), dtype=np.int8)
        self.lib.oracle_unpack(_ptr(wp, _u8p), K, N, _ptr(q, _i8p))
        return q

    def tiled_bytes(self, K: int, N: int) -> int:
        return int(self.lib.oracle_tiled_bytes(K, N))

    def tile(self, q: np.ndarray) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.int8)
        K, N = q.shape
        wt = np.empty(self.tiled_bytes(K, N), dtype=np.uint8)
        self.lib.oracle_tile(_ptr(q, _i8p), K, N, _ptr(wt, _u8p))
        return wt

    # -- the product ------------------------------------------------------
    def gemm(self, A: np.ndarray, wp: np.ndarray, S: np.ndarray, K: int, G: int,
             threads: int = 0) -> np.ndarray:
        """C = fp16(A @ dequant(W)) from canonical packed weights."""
        a = _bits(A)
        s = _bits(S)
        wp = np.ascontiguousarray(wp, dtype=np.uint8)
        M = a.shape[0]
        N = wp.shape[1]
        assert a.shape == (M, K) and s.shape == (-(-K // G), N)
        c = np.zeros((M, N), dtype=np.uint16)
        rc = self.lib.oracle_gemm(_ptr(a, _u16p), _ptr(wp, _u8p), _ptr(s, _u16p), M, N, K, G,
                                  _ptr(c, _u16p), int(threads))
        if rc:
            raise RuntimeError(f"oracle_gemm failed ({rc})")
        return c.view(np.float16)

    def gemm_sample(self, A: np.ndarray, wp: np.ndarray, S: np.ndarray, K: int, G: int,
                    rows: Sequence[int], cols: Sequence[int]) -> np.ndarray:
        a = _bits(A)
        s = _bits(S)
        wp = np.ascontiguousarray(wp, dtype=np.uint8)
        r = np.ascontiguousarray(rows, dtype=np.int64)
        c = np.ascontiguousarray(cols, dtype=np.int64)
        out = np.zeros(len(r), dtype=np.uint16)
        rc = self.lib.oracle_gemm_sample(_ptr(a, _u16p), _ptr(wp, _u8p), _ptr(s, _u16p),
                                         a.shape[0], wp.shape[1], K, G, _ptr(r, _i64p),
                                         _ptr(c, _i64p), len(r), _ptr(out, _u16p))
        if rc:
            raise RuntimeError(f"oracle_gemm_sample failed ({rc})")
        return out.view(np.float16)

    def grouped_gemm(self, A: np.ndarray, wps: Sequence[np.ndarray], Ss: Sequence[np.ndarray],
                     offsets: np.ndarray, K: int, G: int, C: Optional[np.ndarray] = None,
                     threads: int = 0) -> np.ndarray:
        a = _bits(A)
        E = len(wps)
        wps = [np.ascontiguousarray(w, dtype=np.uint8) for w in wps]
        ss = [_bits(s) for s in Ss]
        N = wps[0].shape[1]
        off = np.ascontiguousarray(offsets, dtype=np.int32)
        total = a.shape[0]
        if C is None:
            c = np.zeros((total, N), dtype=np.uint16)
        else:
            c = np.ascontiguousarray(C).view(np.uint16).copy()
        wp_arr = (_u8p * E)(*[_ptr(w, _u8p) for w in wps])
        s_arr = (_u16p * E)(*[_ptr(s, _u16p) for s in ss])
        rc = self.lib.oracle_grouped_gemm(_ptr(a, _u16p), wp_arr, s_arr, _ptr(off, _i32p), E,
                                          total, N, K, G, _ptr(c, _u16p), int(threads))
        if rc:
            raise RuntimeError(f"oracle_grouped_gemm failed ({rc})")
        return c.view(np.float16)


    # -- the 8-bit code variant (W8A16) ----------------------------------
    def tiled_bytes_w8(self, K: int, N: int) -> int:
        return int(self.lib.oracle_tiled_bytes_w8(K, N))

    def tile_w8(self, q8: np.ndarray) -> np.ndarray:
        q8 = np.ascontiguousarray(q8, dtype=np.int8)
        K, N = q8.shape
        wt = np.empty(self.tiled_bytes_w8(K, N), dtype=np.uint8)
        self.lib.oracle_tile_w8(_ptr(q8, _i8p), K, N, _ptr(wt, _u8p))
        return wt

    def gemm_w8(self, A: np.ndarray, q8: np.ndarray, S: np.ndarray, K: int, G: int,
                threads: int = 0) -> np.ndarray:
        """C = fp16(A @ (q8 * s)) for signed 8-bit codes q8 [K, N]."""
        a = _bits(A)
        s = _bits(S)
        q8 = np.ascontiguousarray(q8, dtype=np.int8)
        M = a.shape[0]
        N = q8.shape[1]
        assert a.shape == (M, K) and q8.shape == (K, N) and s.shape == (-(-K // G), N)
        c = np.zeros((M, N), dtype=np.uint16)
        rc = self.lib.oracle_gemm_w8(_ptr(a, _u16p), _ptr(q8, _i8p), _ptr(s, _u16p), M, N, K, G,
                                     _ptr(c, _u16p), int(threads))
        if rc:
            raise RuntimeError(f"oracle_gemm_w8 failed ({rc})")
        return c.view(np.float16)

    def quantize_w8(self, W: np.ndarray, G: int):
        """Group-wise 8-bit quantisation of fp16 W [K, N]: (int8 codes [K, N], fp16 scales)."""
        w = _bits(W)
        K, N = w.shape
        q8 = np.zeros((K, N), dtype=np.int8)
        S = np.zeros(((K + G - 1) // G, N), dtype=np.uint16)
        self.lib.oracle_quantize_w8(_ptr(w, _u16p), K, N, G, _ptr(q8, _i8p), _ptr(S, _u16p))
        return q8, S.view(np.float16)

    def quantize(self, W: np.ndarray, G: int):
        """Group-wise int4 quantisation of fp16 W [K, N]: (canonical packed codes, fp16 scales)."""
        w = _bits(W)
        K, N = w.shape
        wp = np.zeros(((K + 1) // 2, N), dtype=np.uint8)
        S = np.zeros(((K + G - 1) // G, N), dtype=np.uint16)
        self.lib.oracle_quantize(_ptr(w, _u16p), K, N, G, _ptr(wp, _u8p), _ptr(S, _u16p))
        return wp, S.view(np.float16)


_default: Optional[Oracle] = None


def load() -> Oracle:
    """The oracle library, compiled next to its source if missing or stale."""
    global _default
    if _default is None:
        if _needs_build(LIB):
            compile_oracle(LIB)
        _default = Oracle(LIB)
    return _default


def load_mutant(mutant: int, directory: Optional[str] = None) -> Oracle:
    """A copy of the oracle with planted mistake number `mutant` (tests only)."""
    directory = directory or tempfile.mkdtemp(prefix="oracle_mutant_")
    path = os.path.join(directory, f"_liboracle_m{mutant}.so")
    compile_oracle(path, mutant)
    return Oracle(path)
