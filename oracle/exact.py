"""Exact brute force of the W4A16 product, for small shapes — TEST INFRASTRUCTURE ONLY.

Independent of `w4a16_oracle.c`: it reads the int4 codes straight from the
int8 matrix q (no packing), and it never touches floating-point arithmetic.

Every binary16 value is an integer multiple of 2^-24, so each term
A[m,k] * q[k,n] * s[floor(k/G), n] is an integer multiple of 2^-48 and the
whole sum is one exact Python integer T in units of 2^-48. That sum is then
rounded once to binary16 with round-to-nearest, ties-to-even, using integer
arithmetic only (IEEE 754 binary16: 1 sign bit, 5 exponent bits with bias 15,
10 fraction bits; subnormals are multiples of 2^-24; magnitudes at or above
65520 round to infinity).
"""
from __future__ import annotations

import numpy as np


def half_to_units(bits: int) -> int:
    """binary16 bit pattern -> exact value in units of 2^-24 (finite inputs only)."""
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 10) & 0x1F
    f = bits & 0x3FF
    if e == 0x1F:
        raise ValueError("non-finite input")
    if e == 0:
        return sign * f
    return sign * ((1024 + f) << (e - 1))


def round_units_to_half(T: int, unit_exp: int) -> int:
    """Round the exact value T * 2^unit_exp to a binary16 bit pattern (RNE)."""
    sign = 0x8000 if T < 0 else 0
    a = -T if T < 0 else T
    if a == 0:
        return sign

    def rne_shift(x: int, sh: int) -> int:
        """round(x / 2^sh) to nearest, ties to even, for sh >= 0 (else exact)."""
        if sh <= 0:
            return x << (-sh)
        q, r = divmod(x, 1 << sh)
        half = 1 << (sh - 1)
        if r > half or (r == half and (q & 1)):
            q += 1
        return q

    # Largest E with 2^E <= a * 2^unit_exp.
    E = a.bit_length() - 1 + unit_exp
    if E < -14:
        # Subnormal: integer count of 2^-24.
        r = rne_shift(a, -24 - unit_exp)
        return sign | r  # r == 1024 is exactly the smallest normal's pattern
    # Normal: 11 significant bits, value = r * 2^(E-10), r in [1024, 2048].
    r = rne_shift(a, E - 10 - unit_exp)
    if r == 2048:
        r = 1024
        E += 1
    if E > 15:
        return sign | 0x7C00
    return sign | ((E + 15) << 10) | (r - 1024)


def gemm_exact(A: np.ndarray, q: np.ndarray, S: np.ndarray, G: int) -> np.ndarray:
    """C[m, n] = RNE_fp16( sum_k A[m,k] * q[k,n] * S[k // G, n] ), exactly."""
    a = np.ascontiguousarray(A, dtype=np.float16).view(np.uint16)
    s = np.ascontiguousarray(S, dtype=np.float16).view(np.uint16)
    M, K = a.shape
    K2, N = q.shape
    assert K2 == K and s.shape == (-(-K // G), N)
    au = [[half_to_units(int(a[m, k])) for k in range(K)] for m in range(M)]
    su = [[half_to_units(int(s[g, n])) for n in range(N)] for g in range(s.shape[0])]
    out = np.zeros((M, N), dtype=np.uint16)
    for n in range(N):
        w = [int(q[k, n]) * su[k // G][n] for k in range(K)]
        for m in range(M):
            row = au[m]
            T = 0
            for k in range(K):
                T += row[k] * w[k]
            out[m, n] = round_units_to_half(T, -48)
    return out.view(np.float16)
