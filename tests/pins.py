"""Pins of the CPU oracle: checks against things other than the oracle itself.

Each `pin_*` takes a compiled oracle (the real one, or a planted-mistake
mutant) and returns True when the oracle agrees with what the binary16 format,
the packing rule, exact arithmetic or a library routine fixes. The pytest
wrappers in test_oracle_pins.py assert each one on the real oracle; the mutant
test asserts that every planted mistake makes at least one of them fail.
"""
from __future__ import annotations

import json
import os

import numpy as np

import workloads
from oracle import exact

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def python_pack(q: np.ndarray) -> np.ndarray:
    """The canonical packing rule, written independently for cross-checks."""
    K, N = q.shape
    out = np.zeros(((K + 1) // 2, N), dtype=np.uint8)
    u = q.astype(np.int16) & 0xF
    out[:] = u[0::2]
    if K > 1:
        out[: K // 2] |= (u[1::2] << 4).astype(np.uint8)
    return out


def decode_tiled(wt: np.ndarray, K: int, N: int) -> np.ndarray:
    """Read every code back out of the tiled layout by its position formula."""
    KT = (K + 63) // 64
    perm = (0, 2, 4, 6, 1, 3, 5, 7)
    pos = {r: i for i, r in enumerate(perm)}
    q = np.zeros((K, N), dtype=np.int8)
    for k in range(K):
        kt, kl = divmod(k, 64)
        h, r32 = divmod(kl, 32)
        w, r = divmod(r32, 8)
        i = pos[r]
        for n in range(N):
            nt, j = divmod(n, 128)
            b = int(wt[(nt * KT + kt) * 4096 + h * 2048 + j * 16 + w * 4 + i // 2])
            v = (b >> 4) if (i & 1) else (b & 0xF)
            q[k, n] = v - 16 if v >= 8 else v
    return q


# ---------------------------------------------------------------- binary16

def pin_half_widening(o) -> bool:
    """All 65536 binary16 patterns widen exactly as numpy's float16 -> float64 does."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    for b in range(0, 65536, 1):
        got = o.half_to_double(b)
        r = ref[b]
        if np.isnan(r):
            if not np.isnan(got):
                return False
        elif got != r or np.signbit(got) != np.signbit(r):
            return False
    return True


def _rounding_probe_values(seed=7):
    """Doubles at, just above and just below binary16 rounding ties, plus random ones."""
    g = np.random.Generator(np.random.PCG64(seed))
    h = g.integers(0, 0x7BFF, size=3000).astype(np.uint16)  # finite positive patterns
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2.0  # exact in double
    vals = [mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf), lo, -mid,
            g.standard_normal(2000) * 10.0 ** g.integers(-9, 5, size=2000)]
    return np.concatenate(vals)


def pin_half_rounding(o) -> bool:
    """double -> binary16 agrees with exact integer RNE on ties and near-ties."""
    for x in _rounding_probe_values():
        x = float(x)
        if not np.isfinite(x) or x == 0.0:
            continue
        m, e = np.frexp(x)
        # x = mant * 2^(e-53) exactly, mant an integer
        mant = int(np.ldexp(m, 53))
        want = exact.round_units_to_half(mant, int(e) - 53)
        if o.double_to_half(x) != want:
            return False
    return True


def pin_half_rounding_numpy(o) -> bool:
    """double -> binary16 agrees with numpy's direct float64 -> float16 cast."""
    vals = _rounding_probe_values(seed=8)
    want = vals.astype(np.float16).view(np.uint16)
    return all(o.double_to_half(float(x)) == int(w) for x, w in zip(vals, want))


# ----------------------------------------------------------------- packing

def pin_pack_golden(o) -> bool:
    rows = _read_table("pack_bytes.txt")
    q = np.array([[int(r[0]) for r in rows], [int(r[1]) for r in rows]], dtype=np.int8)
    want = np.array([int(r[2], 16) for r in rows], dtype=np.uint8)
    return bool(np.array_equal(o.pack(q)[0], want))


def pin_pack_all_bytes(o) -> bool:
    """Every byte value unpacks to two codes in [-8, 7] and packs back to itself."""
    wp = np.arange(256, dtype=np.uint8).reshape(1, 256)
    q = o.unpack(wp, 2)
    if q.min() < -8 or q.max() > 7:
        return False
    if not np.array_equal(o.pack(q), wp):
        return False
    # low nibble is the even row, as a two's-complement nibble
    lo = np.arange(256) & 0xF
    return bool(np.array_equal(q[0], np.where(lo >= 8, lo - 16, lo)))


def pin_pack_random_odd_k(o) -> bool:
    """Random codes with odd K: pack equals the independent rule, unpack inverts it."""
    g = np.random.Generator(np.random.PCG64(5))
    q = g.integers(-8, 8, size=(37, 29), dtype=np.int8)
    wp = o.pack(q)
    if not np.array_equal(wp, python_pack(q)):
        return False
    if np.any(wp[-1] >> 4):  # no odd row beyond K
        return False
    return bool(np.array_equal(o.unpack(wp, 37), q))


def pin_tiled_positions(o) -> bool:
    """A single code lands at the byte and nibble its position formula gives."""
    K, N = 100, 200
    for k, n, byte, half in _read_table("tiled_positions.txt"):
        q = np.zeros((K, N), dtype=np.int8)
        q[int(k), int(n)] = 5
        wt = o.tile(q)
        nz = np.nonzero(wt)[0]
        want = 0x05 if half == "low" else 0x50
        if len(nz) != 1 or nz[0] != int(byte) or wt[nz[0]] != want:
            return False
    return True


def pin_tiled_roundtrip(o) -> bool:
    """Random codes, ragged K and N: decoding the tiles by formula returns q."""
    g = np.random.Generator(np.random.PCG64(6))
    q = g.integers(-8, 8, size=(72, 136), dtype=np.int8)
    wt = o.tile(q)
    return len(wt) == o.tiled_bytes(72, 136) == 2 * 2 * 4096 and \
        bool(np.array_equal(decode_tiled(wt, 72, 136), q))


# ----------------------------------------------------------------- product

def pin_exact_small(o) -> bool:
    """Bit-exact against the integer brute force on small ragged shapes."""
    for (M, K, N, G, seed) in [(3, 40, 9, 16, 1), (2, 65, 7, 13, 2), (4, 96, 16, 32, 3),
                               (1, 7, 5, 3, 4)]:
        c = workloads.dense(M, K, N, G, seed)
        got = o.gemm(c.A, python_pack(c.q), c.S, K, G)
        want = exact.gemm_exact(c.A, c.q, c.S, G)
        if not np.array_equal(got.view(np.uint16), want.view(np.uint16)):
            return False
    return True


def pin_exact_tiny_config(o, cols=None) -> bool:
    """Bit-exact against the integer brute force on the tiny config (4x512x512, G=128)."""
    c = workloads.make("tiny")
    cols = slice(None) if cols is None else cols
    q = c.q[:, cols]
    S = c.S[:, cols]
    got = o.gemm(c.A, python_pack(q), S, c.K, c.G)
    want = exact.gemm_exact(c.A, q, S, c.G)
    return bool(np.array_equal(got.view(np.uint16), want.view(np.uint16)))


def pin_near_ties(o) -> bool:
    with open(os.path.join(GOLDEN, "near_ties.json")) as f:
        cases = json.load(f)["cases"]
    for cs in cases:
        K, G = cs["K"], cs["G"]
        A = np.array([cs["A"]], dtype=np.float16).reshape(cs["M"], K)
        q = np.array(cs["q"], dtype=np.int8)
        S = np.array(cs["S"], dtype=np.float16)
        got = o.gemm(A, python_pack(q), S, K, G).view(np.uint16)
        want = np.array([[int(x, 16) for x in row] for row in cs["C_bits"]], dtype=np.uint16)
        if not np.array_equal(got, want):
            return False
    return True


def pin_closed_form(o) -> bool:
    """Constant q and s: C[m, n] = fp16(q * s * sum_k A[m, k]) for every n."""
    M, K, N, G = 3, 192, 6, 64
    g = np.random.Generator(np.random.PCG64(9))
    A = g.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    for qv, sv in [(-3, 0.0107421875), (7, 0.003), (-8, 0.019)]:
        s16 = np.float16(sv)
        q = np.full((K, N), qv, dtype=np.int8)
        S = np.full((-(-K // G), N), s16, dtype=np.float16)
        got = o.gemm(A, python_pack(q), S, K, G).view(np.uint16)
        s_units = exact.half_to_units(int(np.array(s16).view(np.uint16)))
        for m in range(M):
            row_units = sum(exact.half_to_units(int(b)) for b in A[m].view(np.uint16))
            want = exact.round_units_to_half(row_units * qv * s_units, -48)
            if not np.all(got[m] == want):
                return False
    return True


def pin_one_hot(o) -> bool:
    """s = 1 and q[k, n] = 1 only at k = pi(n): C[m, n] = A[m, pi(n)] exactly."""
    M, K, N, G = 5, 130, 12, 64
    g = np.random.Generator(np.random.PCG64(10))
    A = g.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    # even and odd rows, rows in the second byte of a group, the last row
    pi = np.array([0, 1, 2, 3, 63, 64, 65, 127, 128, 129, 77, 30])
    q = np.zeros((K, N), dtype=np.int8)
    q[pi, np.arange(N)] = 1
    S = np.ones((-(-K // G), N), dtype=np.float16)
    got = o.gemm(A, python_pack(q), S, K, G)
    return bool(np.array_equal(got.view(np.uint16), A[:, pi].view(np.uint16)))


def pin_scale_duplication(o) -> bool:
    """G = K with scale row s0 equals G = 64 and G = 128 with s0 repeated in every group."""
    M, K, N = 3, 256, 10
    c = workloads.dense(M, K, N, K, 11)
    wp = python_pack(c.q)
    base = o.gemm(c.A, wp, c.S, K, K)
    for G in (64, 128):
        S = np.repeat(c.S, K // G, axis=0)
        if not np.array_equal(o.gemm(c.A, wp, S, K, G).view(np.uint16), base.view(np.uint16)):
            return False
    # and a single nonzero-scale group selects exactly that group's rows
    G = 64
    S = np.zeros((K // G, N), dtype=np.float16)
    S[2] = c.S[0]
    q2 = c.q.copy()
    q2[:128] = 0
    q2[192:] = 0
    want = o.gemm(c.A, python_pack(q2), c.S, K, K)
    return bool(np.array_equal(o.gemm(c.A, wp, S, K, G).view(np.uint16), want.view(np.uint16)))


def dequant_numpy(q: np.ndarray, S: np.ndarray, G: int) -> np.ndarray:
    """float64 dequantised weights from the int8 codes, without the oracle."""
    rows = np.arange(q.shape[0]) // G
    return q.astype(np.float64) * S.astype(np.float64)[rows]


def pin_numpy_blas(o) -> bool:
    """numpy float64 matmul of the dequantised weights, rounded to fp16, agrees to 1 ulp."""
    c = workloads.dense(6, 320, 48, 64, 12)
    got = o.gemm(c.A, python_pack(c.q), c.S, c.K, c.G).view(np.uint16).astype(np.int32)
    ref = (c.A.astype(np.float64) @ dequant_numpy(c.q, c.S, c.G)).astype(np.float16)
    want = ref.view(np.uint16).astype(np.int32)
    # same sign, at most one step apart in the ordered binary16 encoding
    return bool(np.all(np.abs(got - want) <= 1))


def pin_grouped_segments(o) -> bool:
    """Grouped form: each segment (an empty expert included) equals the plain product on its
    rows, and E=1 with one segment over all rows is the plain product."""
    c = workloads.grouped(E=4, top_k=2, tokens=9, K=64, N=24, G=32, seed=13, empty_experts=[2])
    wps = [python_pack(c.q[e]) for e in range(c.E)]
    sentinel = np.full((c.total_rows, c.N), np.float16(-7.5))
    got = o.grouped_gemm(c.A, wps, list(c.S), c.offsets, c.K, c.G, C=sentinel)
    if c.offsets[2] != c.offsets[3]:
        return False
    for e in range(c.E):
        r0, r1 = c.offsets[e], c.offsets[e + 1]
        if r1 > r0:
            want = o.gemm(c.A[r0:r1], wps[e], c.S[e], c.K, c.G)
            if not np.array_equal(got[r0:r1].view(np.uint16), want.view(np.uint16)):
                return False
    one = o.grouped_gemm(c.A, wps[:1], [c.S[0]], np.array([0, c.total_rows]), c.K, c.G)
    plain = o.gemm(c.A, wps[0], c.S[0], c.K, c.G)
    if not np.array_equal(one.view(np.uint16), plain.view(np.uint16)):
        return False
    return True


def pin_grouped_brute(o) -> bool:
    """Grouped form against the integer brute force on each expert's rows."""
    c = workloads.grouped(E=3, top_k=1, tokens=7, K=48, N=10, G=16, seed=14)
    wps = [python_pack(c.q[e]) for e in range(c.E)]
    got = o.grouped_gemm(c.A, wps, list(c.S), c.offsets, c.K, c.G)
    for e in range(c.E):
        r0, r1 = c.offsets[e], c.offsets[e + 1]
        if r1 > r0:
            want = exact.gemm_exact(c.A[r0:r1], c.q[e], c.S[e], c.G)
            if not np.array_equal(got[r0:r1].view(np.uint16), want.view(np.uint16)):
                return False
    return True


def pin_sample_matches_full(o) -> bool:
    """The one-by-one sampler returns the same elements as the full product."""
    c = workloads.dense(5, 200, 33, 40, 15)
    wp = python_pack(c.q)
    full = o.gemm(c.A, wp, c.S, c.K, c.G)
    rows = [0, 4, 2, 3, 1, 4]
    cols = [0, 32, 17, 5, 31, 1]
    got = o.gemm_sample(c.A, wp, c.S, c.K, c.G, rows, cols)
    return bool(np.array_equal(got.view(np.uint16), full[rows, cols].view(np.uint16)))


def _read_quantize_example(name="quantize_example.txt"):
    path = os.path.join(GOLDEN, name)
    sections, cur, dims = {}, None, {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] in ("K", "N", "G"):
                dims[parts[0]] = int(parts[1])
            elif parts[0] in ("W", "S", "Q"):
                cur = parts[0]
                sections[cur] = []
            else:
                sections[cur].append([float(x) for x in parts])
    return dims, {k: np.array(v) for k, v in sections.items()}


def pin_quantize_golden(o) -> bool:
    """The hand-worked example: scales bit for bit, codes exactly (a tie rounds away from zero)."""
    dims, t = _read_quantize_example()
    W = t["W"].astype(np.float16)
    wp, S = o.quantize(W, dims["G"])
    q = o.unpack(wp, dims["K"])
    return (bool(np.array_equal(S.view(np.uint16), t["S"].astype(np.float16).view(np.uint16)))
            and bool(np.array_equal(q, t["Q"].astype(np.int8))))


def _quantize_case(seed=21, K=200, N=24, G=64):
    g = np.random.Generator(np.random.PCG64(seed))
    W = (g.standard_normal((K, N)) * g.uniform(0.01, 3.0, size=(1, N))).astype(np.float16)
    return W, K, N, G


def pin_quantize_properties(o) -> bool:
    """Codes in [-8, 7]; each group's largest |w| gets code +-7; |q s - w| <= s / 2 for every
    weight (the rounding bound, with room for the float division); a partial last group."""
    W, K, N, G = _quantize_case()
    wp, S = o.quantize(W, G)
    q = o.unpack(wp, K).astype(np.float64)
    s = S.astype(np.float64)
    w = W.astype(np.float64)
    if q.min() < -8 or q.max() > 7:
        return False
    for g in range((K + G - 1) // G):
        rows = slice(g * G, min(K, g * G + G))
        for n in range(N):
            col = w[rows, n]
            if s[g, n] <= 0.0:
                return False
            i = int(np.argmax(np.abs(col)))
            if abs(q[rows, n][i]) != 7 or np.sign(q[rows, n][i]) != np.sign(col[i]):
                return False
            if np.max(np.abs(q[rows, n] * s[g, n] - col)) > s[g, n] * (0.5 + 1e-6):
                return False
    return True


def pin_quantize_scale_invariance(o) -> bool:
    """Doubling every weight doubles every scale exactly and leaves the codes unchanged."""
    W, K, N, G = _quantize_case(seed=22)
    wp1, S1 = o.quantize(W, G)
    wp2, S2 = o.quantize((W.astype(np.float32) * 2).astype(np.float16), G)
    return (bool(np.array_equal(wp1, wp2))
            and bool(np.array_equal(S2.astype(np.float32), 2 * S1.astype(np.float32))))


def pin_quantize_groups_independent(o) -> bool:
    """Changing one group's rows changes only that group's codes and scales; an all-zero group
    gets scale 0 and codes 0."""
    W, K, N, G = _quantize_case(seed=23)
    wp1, S1 = o.quantize(W, G)
    W2 = W.copy()
    W2[G:2 * G] = 0
    wp2, S2 = o.quantize(W2, G)
    q1, q2 = o.unpack(wp1, K), o.unpack(wp2, K)
    other = np.ones(K, dtype=bool)
    other[G:2 * G] = False
    return (bool(np.array_equal(q1[other], q2[other])) and bool(np.all(q2[G:2 * G] == 0))
            and bool(np.all(S2[1] == 0)) and bool(np.array_equal(np.delete(S1, 1, 0), np.delete(S2, 1, 0))))


def pin_quantize_edges(o) -> bool:
    """Odd K: the last packed row's high nibbles are 0. A group whose largest |w| is below
    3.5 * 2^-24 (half the smallest fp16 step, times 7) rounds its scale to 0 and its codes to 0."""
    W = np.array([[0.5, -0.25], [0.125, 1.0], [-1.0, 0.0], [2.0, -3.0], [1.5, 0.75]], dtype=np.float16)
    wp, S = o.quantize(W, 2)
    if wp.shape != (3, 2) or np.any(wp[2] >> 4):
        return False
    tiny = np.array([[2.0 ** -24, -2.0 ** -24], [0.0, 2.0 ** -23]], dtype=np.float16)  # max 2^-23 < 3.5 * 2^-24
    wp_t, S_t = o.quantize(tiny, 2)
    return bool(np.all(S_t.view(np.uint16) == 0)) and bool(np.all(wp_t == 0))


# ----------------------------------------------------- 8-bit codes (W8A16)

def decode_tiled_w8(wt: np.ndarray, K: int, N: int) -> np.ndarray:
    """Read every 8-bit code back out of the W8 tiled layout by its position formula."""
    KT = (K + 63) // 64
    q = np.zeros((K, N), dtype=np.int8)
    k = np.arange(K)[:, None]
    n = np.arange(N)[None, :]
    kl = k % 64
    byte = ((n // 128) * KT + k // 64) * 8192 + (kl // 16) * 2048 + (n % 128) * 16 + kl % 16
    q[:, :] = wt[byte].view(np.int8)
    return q


def pin_w8_tiled_positions(o) -> bool:
    """A single 8-bit code lands at the byte its position formula gives, unchanged."""
    K, N = 100, 200
    for k, n, byte in _read_table("tiled_positions_w8.txt"):
        q = np.zeros((K, N), dtype=np.int8)
        q[int(k), int(n)] = -77
        wt = o.tile_w8(q)
        nz = np.nonzero(wt)[0]
        if len(nz) != 1 or nz[0] != int(byte) or wt[nz[0]] != np.uint8(256 - 77):
            return False
    return len(o.tile_w8(np.zeros((K, N), dtype=np.int8))) == 4 * 8192


def pin_w8_tiled_roundtrip(o) -> bool:
    """Random 8-bit codes, ragged K and N: decoding the tiles by formula returns q, and the
    padding past K and N is zero."""
    g = np.random.Generator(np.random.PCG64(16))
    q = g.integers(-128, 128, size=(72, 136), dtype=np.int8)
    wt = o.tile_w8(q)
    if len(wt) != o.tiled_bytes_w8(72, 136) or len(wt) != 2 * 2 * 8192:
        return False
    ones = o.tile_w8(np.full((72, 136), -1, dtype=np.int8))
    return bool(np.array_equal(decode_tiled_w8(wt, 72, 136), q)) and int(np.count_nonzero(ones)) == 72 * 136


def w8_case(M, K, N, G, seed):
    c = workloads.dense8(M, K, N, G, seed)
    return c.A, c.q, c.S


def pin_w8_exact_small(o) -> bool:
    """8-bit codes: bit-exact against the integer brute force on small ragged shapes, with
    the extreme codes -128 and 127 present."""
    for (M, K, N, G, seed) in [(3, 40, 9, 16, 1), (2, 65, 7, 13, 2), (4, 96, 16, 32, 3), (1, 7, 5, 3, 4)]:
        A, q, S = w8_case(M, K, N, G, seed)
        q = q.copy()
        q[0, 0], q[-1, -1] = -128, 127
        got = o.gemm_w8(A, q, S, K, G)
        want = exact.gemm_exact(A, q, S, G)
        if not np.array_equal(got.view(np.uint16), want.view(np.uint16)):
            return False
    return True


def pin_w8_closed_form(o) -> bool:
    """Constant 8-bit codes and scale: C[m, n] = fp16(q * s * sum_k A[m, k])."""
    M, K, N, G = 3, 192, 6, 64
    g = np.random.Generator(np.random.PCG64(19))
    A = g.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    for qv, sv in [(-128, 0.0001220703125), (127, 0.00031), (-1, 0.019)]:
        s16 = np.float16(sv)
        q = np.full((K, N), qv, dtype=np.int8)
        S = np.full((-(-K // G), N), s16, dtype=np.float16)
        got = o.gemm_w8(A, q, S, K, G).view(np.uint16)
        s_units = exact.half_to_units(int(np.array(s16).view(np.uint16)))
        for m in range(M):
            row_units = sum(exact.half_to_units(int(b)) for b in A[m].view(np.uint16))
            want = exact.round_units_to_half(row_units * qv * s_units, -48)
            if not np.all(got[m] == want):
                return False
    return True


def pin_w8_one_hot(o) -> bool:
    """q = -128 only at k = pi(n), s = 2^-7: each weight is -1, so C[m, n] = -A[m, pi(n)] exactly."""
    M, K, N, G = 5, 130, 12, 64
    g = np.random.Generator(np.random.PCG64(20))
    A = g.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    pi = np.array([0, 1, 15, 16, 63, 64, 65, 127, 128, 129, 77, 30])
    q = np.zeros((K, N), dtype=np.int8)
    q[pi, np.arange(N)] = -128
    S = np.full((-(-K // G), N), 2.0 ** -7, dtype=np.float16)
    got = o.gemm_w8(A, q, S, K, G)
    return bool(np.array_equal(got.view(np.uint16), (-A[:, pi]).view(np.uint16)))


def pin_w8_numpy_blas(o) -> bool:
    """numpy float64 matmul of the dequantised 8-bit weights, rounded to fp16, agrees to 1 ulp."""
    A, q, S = w8_case(6, 320, 48, 64, 22)
    got = o.gemm_w8(A, q, S, 320, 64).view(np.uint16).astype(np.int32)
    ref = (A.astype(np.float64) @ dequant_numpy(q, S, 64)).astype(np.float16)
    return bool(np.all(np.abs(got - ref.view(np.uint16).astype(np.int32)) <= 1))


def pin_quantize_w8_golden(o) -> bool:
    """The hand-worked 8-bit example: scales bit for bit (one just above the smallest normal
    fp16), codes exactly (an exact half rounds away from zero, an all-zero group gives 0)."""
    dims, t = _read_quantize_example("quantize_w8_example.txt")
    W = t["W"].astype(np.float16)
    q8, S = o.quantize_w8(W, dims["G"])
    return (bool(np.array_equal(S.view(np.uint16), t["S"].astype(np.float16).view(np.uint16)))
            and bool(np.array_equal(q8, t["Q"].astype(np.int8))))


def pin_quantize_w8_properties(o) -> bool:
    """Random weights: codes within [-127, 127]; each group's largest |w| gets +-127; every
    code reconstructs its weight within half a scale step; 2W gives 2s and the same codes."""
    W, K, N, G = _quantize_case(seed=24)
    q8, S = o.quantize_w8(W, G)
    s = S.astype(np.float64)[np.arange(K) // G]
    w = W.astype(np.float64)
    if q8.min() < -127 or q8.max() > 127:
        return False
    if np.any(np.abs(q8 * s - w) > s / 2 * (1 + 1e-6)):
        return False
    for g in range(-(-K // G)):
        rows = slice(g * G, min(K, (g + 1) * G))
        top = np.argmax(np.abs(w[rows]), axis=0)
        if not np.all(np.abs(q8[rows][top, np.arange(N)]) == 127):
            return False
    q2, S2 = o.quantize_w8((2 * W.astype(np.float32)).astype(np.float16), G)
    return bool(np.array_equal(q2, q8)) and bool(np.array_equal(S2.astype(np.float64), 2 * S.astype(np.float64)))


PINS = [pin_half_widening, pin_half_rounding, pin_half_rounding_numpy, pin_pack_golden,
        pin_pack_all_bytes, pin_pack_random_odd_k, pin_tiled_positions, pin_tiled_roundtrip,
        pin_exact_small, pin_near_ties, pin_closed_form, pin_one_hot, pin_scale_duplication,
        pin_numpy_blas, pin_grouped_segments, pin_grouped_brute, pin_sample_matches_full,
        pin_quantize_golden, pin_quantize_properties, pin_quantize_scale_invariance,
        pin_quantize_groups_independent, pin_quantize_edges, pin_w8_tiled_positions, pin_w8_tiled_roundtrip,
        pin_w8_exact_small, pin_w8_closed_form, pin_w8_one_hot, pin_w8_numpy_blas, pin_quantize_w8_golden,
        pin_quantize_w8_properties]
