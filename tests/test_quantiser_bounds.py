"""The numeric facts the GPU quantiser relies on, checked exhaustively on the host.

The kernel takes the code of w with scale s as the nearest integer of
x = w * (1/s) (float products, round to nearest), falls back to the IEEE
quotient near a half-integer, and reads that integer from the low bits of
x + 1.5 * 2^23. For groups whose fp16 scale is 0 or a normal number it leaves
out the clamp to the code range, because then every |w| <= max rounds into it.
These tests check both facts over every fp16 maximum, in float32 arithmetic as
the kernel does it (numpy float32 operations round to nearest even)."""
import numpy as np
import pytest

F32 = np.float32
MIN_NORMAL = F32(2.0 ** -14)


def all_positive_fp16():
    bits = np.arange(1, 0x7C00, dtype=np.uint16)  # every finite positive fp16 value
    return bits.view(np.float16)


@pytest.mark.parametrize("kmax", [7, 127])
def test_normal_scales_keep_every_code_in_range(kmax):
    # the worst case of a group is w = +-max: check x = max * (1/s) and the
    # exact quotient max / s for every fp16 maximum whose scale is normal
    mx = all_positive_fp16().astype(F32)
    s = (mx / F32(kmax)).astype(np.float16)  # float division, then fp16 rounding
    normal = s.astype(F32) >= MIN_NORMAL
    assert normal.sum() > 20000
    sf = s[normal].astype(F32)
    rs = (F32(1.0) / sf).astype(F32)
    x = (mx[normal] * rs).astype(F32)
    q = mx[normal].astype(np.float64) / sf.astype(np.float64)
    assert np.all(x < kmax + 0.5) and np.all(q < kmax + 0.5)
    assert float(x.max()) < kmax * (1 + 2.0 ** -10)
    # below the normal range the rounding is coarse enough to leave the range
    sub = ~normal & (s.astype(F32) > 0)
    qs = mx[sub].astype(np.float64) / s[sub].astype(np.float64)
    assert np.any(qs >= kmax + 0.5)


def test_magic_sum_gives_the_nearest_integer_in_its_low_bits():
    # x + 1.5 * 2^23 rounds x to an integer (ties to even) for |x| < 2^22; the
    # sum's bit pattern is 0x4B400000 + that integer, and 0x4B400000 is a
    # multiple of 256, so the low 8 bits are the integer's two's-complement bits
    g = np.random.Generator(np.random.PCG64(3))
    x = np.concatenate([g.uniform(-200.0, 200.0, 1 << 20), np.arange(-400, 401) / 2.0]).astype(F32)
    x = np.concatenate([x, np.nextafter(x, F32(np.inf)), np.nextafter(x, F32(-np.inf))])
    m = (x + F32(12582912.0)).astype(F32)
    r = np.rint(x).astype(np.int64)
    bits = m.view(np.int32).astype(np.int64)
    assert np.array_equal(bits - 0x4B400000, r)
    assert np.array_equal(bits & 0xFF, r & 0xFF) and np.array_equal(bits & 0xF, r & 0xF)
    assert np.array_equal((m - F32(12582912.0)).astype(F32), np.rint(x).astype(F32))
