"""The weights pass's dropout keep decision, as float arithmetic.

A weight is kept when the 16-bit field u of its draw is >= thr = ceil(p * 2^16) (the generator's
definition, which the oracle follows with an integer compare). The tcgen05 weights pass takes the
same decision without a compare: u placed under the exponent bits of 2^23 is the float 2^23 + u,
and saturate(2^23 + u + (1 - thr - 2^23)) in float32 is exactly 1 for a kept weight and 0 for a
dropped one, because every term and partial sum is an integer below 2^24. This checks that
identity in IEEE float32 (round to nearest, as the GPU's add) for every u against a spread of
thresholds, and for every threshold against a spread of u."""
import numpy as np


def kept_by_float(u, thr):
    f = (np.uint32(0x4B000000) | u.astype(np.uint32)).view(np.float32)  # 2^23 + u, exactly
    kthr = (np.float32(1.0) - np.float32(thr)) - np.float32(8388608.0)
    s = (f + kthr).astype(np.float32)
    return np.clip(s, np.float32(0.0), np.float32(1.0))


def test_float_keep_equals_integer_compare_all_fields():
    u = np.arange(65536, dtype=np.uint32)
    thresholds = sorted({1, 2, 255, 256, 6554, 16384, 32767, 32768, 32769, 49152, 65535} |
                        set(range(1, 65536, 331)))
    for thr in thresholds:
        got = kept_by_float(u, thr)
        want = (u >= thr).astype(np.float32)
        assert np.array_equal(got, want), thr


def test_float_keep_equals_integer_compare_all_thresholds():
    thr = np.arange(1, 65536, dtype=np.int64)
    for u0 in (0, 1, 2, 6553, 6554, 6555, 32767, 32768, 65534, 65535):
        u = np.full(thr.shape, u0, dtype=np.uint32)
        f = (np.uint32(0x4B000000) | u).view(np.float32)
        kthr = ((np.float32(1.0) - thr.astype(np.float32)) - np.float32(8388608.0)).astype(np.float32)
        got = np.clip((f + kthr).astype(np.float32), 0, 1)
        assert np.array_equal(got, (u0 >= thr).astype(np.float32)), u0
