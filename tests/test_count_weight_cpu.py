"""The fused kernel's integer-to-float shortcut for hash-match counts, checked in float32 (no GPU).

The kernel turns a popcount p (0 <= p <= s <= 64) into the weight s - p without an integer
conversion: the float whose bits are those of 2^23 with p in the low mantissa bits is exactly
2^23 + p, so (2^23 + s) - that float = s - p exactly in float32; a count c stored in a byte
becomes float(c) the same way, minus 2^23.
"""
import numpy as np


def _bits_to_f32(u):
    return np.asarray(u, dtype=np.uint32).view(np.float32)


def test_popcount_to_weight_is_exact():
    for s in range(1, 65):
        p = np.arange(0, s + 1, dtype=np.uint32)
        cs = np.float32(8388608.0 + s)
        w = cs - _bits_to_f32(np.uint32(0x4B000000) | p)
        assert w.dtype == np.float32
        assert np.array_equal(w, (s - p).astype(np.float32)), s


def test_byte_count_to_float_is_exact():
    c = np.arange(0, 256, dtype=np.uint32)
    f = _bits_to_f32(np.uint32(0x4B000000) | c) - np.float32(8388608.0)
    assert np.array_equal(f, c.astype(np.float32))
