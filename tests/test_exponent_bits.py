"""The QUEST metadata kernel turns bytes 1 and 3 of each code word into floats without the
conversion instruction: the code b (int8) with its sign bit flipped is b + 128 in 0..255,
placed as the low mantissa byte under exponent byte 0x4B that is the float 2^23 + b + 128,
and subtracting 2^23 + 128 (one correctly rounded fp32 subtraction) leaves b exactly. The
products code * scale then equal the ones an fp32 multiply of the converted code gives.
Checked here for every byte value, in numpy's IEEE fp32 arithmetic."""
import numpy as np


def test_every_code_byte_is_exact():
    b = np.arange(-128, 128, dtype=np.int32)
    bits = np.uint32(0x4B000000) | ((b.astype(np.uint32) ^ np.uint32(0x80)) & np.uint32(0xFF))
    f = bits.view(np.float32)
    assert np.array_equal(f, (2.0 ** 23 + b + 128).astype(np.float32))
    got = f - np.float32(8388736.0)
    assert got.dtype == np.float32
    assert np.array_equal(got, b.astype(np.float32))


def test_products_match_the_converted_codes():
    rng = np.random.default_rng(0)
    b = np.arange(-128, 128, dtype=np.int32)
    bits = np.uint32(0x4B000000) | ((b.astype(np.uint32) ^ np.uint32(0x80)) & np.uint32(0xFF))
    via_bits = bits.view(np.float32) - np.float32(8388736.0)
    scales = np.concatenate([rng.uniform(-40, 40, 64), [-149, -130, -126, 0, 100, 127]])
    with np.errstate(over="ignore"):  # the largest scales overflow to +-inf on purpose
        for e in scales:
            s = np.float32(2.0 ** e) * np.float32(rng.uniform(1, 2))
            assert np.array_equal((via_bits * s).view(np.uint32),
                                  (b.astype(np.float32) * s).view(np.uint32))
