"""Pins for the oracle's wire packing.

The pages fix the bit count only (LQ-SGD review, "Core claim": b-bit indices
are sent in place of 32-bit floats); the layout is this library's reading:
per worker row, a little-endian bitstream with code j in bits [b*j, b*j + b)
as an excess-2^(b-1) field (4 and 5 bits) or one two's-complement int8/int16
per code, rows padded with code 0 to 128-code blocks of 16*b bytes.  The checks
are a hand-worked example, numpy's own bit packing as an independent
implementation, the round trip over every representable code, and the byte
count.
"""
import numpy as np
import pytest


def test_hand_worked_5bit_example(oracle):
    # codes 1, -1, 15, -15 -> fields (code + 16) 17, 15, 31, 1 at bits 0, 5, 10, 15,
    # then padding code 0 -> field 16 at bits 20 and 25 (bit 4 of each set):
    # 0x11 + 0x1E0 + 0x7C00 + 0x8000 + 0x1000000 + 0x20000000 = 0x2100FDF1
    codes = np.array([[1, -1, 15, -15]], np.int32)
    packed = oracle.pack(codes, 5)
    assert packed.shape == (1, 80)
    word0 = int.from_bytes(packed[0, :4].tobytes(), "little")
    assert word0 == 0x2100FDF1
    # the rest of the block is code 0 everywhere: the 160-bit pattern of
    # 32 fields of 16 repeats every 5 words from word 5 on
    rest = np.frombuffer(packed[0, 20:].tobytes(), dtype="<u4")
    assert np.array_equal(rest, np.tile(rest[:5], 3))


def test_hand_worked_4bit_example(oracle):
    # codes 7, -7, -1, 3 -> fields (code + 8) F, 1, 7, B; padding code 0 -> 8
    packed = oracle.pack(np.array([[7, -7, -1, 3]], np.int32), 4)
    assert packed.shape == (1, 64)
    assert int.from_bytes(packed[0, :4].tobytes(), "little") == 0x8888B71F
    assert np.all(packed[0, 4:] == 0x88)


def numpy_bitstream(codes, bits):
    """Independent packer: numpy bit matrix + np.packbits (little bit order)."""
    W, d = codes.shape
    padded = ((d + 127) // 128) * 128
    full = np.zeros((W, padded), np.int64)
    full[:, :d] = codes
    fields = full + (1 << (bits - 1))
    bitmat = ((fields[:, :, None] >> np.arange(bits)[None, None, :]) & 1).astype(np.uint8)
    stream = bitmat.reshape(W, padded * bits)
    return np.packbits(stream, axis=1, bitorder="little")


@pytest.mark.parametrize("bits", [4, 5, 8, 16])
@pytest.mark.parametrize("d", [1, 3, 31, 32, 33, 127, 128, 129, 1000])
def test_pack_matches_numpy_and_round_trips(oracle, bits, d):
    rng = np.random.default_rng(bits * 1000 + d)
    hi = (1 << (bits - 1)) - 1
    lo = -hi if bits in (4, 5) else -hi - 1
    W = 3
    codes = rng.integers(lo, hi + 1, size=(W, d)).astype(np.int32)
    packed = oracle.pack(codes, bits)
    assert packed.shape == (W, ((d + 127) // 128) * 16 * bits)
    if bits in (4, 5):
        assert np.array_equal(packed, numpy_bitstream(codes, bits))
    elif bits == 8:
        assert np.array_equal(packed[:, :d].view(np.int8), codes.astype(np.int8))
    else:
        assert np.array_equal(packed[:, :2 * d].view("<i2"), codes.astype(np.int16))
    assert np.array_equal(oracle.unpack(packed, W, d, bits), codes)


@pytest.mark.parametrize("bits", [4, 5, 8, 16])
def test_every_code_round_trips(oracle, bits):
    hi = (1 << (bits - 1)) - 1
    lo = -hi if bits in (4, 5) else -hi - 1
    codes = np.arange(lo, hi + 1, dtype=np.int32)[None, :]
    assert np.array_equal(oracle.unpack(oracle.pack(codes, bits), 1, codes.shape[1], bits),
                          codes)


def test_out_of_range_code_rejected(oracle):
    with pytest.raises(ValueError):
        oracle.pack(np.array([[16]], np.int32), 5)
    with pytest.raises(ValueError):
        oracle.pack(np.array([[-16]], np.int32), 5)
    with pytest.raises(ValueError):
        oracle.pack(np.array([[-8]], np.int32), 4)


def test_byte_count_of_wire_codes(oracle):
    # W rows of ceil(d/128) * 16 * bits bytes: bits/8 bytes per code plus padding
    for bits in (4, 5, 8, 16):
        for d in (25_557_032, 124_439_808, 1 << 30):
            rb = oracle.packed_row_bytes(bits, d)
            assert rb == -(-d // 128) * 16 * bits
            assert 0 <= rb - d * bits / 8 < 16 * bits
