"""Pins for the oracle's cache layout (written from the header's prose spec).

Record sizes come from the byte accounting; single-bit placements are
checked against hand-computed byte offsets; pack/unpack round-trips, and the
vectorised reader agrees with the one-record reader.
"""

import numpy as np

from oracle import layout


def test_record_sizes():
    assert layout.record_bytes(128, 3, 2, 32) == 100
    assert layout.record_bytes(128, 3, 3, 32) == 116
    assert layout.record_bytes(128, 4, 2, 32) == 116
    assert layout.tile_bytes(128, 3, 2, 32) == 12800


def _blank(n, d=128, ng=4):
    return ({"idx": np.zeros((n, d), np.int64), "sign": np.zeros((n, d), np.uint8),
             "nk16": np.zeros(n), "rn16": np.zeros(n)},
            {"codes": np.zeros((n, d), np.int64), "scale16": np.zeros((n, ng)),
             "zero16": np.zeros((n, ng))})


def test_single_bit_positions_by_hand():
    spec = layout.CacheSpec(batch=2, h_kv=3, capacity=256, d=128, key_bits=3,
                            value_bits=2, group=32)
    buf = spec.empty()
    kr, vr = _blank(1)
    kr["idx"][0, 13] = 2          # bit 1 of coordinate 13 -> plane 1, byte 1, bit 5
    kr["sign"][0, 127] = 1        # byte 15, bit 7
    vr["codes"][0, 65] = 2        # 2-bit values packed: byte 16, bits 2-3 -> 0b1000
    kr["nk16"][0] = 1.0           # fp16 0x3C00
    kr["rn16"][0] = -2.0          # fp16 0xC000
    vr["scale16"][0, 3] = 0.5     # fp16 0x3800, group 3 scale
    b, h, pos = 1, 2, 130         # tile 1, slot 2
    spec.write(buf, b, h, pos, kr, vr, 0)
    tile_bytes = 12800
    base = ((1 * 3 + 2) * 2 + 1) * tile_bytes
    slot = 2
    assert buf[base + 1 * 2048 + slot * 16 + 1] == 1 << 5
    assert buf[base + 2 * 2048 + slot * 16 + 15] == 1 << 7
    assert buf[base + 3 * 2048 + slot * 32 + 16] == 0b1000
    norms = base + 5 * 2048 + slot * 4
    assert list(buf[norms:norms + 4]) == [0x00, 0x3C, 0x00, 0xC0]
    vsz = base + 5 * 2048 + 512 + slot * 16 + 3 * 4
    assert list(buf[vsz:vsz + 2]) == [0x00, 0x38]
    assert int(np.count_nonzero(buf)) == 6


def test_roundtrip_and_readers_agree():
    rng = np.random.default_rng(0)
    for kb, vb in [(2, 2), (3, 2), (3, 3), (4, 2), (4, 4)]:
        spec = layout.CacheSpec(batch=2, h_kv=2, capacity=384, d=128, key_bits=kb,
                                value_bits=vb, group=32)
        buf = spec.empty()
        n = 300
        kr = {"idx": rng.integers(0, 2 ** (kb - 1), (n, 128)),
              "sign": rng.integers(0, 2, (n, 128)).astype(np.uint8),
              "nk16": np.float16(rng.random(n) * 50).astype(np.float64),
              "rn16": np.float16(rng.random(n)).astype(np.float64)}
        vr = {"codes": rng.integers(0, 2 ** vb, (n, 128)),
              "scale16": np.float16(rng.random((n, 4))).astype(np.float64),
              "zero16": np.float16(-rng.random((n, 4))).astype(np.float64)}
        spec.write_sequence(buf, 1, 0, 50, kr, vr)
        got = spec.read(buf, 1, 0, 50, n)
        one = spec.read_one(buf, 1, 0, 50, n)
        for key in ("idx", "sign", "nk16", "rn16"):
            assert np.array_equal(got[key], kr[key]), key
            assert np.array_equal(one[key], kr[key]), key
        for key in ("codes", "scale16", "zero16"):
            assert np.array_equal(got[key], vr[key]), key
            assert np.array_equal(one[key], vr[key]), key
        # the other (b, h) blocks are untouched
        assert not spec.read(buf, 0, 1, 0, 384)["idx"].any()
        # one-record writer produces the same bytes
        buf2 = spec.empty()
        for i in range(n):
            spec.write(buf2, 1, 0, 50 + i, kr, vr, i)
        assert np.array_equal(buf, buf2)


def test_three_bit_values_stay_bit_planes():
    spec = layout.CacheSpec(batch=1, h_kv=1, capacity=128, d=128, key_bits=3,
                            value_bits=3, group=32)
    buf = spec.empty()
    kr, vr = _blank(1)
    vr["codes"][0, 64] = 5        # 0b101 -> planes 0 and 2, byte 8, bit 0
    spec.write(buf, 0, 0, 1, kr, vr, 0)
    vbase = 3 * 2048              # after 2 key planes and the sign plane
    assert buf[vbase + 0 * 2048 + 1 * 16 + 8] == 1
    assert buf[vbase + 1 * 2048 + 1 * 16 + 8] == 0
    assert buf[vbase + 2 * 2048 + 1 * 16 + 8] == 1
