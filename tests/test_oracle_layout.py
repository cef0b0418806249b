"""Pins of the oracle's packed code layout and storage accounting.

- hand-worked byte layouts (tests/golden/pack_layout.txt);
- round-trip identity, exhaustively: every byte value for INT2 / INT4 / INT8
  and every one of the 2^24 bit patterns of a 4-code INT6 unit;
- storage: group-wise INT4 with one binary16 scale per 32 codes is exactly
  4.50 bits per element ("Preserving Updates in Low-Bit Recurrent State
  Quantization", Table 2, Bits column).
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pack_layout.txt")


def _golden():
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, codes, data = (p.split() for p in line.split("|"))
        bits, dk, dv = map(int, head)
        yield bits, dk, dv, np.array(list(map(int, codes)), np.int8).reshape(dk, dv), \
            np.array([int(h, 16) for h in data], np.uint8)


@pytest.mark.parametrize("case", list(_golden()), ids=lambda c: f"int{c[0]}_{c[1]}x{c[2]}")
def test_golden_layout(orc, case):
    bits, dk, dv, codes, data = case
    assert np.array_equal(orc.pack(bits, codes), data)
    back = orc.unpack(bits, dk, dv, data)
    assert np.array_equal(back, codes)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_roundtrip_every_byte(orc, bits):
    dk, dv = 8, 256 * 8 // bits // 8 * 8   # a tile whose bytes take all 256 values
    nb = orc.tile_bytes(bits, dk, dv)
    data = (np.arange(nb) % 256).astype(np.uint8)
    codes = orc.unpack(bits, dk, dv, data)
    q = 1 << (bits - 1)
    assert codes.min() == -q and codes.max() == q - 1
    assert np.array_equal(orc.pack(bits, codes), data)
    rng = np.random.default_rng(bits)
    c2 = rng.integers(-q, q, size=(dk, dv)).astype(np.int8)
    assert np.array_equal(orc.unpack(bits, dk, dv, orc.pack(bits, c2)), c2)


def test_roundtrip_int6_all_unit_patterns(orc):
    # A unit of 4 consecutive INT6 codes occupies 2 bytes of the nibble plane
    # and 1 byte of the 2-bit plane: 24 bits, enumerated exhaustively.
    dk, dv = 512, 8                # 2 units per row, 1024 units per tile
    units_per_tile = dk * dv // 4
    pats = np.arange(1 << 24, dtype=np.uint32)
    ntiles = (1 << 24) // units_per_tile
    nib_bytes, hi_bytes = dk * dv // 2, dk * dv // 4
    for t in range(0, ntiles, 1):
        p = pats[t * units_per_tile:(t + 1) * units_per_tile]
        data = np.empty(nib_bytes + hi_bytes, np.uint8)
        data[0:nib_bytes:2] = p & 0xFF
        data[1:nib_bytes:2] = (p >> 8) & 0xFF
        data[nib_bytes:] = (p >> 16) & 0xFF
        codes = orc.unpack(6, dk, dv, data)
        assert np.array_equal(orc.pack(6, codes), data)
        if t == 0:
            assert codes.min() >= -32 and codes.max() <= 31


def test_int4_group32_is_4p5_bits(orc):
    cfg = orc.Config(128, 128, orc.GLA, 32)
    bits = (orc.tile_bytes(4, 128, 128) * 8 + cfg.n_scales * 16) / (128 * 128)
    assert bits == 4.5
    # group 64 (the GDN configuration) halves the scale overhead
    cfg64 = orc.Config(128, 128, orc.GDN, 64)
    assert (orc.tile_bytes(4, 128, 128) * 8 + cfg64.n_scales * 16) / (128 * 128) == 4.25
    # the pages' 5.3x memory reduction matches 32 / 6.00 peak bits (Table 6)
    assert round(32 / 6.00, 1) == 5.3
