"""Pins of the oracle's number-format conversions against independent library
routines (numpy's IEEE binary16 cast, torch's bfloat16 cast).

Scales are stored as IEEE binary16: group-wise INT4 costs 4.50 bits per state
element ("Preserving Updates in Low-Bit Recurrent State Quantization",
Table 2, Bits column), i.e. one 16-bit scale per 32 four-bit codes.
"""
import numpy as np
import pytest
import torch


def _np_f16_bits(x):
    return int(np.array([x], np.float32).astype(np.float16).view(np.uint16)[0])


def test_f16_to_f32_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([orc.f16_bits_to_f32(int(b)) for b in bits], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_f16_exact_values_and_ties(orc):
    # every finite binary16 value converts back to itself, and every midpoint
    # between neighbours rounds to the even neighbour (numpy agrees)
    finite = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    for sgn in (1.0, -1.0):
        vals = sgn * finite
        for v in vals[::7]:
            assert orc.f32_to_f16_bits(np.float32(v)) == _np_f16_bits(np.float32(v))
        mids = (vals[:-1] + vals[1:]) / 2.0          # exact in fp64 and fp32
        for m in mids[::5]:
            m32 = np.float32(m)
            assert float(m32) == m
            assert orc.f32_to_f16_bits(m32) == _np_f16_bits(m32), m


def test_f32_to_f16_random_and_edges(orc):
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-30, 17, 20000))).astype(np.float32)
    edges = np.array([0.0, -0.0, 65504.0, 65519.996, 65520.0, 1e9, 2.0 ** -24, 2.0 ** -25,
                      3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, np.inf, -np.inf],
                     np.float32)
    for v in np.concatenate([x, edges, -edges]):
        assert orc.f32_to_f16_bits(v) == _np_f16_bits(v), v


def test_bf16_conversions(orc):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-60, 60, 20000))).astype(np.float32)
    # force ties: low 16 bits exactly 0x8000
    ties = (x.view(np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = np.concatenate([x, ties.view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for v, r in zip(x[::3], ref[::3]):
        assert orc.f32_to_bf16_bits(v) == int(r)
        back = torch.from_numpy(np.array([r], np.uint16).view(np.int16)).view(torch.bfloat16)
        assert orc.bf16_bits_to_f32(int(r)) == float(back.float()[0])
