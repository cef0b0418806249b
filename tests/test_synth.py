"""The seeded input generator: Philox4x32-10 known-answer vectors (Salmon et
al., SC'11, Random123 distribution), determinism, tile-subset consistency and
the shape of the synthetic distributions."""
import numpy as np
import pytest

from bit_recurrent_state_decode_b200 import synth


@pytest.mark.parametrize("ctr,key,expect", [
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
])
def test_philox_known_answers(ctr, key, expect):
    out = synth.philox4x32_10(*ctr, *key)
    assert tuple(int(x) for x in out) == expect


def test_normal_table():
    z = synth.normal_table()
    assert np.all(np.diff(z) > 0)
    assert np.allclose(z, -z[::-1])
    assert abs(z.mean()) < 1e-12 and abs(z.std() - 1) < 1e-3


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_deterministic_and_subset_consistent(name):
    wl = synth.WORKLOADS[name]
    n = min(64, wl.tiles_per_layer)
    pick = [n - 1, n // 2]
    a = synth.gen_step(wl, 5, layer=0, tiles=np.arange(n))
    b = synth.gen_step(wl, 5, layer=0, tiles=np.arange(n))
    sub = synth.gen_step(wl, 5, layer=0, tiles=np.array(pick))
    for fa, fb, fs in zip((a.q, a.k, a.v, a.gates), (b.q, b.k, b.v, b.gates),
                          (sub.q, sub.k, sub.v, sub.gates)):
        if fa is None:
            continue
        assert np.array_equal(fa, fb)
        assert np.array_equal(fa[pick], fs)
    c = synth.gen_step(wl, 6, layer=0, tiles=np.arange(2))
    assert not np.array_equal(a.v[:2], c.v)


def test_distributions():
    wl = synth.WORKLOADS["gdn_l24_b256_h32_d128_int4g64_bdr"]
    x = synth.gen_step(wl, 0, tiles=np.arange(512))
    q, k, v, g = x.as_f32(wl)
    assert np.allclose(np.linalg.norm(k.astype(np.float64), axis=1), 1, atol=1e-2)
    assert abs(v.std() - 1) < 0.02
    alpha, beta = g[:, 0], g[:, 1]
    assert 0.9 < alpha.mean() < 0.96 and 0.45 < beta.mean() < 0.55
    wl2 = synth.WORKLOADS["mamba2_b64_h32_dk128_dv64_int8tok"]
    y = synth.gen_step(wl2, 0)
    assert abs(y.q.std() - 1 / np.sqrt(128)) < 1e-3
    assert 0.45 < y.gates.mean() < 0.55
    wl3 = synth.WORKLOADS["gla_b128_h16_d128_int4g32_persistent"]
    z = synth.gen_step(wl3, 0)
    assert 0.98 < z.gates.mean() < 0.995


def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(5000) * 3).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.f32_to_bf16_bits(x), ref)


def test_mixed_head_bits_mean_four():
    hb = synth.WORKLOADS["gdn_b32_h16_d128_mixed_3modes"].head_bits()
    assert sorted(hb.tolist()) == [2] * 4 + [4] * 9 + [6] * 2 + [8]
    assert hb.mean() == 4.0


@pytest.mark.parametrize("name", ["mamba2_b64_h32_dk128_dv64_int8tok", "gdn_b32_h16_d128_mixed_3modes",
                                  "gla_b128_h16_d128_int4g32_persistent"])
def test_multi_step_generation_matches_single_steps(name):
    wl = synth.WORKLOADS[name]
    tiles = np.arange(6)
    many = synth.gen_step(wl, np.arange(10, 14), layer=2, tiles=tiles)
    for i, s in enumerate(range(10, 14)):
        one = synth.gen_step(wl, s, layer=2, tiles=tiles)
        for f in ("q", "k", "v", "gates"):
            a, b = getattr(many, f), getattr(one, f)
            if b is None:
                assert a is None
            else:
                assert np.array_equal(a[i], b), f
