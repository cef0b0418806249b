"""Pins of the oracle's pure-write sliding window (PW) of "Low-Bit GDN
Recurrent-State Quantization: Global Gradient-aware Allocation and Pure-Write
Sliding Windows" (Abstract).

- The FP8 E4M3 codec against torch's float8_e4m3fn (every code decoded; a
  sweep of binary32 values, every midpoint between neighbouring codes and
  its neighbours encoded) and the saturation at 448.
- With an fp32 history and inputs whose every intermediate value is exact in
  E4M3 (keys +-e_i, beta in {1/2, 1}, alpha in {1/2, 1}, small integer
  values), history + window is exactly the Gated DeltaNet recurrence
  S_t = alpha (I - beta k k^T) S_{t-1} + beta k v^T in fp64, and the output
  is exactly S_t^T q, for window sizes that merge at every step, at some
  steps and never.  A pair propagated without its erase term, a pair merged
  a step late, a window ring index off by one or an output that skips a
  pair all break the equality.
- Nothing leaves a window that is never full: the quantized history stays
  zero and the output is that of the pairs alone.
- With general inputs the windowed state stays within the FP8 rounding of
  its pairs of the fp32 recurrence.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_recurrent_state_decode_b200 import synth


def test_e4m3_decode_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3_to_f32(int(c)) for c in codes], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_e4m3_encode_matches_torch():
    finite = np.array([oracle.e4m3_to_f32(c) for c in range(127)], np.float64)   # ascending
    mids = (finite[:-1] + finite[1:]) / 2
    xs = [mids, np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
          np.nextafter(mids.astype(np.float32), np.float32(-np.inf)), finite,
          np.geomspace(1e-4, 460.0, 4001), np.linspace(0, 460, 4001)]
    x = np.concatenate([np.asarray(a, np.float32) for a in xs])
    x = np.concatenate([x, -x])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.f32_to_e4m3(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_saturates():
    for v, c in [(448.0, 0x7E), (460.0, 0x7E), (464.0, 0x7E), (470.0, 0x7E), (1e30, 0x7E),
                 (np.inf, 0x7E), (-470.0, 0xFE), (-np.inf, 0xFE), (2.0 ** -10, 0x00),
                 (3 * 2.0 ** -11, 0x01)]:
        assert oracle.f32_to_e4m3(v) == c, v


def _exact_stream(d, steps, seed, alphas=(1.0,)):
    rng = np.random.default_rng(seed)
    for _ in range(steps):
        k = np.zeros(d, np.float32)
        k[rng.integers(d)] = rng.choice([-1.0, 1.0])
        q = rng.integers(-3, 4, d).astype(np.float32)
        v = rng.integers(-4, 5, d).astype(np.float32)
        yield q, k, v, np.float32(rng.choice(alphas)), np.float32(rng.choice([0.5, 1.0]))


@pytest.mark.parametrize("W,alphas", [(1, (1.0,)), (2, (0.5, 1.0)), (3, (1.0,)), (8, (1.0,)),
                                      (16, (1.0,))])
def test_exact_recurrence(W, alphas):
    d, T, steps = 16, 3, 14
    cfg = oracle.Config(d, d, synth.GDN, 0, scale_mode=synth.DYNAMIC)
    st = oracle.PwState(cfg, [32] * T, W)
    S = np.zeros((T, d, d))
    streams = [_exact_stream(d, steps, 100 * W + t, alphas) for t in range(T)]
    for s in range(steps):
        xs = [next(g) for g in streams]
        q = np.stack([x[0] for x in xs]); k = np.stack([x[1] for x in xs])
        v = np.stack([x[2] for x in xs])
        al = np.array([x[3] for x in xs], np.float32); be = np.array([x[4] for x in xs], np.float32)
        out = st.step(q, k, v, al[:, None], be)
        for t in range(T):
            kk = k[t].astype(np.float64)
            S[t] = al[t] * (S[t] - be[t] * np.outer(kk, kk @ S[t])) + be[t] * np.outer(kk, v[t])
            assert np.array_equal(st.state(t), S[t]), (W, s, t)
            assert np.array_equal(out[t].astype(np.float64), S[t].T @ q[t]), (W, s, t)
        assert np.all(st.count == min(s + 1, W))


def test_history_untouched_while_the_window_fills():
    wl = synth.WORKLOADS["gdn_l24_b256_h32_d128_int4g64_bdr"].scaled(batch=1, heads=2)
    cfg = oracle.Config(128, 128, synth.GDN, 64, scale_mode=synth.PERSISTENT,
                        round_mode=synth.BDR, eps_b=0.3)
    W = 6
    st = oracle.PwState(cfg, [4, 4], W)
    for s in range(W):
        x = synth.gen_step(wl, s, tiles=np.arange(2))
        q, k, v, g = x.as_f32(wl)
        out = st.step(q, k, v, g[:, :1], g[:, 1])
        assert not st.codes.any() and not st.scales.any()
        for t in range(2):
            a, b = st.pairs(t)
            ref = (a @ q[t].astype(np.float64)) @ b
            assert np.abs(out[t] - ref).max() <= 1e-5 * np.abs(ref).max()
    x = synth.gen_step(wl, W, tiles=np.arange(2))
    q, k, v, g = x.as_f32(wl)
    st.step(q, k, v, g[:, :1], g[:, 1])
    assert st.codes.any() and np.all(st.count == W)


def test_close_to_the_fp32_recurrence():
    """General inputs, fp32 history: the only difference from the fp32
    recurrence is the E4M3 rounding of the window's pairs, re-rounded at
    every step on the key side (up to 2^-4 of a normal element, more for
    the many entries of beta k below 2^-6, which are subnormal), and kept in
    the history once merged.  A sanity band, not a pin (the exact cases
    above are the pins): the states agree to some percent."""
    wl = synth.WORKLOADS["gdn_l24_b256_h32_d128_int4g64_bdr"].scaled(batch=1, heads=4)
    cfg = oracle.Config(128, 128, synth.GDN, 64, scale_mode=synth.DYNAMIC)
    T = 4
    pw = oracle.PwState(cfg, [32] * T, 8)
    ref = oracle.State(cfg, [32] * T)
    for s in range(24):
        x = synth.gen_step(wl, s, tiles=np.arange(T))
        q, k, v, g = x.as_f32(wl)
        pw.step(q, k, v, g[:, :1], g[:, 1])
        ref.step(q, k, v, g[:, :1], g[:, 1])
    for t in range(T):
        e = np.linalg.norm(pw.state(t) - ref.S[t]) / np.linalg.norm(ref.S[t])
        assert 1e-3 < e < 0.15, e
