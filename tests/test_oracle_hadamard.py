"""Pins of the oracle's Hadamard-rotated state (INT4+Had, Table 2 of
"Preserving Updates in Low-Bit Recurrent State Quantization"): the butterfly
against an independent Hadamard matrix, its involution, and the rotated
recurrence against the unrotated one where both are exact up to rounding."""
import numpy as np
import pytest
import scipy.linalg

import oracle
from bit_recurrent_state_decode_b200 import synth

W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)


@pytest.mark.parametrize("n", [2, 8, 64, 128])
def test_fwht_is_the_sylvester_matrix(n, orc):
    rng = np.random.default_rng(n)
    x = rng.integers(-1000, 1000, n).astype(np.float32)     # integer sums: exact in fp32
    ref = scipy.linalg.hadamard(n).astype(np.float64) @ x.astype(np.float64)
    assert np.array_equal(orc.fwht(x).astype(np.float64), ref)


@pytest.mark.parametrize("n", [64, 128])
def test_fwht_twice_is_n_times_identity(n, orc):
    x = np.arange(n, dtype=np.float32) - n / 2
    assert np.array_equal(orc.fwht(orc.fwht(x)), n * x)


def _run(wl, rotate, steps, bits=32, mode=synth.DYNAMIC, tiles=4):
    cfg = oracle.Config(wl.d_k, wl.d_v, wl.kind, wl.group, scale_mode=mode,
                        round_mode=wl.round_mode, scale_f32=wl.scale_dtype == synth.F32,
                        gamma=wl.gamma, eps_b=wl.eps_b, rotate=rotate)
    st = oracle.State(cfg, [bits] * tiles)
    outs = []
    for s in range(steps):
        x = synth.gen_step(wl, s, tiles=np.arange(tiles))
        q, k, v, g = x.as_f32(wl)
        alpha = beta = None
        if wl.kind in (synth.MAMBA2, synth.GLA):
            alpha = g
        elif wl.kind == synth.GDN:
            alpha, beta = g[:, :1], g[:, 1]
        outs.append(st.step(q, k, v, alpha, beta))
    return st, np.array(outs)


@pytest.mark.parametrize("base", [C1, C2, C3, C4], ids=["retnet", "mamba2", "gla", "gdn"])
def test_rotated_recurrence_matches_unrotated_at_32_bits(base, orc):
    """Unquantized, the rotated state is S H and the outputs are those of the
    plain recurrence, up to binary32 rounding (a misplaced transform, a
    missing 1/d_v or a rotation of k instead of v fails by orders of
    magnitude)."""
    wl = base.scaled(d_v=64 if base.d_v == 64 else 128)
    plain, o_plain = _run(wl, 0, 40)
    rot, o_rot = _run(wl, 1, 40)
    H = scipy.linalg.hadamard(wl.d_v).astype(np.float64)
    S = plain.S.astype(np.float64)
    Srot = rot.S.astype(np.float64)
    scale = np.abs(S).max() * wl.d_v
    assert np.abs(Srot - S @ H).max() <= 1e-5 * scale
    assert np.abs(o_rot - o_plain).max() <= 1e-5 * np.abs(o_plain).max()


def test_rotation_halves_the_error_of_a_spiky_row(orc):
    """The purpose of the rotation: a row whose few large entries set its
    one scale (a scale group of the whole row) loses the rest of the row to
    rounding; rotated, the row's mass is spread evenly and the same INT4
    budget reconstructs it with about half the error (0.21-0.24 against
    0.09-0.10 here).  Rank-1 state after one step from zero, v ~ N(0, 1) with
    three entries of 10."""
    H = scipy.linalg.hadamard(128).astype(np.float64)
    for seed in range(5):
        rng = np.random.default_rng(seed)
        k = rng.standard_normal((1, 128)).astype(np.float32) / np.float32(np.sqrt(128))
        v = rng.standard_normal((1, 128)).astype(np.float32)
        v[0, rng.choice(128, 3, replace=False)] = 10.0
        q = np.zeros((1, 128), np.float32)
        alpha = np.ones((1, 128), np.float32)
        S = np.outer(k[0], v[0]).astype(np.float64)
        err = {}
        for rotate in (0, 1):
            cfg = oracle.Config(128, 128, synth.GLA, 128, scale_mode=synth.DYNAMIC, rotate=rotate)
            st = oracle.State(cfg, [4])
            st.step(q, k, v, alpha)
            rec = st.dequant()[0].astype(np.float64)
            if rotate:
                rec = rec @ H / 128.0
            err[rotate] = np.linalg.norm(rec - S) / np.linalg.norm(S)
        assert err[1] < 0.6 * err[0], (seed, err)
