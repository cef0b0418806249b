"""Pins of the oracle's quantizer (scale modes, RTN, BDR, taxonomy).

Sources: "When Dynamic Scaling Fails", Abstract (dynamic scale re-derived from
the state, persistent scale, scale yoked to a full-precision reference);
"Preserving Updates in Low-Bit Recurrent State Quantization", Abstract and
Figure 4 caption (lost / moved / reversed updates; BDR rounds a reversed
element toward its update and enlarges the rounding error), Table 6 (eps_B).

The checks use exact rational arithmetic (fractions.Fraction), numpy's
half-to-even rint and binary16 cast, and invariants of the definitions:
error bounds, symmetry, fixed points, monotonicity, the yoked bound.
"""
from fractions import Fraction

import numpy as np
import pytest


def f16(x):
    return float(np.float32(x).astype(np.float16))


# ------------------------------------------------------------ helpers
def _mamba2_unit_decay_x(orc, st_q, k, v):
    """Pre-rounding state x of a Mamba2 tile with alpha = 1.

    With alpha = 1 the decayed state code * (1 * scale) equals the dequantized
    state exactly, so x = fma(k, v, S_hat) is what an unquantized (32-bit)
    oracle tile computes from S_hat."""
    cfg = st_q.cfg
    c32 = orc.Config(cfg.d_k, cfg.d_v, orc.MAMBA2, 0)
    s32 = orc.State(c32, [32] * st_q.ntiles)
    s32.S[:] = st_q.dequant()
    T = st_q.ntiles
    s32.step(np.zeros((T, cfg.d_k)), k, v, np.ones((T, 1)))
    return s32.S.copy()


def _groups(x, group):
    dk, dv = x.shape
    if group == 0:
        return x.reshape(1, dk * dv)
    return x.reshape(dk, dv // group, group).reshape(-1, group)


def _random_state(orc, cfg, bits, T, rng, steps=3):
    st = orc.State(cfg, [bits] * T)
    for _ in range(steps):
        st.step(rng.standard_normal((T, cfg.d_k)) / 8, rng.standard_normal((T, cfg.d_k)) / 8,
                rng.standard_normal((T, cfg.d_v)), np.ones((T, 1)))
    return st


# ------------------------------------------------------------ RTN
def test_round_rtn_matches_exact_half_even(orc):
    rng = np.random.default_rng(20)
    xs = (rng.standard_normal(4000) * 10).astype(np.float32)
    invs = rng.uniform(0.01, 3, 4000).astype(np.float32)
    # exact ties: x * inv = k + 1/2 with inv a power of two
    tx = (np.arange(-20, 20) + 0.5).astype(np.float32) * 4
    xs = np.concatenate([xs, tx])
    invs = np.concatenate([invs, np.full(40, 0.25, np.float32)])
    for qmax in (1, 7, 31, 127):
        for x, inv in zip(xs, invs):
            w = Fraction(float(x)) * Fraction(float(inv))
            ref = max(-qmax, min(qmax, round(w)))         # round(): half to even
            assert orc.round_rtn(x, inv, qmax) == ref
            assert orc.round_rtn(-x, inv, qmax) == -ref   # symmetry


@pytest.mark.parametrize("bits,group", [(4, 64), (8, 0), (4, 32), (2, 64), (6, 64)])
def test_dynamic_step_definition_and_bounds(orc, bits, group):
    rng = np.random.default_rng(21 + bits + group)
    dk, dv, T = 64, 128, 3
    cfg = orc.Config(dk, dv, orc.MAMBA2, group, scale_mode=orc.DYNAMIC)
    st = _random_state(orc, cfg, bits, T, rng)
    k = (rng.standard_normal((T, dk)) / 8).astype(np.float32)
    v = rng.standard_normal((T, dv)).astype(np.float32)
    x = _mamba2_unit_decay_x(orc, st, k, v)
    st.step(np.zeros((T, dk)), k, v, np.ones((T, 1)))
    qmax = (1 << (bits - 1)) - 1
    for t in range(T):
        xg = _groups(x[t], group)
        cg = _groups(st.codes[t].astype(np.float64), group)
        for g in range(xg.shape[0]):
            m = np.float32(np.abs(xg[g]).max())
            delta = f16(m / np.float32(qmax))
            assert st.scales[t, g] == delta
            inv = np.float32(1) / np.float32(delta)
            ref = np.clip(np.rint(xg[g].astype(np.float64) * np.float64(inv)), -qmax, qmax)
            assert np.array_equal(cg[g], ref)
            # RTN error bound and the max element sitting on the code range edge
            assert np.all(np.abs(xg[g] - cg[g] * delta) <= delta / 2 * (1 + 2 ** -20))
            if m > 0:
                assert np.abs(cg[g]).max() == qmax


@pytest.mark.parametrize("mode", ["dynamic", "persistent", "yoked"])
def test_fixed_point_no_update(orc, mode):
    # alpha = 1 and k = 0 leave codes and scales unchanged in every mode
    sm = {"dynamic": orc.DYNAMIC, "persistent": orc.PERSISTENT, "yoked": orc.YOKED}[mode]
    rng = np.random.default_rng(22)
    dk, dv, T = 64, 64, 2
    cfg = orc.Config(dk, dv, orc.MAMBA2, 64, scale_mode=sm)
    st = orc.State(cfg, [4] * T)
    st.step(rng.standard_normal((T, dk)), rng.standard_normal((T, dk)) / 8,
            rng.standard_normal((T, dv)), np.ones((T, 1)))
    codes, scales = st.codes.copy(), st.scales.copy()
    for _ in range(5):
        st.step(rng.standard_normal((T, dk)), np.zeros((T, dk)), rng.standard_normal((T, dv)),
                np.ones((T, 1)))
        assert np.array_equal(st.codes, codes)
        assert np.array_equal(st.scales, scales)


def test_zero_state_zero_scale(orc):
    cfg = orc.Config(64, 64, orc.RETNET, 64)
    st = orc.State(cfg, [4])
    st.step(np.ones(64), np.zeros(64), np.zeros(64))
    assert not st.codes.any() and not st.scales.any()


def test_persistent_scale_grows_only_on_overflow(orc):
    rng = np.random.default_rng(23)
    dk, dv, T = 64, 128, 2
    cfg = orc.Config(dk, dv, orc.MAMBA2, 32, scale_mode=orc.PERSISTENT)
    st = orc.State(cfg, [4] * T)
    qmax = 7
    for step in range(40):
        prev = st.scales.copy()
        k = (rng.standard_normal((T, dk)) / 8 * (1 + step % 5)).astype(np.float32)
        v = rng.standard_normal((T, dv)).astype(np.float32)
        x = _mamba2_unit_decay_x(orc, st, k, v)
        st.step(np.zeros((T, dk)), k, v, np.ones((T, 1)))
        assert np.all(st.scales >= prev)
        for t in range(T):
            m = np.abs(_groups(x[t], 32)).max(axis=1).astype(np.float32)
            over = m > np.float32(qmax) * prev[t]
            assert np.array_equal(st.scales[t][~over], prev[t][~over])
            assert np.array_equal(st.scales[t][over],
                                  np.array([f16(mm / np.float32(qmax)) for mm in m[over]],
                                           np.float32))


def test_per_token_scale_is_tile_max(orc):
    rng = np.random.default_rng(24)
    dk, dv, T = 128, 64, 2
    cfg = orc.Config(dk, dv, orc.MAMBA2, 0, scale_mode=orc.DYNAMIC)
    st = _random_state(orc, cfg, 8, T, rng)
    k = (rng.standard_normal((T, dk)) / 8).astype(np.float32)
    v = rng.standard_normal((T, dv)).astype(np.float32)
    x = _mamba2_unit_decay_x(orc, st, k, v)
    st.step(np.zeros((T, dk)), k, v, np.ones((T, 1)))
    assert st.scales.shape == (T, 1)
    for t in range(T):
        assert st.scales[t, 0] == f16(np.float32(np.abs(x[t]).max()) / np.float32(127))


def test_f16_scale_saturates_and_counts(orc):
    cfg = orc.Config(64, 64, orc.RETNET, 64)
    st = orc.State(cfg, [4])
    st.step(np.ones(64), np.full(64, 1e4, np.float32), np.full(64, 1e3, np.float32))
    assert np.all(st.scales == 65504.0)
    assert st.counts.saturated == 64
    assert np.all(st.codes == 7)        # clamped at Qmax


def test_yoked_bound_and_reference_matches_fp32(orc):
    rng = np.random.default_rng(25)
    dk, dv, T, steps = 64, 64, 2, 60
    for scale_f32, tol in ((False, 2 ** -10), (True, 2 ** -23)):
        cfg = orc.Config(dk, dv, orc.GDN, 64, scale_mode=orc.YOKED, round_mode=orc.BDR,
                         scale_f32=scale_f32)
        st = orc.State(cfg, [4, 2])
        ref = orc.State(orc.Config(dk, dv, orc.GDN, 0), [32] * T)
        for _ in range(steps):
            q = rng.standard_normal((T, dk)).astype(np.float32)
            k = rng.standard_normal((T, dk)).astype(np.float32)
            k /= np.linalg.norm(k, axis=1, keepdims=True)
            v = rng.standard_normal((T, dv)).astype(np.float32)
            al = (1 / (1 + np.exp(-(3 + rng.standard_normal((T, 1)))))).astype(np.float32)
            be = (1 / (1 + np.exp(-rng.standard_normal(T)))).astype(np.float32)
            st.step(q, k, v, al, be)
            ref.step(q, k, v, al, be)
            # the yoked reference is exactly the unquantized recurrence
            assert np.array_equal(st.ref, ref.S)
            S_hat = st.dequant()
            for t in range(T):
                mq = np.abs(_groups(S_hat[t], 64)).max(axis=1)
                mr = np.abs(_groups(st.ref[t], 64)).max(axis=1)
                assert np.all(mq <= mr * (1 + tol))


# ------------------------------------------------------------ BDR / taxonomy
def _cases():
    """Tiny-state enumeration: prior code, prior scale, decay, new scale and
    an update of a given number of grid steps."""
    updates = [0, 1 / 64, 1 / 16, 0.1, 0.25, 0.3, 0.49, 0.5, 0.51, 0.75, 1.0, 1.5, 3.0]
    for bits in (2, 4):
        qmax = (1 << (bits - 1)) - 1
        for c0 in range(-qmax, qmax + 1):
            for dprev in (0.0625, 0.1, 0.3, 1.0):
                for alpha in (1.0, 0.75, 0.5):
                    for growth in (1.0, 1.25):
                        dnew = f16(dprev * growth)
                        a = np.float32(c0) * (np.float32(alpha) * np.float32(dprev))
                        inv = np.float32(1) / np.float32(dnew)
                        for du in updates:
                            for sgn in (1, -1):
                                x = np.float32(a + np.float32(sgn * du * dnew))
                                yield qmax, np.float32(a), x, inv


def test_bdr_brute_force_enumeration(orc):
    cfg0 = orc.Config(8, 8, orc.GDN, 8, round_mode=orc.BDR, eps_b=0.0)
    cfg3 = orc.Config(8, 8, orc.GDN, 8, round_mode=orc.BDR, eps_b=0.3)
    n_rev = n_enlarged = 0
    for qmax, a, x, inv in _cases():
        d = Fraction(float(x)) - Fraction(float(a))
        u = Fraction(float(a)) * Fraction(float(inv))
        w = Fraction(float(x)) * Fraction(float(inv))
        c_rtn = orc.round_rtn(x, inv, qmax)
        assert c_rtn == max(-qmax, min(qmax, round(w)))
        cls = orc.classify(a, x, inv, qmax)
        # (i) exactly one class for every element with a nonzero update
        if d == 0:
            assert cls == orc.NONE
            assert cfg0.round(a, x, inv, qmax) == c_rtn
            continue
        reversed_ = (c_rtn - u) * d < 0
        lost = c_rtn == max(-qmax, min(qmax, round(u)))
        assert cls == (orc.REVERSED if reversed_ else orc.LOST if lost else orc.MOVED)
        c_bdr = cfg0.round(a, x, inv, qmax)
        saturated = abs(round(w)) >= qmax or abs(round(u)) >= qmax
        if not reversed_:
            assert c_bdr == c_rtn                               # (v)
        elif not saturated:
            n_rev += 1
            assert c_rtn == round(u)                            # (ii) would-be lost
            assert (c_bdr - u) * d >= 0                         # (iii) never against d
            assert abs(c_bdr - w) < 1                           # (iv) bounded
            # (vi) RTN is the nearest code, so BDR never lowers the error, and
            # raises it except at exact half-way ties
            assert abs(c_bdr - w) >= abs(c_rtn - w)
            if abs(c_bdr - w) > abs(c_rtn - w):
                n_enlarged += 1
        if not saturated:
            c3 = cfg3.round(a, x, inv, qmax)
            # against the update by at most eps_B grid steps (up to one fp32 rounding)
            assert (u - c3) * (1 if d > 0 else -1) <= Fraction(0.3) + Fraction(1, 2 ** 20)
            assert abs(c3 - w) < 1
    assert n_rev > 100
    assert n_enlarged > 0.9 * n_rev


def test_bdr_tile_counts(orc):
    # On a GDN tile with eps_B = 0 the number of BDR corrections equals the
    # number of reversed elements under the exact taxonomy.
    rng = np.random.default_rng(26)
    dk, dv, T = 64, 64, 4
    cfg = orc.Config(dk, dv, orc.GDN, 64, scale_mode=orc.PERSISTENT, round_mode=orc.BDR,
                     taxonomy=True)
    st = orc.State(cfg, [4] * T)
    for _ in range(30):
        k = rng.standard_normal((T, dk)).astype(np.float32)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        st.step(k, k, rng.standard_normal((T, dv)),
                np.full((T, 1), 0.95, np.float32), np.full(T, 0.5, np.float32))
    c = st.counts
    assert c.reversed > 0 and c.lost > 0 and c.moved > 0
    assert c.bdr_applied == c.reversed
