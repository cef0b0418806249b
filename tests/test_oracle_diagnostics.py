"""Pins of the oracle's error accounting (``oracle.diagnostics``): the
accumulated error of the rank-1 recurrences against the unquantized
recurrence in fp64, closed forms of the coherent gain, and the rounding
classes against the oracle's own counters."""
from __future__ import annotations

import numpy as np
import pytest


def _inputs(rng, T, dk, dv, kind, steps):
    for _ in range(steps):
        k = (rng.standard_normal((T, dk)) / np.sqrt(dk)).astype(np.float32)
        v = rng.standard_normal((T, dv)).astype(np.float32)
        q = rng.standard_normal((T, dk)).astype(np.float32)
        if kind == 2:      # GLA: one decay per key row
            alpha = rng.uniform(0.90, 0.999, (T, dk)).astype(np.float32)
        else:
            alpha = rng.uniform(0.85, 0.99, (T, 1)).astype(np.float32)
        yield q, k, v, alpha


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("group,mode", [(8, 0), (0, 0), (16, 1)])
def test_accumulated_error_is_the_state_error(orc, kind, group, mode):
    """Rank-1 kinds: E_T = sum a_{tau:T} R_tau equals S_hat_T - S_T, S_T the
    unquantized recurrence in fp64, up to the binary32 rounding of the
    updates (a dropped decay, a shifted decay index or a flipped sign of R
    would miss by the size of the quantization error)."""
    from oracle import diagnostics as D
    rng = np.random.default_rng(7 + kind * 10 + group)
    T, dk, dv, steps = 3, 16, 16, 40
    cfg = orc.Config(dk, dv, kind, group, scale_mode=mode, gamma=0.96875)
    st = orc.State(cfg, np.full(T, 4))
    acc = D.ErrorAccount(st)
    S = np.zeros((T, dk, dv))
    xmax = 0.0
    for q, k, v, alpha in _inputs(rng, T, dk, dv, kind, steps):
        w = (np.full((T, dk), np.float32(0.96875)) if kind == 0
             else alpha.astype(np.float64) if kind == 2 else np.repeat(alpha, dk, 1).astype(np.float64))
        S = w[:, :, None] * S + k.astype(np.float64)[:, :, None] * v.astype(np.float64)[:, None, :]
        acc.step(q, k, v, None if kind == 0 else alpha)
        xmax = max(xmax, float(np.abs(S).max()))
    err = st.dequant().astype(np.float64) - S
    quant = float(np.abs(err).max())
    diff = float(np.abs(acc.E["all"] - err).max())
    assert quant > 1e-3 * xmax                        # the test sees a real quantization error
    assert diff <= steps * 2.0 ** -22 * xmax          # binary32 rounding of the updates only


def test_gain_is_one_for_orthogonal_errors():
    from oracle.diagnostics import accumulate, coherent_gain
    rng = np.random.default_rng(3)
    E, Dr = np.zeros((1, 4, 4)), np.zeros((1, 4))
    for t in range(16):                                # each step errs on its own element
        R = np.zeros((1, 4, 4))
        R[0, t // 4, t % 4] = rng.standard_normal()
        E, Dr = accumulate(E, Dr, R, np.full((1, 4), rng.uniform(0.5, 1.0)))
    assert coherent_gain(E, Dr) == pytest.approx(1.0, rel=1e-12)


@pytest.mark.parametrize("w", [1.0, 0.9, 0.5])
def test_gain_of_identical_errors(w):
    """Identical per-step errors under a constant decay w:
    g_T = (sum_s w^s)^2 / sum_s w^(2s), s = 0 .. T-1 (T for w = 1)."""
    from oracle.diagnostics import accumulate, coherent_gain
    rng = np.random.default_rng(5)
    R = rng.standard_normal((2, 3, 5))
    E, Dr = np.zeros_like(R), np.zeros((2, 3))
    T = 25
    for _ in range(T):
        E, Dr = accumulate(E, Dr, R, np.full((2, 3), w))
    s = np.array([w ** i for i in range(T)])
    assert coherent_gain(E, Dr) == pytest.approx(s.sum() ** 2 / (s * s).sum(), rel=1e-12)


def test_recursion_matches_the_double_sum():
    """||E_T||^2 = sum_{tau, tau'} a_{tau:T} a_{tau':T} <R_tau, R_tau'> with
    per-row decays, and D_T its diagonal."""
    from oracle.diagnostics import accumulate
    rng = np.random.default_rng(11)
    T, dk, dv = 9, 4, 3
    Rs = rng.standard_normal((T, dk, dv))
    ws = rng.uniform(0.3, 1.0, (T, dk))
    E, Dr = np.zeros((dk, dv)), np.zeros(dk)
    for t in range(T):
        E, Dr = accumulate(E, Dr, Rs[t], ws[t])
    a = np.ones((T, dk))                               # a_{tau:T} per row
    for tau in range(T):
        for s in range(tau + 1, T):
            a[tau] *= ws[s]
    full = sum(np.sum(a[t1][:, None] * Rs[t1] * a[t2][:, None] * Rs[t2])
               for t1 in range(T) for t2 in range(T))
    diag = sum(np.sum((a[t][:, None] * Rs[t]) ** 2) for t in range(T))
    assert np.sum(E * E) == pytest.approx(full, rel=1e-10)
    assert np.sum(Dr) == pytest.approx(diag, rel=1e-10)


def test_classes_match_the_oracle_counters(orc):
    from oracle import diagnostics as D
    rng = np.random.default_rng(19)
    T, dk, dv = 2, 16, 16
    cfg = orc.Config(dk, dv, orc.MAMBA2, 8, scale_mode=orc.PERSISTENT, taxonomy=True)
    st = orc.State(cfg, np.full(T, 4))
    acc = D.ErrorAccount(st)
    for q, k, v, alpha in _inputs(rng, T, dk, dv, 1, 30):
        acc.step(q, k * np.float32(0.05), v, alpha)     # small updates: many are lost
    c = st.counts
    assert acc.n_lost == c.lost
    assert acc.n_updates == c.lost + c.moved + c.reversed
    assert 0.0 < acc.lost_fraction() < 1.0
    rep = acc.report()
    assert rep["b_over_delta_q25"] <= rep["b_over_delta_q50"] <= rep["b_over_delta_q75"]


def test_update_ratio_of_a_known_first_step(orc):
    """From the zero state the update is b = k v^T; with k = kappa e_0 and a
    per-token dynamic INT8 scale Delta = f16(max|b| / 127), the ratios are
    |kappa v_j| / Delta on row 0."""
    from oracle import diagnostics as D
    dk = dv = 8
    cfg = orc.Config(dk, dv, orc.MAMBA2, 0, scale_mode=orc.DYNAMIC)
    st = orc.State(cfg, np.full(1, 8))
    acc = D.ErrorAccount(st)
    k = np.zeros((1, dk), np.float32)
    k[0, 0] = 0.5
    v = np.array([[1, -2, 3, -4, 5, -6, 7, -8]], np.float32)
    acc.step(np.ones((1, dk), np.float32), k, v, np.full((1, 1), 0.9, np.float32))
    delta = float(np.float16(4.0 / 127))
    want = np.abs(0.5 * v[0].astype(np.float64)) / delta
    got = np.concatenate(acc.ratios)
    assert np.allclose(np.sort(got), np.sort(want), rtol=0, atol=0)
    assert acc.n_updates == dv
