"""Pins of the oracle's Low-Rank Bypass (LRB) of "Preserving Updates in
Low-Bit Recurrent State Quantization" (Abstract, Figure 3, Tables 6, 8, 9).

- Storage: the bypass occupancy the oracle's own state machine reaches (rank
  k residual plus one fresh column per step, merged every m steps) gives the
  average and peak bits per state element that Tables 6, 8 and 9 print, for
  the pages' state layout (INT4, binary16 scales per 32 elements, d_k = 256,
  d_v = 512; Mamba2 d_k = 128, d_v = 64).
- The rank-k residual is the best rank-k approximation (Eckart-Young),
  against numpy's SVD.
- A bypass merged every step with no residual and threshold 0 is the plain
  quantized step (same codes and scales), with inputs exact in binary16.
- The merge threshold: merged elements are those of the bypass at least
  eps_L grid steps large, and fewer as eps_L grows.
- GLA (a decay factor per key row): the row-factor bits of Table 6's GLA
  row; all gates 1 is RetNet with gamma = 1 bit for bit; a merge every step
  with exact binary16 inputs is the plain GLA step; before the first merge
  the bypass is the unquantized GLA recurrence within binary16 rounding.
- Before the first merge the bypass is the unquantized recurrence (Mamba2
  element by element, Gated DeltaNet in Frobenius norm) within the binary16
  rounding of its columns.
- At a GLA merge the elements that leave are those at least eps_L grid
  steps of their own row's decayed grid (D_i * Delta) large.
"""
import numpy as np
import pytest

import oracle
from bit_recurrent_state_decode_b200 import synth

W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)


def _occupancy(k, m, steps=None):
    """Columns held after each step, and at the peak, from the state
    machine itself (a 64 x 64 RetNet tile; the counts do not depend on it)."""
    cfg = oracle.Config(64, 64, synth.RETNET, 32, scale_mode=synth.DYNAMIC)
    st = oracle.LrbState(cfg, [4], k=k, m=m, eps_l=0.5)
    wl = C1
    held = []
    for s in range(steps or 4 * m + 8):
        x = synth.gen_step(wl, s, tiles=np.arange(1))
        q, kk, v, _ = x.as_f32(wl)
        st.step(q, kk, v)
        held.append(int(st.cols_used()[0]))
    steady = held[2 * m:]                 # after the residual has been filled
    return float(np.mean(steady[: (len(steady) // m) * m])), st.peak_cols


# (k, m, avg, peak) printed for GDN / RetNet (Tables 6, 8, 9)
PAGES_256_512 = [(1, 15, 5.25, 6.00), (0, 16, 5.20, 6.00), (2, 14, 5.30, 6.00),
                 (4, 12, 5.39, 6.00), (8, 8, 5.58, 6.00), (1, 7, 4.88, 5.25),
                 (1, 11, 5.06, 5.63), (1, 23, 5.63, 6.76)]


@pytest.mark.parametrize("k,m,avg,peak", PAGES_256_512)
def test_bits_reproduce_the_pages(k, m, avg, peak, orc):
    mean_cols, peak_cols = _occupancy(k, m)
    assert mean_cols == k + (m - 1) / 2 and peak_cols == k + m
    a = orc.lrb_bits(4, 32, 256, 512, mean_cols)
    p = orc.lrb_bits(4, 32, 256, 512, peak_cols)
    assert abs(a - avg) <= 0.005 and abs(p - peak) <= 0.005, (a, p)


def test_bits_mamba2_layout(orc):
    """Mamba2 (k = 1, m = 5; d_state 128 x head dim 64): the average 5.64 of
    Table 6 to the printed digit; the peak reads 6.773 against 6.78 (within
    one unit of the last digit)."""
    mean_cols, peak_cols = _occupancy(1, 5)
    assert abs(orc.lrb_bits(4, 32, 128, 64, mean_cols) - 5.64) <= 0.005
    assert abs(orc.lrb_bits(4, 32, 128, 64, peak_cols) - 6.78) <= 0.01


@pytest.mark.parametrize("k", [1, 2, 4])
def test_rank_k_is_the_truncated_svd(k, orc):
    rng = np.random.default_rng(k)
    R = rng.standard_normal((64, 48)) @ np.diag(np.linspace(3, 0.1, 48)) @ \
        rng.standard_normal((48, 48))
    s, U, V = orc.rank_k(R, k)
    s_ref = np.linalg.svd(R, compute_uv=False)[:k]
    assert np.allclose(s, s_ref, rtol=1e-10)
    Rk = (U.T * s) @ V
    U0, s0, V0 = np.linalg.svd(R)
    Rk_ref = (U0[:, :k] * s0[:k]) @ V0[:k]
    assert np.allclose(Rk, Rk_ref, atol=1e-9 * np.abs(R).max())


@pytest.mark.parametrize("base", [C1, C2], ids=["retnet", "mamba2"])
def test_merge_every_step_is_the_plain_step(base, orc):
    """k = 0, m = 1, eps_L = 0 merges each update whole at once: with k and v
    exact in binary16 the product u w is exact and a + u w rounds once, as the
    plain step's fma(k, v, a), so codes and scales agree bit for bit."""
    wl = base.scaled(batch=1, heads=4, d_k=64, d_v=64, group=32, bits=4,
                     scale_modes=(synth.DYNAMIC,))
    cfg = oracle.Config(64, 64, wl.kind, 32, scale_mode=synth.DYNAMIC, gamma=wl.gamma)
    lrb = oracle.LrbState(cfg, [4] * 4, k=0, m=1, eps_l=0.0)
    plain = oracle.State(cfg, [4] * 4)
    for s in range(40):
        x = synth.gen_step(wl, s, tiles=np.arange(4))
        q, k, v, g = x.as_f32(wl)
        k = k.astype(np.float16).astype(np.float32)
        v = v.astype(np.float16).astype(np.float32)
        o_l = lrb.step(q, k, v, g)
        o_p = plain.step(q, k, v, g)
        assert np.array_equal(lrb.codes, plain.codes) and np.array_equal(lrb.scales, plain.scales)
        assert np.abs(o_l - o_p).max() <= 1e-5 * np.abs(o_p).max()
    assert int(lrb.merged.sum()) > 0


def test_merge_threshold(orc):
    """At the second merge (the first merges everything: the state is still
    zero, its scales 0) the merged elements are those of the bypass at least
    eps_L grid steps of the decayed grid large: checked against the bypass
    held before the merge step in fp64, up to elements within 1e-5 of the
    threshold; a larger eps_L merges fewer."""
    wl = C4.scaled(batch=1, heads=4, layers=1)
    merged = {}
    for eps in (0.1, 0.5, 2.0):
        cfg = oracle.Config(128, 128, synth.GDN, 64, scale_mode=synth.PERSISTENT,
                            round_mode=synth.BDR, eps_b=0.3)
        st = oracle.LrbState(cfg, [4] * 4, k=1, m=15, eps_l=eps)
        for s in range(30):
            x = synth.gen_step(wl, s, tiles=np.arange(4))
            q, k, v, g = x.as_f32(wl)
            st.step(q, k, v, g[:, :1], g[:, 1])
            if s == 28:
                # the bypass and grid one step before the merge; the merge step
                # decays both by its alpha and adds one column
                P_before = [st.bypass(t) for t in range(4)]
                grid = [st.scales[t].reshape(128, 2).repeat(64, axis=1) * float(st.D[t])
                        for t in range(4)]
        merged[eps] = int(st.merged.sum())
        assert 0 < merged[eps] < 4 * 128 * 128 or eps == 2.0
        # loose check: most elements above the threshold before the merge step
        # are among the merged ones
        above = sum(int(np.count_nonzero(np.abs(P_before[t]) >= 1.2 * eps * grid[t]))
                    for t in range(4))
        assert merged[eps] >= 0.5 * above
    assert merged[0.1] > merged[0.5] > merged[2.0]


def test_lrb_tracks_the_unquantized_state_better(orc):
    """What the bypass is for (Abstract): small updates that INT4 rounding
    loses are kept and merged, so after 240 RetNet steps (gamma = 1 - 2^-5,
    persistent INT4 g32) the state plus bypass is closer to the unquantized
    recurrence than the plain quantized state is.  An observation on these
    synthetic streams, not a claim about the pages' models."""
    wl = C1.scaled(batch=1, heads=8)
    cfgq = oracle.Config(64, 64, synth.RETNET, 32, scale_mode=synth.PERSISTENT, gamma=wl.gamma)
    plain = oracle.State(cfgq, [4] * 8)
    lrb = oracle.LrbState(cfgq, [4] * 8, k=1, m=15, eps_l=0.7)
    ref = oracle.State(oracle.Config(64, 64, synth.RETNET, 32, gamma=wl.gamma), [32] * 8)
    for s in range(240):
        x = synth.gen_step(wl, s, tiles=np.arange(8))
        q, k, v, _ = x.as_f32(wl)
        for st in (plain, lrb, ref):
            st.step(q, k, v)
    S = ref.S.astype(np.float64)
    e_plain = np.linalg.norm(plain.dequant() - S)
    e_lrb = np.linalg.norm(np.stack([lrb.state(t) for t in range(8)]) - S)
    assert e_lrb < 0.8 * e_plain, (e_lrb, e_plain)


def test_residual_output_is_the_unmerged_bypass(orc):
    """With a threshold nothing reaches, the residual handed out at a merge
    is the whole decayed bypass (the fp64 sum of its columns, within fp32
    rounding), and the kept rank-1 pair is numpy's leading singular pair of
    it (within binary16 rounding).  The first merge finds no quantized state
    (all scales 0: a grid step of 0), so everything merges there and the
    residual is zero; the second merge is the one that keeps a residual.
    With threshold 0 everything merges at every merge."""
    wl = C1
    cfg = oracle.Config(64, 64, synth.RETNET, 32, scale_mode=synth.DYNAMIC, gamma=wl.gamma)
    st = oracle.LrbState(cfg, [4], k=1, m=3, eps_l=1e30, keep_resid=True)
    gam = float(np.float32(wl.gamma))
    for s in range(6):
        nb = int(st.nres[0] + st.nnew[0])
        u0 = st.u[0, :nb].view(np.float16).astype(np.float64).copy()
        w0 = st.w[0, :nb].view(np.float16).astype(np.float64).copy()
        g0 = st.g[0, :nb].astype(np.float64).copy()
        x = synth.gen_step(wl, s, tiles=np.arange(1))
        q, kk, v, _ = x.as_f32(wl)
        st.step(q, kk, v)
        if s == 2:
            assert not st.resid.any() and not st.u[0, 0].any() and not st.w[0, 0].any()
    assert nb == 3
    un = st.u[0, nb].view(np.float16).astype(np.float64)
    wn = st.w[0, nb].view(np.float16).astype(np.float64)
    P = np.outer(un, wn)
    for l in range(nb):
        P = P + float(np.float32(gam * g0[l])) * np.outer(u0[l], w0[l])
    R = st.resid[0].astype(np.float64)
    assert np.abs(P).max() > 0 and np.abs(R - P).max() <= 1e-6 * np.abs(P).max()
    U, S, Vt = np.linalg.svd(R)
    best = S[0] * np.outer(U[:, 0], Vt[0])
    kept = float(st.g[0, 0]) * np.outer(st.u[0, 0].view(np.float16).astype(np.float64),
                                        st.w[0, 0].view(np.float16).astype(np.float64))
    assert np.linalg.norm(kept - best) <= 2e-3 * np.linalg.norm(best)

    st0 = oracle.LrbState(cfg, [4], k=1, m=3, eps_l=0.0, keep_resid=True)
    for s in range(6):
        x = synth.gen_step(wl, s, tiles=np.arange(1))
        q, kk, v, _ = x.as_f32(wl)
        st0.step(q, kk, v)
    assert not st0.resid.any() and not st0.u[0, 0].any() and not st0.w[0, 0].any()


# ------------------------------------------------------------------ GLA (reading L7)
def test_bits_gla_row_factors(orc):
    """GLA's row of Table 6 (k = 1, m = 15: 5.31 average, 6.07 peak at the
    256 x 512 layout) is GDN's storage plus one binary32 decay factor per
    key row: 32 / d_v = 1/16 bit per element.  The average matches to the
    printed digit; the peak reads 6.0625 against 6.07 (within one unit of the
    last digit, as the Mamba2 peak)."""
    mean_cols, peak_cols = _occupancy(1, 15)
    row = 32.0 / 512
    assert abs(orc.lrb_bits(4, 32, 256, 512, mean_cols) + row - 5.31) <= 0.005
    assert abs(orc.lrb_bits(4, 32, 256, 512, peak_cols) + row - 6.07) <= 0.01


def _gla_stream(wl, s, T, alpha_fn=None):
    x = synth.gen_step(wl, s, tiles=np.arange(T))
    q, k, v, g = x.as_f32(wl)
    if alpha_fn is not None:
        g = alpha_fn(s, g.shape)
    return q, k, v, g


def test_gla_without_decay_is_retnet_without_decay(orc):
    """With every gate alpha = 1 the per-row factors stay 1 and a GLA bypass
    computes exactly what the scalar-decay bypass of RetNet with gamma = 1
    does: outputs, codes, scales and the bypass itself agree bit for bit,
    through merges and the rank-1 residual."""
    wl = C3.scaled(batch=1, heads=4, d_k=64, d_v=64, group=32,
                   qkv_dtype=synth.F32, gate_dtype=synth.F32)
    T = 4
    ones = lambda s, shape: np.ones(shape, np.float32)
    gla = oracle.LrbState(oracle.Config(64, 64, synth.GLA, 32, scale_mode=synth.PERSISTENT),
                          [4] * T, k=1, m=5, eps_l=0.5)
    ret = oracle.LrbState(oracle.Config(64, 64, synth.RETNET, 32, scale_mode=synth.PERSISTENT,
                                        gamma=1.0), [4] * T, k=1, m=5, eps_l=0.5)
    for s in range(23):
        q, k, v, g = _gla_stream(wl, s, T, ones)
        o1 = gla.step(q, k, v, g)
        o2 = ret.step(q, k, v)
        assert np.array_equal(o1.view(np.uint32), o2.view(np.uint32)), s
        assert np.array_equal(gla.codes, ret.codes) and np.array_equal(gla.scales, ret.scales)
        assert np.array_equal(gla.u, ret.u) and np.array_equal(gla.w, ret.w)
        assert np.all(gla.D == 1.0)


def test_gla_merge_every_step_is_the_plain_step(orc):
    """k = 0, m = 1, eps_L = 0 with gates alpha_i in {1/2, 1} (so k_i / D_i
    and D_i (k_i / D_i) are exact in binary16) and k, v exact in binary16:
    each update merges whole, D_i u_i w_j = k_i v_j exactly, and the codes and
    scales are the plain GLA step's bit for bit."""
    wl = C3.scaled(batch=1, heads=4, d_k=64, d_v=64, group=32,
                   qkv_dtype=synth.F32, gate_dtype=synth.F32)
    T = 4
    rng = np.random.default_rng(3)
    halves = lambda s, shape: rng.choice([0.5, 1.0], shape).astype(np.float32)
    cfg = oracle.Config(64, 64, synth.GLA, 32, scale_mode=synth.DYNAMIC)
    lrb = oracle.LrbState(cfg, [4] * T, k=0, m=1, eps_l=0.0)
    plain = oracle.State(cfg, [4] * T)
    for s in range(30):
        q, k, v, g = _gla_stream(wl, s, T, halves)
        k = k.astype(np.float16).astype(np.float32)
        v = v.astype(np.float16).astype(np.float32)
        o_l = lrb.step(q, k, v, g)
        o_p = plain.step(q, k, v, g)
        assert np.array_equal(lrb.codes, plain.codes) and np.array_equal(lrb.scales, plain.scales), s
        assert np.abs(o_l - o_p).max() <= 1e-5 * np.abs(o_p).max()


def test_gla_lrb_tracks_the_unquantized_state_better(orc):
    """The bypass with per-row decay factors keeps small GLA updates: after
    240 steps of the GLA workload's streams (INT4 g32 persistent) the state
    plus bypass is closer to the unquantized recurrence than the plain
    quantized state is (an observation on these streams)."""
    wl = C3.scaled(batch=1, heads=8, d_k=64, d_v=64)
    T = 8
    cfgq = oracle.Config(64, 64, synth.GLA, 32, scale_mode=synth.PERSISTENT)
    plain = oracle.State(cfgq, [4] * T)
    lrb = oracle.LrbState(cfgq, [4] * T, k=1, m=15, eps_l=0.5)
    ref = oracle.State(oracle.Config(64, 64, synth.GLA, 32), [32] * T)
    for s in range(240):
        q, k, v, g = _gla_stream(wl, s, T)
        for st in (plain, lrb, ref):
            st.step(q, k, v, g)
    S = ref.S.astype(np.float64)
    e_plain = np.linalg.norm(plain.dequant() - S)
    e_lrb = np.linalg.norm(np.stack([lrb.state(t) for t in range(T)]) - S)
    assert e_lrb < 0.8 * e_plain, (e_lrb, e_plain)


def test_gla_bypass_before_its_first_merge_is_the_recurrence(orc):
    """Before its first merge a GLA tile's codes are zero, so the state its
    bypass stands for is Diag(D_t) sum_l fp16(k_l / D_l) fp16(v_l)^T: the
    column added at step l, read at step t, is (D_t / D_l) k_l v_l^T with
    D_t / D_l the product of the gates of steps l+1 .. t.  That is the
    unquantized GLA recurrence S_t = Diag(alpha_t) S_{t-1} + k_t v_t^T (GLA in
    Table 1) up to the binary16 rounding of each column (2^-11 relative per
    side, 2^-25 absolute below the binary16 normal range) and the binary32
    products that form D.  Checked element by element in fp64 at every step,
    and the outputs against S_t^T q_t; the decay the pin checks is far larger
    than its tolerance, so a row factor dropped, applied twice or applied
    along d_v fails it."""
    wl = C3.scaled(batch=1, heads=4, d_k=64, d_v=64, group=32,
                   qkv_dtype=synth.F32, gate_dtype=synth.F32)
    T, m, dk, dv = 4, 31, 64, 64
    cfg = oracle.Config(dk, dv, synth.GLA, 32, scale_mode=synth.PERSISTENT)
    lrb = oracle.LrbState(cfg, [4] * T, k=0, m=m, eps_l=0.5)
    S = np.zeros((T, dk, dv))
    S_nodecay = np.zeros((T, dk, dv))
    A = np.zeros((T, dk, dv))            # the recurrence of |k_l v_l^T|
    K = np.zeros((T, dk))
    V = np.zeros((T, dv))
    for s in range(m - 1):
        q, k, v, g = _gla_stream(wl, s, T)
        o = lrb.step(q, k, v, g).astype(np.float64)
        a = g.astype(np.float64)[:, :, None]
        kv = k.astype(np.float64)[:, :, None] * v.astype(np.float64)[:, None, :]
        S = a * S + kv
        S_nodecay = S_nodecay + kv
        A = a * A + np.abs(kv)
        K += np.abs(k)
        V += np.abs(v)
        assert not lrb.codes.any() and int(lrb.nnew[0]) == s + 1
        P = np.stack([lrb.state(t) for t in range(T)])
        tol = 1.05 * 2.0**-10 * A + 2.0**-24 * (K[:, :, None] + V[:, None, :])
        assert np.all(np.abs(P - S) <= tol), (s, np.abs(P - S).max())
        qa = np.abs(q.astype(np.float64))
        o_ref = np.einsum("tij,ti->tj", S, q.astype(np.float64))
        tol_o = 2.0**-9 * np.einsum("tij,ti->tj", A, qa) + \
            2.0**-23 * (V * qa.sum(1)[:, None] + (K * qa).sum(1)[:, None])
        assert np.all(np.abs(o - o_ref) <= tol_o), (s, np.abs(o - o_ref).max())
    # the readings the pin tells apart: no decay at all, and a key side held
    # undivided (every column decayed by the whole D_t)
    assert np.abs(S_nodecay - S).max() > 100 * tol.max()
    Dt = lrb.D.astype(np.float64)[:, :, None]
    assert np.abs(Dt * S_nodecay - S).max() > 100 * tol.max()


@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_bypass_before_its_first_merge_is_the_recurrence(kind, orc):
    """Before the first merge the codes are zero and the bypass alone holds
    the state, so it must follow the unquantized recurrence of Table 1 up to
    the binary16 rounding of its columns.

    Mamba2 (scalar decay): column l read at step t is g_l fp16(k_l) fp16(v_l)^T
    with g_l the binary32 product of the gates since step l; checked element
    by element against S_t = alpha_t S_{t-1} + k_t v_t^T with the same bound
    as the GLA pin.  Gated DeltaNet: the column is (fp16(beta k), fp16(e)) with
    e = v - r and r over the bypass itself; with unit keys, alpha <= 1 and
    beta <= 1 the transition alpha (I - beta k k^T) has norm at most 1, so the
    rounding of each column adds to the Frobenius distance from
    S_t = alpha_t S_{t-1} + beta_t k_t (v_t - alpha_t S_{t-1}^T k_t)^T and
    never grows: ||P_t - S_t||_F <= 1.1 * 2^-10 * sum_l ||beta_l k_l|| ||e_l||
    plus the binary32 sums.  Outputs are checked against S_t^T q_t."""
    if kind == "mamba2":
        wl = C2.scaled(batch=1, heads=4)
    else:
        wl = C4.scaled(batch=1, heads=4, layers=1)
    T, m, dk, dv = 4, 31, wl.d_k, wl.d_v
    cfg = oracle.Config(dk, dv, wl.kind, wl.group, scale_mode=synth.DYNAMIC,
                        scale_f32=wl.scale_dtype == synth.F32)
    lrb = oracle.LrbState(cfg, [wl.bits] * T, k=0, m=m, eps_l=0.5)
    S = np.zeros((T, dk, dv))
    S_nodecay = np.zeros((T, dk, dv))
    A = np.zeros((T, dk, dv))
    K = np.zeros((T, dk))
    V = np.zeros((T, dv))
    budget = np.zeros(T)
    for s in range(m - 1):
        x = synth.gen_step(wl, s, tiles=np.arange(T))
        q, k, v, g = x.as_f32(wl)
        q64, k64, v64 = (z.astype(np.float64) for z in (q, k, v))
        if kind == "mamba2":
            o = lrb.step(q, k, v, g).astype(np.float64)
            a = g.astype(np.float64)[:, :1, None]
            kv = k64[:, :, None] * v64[:, None, :]
            S = a * S + kv
            A = a * A + np.abs(kv)
            K += np.abs(k64)
            V += np.abs(v64)
        else:
            alpha, beta = g[:, :1], g[:, 1]
            o = lrb.step(q, k, v, alpha, beta).astype(np.float64)
            a = alpha.astype(np.float64)[:, :, None]
            b = beta.astype(np.float64)
            e = v64 - np.einsum("tij,ti->tj", a * S, k64)
            upd = (b[:, None] * k64)[:, :, None] * e[:, None, :]
            S = a * S + upd
            budget += np.linalg.norm(b[:, None] * k64, axis=1) * np.linalg.norm(e, axis=1)
        S_nodecay = S_nodecay + (upd if kind == "gdn" else kv)
        assert not lrb.codes.any() and int(lrb.nnew[0]) == s + 1
        P = np.stack([lrb.state(t) for t in range(T)])
        o_ref = np.einsum("tij,ti->tj", S, q64)
        qa = np.abs(q64)
        if kind == "mamba2":
            tol = 1.05 * 2.0**-10 * A + 2.0**-24 * (K[:, :, None] + V[:, None, :])
            assert np.all(np.abs(P - S) <= tol), (s, np.abs(P - S).max())
            tol_o = 2.0**-9 * np.einsum("tij,ti->tj", A, qa) + \
                2.0**-23 * (V * qa.sum(1)[:, None] + (K * qa).sum(1)[:, None])
            assert np.all(np.abs(o - o_ref) <= tol_o), (s, np.abs(o - o_ref).max())
        else:
            fro = np.linalg.norm((P - S).reshape(T, -1), axis=1)
            tol = 1.1 * 2.0**-10 * budget + 2.0**-20 * (s + 1)
            assert np.all(fro <= tol), (s, fro, tol)
            # |o - S^T q| <= ||P - S||_F ||q|| plus the binary32 sums
            err_o = np.linalg.norm(o - o_ref, axis=1)
            assert np.all(err_o <= 1.05 * tol * np.linalg.norm(q64, axis=1) + 2.0**-20), s
    # the decay the pin resolves is far above its tolerance (for GDN the
    # tolerance is the worst case of the triangle inequality, about 35 times
    # the distance the roundings actually leave)
    if kind == "mamba2":
        assert np.abs(S_nodecay - S).max() > 100 * tol.max()
    else:
        assert np.linalg.norm((S_nodecay - S).reshape(T, -1), axis=1).min() > 50 * tol.max()


def test_gla_merge_threshold_uses_each_rows_factor(orc):
    """At a merge the elements that leave a GLA bypass are those with
    |P_ij| >= eps_L * (D_i * Delta_ij), D_i the row's decay factor of that
    step (reading L7).  The test forms P itself from the bypass the oracle
    held before the merge step (columns read as D_i u_i, the new column
    fp16(k / D) and fp16(v)) and checks which elements the oracle kept as its
    residual, away from a thin band around the threshold where the fp32 and
    fp64 sums may round to opposite sides.  Gates spread over [1/2, 1] make
    the row factors differ by far more than that band, so a threshold
    without D_i, or with one factor for the whole tile, selects other
    elements."""
    wl = C3.scaled(batch=1, heads=4, d_k=64, d_v=64, group=32,
                   qkv_dtype=synth.F32, gate_dtype=synth.F32)
    T, m, eps = 4, 6, 0.5
    cfg = oracle.Config(64, 64, synth.GLA, 32, scale_mode=synth.PERSISTENT)
    st = oracle.LrbState(cfg, [4] * T, k=1, m=m, eps_l=eps, keep_resid=True)
    rng = np.random.default_rng(7)
    spread = lambda s, shape: rng.uniform(0.5, 1.0, shape).astype(np.float32)
    for s in range(2 * m - 1):
        st.step(*_gla_stream(wl, s, T, spread))
    assert np.all(st.nnew == m - 1)
    u0, w0, g0 = st.u.copy(), st.w.copy(), st.g.copy()
    D0, scales0, n0 = st.D.copy(), st.scales.copy(), (st.nres + st.nnew).copy()
    q, k, v, g = _gla_stream(wl, 2 * m - 1, T, spread)
    st.step(q, k, v, g)
    assert np.all(st.nnew == 0)                      # this step merged
    agree = differs = differs_tile = 0
    for t in range(T):
        Dn = g[t] * D0[t]                            # binary32, as the step forms it
        n = int(n0[t])
        U = u0[t, :n].view(np.float16).astype(np.float32) * Dn[None, :]
        u_new = (k[t] / Dn).astype(np.float16).astype(np.float32) * Dn
        Wc = w0[t, :n].view(np.float16).astype(np.float64)
        w_new = v[t].astype(np.float16).astype(np.float64)
        P = np.einsum("l,li,lj->ij", g0[t, :n].astype(np.float64), U.astype(np.float64), Wc) + \
            np.outer(u_new.astype(np.float64), w_new)
        delta = np.repeat(scales0[t].reshape(64, 2), 32, axis=1).astype(np.float64)
        thr = eps * (Dn.astype(np.float64)[:, None] * delta)
        far = (np.abs(np.abs(P) - thr) > 1e-4 * thr) & (P != 0)
        merged = st.resid[t] == 0
        want = np.abs(P) >= thr
        assert np.array_equal(merged[far], want[far]), t
        band = int(((~far) & (P != 0)).sum())
        assert abs(int(st.merged[t]) - int(want.sum())) <= band, t
        agree += int(far.sum())
        alt = np.abs(P) >= eps * delta                             # no D_i
        alt_tile = np.abs(P) >= eps * (float(Dn.mean()) * delta)  # one factor per tile
        differs += int((alt[far] != want[far]).sum())
        differs_tile += int((alt_tile[far] != want[far]).sum())
    assert agree > 0.95 * T * 64 * 64 and differs > 100 and differs_tile > 10
