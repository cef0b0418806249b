"""Pins of the oracle's key-row x value-column scales (readings R1-R5 of the
C code; "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent
State Quantization", Abstract).

- A state whose magnitudes are a rank-1 product |x_ij| = |u_i| |w_j| is
  exactly what two-factor scales fit: every code lands on +-Qmax with the
  sign of x, and the dequantized state equals x within the binary16
  rounding of the scales.  A single scale per row, per column or per tile,
  a transposed (row <-> column) layout, or a dropped factor all fail it on
  a d_k != d_v tile with unequal magnitudes.
- Round to nearest: |x - S_hat| <= Delta_ij / 2 wherever x * inv is inside
  the code range, all codes within +-Qmax, and every non-zero row reaches
  Qmax - 1 or more (its largest column-normalised element is spread over
  the code range).
- The update and the output are the plain step's: the first step from a zero
  state gives the same outputs, bit for bit, as the per-group oracle.
- On states whose magnitudes vary along both axes the two-factor grid has
  less error than one scale per tile.
"""
import numpy as np
import pytest

import oracle
from bit_recurrent_state_decode_b200 import synth

W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
def test_rank1_magnitudes_land_on_qmax(bits, dk, dv):
    rng = np.random.default_rng(bits * 1000 + dk)
    cfg = oracle.Config(dk, dv, synth.RETNET, 0, scale_mode=synth.DYNAMIC)
    st = oracle.RcState(cfg, [bits] * 2)
    k = (rng.choice([-1, 1], (2, dk)) * 2.0 ** rng.integers(-6, 3, (2, dk))).astype(np.float32)
    v = (rng.choice([-1, 1], (2, dv)) * 2.0 ** rng.integers(-4, 5, (2, dv))).astype(np.float32)
    q = np.ones((2, dk), np.float32)
    st.step(q, k, v)
    qmax = (1 << (bits - 1)) - 1
    x = k[:, :, None].astype(np.float64) * v[:, None, :]
    assert np.array_equal(st.codes, (np.sign(x) * qmax).astype(np.int8))
    deq = st.dequant().astype(np.float64)
    assert np.all(np.abs(deq - x) <= 2.0 ** -10 * np.abs(x))


def _run(wl, steps, bits, tiles=4):
    cfg = oracle.Config(wl.d_k, wl.d_v, wl.kind, 0, scale_mode=synth.DYNAMIC,
                        round_mode=synth.RTN, gamma=wl.gamma)
    st = oracle.RcState(cfg, [bits] * tiles)
    for s in range(steps):
        x = synth.gen_step(wl, s, tiles=np.arange(tiles))
        q, k, v, g = x.as_f32(wl)
        alpha = beta = None
        if wl.kind in (synth.MAMBA2, synth.GLA):
            alpha = g
        elif wl.kind == synth.GDN:
            alpha, beta = g[:, :1], g[:, 1]
        st.step(q, k, v, alpha, beta)
    return st, cfg


@pytest.mark.parametrize("base", ["C1", "C2", "C3", "C4"])
@pytest.mark.parametrize("bits", [4, 8])
def test_rounding_error_bound(base, bits):
    wl = {"C1": C1, "C2": C2, "C3": C3, "C4": C4}[base]
    st, cfg = _run(wl, 6, bits)
    dk, dv = cfg.d_k, cfg.d_v
    qmax = (1 << (bits - 1)) - 1
    # one more step; its state before rounding x is re-derived in fp64 from
    # the stored state and the inputs (within fp32 rounding of the oracle's
    # own x, covered by the slack of the bound)
    x_in = synth.gen_step(wl, 6, tiles=np.arange(4))
    q, k, v, g = x_in.as_f32(wl)
    alpha = beta = None
    if wl.kind in (synth.MAMBA2, synth.GLA):
        alpha = g
    elif wl.kind == synth.GDN:
        alpha, beta = g[:, :1], g[:, 1]
    prev = st.dequant().astype(np.float64)
    st.step(q, k, v, alpha, beta)
    assert np.abs(st.codes).max() <= qmax
    deq = st.dequant().astype(np.float64)
    for t in range(4):
        rho, kap = st.scales[t, :dk].astype(np.float64), st.scales[t, dk:].astype(np.float64)
        step = np.outer(rho, kap)
        if wl.kind == synth.GLA:
            al = alpha[t].astype(np.float64)[:, None]
        elif wl.kind == synth.RETNET:
            al = np.float64(np.float32(wl.gamma))
        else:
            al = np.float64(alpha[t, 0])
        a = al * prev[t]
        if wl.kind == synth.GDN:
            kk = k[t].astype(np.float64)
            x = a + np.outer(beta[t] * kk, v[t] - kk @ a)
        else:
            x = a + np.outer(k[t], v[t])
        inside = np.abs(x) <= (qmax + 0.25) * step
        assert np.all(np.abs(x - deq[t])[inside] <= 0.5 * step[inside] * (1 + 1e-3) + 1e-6 * np.abs(x).max())
        rows = np.abs(st.codes[t]).max(axis=1)
        assert np.all(rows[np.abs(x).max(axis=1) > 0] >= qmax - 1)


@pytest.mark.parametrize("base", ["C1", "C3", "C4"])
def test_first_step_outputs_are_the_plain_steps(base):
    wl = {"C1": C1, "C3": C3, "C4": C4}[base]
    cfg_rc = oracle.Config(wl.d_k, wl.d_v, wl.kind, 0, scale_mode=synth.DYNAMIC, gamma=wl.gamma)
    cfg_pl = oracle.Config(wl.d_k, wl.d_v, wl.kind, wl.group, scale_mode=synth.DYNAMIC,
                           gamma=wl.gamma)
    rc = oracle.RcState(cfg_rc, [4] * 3)
    pl = oracle.State(cfg_pl, [4] * 3)
    x = synth.gen_step(wl, 0, tiles=np.arange(3))
    q, k, v, g = x.as_f32(wl)
    alpha = beta = None
    if wl.kind in (synth.MAMBA2, synth.GLA):
        alpha = g
    elif wl.kind == synth.GDN:
        alpha, beta = g[:, :1], g[:, 1]
    o1 = rc.step(q, k, v, alpha, beta)
    o2 = pl.step(q, k, v, alpha, beta)
    assert np.array_equal(o1.view(np.uint32), o2.view(np.uint32))


def test_beats_one_scale_per_tile_on_two_axis_magnitudes():
    """Updates whose rows and columns carry magnitudes spread over 2^8: the
    two-factor grid tracks the unquantized recurrence (fp64) with far less
    error than one scale per tile."""
    rng = np.random.default_rng(7)
    dk = dv = 64
    T = 4
    cfg = oracle.Config(dk, dv, synth.RETNET, 0, scale_mode=synth.DYNAMIC)
    rc = oracle.RcState(cfg, [4] * T)
    pt = oracle.State(cfg, [4] * T)
    gam = np.float64(np.float32(cfg.c.gamma))
    ref = np.zeros((T, dk, dv))
    ru = 2.0 ** rng.uniform(-4, 4, (T, dk))
    rv = 2.0 ** rng.uniform(-4, 4, (T, dv))
    for s in range(4):
        k = (rng.standard_normal((T, dk)) * ru).astype(np.float32)
        v = (rng.standard_normal((T, dv)) * rv).astype(np.float32)
        q = np.zeros((T, dk), np.float32)
        rc.step(q, k, v)
        pt.step(q, k, v)
        ref = gam * ref + k[:, :, None].astype(np.float64) * v[:, None, :]
    e_rc = np.linalg.norm(rc.dequant() - ref)
    e_pt = np.linalg.norm(pt.dequant() - ref)
    assert e_rc < 0.5 * e_pt, (e_rc, e_pt)
