"""Long horizons of the layout variants on a few tiles of the 24-layer Gated
DeltaNet workload's own streams: the errors of a quantized recurrence compound
over time ("Preserving Updates in Low-Bit Recurrent State Quantization",
Abstract), so each variant is stepped for hundreds of steps and compared with
the oracle bit for bit at checkpoints (outputs, codes, scales and the
variant's side state).  The bypass runs with no residual (k = 0), where every
result is exact, through many merge cycles."""
import numpy as np
import pytest
import torch

import oracle
from bit_recurrent_state_decode_b200 import synth

from parity_util import GpuView, gpu_inputs, gpu_object, oracle_inputs, oracle_state

pytestmark = [pytest.mark.gpu, pytest.mark.long]
STEPS = 256
EVERY = 32


def _cfg(wl, mode):
    return oracle.Config(wl.d_k, wl.d_v, wl.kind, wl.group, scale_mode=mode,
                         round_mode=wl.round_mode, scale_f32=wl.scale_dtype == synth.F32,
                         gamma=wl.gamma, eps_b=wl.eps_b, rotate=wl.rotation)


def _run(name, make, check, steps=STEPS):
    wl = synth.workload(name).scaled(batch=1, heads=4, layers=1)
    mode = wl.scale_modes[0]
    gpu, orc = make(wl, mode)
    T = gpu.tiles
    out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
    for step in range(steps):
        x = synth.gen_step(wl, step, tiles=np.arange(T))
        gpu.step(*gpu_inputs(wl, x), out)
        o_orc = orc.step(*oracle_inputs(wl, x))
        if (step + 1) % EVERY == 0:
            torch.cuda.synchronize()
            o_gpu = out.cpu().numpy()
            assert np.array_equal(o_gpu.view(np.uint32), o_orc.view(np.uint32)), (name, step)
            view = GpuView(gpu)
            for t in range(T):
                assert np.array_equal(view.tile_codes(t), orc.codes[t]), (name, step, t)
                assert np.array_equal(view.scales[t], orc.scales[t]), (name, step, t)
            check(gpu, orc, step)
    st = gpu.status()
    assert st["nonfinite"] == 0 and st["pipeline_timeouts"] == 0, st
    gpu.close()


def test_hadamard_horizon():
    def make(wl, mode):
        return gpu_object(wl, mode, 1, 1), oracle_state(wl, mode, np.arange(wl.heads))
    _run("gdn_l24_b256_h32_d128_int4g32_had", make, lambda g, o, s: None)


def test_rowcol_horizon():
    def make(wl, mode):
        g = gpu_object(wl, mode, 1, 1)
        g.set_rowcol()
        return g, oracle.RcState(_cfg(wl, mode), np.full(g.tiles, wl.bits))
    _run("gdn_l24_b256_h32_d128_int4rc", make, lambda g, o, s: None)


def test_pw_horizon():
    def make(wl, mode):
        g = gpu_object(wl, mode, 1, 1)
        g.set_pw(wl.pw)
        return g, oracle.PwState(_cfg(wl, mode), np.full(g.tiles, wl.bits), wl.pw)

    def check(g, o, step):
        w = {n: t.cpu().numpy() for n, t in g.pw_export().items()}
        assert np.array_equal(w["A"], o.A) and np.array_equal(w["B"], o.B), step
        assert np.array_equal(w["head"], o.head) and np.array_equal(w["count"], o.count), step
    _run("gdn_l24_b256_h32_d128_int4g64_pw8", make, check)


def test_lrb_no_residual_horizon():
    m = 15

    def make(wl, mode):
        g = gpu_object(wl, mode, 1, 1)
        g.set_lrb(0, m, wl.lrb[2])
        return g, oracle.LrbState(_cfg(wl, mode), np.full(g.tiles, wl.bits), k=0, m=m,
                                  eps_l=wl.lrb[2])

    def check(g, o, step):
        b = {n: t.cpu().numpy() for n, t in g.lrb_export().items()}
        assert np.array_equal(b["n"][:, 0], o.nres) and np.array_equal(b["n"][:, 1], o.nnew)
        assert np.array_equal(b["D"].view(np.uint32), o.D.view(np.uint32))
        for t in range(g.tiles):
            n = int(o.nnew[t])
            assert np.array_equal(b["u"][t, :n].view(np.uint16), o.u[t, :n]), (step, t)
            assert np.array_equal(b["w"][t, :n].view(np.uint16), o.w[t, :n]), (step, t)
    _run("gdn_l24_b256_h32_d128_int4g32_lrb", make, check, steps=8 * m + 7)


def test_lrb_gla_no_residual_horizon():
    """GLA's bypass (a decay factor per key row) through eight merge cycles of
    the 16-head GLA workload's streams (d 128, INT4 g32, persistent scales)."""
    m = 15

    def make(wl, mode):
        g = gpu_object(wl, mode, 1, 1)
        g.set_lrb(0, m, 0.5)
        return g, oracle.LrbState(_cfg(wl, mode), np.full(g.tiles, wl.bits), k=0, m=m, eps_l=0.5)

    def check(g, o, step):
        b = {n: t.cpu().numpy() for n, t in g.lrb_export().items()}
        assert np.array_equal(b["n"][:, 1], o.nnew)
        assert np.array_equal(b["D"].view(np.uint32), o.D.view(np.uint32)), step
        for t in range(g.tiles):
            n = int(o.nnew[t])
            assert np.array_equal(b["u"][t, :n].view(np.uint16), o.u[t, :n]), (step, t)
    _run("gla_b128_h16_d128_int4g32_persistent", make, check, steps=8 * m + 7)
