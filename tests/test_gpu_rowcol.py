"""GPU parity of the decode step with key-row x value-column scales
("STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State
Quantization", Abstract; readings R1-R5 of the oracle) against the oracle's
row x column step: the scales are fitted from the state element by element
(maxima, one correctly rounded reciprocal and division each), so outputs,
codes, both scale vectors and the dequantized state are bit-exact at every
step, for all four kinds, both tile shapes, 4 and 8 bits, RTN and BDR,
binary16 and binary32 scales."""
import numpy as np
import pytest
import torch

import oracle
from bit_recurrent_state_decode_b200 import qstate as Q
from bit_recurrent_state_decode_b200 import synth

from parity_util import GpuView, gpu_inputs, gpu_object, oracle_inputs, rel_err

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)
DYN = (synth.DYNAMIC,)

CASES = {
    "retnet_d64_int4_f32in": C1.scaled(batch=3, heads=4),
    "mamba2_dk128_dv64_int8": C2.scaled(batch=2, heads=4),
    "gla_d128_int4_bf16": C3.scaled(batch=2, heads=4, scale_modes=DYN),
    "gdn_d128_int4_bdr": C4.scaled(batch=2, heads=4, layers=1, scale_modes=DYN, eps_b=0.3),
    "gdn_dk64_dv128_int8_rtn": C4.scaled(batch=2, heads=4, layers=1, d_k=64, bits=8,
                                         scale_modes=DYN, round_mode=synth.RTN),
    "gla_d128_int8_f32scales": C3.scaled(batch=2, heads=2, bits=8, scale_modes=DYN,
                                         scale_dtype=synth.F32),
}


def _objects(wl):
    gpu = gpu_object(wl, synth.DYNAMIC, wl.batch, wl.layers)
    gpu.set_rowcol()
    cfg = oracle.Config(wl.d_k, wl.d_v, wl.kind, 0, scale_mode=synth.DYNAMIC,
                        round_mode=wl.round_mode, scale_f32=wl.scale_dtype == synth.F32,
                        gamma=wl.gamma, eps_b=wl.eps_b)
    return gpu, oracle.RcState(cfg, np.full(gpu.tiles, wl.bits))


def _run(wl, steps):
    gpu, orc = _objects(wl)
    assert gpu.kernel == "rc_kernel"
    assert gpu.sizes["scale_bytes"] == gpu.tiles * (wl.d_k + wl.d_v) * (
        4 if wl.scale_dtype == synth.F32 else 2)
    out = torch.empty((gpu.tiles, wl.d_v), dtype=torch.float32, device="cuda")
    tiles = np.arange(wl.batch * wl.heads)
    for step in range(steps):
        x = synth.gen_step(wl, step, layer=0, tiles=tiles)
        dq, dk, dv, dg = gpu_inputs(wl, x)
        gpu.step(dq, dk, dv, dg, out)
        oq, ok_, ov, oa, ob = oracle_inputs(wl, x)
        o_orc = orc.step(oq, ok_, ov, oa, ob)
        torch.cuda.synchronize()
        o_gpu = out.cpu().numpy()
        view = GpuView(gpu)
        for t in range(gpu.tiles):
            assert np.array_equal(view.scales[t], orc.scales[t]), (step, t)
            assert np.array_equal(view.tile_codes(t), orc.codes[t]), (step, t)
        assert np.array_equal(o_gpu.view(np.uint32), o_orc.view(np.uint32)), \
            (step, rel_err(o_gpu, o_orc))
    deq = gpu.dequant().cpu().numpy()
    assert np.array_equal(deq.view(np.uint32), orc.dequant().view(np.uint32))
    st = gpu.status()
    assert st["nonfinite"] == 0 and st["pipeline_timeouts"] == 0, st
    gpu.close()
    return orc


@pytest.mark.parametrize("name", list(CASES))
def test_rowcol_bit_exact(name):
    orc = _run(CASES[name], 8)
    assert np.abs(orc.codes).max() == (1 << (CASES[name].bits - 1)) - 1


def test_rowcol_many_tiles():
    """More tiles than CTAs (each CTA loops over tiles)."""
    _run(C1.scaled(batch=600, heads=4), 3)


def test_rowcol_rejects():
    bad = [C4.scaled(batch=1, heads=2, layers=1),                                  # persistent
           C5.scaled(batch=1, scale_modes=DYN),                                    # mixed widths
           C4.scaled(batch=1, heads=2, layers=1, bits=2, scale_modes=DYN),         # 2 bits
           C4.scaled(batch=1, heads=2, layers=1, rotation=1, scale_modes=DYN,
                     round_mode=synth.RTN)]                                        # rotated
    for wl in bad:
        g = gpu_object(wl, wl.scale_modes[0], wl.batch, 1)
        with pytest.raises(Q.QStateError):
            g.set_rowcol()
        g.close()
    wl = C4.scaled(batch=1, heads=2, layers=1, scale_modes=DYN)
    g = gpu_object(wl, synth.DYNAMIC, 1, 1)
    g.set_rowcol()
    with pytest.raises(Q.QStateError):
        g.set_rowcol()
    with pytest.raises(Q.QStateError):
        g.set_pw(4)
    with pytest.raises(Q.QStateError):
        g.set_lrb(0, 4, 0.5)
    g.close()
