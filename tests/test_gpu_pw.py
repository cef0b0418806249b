"""GPU parity of the Gated DeltaNet decode step with a pure-write sliding
window (PW) of "Low-Bit GDN Recurrent-State Quantization: Global
Gradient-aware Allocation and Pure-Write Sliding Windows" (Abstract) against
the oracle's PW step.

Every result is defined element by element (canonical sums, one fma per pair
and element, E4M3 nearest-even saturating), so the outputs, the history's
codes and scales, both sides of every pair (E4M3 bytes), the slot of the
oldest pair and the pair counts are bit-exact at every step: while the
window fills, once it is full (a pair leaves into the history every step)
and for a window of one pair.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_recurrent_state_decode_b200 import qstate as Q
from bit_recurrent_state_decode_b200 import synth

from parity_util import GpuView, gpu_inputs, gpu_object, oracle_inputs, rel_err

pytestmark = pytest.mark.gpu

C4 = synth.WORKLOADS["gdn_l24_b256_h32_d128_int4g64_bdr"]

# (workload, W): INT4 g64 persistent BDR bf16 (the 24-layer GDN layout) with
# the PW-S8 window and others; INT8 g32 dynamic RTN fp32 at d = 64; INT4
# per-token scales
CASES = {
    "d128_int4g64_bdr_W8": (C4.scaled(batch=2, heads=4, layers=1, eps_b=0.3), 8),
    "d128_int4g64_bdr_W1": (C4.scaled(batch=2, heads=4, layers=1), 1),
    "d128_int4g64_bdr_W16": (C4.scaled(batch=1, heads=4, layers=1, eps_b=0.3), 16),
    "d64_int8g32_rtn_f32_W3": (C4.scaled(batch=2, heads=4, layers=1, d_k=64, d_v=64, bits=8,
                                         group=32, scale_modes=(synth.DYNAMIC,),
                                         round_mode=synth.RTN, qkv_dtype=synth.F32,
                                         gate_dtype=synth.F32), 3),
    "d128_int4tok_dynamic_W5": (C4.scaled(batch=2, heads=4, layers=1, group=0,
                                          scale_modes=(synth.DYNAMIC,)), 5),
}


def _objects(wl, W):
    mode = wl.scale_modes[0]
    gpu = gpu_object(wl, mode, wl.batch, wl.layers)
    gpu.set_pw(W)
    cfg = oracle.Config(wl.d_k, wl.d_v, wl.kind, wl.group, scale_mode=mode,
                        round_mode=wl.round_mode, scale_f32=wl.scale_dtype == synth.F32,
                        gamma=wl.gamma, eps_b=wl.eps_b)
    return gpu, oracle.PwState(cfg, np.full(gpu.tiles, wl.bits), W)


def _step(wl, gpu, orc, step, out):
    x = synth.gen_step(wl, step, layer=0, tiles=np.arange(wl.batch * wl.heads))
    dq, dk, dv, dg = gpu_inputs(wl, x)
    gpu.step(dq, dk, dv, dg, out)
    oq, ok_, ov, oa, ob = oracle_inputs(wl, x)
    o_orc = orc.step(oq, ok_, ov, oa, ob)
    torch.cuda.synchronize()
    return out.cpu().numpy(), o_orc


def _assert_exact(gpu, orc, o_gpu, o_orc, step):
    w = {n: x.cpu().numpy() for n, x in gpu.pw_export().items()}
    assert np.array_equal(w["head"], orc.head) and np.array_equal(w["count"], orc.count), step
    for t in range(gpu.tiles):
        h, n = int(orc.head[t]), int(orc.count[t])
        held = [(h + l) % orc.W for l in range(n)]
        for sl in held:
            bad = np.nonzero(w["A"][t, sl] != orc.A[t, sl])[0]
            assert bad.size == 0, (step, t, sl, bad[:8].tolist(), w["A"][t, sl, bad[:8]].tolist(),
                                   orc.A[t, sl, bad[:8]].tolist())
        assert np.array_equal(w["B"][t, held], orc.B[t, held]), (step, t)
    view = GpuView(gpu)
    for t in range(gpu.tiles):
        assert np.array_equal(view.tile_codes(t), orc.codes[t]), (step, t)
        assert np.array_equal(view.scales[t], orc.scales[t]), (step, t)
    assert np.array_equal(o_gpu.view(np.uint32), o_orc.view(np.uint32)), \
        (step, rel_err(o_gpu, o_orc))


@pytest.mark.parametrize("name", list(CASES))
def test_pw_bit_exact(name):
    wl, W = CASES[name]
    gpu, orc = _objects(wl, W)
    assert gpu.kernel == "pw_kernel"
    out = torch.empty((gpu.tiles, wl.d_v), dtype=torch.float32, device="cuda")
    for step in range(W + 6):
        o_gpu, o_orc = _step(wl, gpu, orc, step, out)
        _assert_exact(gpu, orc, o_gpu, o_orc, step)
    assert np.all(orc.count == W) and orc.codes.any()
    st = gpu.status()
    assert st["pipeline_timeouts"] == 0 and st["nonfinite"] == 0, st
    gpu.close()


def test_pw_many_tiles():
    """More tiles than CTAs (each CTA loops over tiles)."""
    wl = C4.scaled(batch=48, heads=4, layers=1, eps_b=0.3)
    gpu, orc = _objects(wl, 2)
    out = torch.empty((gpu.tiles, wl.d_v), dtype=torch.float32, device="cuda")
    for step in range(4):
        o_gpu, o_orc = _step(wl, gpu, orc, step, out)
        _assert_exact(gpu, orc, o_gpu, o_orc, step)
    gpu.close()


def test_pw_rejects():
    bad = [
        synth.WORKLOADS["retnet_b1_h2_d64_int4g64"],                           # not GDN
        C4.scaled(batch=1, heads=2, layers=1, scale_modes=(synth.YOKED,)),     # yoked
        C4.scaled(batch=1, heads=2, layers=1, d_v=64),                         # d_k != d_v
        C4.scaled(batch=1, heads=2, layers=1, bits=2),                         # 2-bit codes
    ]
    for wl in bad:
        g = gpu_object(wl, wl.scale_modes[0], wl.batch, 1)
        with pytest.raises(Q.QStateError):
            g.set_pw(4)
        g.close()
    wl = C4.scaled(batch=1, heads=2, layers=1)
    for W in (0, -1, 17):
        g = gpu_object(wl, wl.scale_modes[0], wl.batch, 1)
        with pytest.raises(Q.QStateError):
            g.set_pw(W)
        g.close()
    g = gpu_object(wl, wl.scale_modes[0], wl.batch, 1)
    g.set_pw(16)
    with pytest.raises(Q.QStateError):
        g.set_pw(4)                                # already set
    with pytest.raises(Q.QStateError):
        g.set_lrb(0, 4, 0.5)                       # a window and a bypass exclude each other
    g.close()


def test_pw_reset_and_import_empty_the_window():
    wl = C4.scaled(batch=1, heads=4, layers=1)
    gpu, orc = _objects(wl, 3)
    out = torch.empty((gpu.tiles, wl.d_v), dtype=torch.float32, device="cuda")
    for step in range(5):
        _step(wl, gpu, orc, step, out)
    w = gpu.pw_export()
    assert int(w["count"].sum()) == 3 * gpu.tiles
    codes, scales, ref = gpu.export()
    gpu.import_(codes, scales, ref)
    w = gpu.pw_export()
    assert int(w["count"].sum()) == 0 and int(w["head"].sum()) == 0
    gpu.reset()
    w = gpu.pw_export()
    assert int(w["count"].sum()) == 0 and not gpu.dequant().any()
    gpu.close()
