"""Write bounds and isolation of every kernel, and allocation failure.

- Guard bands: the caller's out buffer sits between bands of canary words,
  and is itself filled with the canary before each step.  Every kernel (the
  step kernel with one code width, its generic body for per-head widths and
  yoked scales, the row-batched kernel, the diagnostic step kernel, and the
  bypass, window and row x column kernels) must write every element of out
  (no canary left inside) and nothing outside it (the bands intact), step
  after step.
- Isolation: stepping one object leaves another object's state as it was.
- An allocation that cannot succeed returns QSTATE_ENOMEM, and the CUDA
  context stays usable.
"""
import numpy as np
import pytest
import torch

from bit_recurrent_state_decode_b200 import qstate as Q
from bit_recurrent_state_decode_b200 import synth

from parity_util import gpu_inputs, gpu_object

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)
BAND = 64                        # floats on each side (256 bytes: keeps out 16-byte aligned)
CANARY = 0x7FBADBAD              # a NaN pattern no step produces from finite inputs


def _rowcol(wl):
    return wl.scaled(scale_modes=(synth.DYNAMIC,))


CASES = {
    # name: (workload, scale mode, setup, kernel)
    "step_gdn_bdr": (C4.scaled(batch=2, heads=4, layers=1), None, None, "step_kernel"),
    "step_mamba2_tok": (C2.scaled(batch=2, heads=4), None, None, None),
    "step_retnet_d64": (C1.scaled(batch=3, heads=4), None, None, None),
    "rows_gla": (C3.scaled(batch=2, heads=4), None, None, "rows_kernel"),
    "generic_mixed_yoked": (C5.scaled(batch=1), synth.YOKED, None, "step_kernel"),
    "diagnostic_taxonomy": (C4.scaled(batch=2, heads=4, layers=1), None,
                            lambda g: g.set_taxonomy(True), "step_kernel"),
    "lrb_gdn": (C4.scaled(batch=2, heads=4, layers=1, eps_b=0.3), None,
                lambda g: g.set_lrb(1, 3, 0.5), "lrb_kernel"),
    "lrb_gla": (C3.scaled(batch=2, heads=4), None, lambda g: g.set_lrb(0, 3, 0.5), "lrb_kernel"),
    "pw": (C4.scaled(batch=2, heads=4, layers=1), None, lambda g: g.set_pw(4), "pw_kernel"),
    "rowcol": (_rowcol(C4.scaled(batch=2, heads=4, layers=1)), None, lambda g: g.set_rowcol(),
               "rc_kernel"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_out_written_exactly(name):
    wl, mode, setup, kernel = CASES[name]
    mode = wl.scale_modes[0] if mode is None else mode
    gpu = gpu_object(wl, mode, wl.batch, wl.layers)
    if setup is not None:
        setup(gpu)
    if kernel is not None:
        assert gpu.kernel == kernel, gpu.kernel
    T, dv = gpu.tiles, wl.d_v
    full = torch.empty(T * dv + 2 * BAND, dtype=torch.int32, device="cuda")
    out = full[BAND:BAND + T * dv].view(torch.float32).view(T, dv)
    canary = np.int32(np.uint32(CANARY).view(np.int32))
    tiles = np.arange(wl.batch * wl.heads)
    for step in range(7):
        full.fill_(int(canary))
        x = synth.gen_step(wl, step, layer=0, tiles=tiles)
        gpu.step(*gpu_inputs(wl, x), out)
        torch.cuda.synchronize()
        f = full.cpu().numpy()
        assert np.all(f[:BAND] == canary) and np.all(f[BAND + T * dv:] == canary), (name, step)
        inside = f[BAND:BAND + T * dv]
        assert not np.any(inside == canary), (name, step, int(np.sum(inside == canary)))
    st = gpu.status()
    assert st["nonfinite"] == 0 and st["pipeline_timeouts"] == 0, st
    gpu.close()


def test_objects_are_isolated():
    """Steps of one object change neither the codes nor the scales of
    another object of the same layout, before or after that one's own steps."""
    wl = C4.scaled(batch=2, heads=4, layers=1)
    mode = wl.scale_modes[0]
    a = gpu_object(wl, mode, wl.batch, wl.layers)
    b = gpu_object(wl, mode, wl.batch, wl.layers)
    out = torch.empty((a.tiles, wl.d_v), dtype=torch.float32, device="cuda")
    tiles = np.arange(wl.batch * wl.heads)
    for step in range(5):
        a.step(*gpu_inputs(wl, synth.gen_step(wl, step, layer=0, tiles=tiles)), out)
    codes_b, scales_b, _ = b.export()
    torch.cuda.synchronize()
    assert not codes_b.any() and not scales_b.float().any()
    codes_a, scales_a, _ = a.export()
    for step in range(5, 9):
        b.step(*gpu_inputs(wl, synth.gen_step(wl, step, layer=0, tiles=tiles)), out)
    codes_a2, scales_a2, _ = a.export()
    torch.cuda.synchronize()
    assert torch.equal(codes_a, codes_a2) and torch.equal(scales_a.float(), scales_a2.float())
    a.close()
    b.close()


def test_allocation_failure_is_reported():
    """A state of 2^26 tiles of 128 x 128 INT8 codes (1.1 TB) cannot be
    allocated: qstate_create returns QSTATE_ENOMEM, releases what it took,
    and the next object is created and stepped as usual."""
    with pytest.raises(Q.QStateError) as e:
        Q.QState(1 << 20, 64, 128, 128, Q.GDN, bits=8, group=0, qkv_dtype=Q.BF16,
                 gate_dtype=Q.BF16)
    assert e.value.code == -2
    wl = C4.scaled(batch=1, heads=4, layers=1)
    g = gpu_object(wl, wl.scale_modes[0], wl.batch, wl.layers)
    out = torch.empty((g.tiles, wl.d_v), dtype=torch.float32, device="cuda")
    g.step(*gpu_inputs(wl, synth.gen_step(wl, 0, layer=0, tiles=np.arange(4))), out)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    g.close()
