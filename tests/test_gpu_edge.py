"""GPU edge cases of the decode step, each against the CPU oracle.

- the most negative two's-complement code of every width, which the pages'
  symmetric code range never produces but an imported state may hold;
- per-head widths with a rank-1 update (RetNet, Mamba2, GLA) and the yoked
  reference state on both non-square tile shapes;
- objects of different stage sizes that share one kernel (the dynamic
  shared-memory limit of that kernel is only ever raised);
- the yoked bound on the GPU state: no group of the quantized state exceeds
  the reference state's group maximum ("When Dynamic Scaling Fails",
  Abstract: the yoked scale follows the full-precision reference).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_recurrent_state_decode_b200 import qstate as Q
from bit_recurrent_state_decode_b200 import synth

from parity_util import (GpuView, compare, gpu_inputs, gpu_object, import_oracle_state,
                         oracle_inputs, oracle_state, run_pair)

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_recurrent_state_decode_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
@pytest.mark.parametrize("mode", [synth.DYNAMIC, synth.PERSISTENT])
def test_imported_most_negative_code(bits, mode):
    """A state holding -2^(b-1) (and every other code of the width) is
    unpacked, decayed, updated, requantized and repacked like the oracle."""
    wl = C4.scaled(batch=2, heads=4, layers=1, bits=bits, group=64, scale_modes=(mode,))
    rng = np.random.default_rng(100 + bits)
    T = wl.batch * wl.heads
    st = oracle_state(wl, mode, np.tile(np.arange(wl.heads), wl.batch))
    lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    st.codes[:] = rng.integers(lo, hi + 1, size=st.codes.shape).astype(np.int8)
    st.codes[:, 0, :8] = lo                      # certainly present
    # binary16 scales around the state magnitudes of the workload
    sc = rng.uniform(0.01, 0.2, size=st.scales.shape).astype(np.float16)
    st.scales[:] = sc.astype(np.float32)
    obj = gpu_object(wl, mode, wl.batch, 1)
    import_oracle_state(obj, st)
    for step in range(3):
        x = synth.gen_step(wl, step, tiles=np.arange(T))
        qd, kd, vd, gd = gpu_inputs(wl, x)
        out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
        obj.step(qd, kd, vd, gd, out)
        o_orc = st.step(*oracle_inputs(wl, x))
        compare(GpuView(obj), out.cpu().numpy(), st, o_orc, range(T), range(T))
    obj.close()


@pytest.mark.parametrize("kind", [synth.RETNET, synth.MAMBA2, synth.GLA])
def test_mixed_widths_rank1(kind):
    base = {synth.RETNET: C1, synth.MAMBA2: C2, synth.GLA: C3}[kind]
    wl = base.scaled(batch=2, heads=4, layers=1, d_k=128, d_v=128, bits=0, group=32,
                     head_bits_multiset=((2, 1), (4, 1), (6, 1), (8, 1)),
                     scale_modes=(synth.DYNAMIC, synth.PERSISTENT),
                     q_sigma=base.q_sigma or 0.1, k_sigma=base.k_sigma or 0.1)
    stats, _, _ = run_pair(wl, steps=12, check_every=4)
    assert all(s["flips"] == 0 for s in stats)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
@pytest.mark.parametrize("kind", [synth.GLA, synth.GDN])
def test_yoked_non_square(dk, dv, kind):
    base = C3 if kind == synth.GLA else C4
    wl = base.scaled(batch=2, heads=3, layers=1, d_k=dk, d_v=dv, bits=4, group=dv // 2,
                     scale_modes=(synth.YOKED,), scale_dtype=synth.F32,
                     round_mode=synth.BDR if kind == synth.GDN else synth.RTN)
    stats, _, _ = run_pair(wl, steps=12, check_every=4)
    assert all(s["flips"] == 0 for s in stats)


def test_stage_sizes_sharing_one_kernel():
    """A GLA INT8 g16 object (group scales and the gate vector staged) is
    created before a Mamba2 INT8 per-token object (neither staged): both
    launch the same kernel.  Creating the second must not lower the
    kernel's shared-memory limit below what the first launches with."""
    gla = C3.scaled(batch=2, heads=2, layers=1, bits=8, group=16, qkv_dtype=synth.F32,
                    scale_modes=(synth.PERSISTENT,))
    mam = C2.scaled(batch=2, heads=2, layers=1, d_v=128)
    first = gpu_object(gla, synth.PERSISTENT, 2, 1)
    second = gpu_object(mam, synth.DYNAMIC, 2, 1)
    T = 4
    for wl, obj, mode in ((gla, first, synth.PERSISTENT), (mam, second, synth.DYNAMIC)):
        st = oracle_state(wl, mode, np.tile(np.arange(2), 2))
        for step in range(3):
            x = synth.gen_step(wl, step, tiles=np.arange(T))
            qd, kd, vd, gd = gpu_inputs(wl, x)
            out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
            obj.step(qd, kd, vd, gd, out)
            o_orc = st.step(*oracle_inputs(wl, x))
        compare(GpuView(obj), out.cpu().numpy(), st, o_orc, range(T), range(T))
    first.close()
    second.close()


def test_yoked_group_bound_on_gpu():
    """Over 320 steps of the long-horizon mixed-width workload (yoked, fp32
    scales): every group of the dequantized GPU state stays within the
    reference state's group maximum times (1 + 2^-23)."""
    wl = C5.scaled(batch=2)
    obj = gpu_object(wl, synth.YOKED, 2, 1)
    T = obj.tiles
    worst = 0.0
    for step in range(320):
        x = synth.gen_step(wl, step, tiles=np.arange(T))
        qd, kd, vd, gd = gpu_inputs(wl, x)
        out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
        obj.step(qd, kd, vd, gd, out)
        if (step + 1) % 40 == 0:
            deq = obj.dequant().cpu().numpy().reshape(T, wl.d_k, wl.d_v // 64, 64)
            ref = GpuView(obj).ref.reshape(T, wl.d_k, wl.d_v // 64, 64)
            mq = np.abs(deq).max(axis=-1).astype(np.float64)
            mr = np.abs(ref).max(axis=-1).astype(np.float64)
            assert np.all(mq <= mr * (1 + 2.0 ** -23)), step
            worst = max(worst, float(np.max(np.where(mr > 0, mq / np.where(mr > 0, mr, 1), 0))))
    assert 0.5 < worst <= 1 + 2.0 ** -23
    obj.close()
