"""GPU error-accounting counters against the CPU oracle.

The rounding taxonomy of Figure 4 of "Preserving Updates in Low-Bit Recurrent
State Quantization" (an update lost in rounding, moved to another grid point,
or reversed) and the lost fraction of its Table 5, counted by the decode step
itself (qstate_set_taxonomy), equal the oracle's counts on the same inputs
exactly; and the counter of warps that rounded element by element shows which
rounding form ran, so both forms are proven against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.diagnostics import ErrorAccount
from bit_recurrent_state_decode_b200 import synth

from parity_util import (GpuView, compare, gpu_inputs, gpu_object, oracle_inputs, oracle_state,
                         run_pair)

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_recurrent_state_decode_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _oracle_taxonomy_state(wl, mode, heads):
    cfg = oracle.Config(wl.d_k, wl.d_v, wl.kind, wl.group, scale_mode=mode,
                        round_mode=wl.round_mode, scale_f32=wl.scale_dtype == synth.F32,
                        gamma=wl.gamma, eps_b=wl.eps_b, taxonomy=True)
    hb = wl.head_bits()
    bits = hb[heads] if hb is not None else np.full(len(heads), wl.bits)
    return oracle.State(cfg, bits)


@pytest.mark.parametrize("name", ["gdn", "gdn_eps", "mixed", "gla", "mamba2", "retnet"])
def test_taxonomy_counts_equal_oracle(name):
    wl = {"gdn": C4.scaled(batch=2, layers=1), "gdn_eps": C4.scaled(batch=2, layers=1, eps_b=0.3),
          "mixed": C5.scaled(batch=2), "gla": C3.scaled(batch=2),
          "mamba2": C2.scaled(batch=2), "retnet": C1}[name]
    T = wl.batch * wl.heads
    heads = np.tile(np.arange(wl.heads), wl.batch)
    for mode in wl.scale_modes:
        gpu = gpu_object(wl, mode, wl.batch, 1)
        gpu.set_taxonomy(True)
        orc = _oracle_taxonomy_state(wl, mode, heads)
        acc = ErrorAccount(oracle_state(wl, mode, heads))
        for step in range(24):
            x = synth.gen_step(wl, step, tiles=np.arange(T))
            qd, kd, vd, gd = gpu_inputs(wl, x)
            out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
            gpu.step(qd, kd, vd, gd, out)
            o_orc = orc.step(*oracle_inputs(wl, x))
            acc.step(*oracle_inputs(wl, x))
        compare(GpuView(gpu), out.cpu().numpy(), orc, o_orc, range(T), range(T))
        st = gpu.status()
        oc = orc.counts.as_dict()
        for key in ("lost", "moved", "reversed", "bdr_applied"):
            assert st[key] == oc[key], (name, mode, key, st[key], oc[key])
        assert st["lost"] + st["moved"] + st["reversed"] > 0
        n = st["lost"] + st["moved"] + st["reversed"]
        assert n == acc.n_updates and st["lost"] / n == acc.lost_fraction()
        gpu.close()


def test_taxonomy_off_counts_nothing():
    wl = C4.scaled(batch=2, layers=1)
    stats, status, _ = run_pair(wl, steps=6)
    for m in status:
        assert status[m]["lost"] == status[m]["moved"] == status[m]["reversed"] == 0


def test_both_rounding_forms_against_the_oracle():
    """With the workload's inputs the fast rounding form runs for nearly every
    warp; with a vanishing beta (updates below the state's resolution, so the
    sign of x - a is no longer the sign of the update term) the element-wise
    form runs.  Both agree with the oracle code for code."""
    wl = C4.scaled(batch=2, layers=1)
    T = wl.batch * wl.heads
    heads = np.tile(np.arange(wl.heads), wl.batch)
    for tiny in (False, True):
        gpu = gpu_object(wl, synth.PERSISTENT, wl.batch, 1)
        gpu.set_taxonomy(True)             # the path counter is kept with the taxonomy
        orc = oracle_state(wl, synth.PERSISTENT, heads)
        for step in range(16):
            x = synth.gen_step(wl, step, tiles=np.arange(T))
            if tiny and step >= 8:
                g = synth.bf16_bits_to_f32(x.gates).copy()
                g[:, 1] = 1e-30
                x = synth.StepInputs(x.q, x.k, x.v, synth.f32_to_bf16_bits(g))
            qd, kd, vd, gd = gpu_inputs(wl, x)
            out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
            gpu.step(qd, kd, vd, gd, out)
            o_orc = orc.step(*oracle_inputs(wl, x))
            compare(GpuView(gpu), out.cpu().numpy(), orc, o_orc, range(T), range(T))
        exact = gpu.status()["exact_path_warps"]
        warp_tiles = 16 * T * 8              # 8 warps per 128 x 128 tile
        if tiny:
            assert exact >= 8 * T * 8        # every warp of the vanishing steps
        else:
            assert exact < 0.05 * warp_tiles
        gpu.close()
