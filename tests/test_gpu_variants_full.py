"""Full-size parity of the layout variants of the 24-layer Gated DeltaNet
decode (B256 H32 d128, 196 608 tiles), in the launch configuration the
benchmark times (one launch over every tile of every layer): the oracle
steps 48 sampled tiles from the same zero state with the same inputs, and
the sampled tiles' outputs, codes, scales and side state are compared.

- INT4+Had and key-row x value-column scales: bit-exact after 3 steps.
- PW-S8: bit-exact after 10 steps (the window full, two pairs merged).
- LRB+BDR (k = 1, m = 15), and the same bypass on the GLA decode (a decay
  factor per key row; as many replicas of the L2-sized B128 H16 layer as
  the benchmark steps, 32 x 2 048 tiles on B200): bit-exact through the first merge and
  up to the second; at the second merge outputs, codes, scales and counts
  are still bit-exact and the kept rank-1 residual is within the tolerance
  of the small-case test of its optimum (the oracle's truncated SVD).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_recurrent_state_decode_b200 import synth

from parity_util import (GpuView, bench_layers, compare, concat_inputs, gpu_inputs, gpu_object,
                         oracle_inputs, oracle_state)

pytestmark = pytest.mark.gpu
THREADS = 16


def _sample(wl):
    T = wl.tiles_per_layer * wl.layers
    rng = np.random.default_rng(11)
    return np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 46)])), T


def _step(wl, gpu, step, sample, T):
    x = concat_inputs([synth.gen_step(wl, step, layer=l) for l in range(wl.layers)])
    qd, kd, vd, gd = gpu_inputs(wl, x)
    out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
    gpu.step(qd, kd, vd, gd, out)
    sub = synth.StepInputs(x.q[sample], x.k[sample], x.v[sample],
                           None if x.gates is None else x.gates[sample])
    torch.cuda.synchronize()
    return out[torch.from_numpy(sample).cuda()].cpu().numpy(), oracle_inputs(wl, sub)


def _cfg(wl, mode):
    return oracle.Config(wl.d_k, wl.d_v, wl.kind, wl.group, scale_mode=mode,
                         round_mode=wl.round_mode, scale_f32=wl.scale_dtype == synth.F32,
                         gamma=wl.gamma, eps_b=wl.eps_b, rotate=wl.rotation)


@pytest.mark.parametrize("name,steps", [("gdn_l24_b256_h32_d128_int4g32_had", 3),
                                        ("gdn_l24_b256_h32_d128_int4rc", 3)])
def test_full_size_sampled_had_and_rowcol(name, steps):
    wl = synth.workload(name)
    sample, T = _sample(wl)
    mode = wl.scale_modes[0]
    gpu = gpu_object(wl, mode, wl.batch, wl.layers)
    if wl.rowcol:
        gpu.set_rowcol()
        orc = oracle.RcState(_cfg(wl, mode), np.full(len(sample), wl.bits))
    else:
        orc = oracle_state(wl, mode, sample % wl.heads)
    for step in range(steps):
        o_gpu, oin = _step(wl, gpu, step, sample, T)
        o_orc = orc.step(*oin) if wl.rowcol else orc.step(*oin, threads=THREADS)
    out_full = np.zeros((T, wl.d_v), np.float32)
    out_full[sample] = o_gpu
    stats = compare(GpuView(gpu), out_full, orc, o_orc, sample, range(len(sample)))
    assert stats["flips"] == 0 and np.array_equal(o_gpu.view(np.uint32), o_orc.view(np.uint32)), stats
    assert gpu.status()["nonfinite"] == 0
    gpu.close()


def test_full_size_sampled_pw():
    wl = synth.workload("gdn_l24_b256_h32_d128_int4g64_pw8")
    sample, T = _sample(wl)
    mode = wl.scale_modes[0]
    gpu = gpu_object(wl, mode, wl.batch, wl.layers)
    gpu.set_pw(wl.pw)
    orc = oracle.PwState(_cfg(wl, mode), np.full(len(sample), wl.bits), wl.pw)
    for step in range(wl.pw + 2):
        o_gpu, oin = _step(wl, gpu, step, sample, T)
        o_orc = orc.step(*oin)
        assert np.array_equal(o_gpu.view(np.uint32), o_orc.view(np.uint32)), step
    idx = torch.from_numpy(sample).cuda()
    w = {n: t[idx].cpu().numpy() for n, t in gpu.pw_export().items()}
    assert np.array_equal(w["head"], orc.head) and np.array_equal(w["count"], orc.count)
    assert np.array_equal(w["A"], orc.A) and np.array_equal(w["B"], orc.B)
    view = GpuView(gpu)
    for i, t in enumerate(sample):
        assert np.array_equal(view.tile_codes(t), orc.codes[i]), t
        assert np.array_equal(view.scales[t], orc.scales[i]), t
    gpu.close()


@pytest.mark.parametrize("name", ["gdn_l24_b256_h32_d128_int4g32_lrb",
                                  "gla_b128_h16_d128_int4g32_lrb"])
def test_full_size_sampled_lrb(name):
    wl = synth.workload(name)
    wl = wl.scaled(layers=bench_layers(wl))
    k, m, eps_l = wl.lrb
    sample, T = _sample(wl)
    mode = wl.scale_modes[0]
    gpu = gpu_object(wl, mode, wl.batch, wl.layers)
    gpu.set_lrb(k, m, eps_l)
    orc = oracle.LrbState(_cfg(wl, mode), np.full(len(sample), wl.bits), k=k, m=m, eps_l=eps_l,
                          keep_resid=True)
    idx = torch.from_numpy(sample).cuda()
    for step in range(2 * m):
        o_gpu, oin = _step(wl, gpu, step, sample, T)
        o_orc = orc.step(*oin)
        assert np.array_equal(o_gpu.view(np.uint32), o_orc.view(np.uint32)), step
    b = {n: t[idx].cpu().numpy() for n, t in gpu.lrb_export().items()}
    assert np.array_equal(b["n"][:, 0], orc.nres) and np.array_equal(b["n"][:, 1], orc.nnew)
    assert np.all(b["D"] == 1.0) and np.all(orc.D == 1.0)
    view = GpuView(gpu)
    for i, t in enumerate(sample):
        assert np.array_equal(view.tile_codes(t), orc.codes[i]), t
        assert np.array_equal(view.scales[t], orc.scales[i]), t
        R = orc.resid[i].astype(np.float64)
        Pg = float(b["g"][i, 0]) * np.outer(b["u"][i, 0].astype(np.float64),
                                            b["w"][i, 0].astype(np.float64))
        e_g, e_o, nr = np.linalg.norm(R - Pg), np.linalg.norm(R - orc.bypass(i)), np.linalg.norm(R)
        assert e_g <= (1 + 1e-2) * e_o + 4e-3 * nr, (t, e_g, e_o, nr)
    assert any(np.any(orc.resid[i]) for i in range(len(sample)))
    gpu.close()
