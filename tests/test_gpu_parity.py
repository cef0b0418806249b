"""GPU parity: the CUDA step (called through the C ABI) against the CPU oracle
on the same seeded synthetic inputs.

Bars: packed codes bit-exact (at most 1e-5 of codes one level off), scales
bit-exact, outputs within 1e-3 max relative error per tile; the fp32 state
(quantization disabled) and the yoked reference state bit-exact.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from bit_recurrent_state_decode_b200 import qstate as Q
from bit_recurrent_state_decode_b200 import synth

from parity_util import (GpuView, bench_layers, compare, concat_inputs, gpu_inputs, gpu_object,
                         import_oracle_state, oracle_inputs, oracle_state, rel_err, run_pair)

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)
THREADS = os.cpu_count() or 4


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_recurrent_state_decode_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


# ------------------------------------------------------------ 32-bit recurrence
@pytest.mark.parametrize("kind", [synth.RETNET, synth.MAMBA2, synth.GLA, synth.GDN])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("dt", [synth.F32, synth.BF16])
def test_fp32_recurrence_bit_exact(kind, dk, dv, dt):
    base = {synth.RETNET: C1, synth.MAMBA2: C2, synth.GLA: C3, synth.GDN: C4}[kind]
    wl = base.scaled(batch=3, heads=5, d_k=dk, d_v=dv, bits=32, group=0, layers=1,
                     scale_modes=(synth.DYNAMIC,), round_mode=synth.RTN, qkv_dtype=dt,
                     gate_dtype=dt, head_bits_multiset=(), q_sigma=base.q_sigma or 0.1,
                     k_sigma=base.k_sigma or 0.1)
    stats, status, _ = run_pair(wl, steps=12)
    assert all(s["out_rel"] == 0.0 for s in stats)   # identical order: bit-exact outputs
    assert status[synth.DYNAMIC]["nonfinite"] == 0


# ------------------------------------------------------------ the five workloads
def test_retnet_full_horizon():
    stats, status, _ = run_pair(C1, steps=C1.steps, check_every=16)
    assert all(s["flips"] == 0 for s in stats)
    st = status[synth.DYNAMIC]
    assert (st["nonfinite"], st["saturated"], st["pipeline_timeouts"]) == (0, 0, 0)


@pytest.mark.parametrize("name,batch_sel,layers,steps", [
    ("mamba2", [0, 9], 1, 96),
    ("gla", [0, 3, 127], 1, 96),
    ("gdn", [0, 255], 2, 64),
    ("mixed", [0, 31], 1, 96),
])
def test_workload_reduced_batch(name, batch_sel, layers, steps):
    wl = {"mamba2": C2, "gla": C3, "gdn": C4, "mixed": C5}[name]
    stats, status, ocounts = run_pair(wl, batch_sel=batch_sel, layers=layers, steps=steps,
                                      check_every=8)
    assert all(s["flips"] == 0 for s in stats), [s for s in stats if s["flips"]]
    for m in status:
        assert status[m]["nonfinite"] == 0 and status[m]["pipeline_timeouts"] == 0
        assert status[m]["saturated"] == ocounts[m]["saturated"]


def test_gdn_teacher_forced():
    stats, _, _ = run_pair(C4, batch_sel=[7], layers=1, steps=24, start_step=100,
                           teacher_forced=True)
    assert all(s["flips"] == 0 for s in stats)


# ------------------------------------------------------------ full sizes, sampled tiles
@pytest.mark.parametrize("name,steps", [("mamba2", 3), ("gla", 3), ("gdn", 2), ("mixed", 3)])
def test_full_size_sampled_tiles(name, steps):
    """The full-size object in the launch configuration the benchmark times
    (one launch over every tile of every layer, the layer replicas of the
    L2-sized configurations included); the oracle steps 48 sampled tiles
    from the same zero state with the same inputs."""
    wl = {"mamba2": C2, "gla": C3, "gdn": C4, "mixed": C5}[name]
    layers = bench_layers(wl)
    assert layers > 1
    rng = np.random.default_rng(7)
    T = wl.tiles_per_layer * layers
    sample = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 46)]))
    heads = sample % wl.heads
    for mode in wl.scale_modes:
        gpu = gpu_object(wl, mode, wl.batch, layers)
        orc = oracle_state(wl, mode, heads)
        for step in range(steps):
            x = concat_inputs([synth.gen_step(wl, step, layer=l) for l in range(layers)])
            qd, kd, vd, gd = gpu_inputs(wl, x)
            out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
            gpu.step(qd, kd, vd, gd, out)
            sub = synth.StepInputs(x.q[sample], x.k[sample], x.v[sample],
                                   None if x.gates is None else x.gates[sample])
            o_orc = orc.step(*oracle_inputs(wl, sub), threads=THREADS)
            del qd, kd, vd, gd
        view = GpuView(gpu)
        compare(view, out.cpu().numpy(), orc, o_orc, sample, range(len(sample)))
        assert gpu.status()["nonfinite"] == 0
        gpu.close()


# ------------------------------------------------------------ long horizons, few tiles
@pytest.mark.parametrize("name,batch_sel,steps", [
    ("mamba2", [3], 1024),
    ("gla", [11], 1024),
    ("gdn", [5], 512),
    ("mixed", [2], 1024),
])
def test_long_horizon_few_tiles(name, batch_sel, steps):
    wl = {"mamba2": C2, "gla": C3, "gdn": C4, "mixed": C5}[name]
    stats, status, _ = run_pair(wl, batch_sel=batch_sel, layers=1, steps=steps,
                                check_every=128)
    flips = sum(s["flips"] for s in stats)
    assert flips == 0, stats


# ------------------------------------------------------------ edge cases
def test_empty_batch_is_noop():
    obj = Q.QState(0, 4, 128, 128, Q.GDN, bits=4, group=64, qkv_dtype=Q.BF16, gate_dtype=Q.BF16)
    assert obj.tiles == 0 and obj.bytes_per_step() == 0
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(16, dtype=torch.float32, device="cuda")
    obj.step(x, x, x, x, o)
    obj.close()


@pytest.mark.parametrize("variant", ["lrb", "lrb_gla", "pw", "rowcol"])
def test_empty_batch_with_a_variant(variant):
    """An object of no tiles takes every layout variant; its steps, dequant
    and exports are no-ops that return empty tensors."""
    kind = Q.GLA if variant == "lrb_gla" else Q.GDN
    obj = Q.QState(0, 4, 128, 128, kind, bits=4, group=32, qkv_dtype=Q.BF16,
                   gate_dtype=Q.F32 if kind == Q.GLA else Q.BF16)
    if variant.startswith("lrb"):
        obj.set_lrb(1, 15, 0.5)
        side = obj.lrb_export()
    elif variant == "pw":
        obj.set_pw(8)
        side = obj.pw_export()
    else:
        obj.set_rowcol()
        side = None
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(16, dtype=torch.float32 if kind == Q.GLA else torch.bfloat16, device="cuda")
    o = torch.zeros(16, dtype=torch.float32, device="cuda")
    obj.step(x, x, x, g, o)
    assert obj.bytes_per_step() == 0 and not o.any()
    assert obj.dequant().shape == (0, 128, 128)
    codes, scales, _ = obj.export()
    assert codes.numel() == 0 and scales.numel() == 0
    if side is not None:
        assert all(t.shape[0] == 0 for t in side.values())
    torch.cuda.synchronize()
    obj.close()


def test_zero_update_gives_zero_state():
    obj = Q.QState(2, 3, 64, 64, Q.RETNET, bits=4, group=64)
    q, k, v, g, out = obj.alloc_inputs()
    for t in (q, k, v):
        t.zero_()
    obj.step(q, k, v, g, out)
    codes, scales, _ = obj.export()
    assert int(codes.abs().sum()) == 0 and float(scales.float().abs().sum()) == 0.0
    assert float(out.abs().sum()) == 0.0
    obj.close()


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
@pytest.mark.parametrize("group", [8, 16, 32, 64, 128, 0])
@pytest.mark.parametrize("kind", [synth.GLA, synth.GDN])
def test_bits_and_groups(bits, group, kind):
    base = C3 if kind == synth.GLA else C4
    wl = base.scaled(batch=2, heads=3, layers=1, bits=bits, group=group,
                     scale_modes=(synth.DYNAMIC, synth.PERSISTENT, synth.YOKED),
                     round_mode=synth.BDR if kind == synth.GDN else synth.RTN)
    stats, _, _ = run_pair(wl, steps=10, check_every=5)
    assert all(s["flips"] == 0 for s in stats)


@pytest.mark.parametrize("kind", [synth.RETNET, synth.MAMBA2, synth.GLA, synth.GDN])
@pytest.mark.parametrize("group", [0, 32])
@pytest.mark.parametrize("sdt", [synth.F16, synth.F32])
@pytest.mark.parametrize("rm", [synth.RTN, synth.BDR])
def test_tile_bodies(kind, group, sdt, rm):
    """Every compiled tile body of a uniform-width object: one scale per tile or
    row groups, scalar or per-row decay, binary16 or binary32 scales, RTN or
    BDR, over both warp geometries."""
    base = {synth.RETNET: C1, synth.MAMBA2: C2, synth.GLA: C3, synth.GDN: C4}[kind]
    dk, dv = (128, 64) if (kind + group // 32) % 2 == 0 else (64, 128)
    wl = base.scaled(batch=2, heads=3, layers=1, d_k=dk, d_v=dv, bits=8 if group == 0 else 4,
                     group=group, scale_dtype=sdt, round_mode=rm,
                     scale_modes=(synth.DYNAMIC, synth.PERSISTENT), head_bits_multiset=(),
                     q_sigma=base.q_sigma or 0.1, k_sigma=base.k_sigma or 0.1)
    stats, status, _ = run_pair(wl, steps=8, check_every=4)
    assert all(s["flips"] == 0 for s in stats)


@pytest.mark.parametrize("eps", [0.0, 0.3])
def test_bdr_eps(eps):
    wl = C4.scaled(batch=2, heads=4, layers=1, eps_b=eps)
    stats, _, _ = run_pair(wl, steps=16, check_every=4)
    assert all(s["flips"] == 0 for s in stats)


@pytest.mark.parametrize("dv", [64, 128])      # the general kernel; the row-batched one
def test_saturation_and_nonfinite_counters(dv):
    obj = Q.QState(1, 2, 64, dv, Q.RETNET, bits=4, group=64)
    q, k, v, g, out = obj.alloc_inputs()
    q.fill_(1.0)
    k.fill_(1e4)
    v.fill_(1e3)
    obj.step(q, k, v, g, out)
    st = obj.status()
    assert st["saturated"] == 2 * 64 * (dv // 64) and st["nonfinite"] == 0
    codes, scales, _ = obj.export()
    assert torch.all(scales.float() == 65504.0)
    k.fill_(float("nan"))
    obj.step(q, k, v, g, out)
    assert obj.status()["nonfinite"] == 2
    obj.close()


def test_step_host_matches_step_and_dequant():
    wl = C4.scaled(batch=2, heads=4, layers=2)
    a = gpu_object(wl, synth.PERSISTENT, 2, 2)
    b = gpu_object(wl, synth.PERSISTENT, 2, 2)
    T = a.tiles
    for step in range(6):
        x = concat_inputs([synth.gen_step(wl, step, layer=l, tiles=np.arange(8)) for l in range(2)])
        qd, kd, vd, gd = gpu_inputs(wl, x)
        out_a = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
        a.step(qd, kd, vd, gd, out_a)
        hq, hk, hv, hg = (t.cpu().pin_memory() for t in (qd, kd, vd, gd))
        out_b = torch.empty((T, wl.d_v), dtype=torch.float32).pin_memory()
        b.step_host(hq, hk, hv, hg, out_b)
        torch.cuda.synchronize()
        assert torch.equal(out_a.cpu(), out_b)
    ca, sa, _ = a.export()
    cb, sb, _ = b.export()
    assert torch.equal(ca, cb) and torch.equal(sa, sb)
    # dequant against the oracle definition code * scale
    view = GpuView(a)
    deq = a.dequant().cpu().numpy()
    for t in range(T):
        codes = view.tile_codes(t).astype(np.float32)
        sc = np.repeat(view.scales[t].reshape(wl.d_k, -1), wl.group, axis=1)
        assert np.array_equal(deq[t], codes * sc)
    a.close()
    b.close()


def test_step_host_stream_of_calls():
    """Host-buffer calls issued back to back with no synchronisation between
    them (the copies of consecutive calls overlap the steps): plain calls are
    complete once the stream is, pipelined ones once the stream has also
    completed step_host_sync; every output equals the device-buffer step's."""
    wl = C4.scaled(batch=2, heads=4, layers=2)
    T = wl.batch * wl.heads * 2
    steps = 7
    xs = [concat_inputs([synth.gen_step(wl, s_, layer=l, tiles=np.arange(8)) for l in range(2)])
          for s_ in range(steps)]
    ref = gpu_object(wl, synth.PERSISTENT, 2, 2)
    want = []
    for x in xs:
        out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
        ref.step(*gpu_inputs(wl, x), out)
        want.append(out.cpu())
    ref.close()
    host_in = [tuple(t.cpu().pin_memory() for t in gpu_inputs(wl, x)) for x in xs]
    stream = torch.cuda.current_stream()
    for pipelined in (False, True):
        obj = gpu_object(wl, synth.PERSISTENT, 2, 2)
        outs = [torch.full((T, wl.d_v), float("nan")).pin_memory() for _ in range(steps)]
        for i in range(steps):
            if pipelined:
                obj.step_host_pipelined(*host_in[i], outs[i])
            else:
                obj.step_host(*host_in[i], outs[i])
        if pipelined:
            obj.step_host_sync()
        stream.synchronize()
        for i in range(steps):
            assert torch.equal(outs[i], want[i]), (pipelined, i)
        obj.close()


def test_export_import_roundtrip_and_reset():
    wl = C5.scaled(batch=2)
    a = gpu_object(wl, synth.YOKED, 2, 1)
    for step in range(5):
        x = synth.gen_step(wl, step, tiles=np.arange(32))
        qd, kd, vd, gd = gpu_inputs(wl, x)
        out = torch.empty((32, 128), dtype=torch.float32, device="cuda")
        a.step(qd, kd, vd, gd, out)
    codes, scales, ref = a.export()
    b = gpu_object(wl, synth.YOKED, 2, 1)
    b.import_(codes, scales, ref)
    out_a = torch.empty((32, 128), dtype=torch.float32, device="cuda")
    out_b = torch.empty_like(out_a)
    a.step(qd, kd, vd, gd, out_a)
    b.step(qd, kd, vd, gd, out_b)
    assert torch.equal(out_a, out_b)
    for x_, y_ in zip(a.export(), b.export()):
        assert torch.equal(x_, y_)
    a.reset()
    c2, s2, r2 = a.export()
    assert int(c2.abs().sum()) == 0 and float(r2.abs().sum()) == 0
    a.close()
    b.close()


def test_invalid_pointer_alignment_rejected():
    obj = Q.QState(1, 2, 64, 64, Q.RETNET, bits=4, group=64)
    q, k, v, g, out = obj.alloc_inputs()
    buf = torch.zeros(200, dtype=torch.float32, device="cuda")
    with pytest.raises(Q.QStateError):
        obj.step(buf[1:], k, v, g, out)
    obj.close()


@pytest.mark.parametrize("name", ["gdn", "gla"])      # the general kernel; the row-batched one
def test_bounded_wait_runs_out_and_context_survives(name):
    """Fault injection on the host: the copies of tiles >= 100 are never
    issued, so their bounded waits run out.  The kernel reports pipeline
    timeouts instead of hanging, and the device stays usable."""
    base = {"gdn": C4, "gla": C3}[name]
    wl = base.scaled(batch=8, heads=32, layers=1, scale_modes=(synth.PERSISTENT,))  # 256 tiles
    obj = gpu_object(wl, synth.PERSISTENT, 8, 1)
    obj.debug_set(drop_from_tile=100, wait_polls=4096)
    x = synth.gen_step(wl, 0)
    qd, kd, vd, gd = gpu_inputs(wl, x)
    out = torch.empty((obj.tiles, wl.d_v), dtype=torch.float32, device="cuda")
    obj.step(qd, kd, vd, gd, out)
    torch.cuda.synchronize()
    st = obj.status()
    assert st["pipeline_timeouts"] > 0
    obj.debug_set(-1, 1 << 24)
    obj.reset()
    obj.step(qd, kd, vd, gd, out)
    torch.cuda.synchronize()
    assert obj.status()["pipeline_timeouts"] == 0
    obj.close()
    stats, status, _ = run_pair(wl.scaled(batch=1), steps=4)
    assert all(s["flips"] == 0 for s in stats)
