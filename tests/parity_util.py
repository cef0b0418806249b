"""Helpers of the GPU parity tests: run the CUDA path (through the C ABI) and
the CPU oracle on the same seeded synthetic inputs and compare them.

Bars (the decode-step contract):
  - packed codes bit-exact, allowing at most 1e-5 of the codes to differ by
    one level (a round-half tie flipped by a different fp32 FMA order);
  - scales bit-exact;
  - outputs and dequantized state within a max relative error of 1e-3 per
    tile, measured as max|y - y_oracle| / max|y_oracle|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_recurrent_state_decode_b200 import qstate as Q
from bit_recurrent_state_decode_b200 import synth

CODE_FLIP_FRACTION = 1e-5
REL_TOL = 1e-3


def to_device(x: np.ndarray | None, bf16: bool):
    if x is None:
        return None
    if bf16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def gpu_object(wl: synth.Workload, mode: int, batch: int, layers: int) -> Q.QState:
    hb = wl.head_bits()
    return Q.QState(batch, wl.heads, wl.d_k, wl.d_v, wl.kind, bits=wl.bits or 4, group=wl.group,
                    scale_mode=mode, round_mode=wl.round_mode, eps_b=wl.eps_b, layers=layers,
                    gamma=wl.gamma, qkv_dtype=wl.qkv_dtype, gate_dtype=wl.gate_dtype,
                    scale_dtype=wl.scale_dtype, head_bits=hb, rotation=wl.rotation)


def bench_layers(wl: synth.Workload) -> int:
    """The layers the benchmark steps in one launch: the workload's own, or,
    for a one-layer state that fits in L2, as many independent replicas of
    the layer as take state and inputs past 4x L2 (bench.pick_replicas on
    the per-layer byte count bench.py forms, layout variant included)."""
    import bench
    probe = gpu_object(wl, wl.scale_modes[0], wl.batch, 1)
    if wl.lrb:
        probe.set_lrb(*wl.lrb)
    if wl.pw:
        probe.set_pw(wl.pw)
    if wl.rowcol:
        probe.set_rowcol()
    z = probe.sizes
    resident = z["code_bytes"] + z["scale_bytes"] + z["ref_bytes"]
    per_layer = resident + probe.bytes_per_step() - 2 * resident
    probe.close()
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    return wl.layers * bench.pick_replicas(wl, l2, per_layer)


def oracle_state(wl: synth.Workload, mode: int, tile_heads: np.ndarray, bits=None):
    cfg = oracle.Config(wl.d_k, wl.d_v, wl.kind, wl.group, scale_mode=mode,
                        round_mode=wl.round_mode, scale_f32=wl.scale_dtype == synth.F32,
                        gamma=wl.gamma, eps_b=wl.eps_b, rotate=wl.rotation)
    hb = wl.head_bits()
    if bits is None:
        bits = wl.bits
    tile_bits = hb[tile_heads] if hb is not None else np.full(len(tile_heads), bits)
    return oracle.State(cfg, tile_bits)


def oracle_inputs(wl, x: synth.StepInputs):
    q, k, v, g = x.as_f32(wl)
    alpha = beta = None
    if wl.kind == synth.MAMBA2:
        alpha = g
    elif wl.kind == synth.GLA:
        alpha = g
    elif wl.kind == synth.GDN:
        alpha, beta = g[:, :1], g[:, 1]
    return q, k, v, alpha, beta


def concat_inputs(parts):
    def cat(name):
        arrs = [getattr(p, name) for p in parts]
        return None if arrs[0] is None else np.concatenate(arrs, axis=0)
    return synth.StepInputs(cat("q"), cat("k"), cat("v"), cat("gates"))


def gpu_inputs(wl, x: synth.StepInputs):
    bf = wl.qkv_dtype == synth.BF16
    gbf = wl.gate_dtype == synth.BF16
    return (to_device(x.q, bf), to_device(x.k, bf), to_device(x.v, bf),
            to_device(x.gates, gbf))


class GpuView:
    """Exported GPU state of one object, indexable per tile."""

    def __init__(self, obj: Q.QState):
        self.obj = obj
        codes, scales, ref = obj.export()
        torch.cuda.synchronize()
        self.codes = codes.cpu().numpy()
        self.scales = scales.float().cpu().numpy().reshape(obj.tiles, -1) if scales.numel() else None
        self.ref = None if ref is None else ref.cpu().numpy().reshape(obj.tiles, obj.d_k, obj.d_v)
        hb = obj.head_bits
        self.tile_bits = ([hb[t % obj.heads] for t in range(obj.tiles)] if hb
                          else [obj.bits] * obj.tiles)
        tb = [oracle.tile_bytes(b, obj.d_k, obj.d_v) for b in (hb or [obj.bits] * obj.heads)]
        self.head_off = np.concatenate([[0], np.cumsum(tb)[:-1]]).astype(np.int64)
        self.row_bytes = int(np.sum(tb))

    def tile_codes(self, t: int) -> np.ndarray:
        o = self.obj
        b = self.tile_bits[t]
        nb = oracle.tile_bytes(b, o.d_k, o.d_v)
        start = (t // o.heads) * self.row_bytes + int(self.head_off[t % o.heads])
        raw = self.codes[start:start + nb]
        if b == 32:
            return raw.view(np.float32).reshape(o.d_k, o.d_v)
        return oracle.unpack(b, o.d_k, o.d_v, raw)


def rel_err(y, ref):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.abs(ref).max()
    num = np.abs(y - ref).max()
    if den == 0:
        return float(num)
    return float(num / den)


def compare(view: GpuView, out_gpu: np.ndarray, st: oracle.State, out_orc: np.ndarray,
            gpu_tiles, orc_tiles, check_dequant=None):
    """Compare sampled tiles; returns a stats dict and raises AssertionError on
    a breach of the bars."""
    n_codes = n_flip = n_big = 0
    worst_out = 0.0
    scale_mismatch = 0
    for gt, ot in zip(gpu_tiles, orc_tiles):
        b = int(st.tile_bits[ot])
        got = view.tile_codes(gt)
        if b == 32:
            assert np.array_equal(got.view(np.uint32), st.S[ot].view(np.uint32)), \
                f"fp32 state differs at tile {gt}"
        else:
            d = np.abs(got.astype(np.int32) - st.codes[ot].astype(np.int32))
            n_codes += d.size
            n_flip += int(np.count_nonzero(d))
            n_big += int(np.count_nonzero(d > 1))
            if view.scales is not None:
                scale_mismatch += int(np.count_nonzero(view.scales[gt] != st.scales[ot]))
            if view.ref is not None and st.ref is not None:
                assert np.array_equal(view.ref[gt].view(np.uint32), st.ref[ot].view(np.uint32)), \
                    f"yoked reference differs at tile {gt}"
        worst_out = max(worst_out, rel_err(out_gpu[gt], out_orc[ot]))
    stats = dict(codes=n_codes, flips=n_flip, big=n_big, scale_mismatch=scale_mismatch,
                 out_rel=worst_out)
    assert n_big == 0, stats
    assert n_flip <= CODE_FLIP_FRACTION * max(n_codes, 1) + 0, stats
    assert scale_mismatch == 0, stats
    assert worst_out <= REL_TOL, stats
    return stats


def _gen_chunk(wl, steps, layer_ids, orig_tiles):
    """Inputs of several consecutive steps at once (a leading step axis), the
    layers' tiles concatenated in object order."""
    parts = [synth.gen_step(wl, np.asarray(steps), layer=l, tiles=orig_tiles) for l in layer_ids]

    def cat(name):
        arrs = [getattr(p, name) for p in parts]
        return None if arrs[0] is None else np.concatenate(arrs, axis=1)
    return synth.StepInputs(cat("q"), cat("k"), cat("v"), cat("gates"))


def _chunk_to_device(a, bf16):
    """[steps, T, n] host array -> list of per-step CUDA views, each starting
    on a 16-byte boundary (the step's operand alignment)."""
    if a is None:
        return None
    S, T, n = a.shape
    esize = 2 if bf16 else 4
    Tp = T
    while (Tp * n * esize) % 16:
        Tp += 1
    dt = torch.bfloat16 if bf16 else torch.float32
    host = np.zeros((S, Tp, n), np.uint16 if bf16 else np.float32)
    host[:, :T] = a
    t = torch.from_numpy(host.view(np.int16) if bf16 else host)
    d = (t.view(torch.bfloat16) if bf16 else t).to("cuda")
    assert d.dtype == dt
    return [d[i, :T] for i in range(S)]


def run_pair(wl: synth.Workload, modes=None, batch_sel=None, layers=1, steps=8, start_step=0,
             check_every=1, teacher_forced=False, layer_ids=None, threads=1, chunk=64,
             final_dequant=False):
    """Step the GPU and the oracle side by side on batch rows ``batch_sel`` of
    ``layers`` layers (seeded as layers ``layer_ids``, default 0 .. layers-1);
    compare every ``check_every`` steps and after the last.  Inputs are drawn
    ``chunk`` steps at a time; ``threads`` host threads step the oracle.
    Returns (stats, status, oracle counters)."""
    modes = modes or wl.scale_modes
    batch_sel = np.arange(wl.batch) if batch_sel is None else np.asarray(batch_sel)
    layer_ids = list(range(layers)) if layer_ids is None else list(layer_ids)
    layers = len(layer_ids)
    H = wl.heads
    B = len(batch_sel)
    orig_tiles = (batch_sel[:, None] * H + np.arange(H)[None, :]).reshape(-1)
    tile_heads = np.tile(np.arange(H), B * layers)
    gpu = {m: gpu_object(wl, m, B, layers) for m in modes}
    orc = {m: oracle_state(wl, m, tile_heads) for m in modes}
    T = B * H * layers
    all_stats = []
    out = {m: torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda") for m in modes}
    end = start_step + steps
    for c0 in range(start_step, end, chunk):
        c1 = min(end, c0 + chunk)
        xs = _gen_chunk(wl, range(c0, c1), layer_ids, orig_tiles)
        dq, dk, dv, dg = (_chunk_to_device(a, bf) for a, bf in
                          zip((xs.q, xs.k, xs.v, xs.gates),
                              (wl.qkv_dtype == synth.BF16,) * 3 + (wl.gate_dtype == synth.BF16,)))
        for i, step in enumerate(range(c0, c1)):
            x = synth.StepInputs(xs.q[i], xs.k[i], xs.v[i], None if xs.gates is None else xs.gates[i])
            oq, ok_, ov, oa, ob = oracle_inputs(wl, x)
            for m in modes:
                if teacher_forced:
                    import_oracle_state(gpu[m], orc[m])
                gpu[m].step(dq[i], dk[i], dv[i], None if dg is None else dg[i], out[m])
            o_all = oracle.step_many([(orc[m], (oq, ok_, ov, oa, ob)) for m in modes], threads)
            for m, o_orc in zip(modes, o_all):
                if (step - start_step + 1) % check_every == 0 or step == end - 1:
                    view = GpuView(gpu[m])
                    s = compare(view, out[m].cpu().numpy(), orc[m], o_orc, range(T), range(T))
                    s.update(step=step, mode=m)
                    all_stats.append(s)
    status = {m: gpu[m].status() for m in modes}
    if final_dequant:
        # the dequantized state after the last step, tile by tile (c15 metric)
        for m in modes:
            deq = gpu[m].dequant().cpu().numpy()
            ref = orc[m].dequant()
            worst = max(rel_err(deq[t], ref[t]) for t in range(T))
            assert worst <= REL_TOL, (m, worst)
            all_stats.append(dict(mode=m, dequant_rel=worst))
    for m in modes:
        gpu[m].close()
        assert status[m]["pipeline_timeouts"] == 0, status
    return all_stats, status, {m: orc[m].counts.as_dict() for m in modes}


def import_oracle_state(obj: Q.QState, st: oracle.State):
    """Pack the oracle state into the GPU layout and import it."""
    view_bits = [obj.head_bits[t % obj.heads] for t in range(obj.tiles)] if obj.head_bits \
        else [obj.bits] * obj.tiles
    chunks = []
    for t in range(obj.tiles):
        if view_bits[t] == 32:
            chunks.append(st.S[t].view(np.uint8).reshape(-1))
        else:
            chunks.append(oracle.pack(view_bits[t], st.codes[t]))
    codes = torch.from_numpy(np.concatenate(chunks)).cuda()
    sdt = np.float32 if obj.scale_dtype == Q.F32 else np.float16
    scales = torch.from_numpy(st.scales.astype(sdt).reshape(-1)).cuda()
    ref = None if st.ref is None else torch.from_numpy(st.ref.reshape(-1)).cuda()
    obj.import_(codes, scales, ref)
