#!/usr/bin/env python
"""Throughput of the fused quantized recurrent-state decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

A step is one decode step of every tile of the workload (one kernel launch per
state object).  Metric: quantized state-updates/s = tiles x steps / time, where
tiles = layers x batch x heads; also tokens/s = batch x steps / time and the
achieved HBM bandwidth of the step kernel against the measured copy peak.

Inputs are seeded synthetic decode streams (bit_recurrent_state_decode_b200.synth),
resident in HBM before the timed region (a ring of 16 steps).  Workloads whose
state fits in L2 are stepped as several independent layer replicas so that the
state, not L2, is what each step reads (the replica count is in `config`).

Multi-GPU: one process per GPU (torchrun); the tiles are independent, so every
rank steps its own shard (the full workload, different layer seeds) with no
collective on the data path ("scaling": "weak"); the time is the max over
ranks.  ``--impl reference`` times the plain CPU oracle on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "gdn_l24_b256_h32_d128_int4g64_bdr"
# workloads at batch >= 64 (the bandwidth goal applies to these) and the
# long-horizon mixed-width one (reported only)
ALL_WORKLOADS = ("gdn_l24_b256_h32_d128_int4g64_bdr", "mamba2_b64_h32_dk128_dv64_int8tok",
                 "gla_b128_h16_d128_int4g32_persistent", "gdn_b32_h16_d128_mixed_3modes")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="a workload name, 'all' for one line per workload in ALL_WORKLOADS, "
                         "or 'variants' for one line per layout variant (synth.VARIANTS)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--replicas", type=int, default=0,
                    help="independent layer replicas (0: enough to exceed 4x L2)")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the number of layers stepped (small profiling cases)")
    ap.add_argument("--launch-samples", type=int, default=200,
                    help="launches timed one by one for the roofline figure")
    ap.add_argument("--ring", type=int, default=16,
                    help="decode steps of resident inputs the timed steps cycle through")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ helpers
def pick_replicas(wl, l2_bytes, per_layer_bytes):
    if wl.layers > 1:
        return 1
    return max(1, math.ceil(4 * l2_bytes / per_layer_bytes))


def rank_layer_ids(rank, layers):
    """Layer seeds of one rank's shard: disjoint across ranks, so every rank
    steps its own independent tiles (no data-path exchange)."""
    return [rank * layers + l for l in range(layers)]


def max_over_ranks(value, device=None):
    """Max of a per-rank float over the process group (identity when not
    distributed).  Used only outside the timed region."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def default_steps(step_seconds_estimate):
    # about 3 s of timed work, never fewer than 50 steps
    return max(50, int(3.0 / max(step_seconds_estimate, 1e-7)))


def cpu_oracle_rate(wl, seconds=10.0, threads=None, max_steps=None, tiles=None, warmup=0):
    """State-updates/s of the CPU oracle on a bounded sample of the workload;
    the first `warmup` steps run untimed."""
    import numpy as np

    import oracle
    from bit_recurrent_state_decode_b200 import synth
    threads = threads or os.cpu_count() or 1
    cycle = 1
    if wl.pw or wl.rowcol:
        tiles = tiles or 32
    if wl.lrb:
        # whole merge cycles (m steps, one of them a merge), after one cycle
        # that fills the residual; the bypass step is single-threaded
        cycle = wl.lrb[1]
        warmup = max(warmup, cycle)
        tiles = tiles or 32
    # enough tiles per step that the worker threads, not their dispatch, set the rate
    tiles = tiles or max(threads * 64, 8)
    tiles = min(tiles, wl.tiles_per_layer)
    hb = wl.head_bits()
    sel = np.arange(tiles)
    tile_bits = hb[sel % wl.heads] if hb is not None else np.full(tiles, wl.bits)
    states = []
    for mode in wl.scale_modes:
        cfg = oracle.Config(wl.d_k, wl.d_v, wl.kind, wl.group, scale_mode=mode,
                            round_mode=wl.round_mode, scale_f32=wl.scale_dtype == synth.F32,
                            gamma=wl.gamma, eps_b=wl.eps_b, rotate=wl.rotation)
        if wl.lrb:
            # the oracle's bypass step runs its tiles on one host thread
            states.append(oracle.LrbState(cfg, tile_bits, *wl.lrb))
            threads = 1
        elif wl.pw:
            # so does its windowed step
            states.append(oracle.PwState(cfg, tile_bits, wl.pw))
            threads = 1
        elif wl.rowcol:
            # and its row x column step
            states.append(oracle.RcState(cfg, tile_bits))
            threads = 1
        else:
            states.append(oracle.State(cfg, tile_bits))
    steps = 0
    busy = 0.0
    for w in range(warmup):
        x = synth.gen_step(wl, w, tiles=sel)
        q, k, v, g = x.as_f32(wl)
        alpha = beta = None
        if wl.kind in (synth.MAMBA2, synth.GLA):
            alpha = g
        elif wl.kind == synth.GDN:
            alpha, beta = g[:, :1], g[:, 1]
        for st in states:
            st.step(q, k, v, alpha, beta, threads=threads)
    t_end = time.perf_counter() + seconds
    while ((time.perf_counter() < t_end or steps % cycle) and
           (max_steps is None or steps < max_steps)):
        x = synth.gen_step(wl, warmup + steps, tiles=sel)
        q, k, v, g = x.as_f32(wl)
        alpha = beta = None
        if wl.kind in (synth.MAMBA2, synth.GLA):
            alpha = g
        elif wl.kind == synth.GDN:
            alpha, beta = g[:, :1], g[:, 1]
        t0 = time.perf_counter()
        for st in states:
            st.step(q, k, v, alpha, beta, threads=threads)
        busy += time.perf_counter() - t0
        steps += 1
    return {"value": tiles * steps / busy, "steps": steps, "tiles": tiles, "threads": threads,
            "seconds": busy}


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    from bit_recurrent_state_decode_b200 import build as qbuild
    from bit_recurrent_state_decode_b200 import qstate as Q
    from bit_recurrent_state_decode_b200 import synth

    qbuild.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    props = torch.cuda.get_device_properties(dev)
    wl0 = synth.workload(args.workload)
    hb = wl0.head_bits()

    def make(mode, layers):
        o = Q.QState(wl0.batch, wl0.heads, wl0.d_k, wl0.d_v, wl0.kind, bits=wl0.bits or 4,
                     group=wl0.group, scale_mode=mode, round_mode=wl0.round_mode,
                     eps_b=wl0.eps_b, layers=layers, gamma=wl0.gamma,
                     qkv_dtype=wl0.qkv_dtype, gate_dtype=wl0.gate_dtype,
                     scale_dtype=wl0.scale_dtype, head_bits=hb, rotation=wl0.rotation)
        if wl0.lrb:
            o.set_lrb(*wl0.lrb)
        if wl0.pw:
            o.set_pw(wl0.pw)
        if wl0.rowcol:
            o.set_rowcol()
        return o

    probe = make(wl0.scale_modes[0], 1)
    per_layer = sum(probe.sizes[k] for k in ("code_bytes", "scale_bytes", "ref_bytes")) \
        + probe.bytes_per_step() - 2 * (probe.sizes["code_bytes"] + probe.sizes["scale_bytes"]
                                        + probe.sizes["ref_bytes"])
    probe.close()
    replicas = args.replicas or pick_replicas(wl0, props.L2_cache_size, per_layer)
    layers = wl0.layers * replicas
    if args.layers:
        layers, replicas = args.layers, max(1, args.layers // wl0.layers)
    objs = [make(m, layers) for m in wl0.scale_modes]
    T = objs[0].tiles
    bytes_per_step = sum(o.bytes_per_step() for o in objs)

    # ring of resident inputs (distinct layer seeds per rank)
    ring_n = max(2, args.ring)
    bf = wl0.qkv_dtype == synth.BF16
    gbf = wl0.gate_dtype == synth.BF16

    def to_dev(a, is_bf):
        if a is None:
            return None
        if is_bf:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    ring = []
    host_ring = []
    for s in range(ring_n):
        parts = [synth.gen_step(wl0, s, layer=lid) for lid in rank_layer_ids(rank, layers)]
        cat = lambda name: (None if getattr(parts[0], name) is None
                            else np.concatenate([getattr(p, name) for p in parts]))
        x = synth.StepInputs(cat("q"), cat("k"), cat("v"), cat("gates"))
        ring.append((to_dev(x.q, bf), to_dev(x.k, bf), to_dev(x.v, bf), to_dev(x.gates, gbf)))
        if s < 2:
            host_ring.append(x)
    out = torch.empty((T, wl0.d_v), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        qd, kd, vd, gd = ring[i % ring_n]
        for o in objs:
            o.step(qd, kd, vd, gd, out, stream)

    # estimate the step time, then size K
    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(10):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    est = e0.elapsed_time(e1) / 10 / 1e3
    dist = world > 1
    if dist:
        import torch.distributed as tdist
        # every rank sizes its loops from the same estimate (same K, same e2e steps)
        est = max_over_ranks(est, dev)
    K = args.steps or default_steps(est)
    W = args.warmup

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    if dist:
        tdist.barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(K):
        step(W + i)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dev)
    if dist:
        tdist.barrier()
    ms_step = ms_total / K

    # per-launch durations of the dominant kernel, events on its stream
    dom = max(objs, key=lambda o: o.bytes_per_step())
    dom_bytes = dom.bytes_per_step()
    nlaunch = max(1, min(K, args.launch_samples))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(nlaunch)]
    for i in range(nlaunch):
        qd, kd, vd, gd = ring[i % ring_n]
        evs[i][0].record(stream)
        dom.step(qd, kd, vd, gd, out, stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)

    # end to end through the host-buffer entry point (copies in the timed region)
    e2e = None
    if not args.no_e2e:
        pin = []
        for x in host_ring:
            def pinned(a):
                if a is None:
                    return None
                t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16
                                     else np.ascontiguousarray(a))
                return t.pin_memory()
            pin.append((pinned(x.q), pinned(x.k), pinned(x.v), pinned(x.gates)))
        # one pinned output per object and step parity (the output copies of
        # consecutive calls are in flight together)
        houts = [[torch.empty((T, wl0.d_v), dtype=torch.float32).pin_memory() for _ in range(2)]
                 for _ in objs]
        h2d = sum(t.numel() * t.element_size() for t in pin[0] if t is not None)
        d2h = houts[0][0].numel() * 4 * len(objs)
        Ke = max(3, min(K, int(2.0 / max(est + (h2d + d2h) / 20e9, 1e-6))))
        # the host-buffer calls of a stream of steps: each call's output copy
        # overlaps the next call's step; the last one is waited for inside
        # the timed region
        for i in range(2):
            for o, ho in zip(objs, houts):
                o.step_host_pipelined(*pin[i % len(pin)], ho[i & 1], stream)
        for o in objs:
            o.step_host_sync(stream)
        torch.cuda.synchronize()
        if dist:
            tdist.barrier()
        e0.record(stream)
        for i in range(Ke):
            for o, ho in zip(objs, houts):
                o.step_host_pipelined(*pin[i % len(pin)], ho[i & 1], stream)
        for o in objs:
            o.step_host_sync(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e = {"value": world * T * Ke / (ems / 1e3), "unit": "state-updates/s",
               "h2d_bytes_per_step": int(h2d * len(objs)), "d2h_bytes_per_step": int(d2h),
               "steps": Ke}

    status = [o.status() for o in objs]
    kernel_name = dom.kernel
    for o in objs:
        o.close()

    peak, peak_kind = measured_peaks()
    achieved = dom_bytes / (launch_ms / 1e3) / 1e9
    footprint = per_layer * layers            # state + step operands of one step
    cold = footprint > 4 * props.L2_cache_size
    # DRAM traffic per launch from the committed ncu summary, scaled to this
    # launch by tiles (traffic grows in proportion once the launch is L2-cold)
    traffic = read_traffic(wl0.name, T, kernel_name) if cold else None
    result = {
        "metric": "quantized state-updates/s",
        "value": world * T * K / (ms_total / 1e3),
        "unit": "state-updates/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int%d/f32" % (wl0.bits or 4) if wl0.bits != 32 else "f32",
        "data": "synthetic (seeded Philox4x32-10 decode streams)",
        "config": {
            "workload": wl0.name, "description": wl0.description, "batch": wl0.batch,
            "heads": wl0.heads, "d_k": wl0.d_k, "d_v": wl0.d_v, "layers": layers,
            "layer_replicas": replicas, "tiles_per_gpu": T,
            "objects": len(objs), "scale_modes": list(wl0.scale_modes),
            "l2": (f"cold: state + inputs of {layers} layers ({footprint / 1e6:.0f} MB) "
                   f"> 4x L2 ({props.L2_cache_size / 1e6:.0f} MB) per step" if cold else
                   f"warm: state + inputs of {layers} layers ({footprint / 1e6:.0f} MB) "
                   f"<= 4x L2 ({props.L2_cache_size / 1e6:.0f} MB); L2-resident between steps"),
            "parallelism": f"dp{world} (tile shards, no collective)",
        },
        "tokens_per_s": world * wl0.batch * K / (ms_total / 1e3),
        "achieved_GBps": bytes_per_step / (ms_step / 1e3) / 1e9,
        "bytes_per_step": bytes_per_step,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind,
                     "frac_of_nominal_8TBps": achieved / NOMINAL_HBM_GBS,
                     "traffic": traffic, "kernel": "qs::" + kernel_name,
                     "bytes_per_launch": dom_bytes, "launch_ms": launch_ms},
        "gpu_launches": K * len(objs),
        "clocks": clk,
        "e2e": e2e,
        "status": status,
    }
    return result


def source_digest(src):
    """First 16 hex digits of a sha256 over the kernel sources in `src` as
    code: in file-name order, each file's name and its text with comments
    removed and whitespace runs collapsed (string and character literals
    kept).  The committed ncu counters are tied to the code they were taken
    on, so an edit of a comment leaves them valid and any other edit does not."""
    import hashlib
    import re
    token = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'', re.S)
    h = hashlib.sha256()
    for f in sorted(os.listdir(src)):
        if f.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(src, f), encoding="utf-8", errors="surrogateescape") as fh:
                text = fh.read()
            code = token.sub(lambda m: " " if m.group(0)[0] == "/" else m.group(0), text)
            h.update(f.encode() + b"\0" + " ".join(code.split()).encode("utf-8", "surrogateescape")
                     + b"\0")
    return h.hexdigest()[:16]


def read_traffic(workload, tiles=None, kernel="step_kernel"):
    """DRAM bytes per launch from the committed ncu summary of this kernel on
    this workload (profiles/<kernel>_<workload>.md), if its recorded
    kernel-source digest (source_digest) matches the current sources; scaled
    from the summary's full-size launch to `tiles` tiles when given."""
    digest = source_digest(os.path.join(ROOT, "bit_recurrent_state_decode_b200", "csrc"))
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha256_16") != digest:
        return None
    try:
        full = float(vals["dram_bytes_per_launch_full_size"])
        full_tiles = float(vals["tiles_per_launch_full_size"])
    except (KeyError, ValueError):
        return None
    return full if tiles is None else full * tiles / full_tiles


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    from bit_recurrent_state_decode_b200 import synth
    wl = synth.workload(DEFAULT_WORKLOAD if args.workload in ("all", "variants") else args.workload)
    K = args.steps or 50
    W = args.warmup
    threads = os.cpu_count() or 1
    # size the per-step sample so that the whole run stays within ~2 minutes
    probe = cpu_oracle_rate(wl, seconds=1.0, threads=threads, max_steps=2)
    per_tile = 1.0 / probe["value"]
    tiles = max(1, min(wl.tiles_per_layer, int(100.0 / max(K + W, 1) / per_tile)))
    r = cpu_oracle_rate(wl, seconds=1e9, threads=threads, max_steps=K, tiles=tiles, warmup=W)
    return {
        "impl": "reference", "metric": "quantized state-updates/s", "value": r["value"],
        "unit": "state-updates/s", "n_gpus": 0, "steps": K, "warmup": W,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int%d/f32" % (wl.bits or 4), "data": "synthetic (seeded Philox4x32-10 decode streams)",
        "config": {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "d_k": wl.d_k,
                   "d_v": wl.d_v},
        "cpu_baseline": {"value": r["value"], "unit": "state-updates/s", "cores": r["threads"],
                         "kind": "oracle",
                         "sample": f"{r['tiles']} tiles x {r['steps']} steps of {wl.name}"},
        "e2e": {"value": r["value"], "unit": "state-updates/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
    if args.workload == "all":
        names = ALL_WORKLOADS
    elif args.workload == "variants":
        from bit_recurrent_state_decode_b200 import synth
        names = tuple(synth.VARIANTS)
    else:
        names = (args.workload,)
    for name in names:
        args.workload = name
        res = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu:     # the CPU baseline at N = 1 only
            from bit_recurrent_state_decode_b200 import synth
            r = cpu_oracle_rate(synth.workload(name), seconds=10.0)
            res["cpu_baseline"] = {"value": r["value"], "unit": "state-updates/s",
                                   "cores": r["threads"], "kind": "oracle",
                                   "sample": f"{r['tiles']} tiles x {r['steps']} steps of "
                                             f"{name} ({r['seconds']:.1f} s)"}
        if rank == 0:
            print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()
        tdist.destroy_process_group()


if __name__ == "__main__":
    main()
