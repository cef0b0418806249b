"""Norm growth of the quantized state under the three scale modes.

    python norm_growth.py [--steps 32768] [--every 64]

"When Dynamic Scaling Fails" (Abstract) reports that a scale re-derived from
the state at every step forms a loop with the state that can make its norm
grow without bound, and that tying the scale to an unquantized copy of the
state prevents that.  This runs the long-horizon Gated DeltaNet workload (batch 32,
16 heads, d_k = d_v = 128, per-head widths {2, 4, 6, 8} with mean 4, group 64,
binary32 scales, BDR) with the three scale modes side by side on the same
seeded inputs and reports, every `--every` steps,

    rho_t = ||S_hat_t||_F / ||S_ref_t||_F

per mode, where S_ref is the unquantized recurrence (the yoked object's
reference state, stepped with the same fp32 arithmetic) and S_hat the
dequantized state.  It is an observation: the inputs are not tuned to force
either outcome.  Output: one JSON object with the per-1024-step medians and
maxima of rho for each mode.
"""
from __future__ import annotations

import argparse
import json
import sys
import time

import numpy as np
import torch

import os

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from bit_recurrent_state_decode_b200 import qstate as Q  # noqa: E402
from bit_recurrent_state_decode_b200 import synth  # noqa: E402


def run(steps: int, every: int, batch: int | None = None) -> dict:
    wl = synth.WORKLOADS["gdn_b32_h16_d128_mixed_3modes"]
    if batch:
        wl = wl.scaled(batch=batch)
    hb = wl.head_bits()
    objs = {m: Q.QState(wl.batch, wl.heads, wl.d_k, wl.d_v, wl.kind, bits=4, group=wl.group,
                        scale_mode=m, round_mode=wl.round_mode, eps_b=wl.eps_b, layers=1,
                        qkv_dtype=wl.qkv_dtype, gate_dtype=wl.gate_dtype,
                        scale_dtype=wl.scale_dtype, head_bits=hb)
            for m in (synth.DYNAMIC, synth.PERSISTENT, synth.YOKED)}
    T = wl.tiles_per_layer
    out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
    names = {synth.DYNAMIC: "dynamic", synth.PERSISTENT: "persistent", synth.YOKED: "yoked"}
    rho = {n: [] for n in names.values()}
    t0 = time.time()
    for step in range(steps):
        x = synth.gen_step(wl, step)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
            torch.bfloat16).cuda(non_blocking=True)
        q, k, v, g = dev(x.q), dev(x.k), dev(x.v), dev(x.gates)
        for o in objs.values():
            o.step(q, k, v, g, out)
        if (step + 1) % every == 0:
            _, _, ref = objs[synth.YOKED].export()
            rn = float(torch.linalg.vector_norm(ref.view(T, -1), dim=1).sum())
            ref_tiles = torch.linalg.vector_norm(ref.view(T, -1), dim=1)
            for m, o in objs.items():
                s = o.dequant()
                st = torch.linalg.vector_norm(s.view(T, -1), dim=1)
                # per-tile ratio, summarised by the median over tiles
                r = (st / ref_tiles.clamp_min(1e-30)).median().item()
                rho[names[m]].append((step + 1, r))
            del rn
    torch.cuda.synchronize()
    status = {names[m]: o.status() for m, o in objs.items()}
    for o in objs.values():
        o.close()
    summary = {}
    for n, series in rho.items():
        blocks = {}
        for s, r in series:
            blocks.setdefault((s - 1) // 1024, []).append(r)
        summary[n] = [{"steps": f"{b * 1024 + 1}-{(b + 1) * 1024}",
                       "rho_median": float(np.median(v)), "rho_max": float(np.max(v))}
                      for b, v in sorted(blocks.items())]
    return {"workload": wl.name, "steps": steps, "every": every, "batch": wl.batch,
            "seconds": time.time() - t0, "status": status, "rho": summary}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--steps", type=int, default=32768)
    ap.add_argument("--every", type=int, default=64)
    ap.add_argument("--batch", type=int, default=0)
    a = ap.parse_args(argv)
    from bit_recurrent_state_decode_b200 import build
    build.build()
    print(json.dumps(run(a.steps, a.every, a.batch or None)))


if __name__ == "__main__":
    sys.exit(main())
