"""GPU parity over the full decode horizon of each workload.

The error of a quantized recurrence compounds over time ("When Dynamic Scaling
Fails", Abstract; "Preserving Updates in Low-Bit Recurrent State
Quantization", Abstract), so the decode step is compared with the CPU oracle
after every step count the workloads name, not a prefix of it: packed codes
and scales bit-exact at every checkpoint, outputs within 1e-3 max relative
error per tile, and the dequantized state within 1e-3 after the last step.
A few tiles of each workload are stepped (their inputs are the workload's own
seeded streams); the sampled full-size launches are covered in
test_gpu_parity.py.
"""
import os

import pytest
import torch

import oracle
from bit_recurrent_state_decode_b200 import synth

from parity_util import run_pair

pytestmark = [pytest.mark.gpu, pytest.mark.long]
W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)
THREADS = min(16, os.cpu_count() or 4)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_recurrent_state_decode_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _no_flips(stats):
    flips = [s for s in stats if s.get("flips")]
    assert not flips, flips


def test_gla_full_horizon():
    """GLA, B128 H16 d128, INT4 g32 persistent: all 4096 steps, batch rows 0
    and 127 (32 tiles)."""
    stats, status, ocounts = run_pair(C3, batch_sel=[0, 127], steps=C3.steps, check_every=512,
                                      threads=THREADS, final_dequant=True)
    _no_flips(stats)
    for m in status:
        assert status[m]["nonfinite"] == 0
        assert status[m]["saturated"] == ocounts[m]["saturated"]


def test_gdn_24_layers_full_horizon():
    """Gated DeltaNet x24, B256 H32 d128, INT4 g64 persistent BDR: all 2048
    steps of the first and the last layer's streams (layers 0 and 23), batch
    rows 0 and 255 of each (128 tiles)."""
    stats, status, ocounts = run_pair(C4, batch_sel=[0, 255], layer_ids=[0, 23], steps=C4.steps,
                                      check_every=512, threads=THREADS, final_dequant=True)
    _no_flips(stats)
    for m in status:
        assert status[m]["nonfinite"] == 0
        assert status[m]["saturated"] == ocounts[m]["saturated"]


def test_mixed_bits_three_modes_full_horizon():
    """Gated DeltaNet, B32 H16 d128, per-head widths {2,4,6,8}, fp32 scales,
    dynamic + persistent + yoked side by side: all 32768 steps of batch row 0
    (16 tiles per mode)."""
    stats, status, ocounts = run_pair(C5, batch_sel=[0], steps=C5.steps, check_every=1024,
                                      threads=THREADS, chunk=256, final_dequant=True)
    _no_flips(stats)
    for m in status:
        assert status[m]["nonfinite"] == 0
