"""GPU parity of the Hadamard-rotated state (INT4+Had of Table 2 of
"Preserving Updates in Low-Bit Recurrent State Quantization") against the CPU
oracle: the stored state is S H, the step rotates v and the output, and the
codes, scales and outputs match the oracle's rotated recurrence."""
import pytest
import torch

import oracle
from bit_recurrent_state_decode_b200 import synth

from parity_util import run_pair

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_recurrent_state_decode_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("kind", [synth.RETNET, synth.MAMBA2, synth.GLA, synth.GDN])
@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128)])
def test_rotated_fp32_recurrence_bit_exact(kind, dk, dv):
    base = {synth.RETNET: C1, synth.MAMBA2: C2, synth.GLA: C3, synth.GDN: C4}[kind]
    wl = base.scaled(batch=2, heads=3, d_k=dk, d_v=dv, bits=32, group=0, layers=1,
                     scale_modes=(synth.DYNAMIC,), round_mode=synth.RTN, head_bits_multiset=(),
                     q_sigma=base.q_sigma or 0.1, k_sigma=base.k_sigma or 0.1, rotation=1)
    stats, status, _ = run_pair(wl, steps=10)
    assert all(s["out_rel"] == 0.0 for s in stats)      # same butterflies: bit-exact


@pytest.mark.parametrize("name", ["gdn_had", "gdn_bdr", "gla", "mixed_yoked"])
def test_rotated_int4_matches_oracle(name):
    wl = {"gdn_had": synth.VARIANTS["gdn_l24_b256_h32_d128_int4g32_had"].scaled(batch=2, layers=1),
          "gdn_bdr": C4.scaled(batch=2, layers=1, rotation=1),
          "gla": C3.scaled(batch=2, rotation=1),
          "mixed_yoked": C5.scaled(batch=1, rotation=1)}[name]
    stats, status, ocounts = run_pair(wl, steps=24, check_every=8, final_dequant=True)
    assert all(s.get("flips", 0) == 0 for s in stats), stats
    for m in status:
        assert status[m]["nonfinite"] == 0
