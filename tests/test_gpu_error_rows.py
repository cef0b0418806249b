"""The per-step rounding error kept by the GPU step with the taxonomy on
(qstate_error_rows) against the oracle's error accounting ("Preserving
Updates in Low-Bit Recurrent State Quantization", Figures 1 and 2, Table 5;
oracle/diagnostics.py).

Per tile and key row the kernel writes sum_j (S_hat_t - x_t)_ij^2 in binary32
(each R one rounded subtraction of binary32 values, squares summed by fma,
the row's lanes by a butterfly); the oracle forms R_t exactly in fp64.  So
every row agrees to 1e-5 relative (plus 1e-30 absolute for rows without
error), and the diagonal terms D_T = sum_t ||a_{t:T} R_t||^2 accumulated
from the GPU rows, and the coherent gain g_T = ||E_T||^2 / D_T, agree with
the oracle's to the same bound.  The state stays bit-exact (the rows are a
by-product of the taxonomy pass)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import diagnostics
from bit_recurrent_state_decode_b200 import synth

from parity_util import GpuView, gpu_inputs, gpu_object, oracle_inputs, oracle_state

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
C1, C2, C3, C4, C5 = (W[n] for n in W)

CASES = {
    "gdn_int4g64_bdr_persistent": (C4.scaled(batch=2, heads=4, layers=1, eps_b=0.3), synth.PERSISTENT),
    "gla_int4g32_persistent": (C3.scaled(batch=2, heads=4), synth.PERSISTENT),
    "mamba2_int8_per_token": (C2.scaled(batch=2, heads=4), synth.DYNAMIC),
    "gdn_mixed_bits_yoked": (C5.scaled(batch=1), synth.YOKED),
    "retnet_int4g64": (C1.scaled(batch=3, heads=4), synth.DYNAMIC),
}


@pytest.mark.parametrize("name", list(CASES))
def test_error_rows_match_the_oracle(name):
    wl, mode = CASES[name]
    gpu = gpu_object(wl, mode, wl.batch, wl.layers)
    gpu.set_taxonomy(True)
    T = gpu.tiles
    st = oracle_state(wl, mode, np.tile(np.arange(wl.heads), wl.batch))
    ea = diagnostics.ErrorAccount(st, gamma=wl.gamma)
    drow = np.zeros((T, wl.d_k))
    out = torch.empty((T, wl.d_v), dtype=torch.float32, device="cuda")
    tiles = np.arange(wl.batch * wl.heads)
    for step in range(12):
        x = synth.gen_step(wl, step, layer=0, tiles=tiles)
        gpu.step(*gpu_inputs(wl, x), out)
        q, k, v, alpha, beta = oracle_inputs(wl, x)
        prev = {m: ea.Drow[m].copy() for m in ea.Drow}
        ea.step(q, k, v, alpha, beta)
        rows = gpu.error_rows().double().cpu().numpy()
        w = ea._decay(alpha)
        # this step's rows from the oracle: D_t - w^2 D_{t-1}
        ref = ea.Drow["all"] - w * w * prev["all"]
        tol = 1e-5 * np.abs(ref) + 1e-30 + 1e-6 * np.abs(ref).max()
        assert np.all(np.abs(rows - ref) <= tol), (step, np.abs(rows - ref).max(), np.abs(ref).max())
        drow = w * w * drow + rows
    assert np.all(np.abs(drow - ea.Drow["all"]) <= 1e-5 * np.abs(ea.Drow["all"]) + 1e-30)
    g_gpu = diagnostics.coherent_gain(ea.E["all"], drow)
    assert abs(g_gpu - ea.gain()) <= 1e-5 * ea.gain(), (g_gpu, ea.gain())
    # the state itself is untouched by the extra pass
    view = GpuView(gpu)
    for t in range(T):
        assert np.array_equal(view.tile_codes(t), st.codes[t]), t
    gpu.close()


def test_error_rows_need_the_taxonomy():
    from bit_recurrent_state_decode_b200 import qstate as Q
    wl = C1.scaled(batch=1)
    gpu = gpu_object(wl, synth.DYNAMIC, 1, 1)
    with pytest.raises(Q.QStateError):
        gpu.error_rows()
    gpu.close()
