"""qstate_step_host_static, the host-buffer step that allocates nothing.

Some callers of this library cannot call cudaMalloc during decoding (a
serving process whose device memory belongs to its own pool allocator, or a
loop that must not stall on the device synchronisation cudaMalloc may cause).
For them the step's operands are staged in a fixed device array inside the
library instead of buffers allocated on first use.  This file checks, through
the C ABI, that two calls in a row give the same outputs and state as the
allocating entry point qstate_step_host, and that an object whose operands do
not fit the array is refused.  It is collected last (its name sorts last), so
a run that stops at the first failure has run every other test first; it
also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_recurrent_state_decode_b200 import qstate as Q
from bit_recurrent_state_decode_b200 import synth

from parity_util import REL_TOL, gpu_object, rel_err

pytestmark = pytest.mark.gpu
C4 = synth.WORKLOADS["gdn_l24_b256_h32_d128_int4g64_bdr"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_recurrent_state_decode_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _pinned(a):
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    return t.pin_memory()


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_static_staging_matches_allocating_host_step():
    wl = C4.scaled(batch=8, layers=1)                   # 256 tiles, 0.3 MB of operands
    a = gpu_object(wl, synth.PERSISTENT, 8, 1)           # stepped by qstate_step_host
    b = gpu_object(wl, synth.PERSISTENT, 8, 1)           # stepped by qstate_step_host_static
    T = a.tiles
    stream = torch.cuda.current_stream()
    for step in range(2):                               # two calls in a row
        x = synth.gen_step(wl, step, tiles=np.arange(T))
        hq, hk, hv, hg = (_pinned(t) for t in (x.q, x.k, x.v, x.gates))
        out_a = torch.zeros((T, wl.d_v), dtype=torch.float32).pin_memory()
        out_b = torch.full((T, wl.d_v), float("nan"), dtype=torch.float32).pin_memory()
        a.step_host(hq, hk, hv, hg, out_a, stream)
        rc = Q.lib().qstate_step_host_static(b._h, _ptr(hq), _ptr(hk), _ptr(hv), _ptr(hg),
                                             _ptr(out_b), ctypes.c_void_p(stream.cuda_stream))
        assert rc == Q.OK, Q.error_string(rc)
        torch.cuda.synchronize()
        for t in range(T):
            assert rel_err(out_b[t].numpy(), out_a[t].numpy()) <= REL_TOL, (step, t)
        assert torch.equal(out_a, out_b)                # the same kernel on the same data
    for x_, y_ in zip(a.export(), b.export()):
        if x_ is not None:
            assert torch.equal(x_, y_)
    st = b.status()
    assert (st["nonfinite"], st["saturated"], st["pipeline_timeouts"]) == (0, 0, 0)
    a.close()
    b.close()


def test_static_staging_refuses_operands_beyond_its_size():
    wl = C4.scaled(batch=256, layers=1)                 # 8192 tiles, 10.5 MB of operands
    big = gpu_object(wl, synth.PERSISTENT, 256, 2)       # 21 MB > 16 MiB
    z = big.sizes
    assert 2 * z["q_bytes"] + z["v_bytes"] + z["gate_bytes"] + z["out_bytes"] > 16 << 20
    h = [torch.zeros(n, dtype=torch.uint8).pin_memory()
         for n in (z["q_bytes"], z["q_bytes"], z["v_bytes"], z["gate_bytes"], z["out_bytes"])]
    rc = Q.lib().qstate_step_host_static(big._h, *(_ptr(t) for t in h), None)
    assert rc == Q.EINVAL
    big.close()
