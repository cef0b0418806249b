"""The ctypes binding rejects step operands the kernels would read or write
out of bounds (wrong device, dtype, layout or size) before the C call: the C
layer receives bare pointers and cannot tell.  No GPU needed: the checks run
on a binding object whose sizes are set by hand."""
import numpy as np
import pytest
import torch

from bit_recurrent_state_decode_b200 import qstate as Q


def _obj(qkv=Q.BF16, gate=Q.BF16, tiles=8, dk=128, dv=128, n_gate=2):
    o = object.__new__(Q.QState)
    o._h = None
    o.device = 0
    o.qkv_dtype, o.gate_dtype = qkv, gate
    isz = 2 if qkv == Q.BF16 else 4
    gsz = 2 if gate == Q.BF16 else 4
    o.sizes = dict(tiles=tiles, q_bytes=tiles * dk * isz, v_bytes=tiles * dv * isz,
                   gate_bytes=tiles * n_gate * gsz, out_bytes=tiles * dv * 4, n_gate=n_gate)
    return o


def _host_ops(o, tiles=8, dk=128, dv=128, n_gate=2):
    dt = o.qkv_torch_dtype
    return [torch.zeros(tiles, dk, dtype=dt), torch.zeros(tiles, dk, dtype=dt),
            torch.zeros(tiles, dv, dtype=dt), torch.zeros(tiles, n_gate, dtype=o.gate_torch_dtype),
            torch.zeros(tiles, dv, dtype=torch.float32)]


def test_host_operands_accepted():
    o = _obj()
    o._check_operands("step_host", _host_ops(o), host=True)
    # bf16 operands given as raw 16-bit patterns, and numpy arrays
    ops = _host_ops(o)
    ops[0] = ops[0].view(torch.int16)
    ops[4] = ops[4].numpy()
    o._check_operands("step_host", ops, host=True)


@pytest.mark.parametrize("idx,bad,msg", [
    (0, torch.zeros(7, 128, dtype=torch.bfloat16), "holds"),          # undersized q
    (2, torch.zeros(8, 128, dtype=torch.float32), "dtype"),           # f32 v for bf16
    (4, torch.zeros(8, 128, dtype=torch.bfloat16), "dtype"),          # out must be f32
    (1, torch.zeros(128, 8, dtype=torch.bfloat16).t(), "contiguous"),  # strided k
    (3, None, "required"),                                           # missing gates
])
def test_bad_host_operand_rejected(idx, bad, msg):
    o = _obj()
    ops = _host_ops(o)
    ops[idx] = bad
    with pytest.raises(ValueError, match=msg):
        o._check_operands("step_host", ops, host=True)


def test_device_step_rejects_host_tensors():
    o = _obj()
    with pytest.raises(ValueError, match="CUDA tensor"):
        o._check_operands("step", _host_ops(o), host=False)


def test_numpy_item_size_checked():
    o = _obj(qkv=Q.F32, gate=Q.F32)
    ops = [a.numpy() for a in _host_ops(o)]
    ops[0] = np.zeros((8, 128), np.float64)
    with pytest.raises(ValueError, match="item size"):
        o._check_operands("step_host", ops, host=True)


def test_retnet_needs_no_gates():
    o = _obj(qkv=Q.F32, gate=Q.F32, n_gate=0)
    ops = _host_ops(o, n_gate=0)
    ops[3] = None
    o._check_operands("step_host", ops, host=True)
