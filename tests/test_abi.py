"""The C ABI (include/qstate.h) without a GPU: the library loads, exports every
declared symbol, and rejects invalid arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def q():
    from bit_recurrent_state_decode_b200 import build, qstate
    build.build()
    return qstate


def _declared():
    text = open(os.path.join(ROOT, "include", "qstate.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qstate_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(q):
    declared = _declared()
    assert len(declared) == 24
    assert sorted(q.EXPORTS) == declared
    lib = q.lib()
    for name in declared:
        assert hasattr(lib, name), name


def test_error_strings(q):
    assert q.error_string(0) == "ok"
    assert q.error_string(-1) == "invalid argument"
    assert q.error_string(-99) == "unknown error"


def _layout(q, **kw):
    d = dict(batch=2, heads=4, d_k=128, d_v=128, layers=1, kind=q.GDN, gamma=0.9,
             qkv_dtype=q.BF16, gate_dtype=q.BF16, scale_dtype=q.F16, head_bits=None)
    d.update(kw)
    return q.Layout(**d)


@pytest.mark.parametrize("kw,args", [
    ({}, dict(bits=5)),
    ({}, dict(bits=4, group=12)),
    ({}, dict(bits=4, group=256)),
    ({}, dict(bits=4, group=-8)),
    ({}, dict(bits=4, sm=3)),
    ({}, dict(bits=4, rm=2)),
    ({}, dict(bits=4, eps=-0.1)),
    ({}, dict(bits=4, eps=float("nan"))),
    ({}, dict(bits=32, sm=2)),                   # yoked needs a quantized state
    (dict(batch=-1), dict(bits=4)),
    (dict(heads=0), dict(bits=4)),
    (dict(layers=0), dict(bits=4)),
    (dict(d_k=60), dict(bits=4)),
    (dict(kind=7), dict(bits=4)),
    (dict(qkv_dtype=2), dict(bits=4)),
    (dict(scale_dtype=1), dict(bits=4)),
    (dict(kind=0, gamma=float("inf")), dict(bits=4)),
    (dict(batch=1 << 20, heads=1 << 8, layers=8), dict(bits=4)),   # 2^31 tiles
])
def test_create_rejects_invalid(q, kw, args):
    L = _layout(q, **kw)
    h = ctypes.c_void_p()
    rc = q.lib().qstate_create(ctypes.byref(L), args.get("bits", 4), args.get("group", 64),
                               args.get("sm", 0), args.get("rm", 0), args.get("eps", 0.0),
                               ctypes.byref(h))
    assert rc == q.EINVAL
    assert not h.value


def test_create_rejects_bad_head_bits(q):
    hb = (ctypes.c_uint8 * 4)(2, 4, 5, 8)
    L = _layout(q, head_bits=ctypes.cast(hb, ctypes.POINTER(ctypes.c_uint8)))
    h = ctypes.c_void_p()
    assert q.lib().qstate_create(ctypes.byref(L), 4, 64, 0, 0, 0.0, ctypes.byref(h)) == q.EINVAL


def test_unsupported_shape(q):
    L = _layout(q, d_k=256)
    h = ctypes.c_void_p()
    assert q.lib().qstate_create(ctypes.byref(L), 4, 64, 0, 0, 0.0,
                                 ctypes.byref(h)) == q.EUNSUPPORTED


def test_null_object_calls(q):
    lib = q.lib()
    assert lib.qstate_create(None, 4, 64, 0, 0, 0.0, None) == q.EINVAL
    assert lib.qstate_step(None, None, None, None, None, None, None) == q.EINVAL
    assert lib.qstate_step_host(None, None, None, None, None, None, None) == q.EINVAL
    assert lib.qstate_step_host_static(None, None, None, None, None, None, None) == q.EINVAL
    assert lib.qstate_dequant(None, None, None) == q.EINVAL
    assert lib.qstate_export(None, None, None, None, None) == q.EINVAL
    assert lib.qstate_import(None, None, None, None, None) == q.EINVAL
    assert lib.qstate_get_sizes(None, None) == q.EINVAL
    assert lib.qstate_bytes_per_step(None) == -1
    assert lib.qstate_status(None, None, None) == q.EINVAL
    assert lib.qstate_reset(None, None) == q.EINVAL
    assert lib.qstate_debug_set(None, -1, 1) == q.EINVAL
    assert lib.qstate_set_taxonomy(None, 1) == q.EINVAL
    assert lib.qstate_destroy(None) == q.EINVAL
    # the layout variants, their side state and the host pipeline
    assert lib.qstate_set_lrb(None, 1, 15, 0.5) == q.EINVAL
    assert lib.qstate_lrb_export(None, None, None, None, None, None, None) == q.EINVAL
    assert lib.qstate_set_pw(None, 8) == q.EINVAL
    assert lib.qstate_pw_export(None, None, None, None, None, None) == q.EINVAL
    assert lib.qstate_set_rowcol(None) == q.EINVAL
    assert lib.qstate_error_rows(None, None, None) == q.EINVAL
    assert lib.qstate_step_host_pipelined(None, None, None, None, None, None, None) == q.EINVAL
    assert lib.qstate_step_host_sync(None, None) == q.EINVAL
    assert lib.qstate_kernel(None) == b""


def test_product_never_imports_oracle():
    pkg = os.path.join(ROOT, "bit_recurrent_state_decode_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "qstate_oracle" not in text, f
