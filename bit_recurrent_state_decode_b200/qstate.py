"""Thin ctypes binding of the C ABI in include/qstate.h (libqstate.so).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of the library.  PyTorch supplies device memory (tensors whose
``data_ptr()`` is passed) and streams (``torch.cuda.current_stream()``).
The library must have been built (``python -m bit_recurrent_state_decode_b200.build``);
loading fails loudly otherwise -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libqstate.so")

OK, EINVAL, ENOMEM, ECUDA, EUNSUPPORTED = 0, -1, -2, -3, -4
RETNET, MAMBA2, GLA, GDN = 0, 1, 2, 3
DYNAMIC, PERSISTENT, YOKED = 0, 1, 2
RTN, BDR = 0, 1
F32, BF16, F16 = 0, 1, 2

# every symbol include/qstate.h declares
EXPORTS = ("qstate_create", "qstate_destroy", "qstate_reset", "qstate_step", "qstate_step_host",
           "qstate_step_host_pipelined", "qstate_step_host_sync", "qstate_step_host_static",
           "qstate_dequant", "qstate_export", "qstate_import", "qstate_get_sizes",
           "qstate_bytes_per_step", "qstate_status", "qstate_set_taxonomy", "qstate_set_lrb",
           "qstate_lrb_export", "qstate_set_pw", "qstate_pw_export", "qstate_set_rowcol",
           "qstate_error_rows", "qstate_kernel", "qstate_debug_set", "qstate_error_string")


class QStateError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {code} ({error_string(code)})")
        self.code = code


class Layout(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("d_k", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("layers", ctypes.c_int32), ("kind", ctypes.c_int32),
                ("gamma", ctypes.c_float), ("qkv_dtype", ctypes.c_int32),
                ("gate_dtype", ctypes.c_int32), ("scale_dtype", ctypes.c_int32),
                ("head_bits", ctypes.POINTER(ctypes.c_uint8)), ("rotation", ctypes.c_int32)]


class Counters(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in ("nonfinite", "saturated", "pipeline_timeouts",
                                               "exact_path_warps", "lost", "moved", "reversed",
                                               "bdr_applied")]


class Sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("tiles", "code_bytes", "scale_bytes", "ref_bytes",
                                              "n_scales", "n_gate", "q_bytes", "v_bytes",
                                              "gate_bytes", "out_bytes")]


_lib = None


def lib():
    """Load libqstate.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m bit_recurrent_state_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
        L.qstate_create.argtypes = [ctypes.POINTER(Layout), I, I, I, I, ctypes.c_float,
                                    ctypes.POINTER(P)]
        L.qstate_destroy.argtypes = [P]
        L.qstate_reset.argtypes = [P, S]
        L.qstate_step.argtypes = [P, P, P, P, P, P, S]
        L.qstate_step_host.argtypes = [P, P, P, P, P, P, S]
        L.qstate_step_host_static.argtypes = [P, P, P, P, P, P, S]
        L.qstate_step_host_pipelined.argtypes = [P, P, P, P, P, P, S]
        L.qstate_step_host_sync.argtypes = [P, S]
        L.qstate_dequant.argtypes = [P, P, S]
        L.qstate_export.argtypes = [P, P, P, P, S]
        L.qstate_import.argtypes = [P, P, P, P, S]
        L.qstate_get_sizes.argtypes = [P, ctypes.POINTER(Sizes)]
        L.qstate_bytes_per_step.argtypes = [P]
        L.qstate_bytes_per_step.restype = ctypes.c_int64
        L.qstate_status.argtypes = [P, ctypes.POINTER(Counters), S]
        L.qstate_debug_set.argtypes = [P, ctypes.c_int64, ctypes.c_uint32]
        L.qstate_set_taxonomy.argtypes = [P, I]
        L.qstate_set_lrb.argtypes = [P, I, I, ctypes.c_float]
        L.qstate_lrb_export.argtypes = [P, P, P, P, P, P, S]
        L.qstate_set_pw.argtypes = [P, I]
        L.qstate_pw_export.argtypes = [P, P, P, P, P, S]
        L.qstate_set_rowcol.argtypes = [P]
        L.qstate_error_rows.argtypes = [P, P, S]
        L.qstate_kernel.argtypes = [P]
        L.qstate_kernel.restype = ctypes.c_char_p
        L.qstate_error_string.argtypes = [I]
        L.qstate_error_string.restype = ctypes.c_char_p
        for name in EXPORTS:
            if name not in ("qstate_bytes_per_step", "qstate_error_string", "qstate_kernel"):
                getattr(L, name).restype = I
        _lib = L
    return _lib


def error_string(code: int) -> str:
    return lib().qstate_error_string(int(code)).decode()


def _check(fn, rc):
    if rc != OK:
        raise QStateError(fn, rc)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return ctypes.c_void_p(t.data_ptr())
    return ctypes.c_void_p(t.ctypes.data)   # numpy array (host buffers)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


_TORCH_OF = {F32: torch.float32, BF16: torch.bfloat16, F16: torch.float16}


class QState:
    """A quantized recurrent state of layers x batch x heads tiles of d_k x d_v.

    Mirrors ``qstate_create``; the object owns its device memory until
    ``close()`` (also called on garbage collection)."""

    def __init__(self, batch, heads, d_k, d_v, kind, bits=4, group=64, scale_mode=DYNAMIC,
                 round_mode=RTN, eps_b=0.0, layers=1, gamma=1.0 - 2.0 ** -5, qkv_dtype=F32,
                 gate_dtype=F32, scale_dtype=F16, head_bits=None, rotation=0):
        self._h = None
        self._hb = None
        L = Layout(batch, heads, d_k, d_v, layers, kind, gamma, qkv_dtype, gate_dtype,
                   scale_dtype, None, int(rotation))
        if head_bits is not None:
            self._hb = (ctypes.c_uint8 * heads)(*[int(b) for b in head_bits])
            L.head_bits = ctypes.cast(self._hb, ctypes.POINTER(ctypes.c_uint8))
        h = ctypes.c_void_p()
        self.device = torch.cuda.current_device() if torch.cuda.is_available() else 0
        _check("qstate_create", lib().qstate_create(ctypes.byref(L), int(bits), int(group),
                                                    int(scale_mode), int(round_mode),
                                                    float(eps_b), ctypes.byref(h)))
        self._h = h
        self.batch, self.heads, self.d_k, self.d_v, self.layers = batch, heads, d_k, d_v, layers
        self.kind, self.bits, self.group = kind, bits, group
        self.scale_mode, self.round_mode, self.eps_b = scale_mode, round_mode, eps_b
        self.qkv_dtype, self.gate_dtype, self.scale_dtype = qkv_dtype, gate_dtype, scale_dtype
        self.head_bits = None if head_bits is None else [int(b) for b in head_bits]
        self.rotation = int(rotation)
        self.lrb = None
        self.pw = None
        self.rowcol = False
        z = Sizes()
        _check("qstate_get_sizes", lib().qstate_get_sizes(self._h, ctypes.byref(z)))
        self.sizes = {n: int(getattr(z, n)) for n, _ in Sizes._fields_}

    # ------------------------------------------------------------ lifetime
    def close(self):
        if self._h is not None and _lib is not None:
            lib().qstate_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------ properties
    @property
    def tiles(self) -> int:
        return self.sizes["tiles"]

    @property
    def n_gate(self) -> int:
        return self.sizes["n_gate"]

    @property
    def qkv_torch_dtype(self):
        return _TORCH_OF[self.qkv_dtype]

    @property
    def gate_torch_dtype(self):
        return _TORCH_OF[self.gate_dtype]

    def bytes_per_step(self) -> int:
        return int(lib().qstate_bytes_per_step(self._h))

    # ------------------------------------------------------------ argument checks
    def _operand_specs(self):
        """(name, bytes, dtype) of q, k, v, gates, out for one step."""
        z = self.sizes
        return (("q", z["q_bytes"], self.qkv_torch_dtype), ("k", z["q_bytes"], self.qkv_torch_dtype),
                ("v", z["v_bytes"], self.qkv_torch_dtype),
                ("gates", z["gate_bytes"], self.gate_torch_dtype),
                ("out", z["out_bytes"], torch.float32))

    def _check_operands(self, fn, tensors, host):
        """Reject, before the C call, operands the kernels would read or write
        out of bounds: wrong device, dtype, layout or size.  The C layer sees
        only pointers and cannot tell."""
        for (name, nbytes, dtype), t in zip(self._operand_specs(), tensors):
            if nbytes == 0 and t is None:
                continue
            if t is None:
                raise ValueError(f"{fn}: {name} is required for this layer kind")
            if isinstance(t, torch.Tensor):
                if host and t.is_cuda:
                    raise ValueError(f"{fn}: {name} must be a host tensor")
                if not host:
                    if not t.is_cuda:
                        raise ValueError(f"{fn}: {name} must be a CUDA tensor")
                    if t.device.index != self.device:
                        raise ValueError(f"{fn}: {name} is on cuda:{t.device.index}, "
                                         f"the object on cuda:{self.device}")
                # bf16 operands may also come as raw 16-bit patterns
                ok_dtypes = {dtype} | ({torch.int16, torch.uint16} if dtype == torch.bfloat16
                                       else set())
                if t.dtype not in ok_dtypes:
                    raise ValueError(f"{fn}: {name} has dtype {t.dtype}, expected {dtype}")
                if not t.is_contiguous():
                    raise ValueError(f"{fn}: {name} must be contiguous")
                have = t.numel() * t.element_size()
            else:
                import numpy as np
                a = np.asarray(t)
                if not a.flags["C_CONTIGUOUS"]:
                    raise ValueError(f"{fn}: {name} must be contiguous")
                if a.dtype.itemsize != torch.tensor([], dtype=dtype).element_size():
                    raise ValueError(f"{fn}: {name} has item size {a.dtype.itemsize}")
                have = a.nbytes
            if have < nbytes:
                raise ValueError(f"{fn}: {name} holds {have} bytes, the step needs {nbytes}")

    # ------------------------------------------------------------ calls
    def reset(self, stream=None):
        _check("qstate_reset", lib().qstate_reset(self._h, _stream(stream)))

    def step(self, q, k, v, gates, out, stream=None):
        """One decode step; q, k, v, gates, out are CUDA tensors in the
        layouts of include/qstate.h (gates None for RetNet)."""
        self._check_operands("step", (q, k, v, gates, out), host=False)
        _check("qstate_step", lib().qstate_step(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(gates),
                                                _ptr(out), _stream(stream)))

    def step_host(self, q, k, v, gates, out, stream=None):
        """The same step from host buffers (pinned CPU tensors or numpy arrays).
        Calls on one object must be issued on one stream: they share the
        object's device staging buffers."""
        self._check_operands("step_host", (q, k, v, gates, out), host=True)
        _check("qstate_step_host", lib().qstate_step_host(self._h, _ptr(q), _ptr(k), _ptr(v),
                                                          _ptr(gates), _ptr(out), _stream(stream)))

    def step_host_pipelined(self, q, k, v, gates, out, stream=None):
        """step_host whose output copy overlaps the next call's step
        (qstate_step_host_pipelined): the last call's output is complete
        after step_host_sync and the stream."""
        self._check_operands("step_host_pipelined", (q, k, v, gates, out), host=True)
        _check("qstate_step_host_pipelined",
               lib().qstate_step_host_pipelined(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(gates),
                                                _ptr(out), _stream(stream)))

    def step_host_sync(self, stream=None):
        """The stream waits for the last host-buffer call's output copy."""
        _check("qstate_step_host_sync", lib().qstate_step_host_sync(self._h, _stream(stream)))

    def step_host_static(self, q, k, v, gates, out, stream=None):
        """The host-buffer step that allocates no device memory: the operands
        are staged in the library's fixed device array (see
        qstate_step_host_static in include/qstate.h for its size limit and
        sharing rules)."""
        self._check_operands("step_host_static", (q, k, v, gates, out), host=True)
        _check("qstate_step_host_static",
               lib().qstate_step_host_static(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(gates),
                                             _ptr(out), _stream(stream)))

    def dequant(self, out=None, stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty((self.tiles, self.d_k, self.d_v), dtype=torch.float32, device="cuda")
        if self.tiles == 0:             # nothing to write (an empty tensor has no address)
            return out
        _check("qstate_dequant", lib().qstate_dequant(self._h, _ptr(out), _stream(stream)))
        return out

    def export(self, stream=None):
        """(codes uint8, scales, ref) as new CUDA tensors."""
        z = self.sizes
        codes = torch.empty(z["code_bytes"], dtype=torch.uint8, device="cuda")
        sdt = torch.float32 if self.scale_dtype == F32 else torch.float16
        scales = torch.empty(z["scale_bytes"] // (4 if self.scale_dtype == F32 else 2),
                             dtype=sdt, device="cuda")
        ref = (torch.empty(z["ref_bytes"] // 4, dtype=torch.float32, device="cuda")
               if z["ref_bytes"] else None)
        if self.tiles == 0:
            return codes, scales, ref
        _check("qstate_export", lib().qstate_export(self._h, _ptr(codes), _ptr(scales), _ptr(ref),
                                                    _stream(stream)))
        return codes, scales, ref

    def import_(self, codes, scales, ref=None, stream=None):
        if self.tiles == 0:
            return
        _check("qstate_import", lib().qstate_import(self._h, _ptr(codes), _ptr(scales), _ptr(ref),
                                                    _stream(stream)))

    def status(self, stream=None) -> dict:
        c = Counters()
        _check("qstate_status", lib().qstate_status(self._h, ctypes.byref(c), _stream(stream)))
        return {n: int(getattr(c, n)) for n, _ in Counters._fields_}

    def set_taxonomy(self, on: bool = True):
        """Count lost / moved / reversed elements of the following steps
        (qstate_set_taxonomy)."""
        _check("qstate_set_taxonomy", lib().qstate_set_taxonomy(self._h, 1 if on else 0))

    @property
    def kernel(self) -> str:
        """The kernel the next step launches (qstate_kernel)."""
        return lib().qstate_kernel(self._h).decode()

    def error_rows(self, stream=None) -> torch.Tensor:
        """Per tile and key row, the squared rounding error of the last step
        taken with the taxonomy on (qstate_error_rows), [tiles, d_k]."""
        out = torch.empty((self.tiles, self.d_k), dtype=torch.float32, device=f"cuda:{self.device}")
        if self.tiles == 0:
            return out
        _check("qstate_error_rows", lib().qstate_error_rows(self._h, _ptr(out), _stream(stream)))
        return out

    def set_rowcol(self):
        """Key-row x value-column scales (qstate_set_rowcol); before the
        first step.  The scales become [tiles, d_k + d_v] (rho, then kappa)."""
        _check("qstate_set_rowcol", lib().qstate_set_rowcol(self._h))
        self.rowcol = True
        z = Sizes()
        _check("qstate_get_sizes", lib().qstate_get_sizes(self._h, ctypes.byref(z)))
        self.sizes = {n: int(getattr(z, n)) for n, _ in Sizes._fields_}

    def set_pw(self, W: int):
        """Gated DeltaNet steps with a pure-write sliding window of W FP8
        pairs (qstate_set_pw); before the first step."""
        _check("qstate_set_pw", lib().qstate_set_pw(self._h, int(W)))
        self.pw = int(W)

    def pw_export(self, stream=None) -> dict:
        """The window as new CUDA tensors: A [tiles, W, d_k], B [tiles, W, d_v]
        (E4M3 bytes, uint8, by slot), head and count [tiles] (int32)."""
        if self.pw is None:
            raise QStateError("qstate_pw_export", 1)
        T, W = self.tiles, self.pw
        dev = f"cuda:{self.device}"
        A = torch.empty((T, W, self.d_k), dtype=torch.uint8, device=dev)
        B = torch.empty((T, W, self.d_v), dtype=torch.uint8, device=dev)
        head = torch.empty((T,), dtype=torch.int32, device=dev)
        count = torch.empty((T,), dtype=torch.int32, device=dev)
        if T == 0:
            return {"A": A, "B": B, "head": head, "count": count}
        _check("qstate_pw_export", lib().qstate_pw_export(self._h, _ptr(A), _ptr(B), _ptr(head),
                                                          _ptr(count), _stream(stream)))
        return {"A": A, "B": B, "head": head, "count": count}

    def set_lrb(self, k: int, m: int, eps_l: float):
        """Low-Rank Bypass with a rank-k residual, a merge every m steps and
        the merge threshold eps_l (qstate_set_lrb); before the first step."""
        _check("qstate_set_lrb", lib().qstate_set_lrb(self._h, int(k), int(m), float(eps_l)))
        self.lrb = (int(k), int(m), float(eps_l))

    def lrb_export(self, stream=None) -> dict:
        """The bypass as new CUDA tensors: u [tiles, k+m, d_k] and
        w [tiles, k+m, d_v] (float16), g [tiles, k+m], n [tiles, 2]
        (residual and fresh columns held), D [tiles] (GLA: [tiles, d_k])."""
        if self.lrb is None:
            raise QStateError("qstate_lrb_export", 1)
        K = self.lrb[0] + self.lrb[1]
        T = self.tiles
        dev = f"cuda:{self.device}"
        u = torch.empty((T, K, self.d_k), dtype=torch.float16, device=dev)
        w = torch.empty((T, K, self.d_v), dtype=torch.float16, device=dev)
        g = torch.empty((T, K), dtype=torch.float32, device=dev)
        n = torch.empty((T, 2), dtype=torch.int32, device=dev)
        D = torch.empty((T, self.d_k) if self.kind == GLA else (T,), dtype=torch.float32, device=dev)
        if T == 0:
            return {"u": u, "w": w, "g": g, "n": n, "D": D}
        _check("qstate_lrb_export", lib().qstate_lrb_export(self._h, _ptr(u), _ptr(w), _ptr(g), _ptr(n),
                                                            _ptr(D), _stream(stream)))
        return {"u": u, "w": w, "g": g, "n": n, "D": D}

    def debug_set(self, drop_from_tile=-1, wait_polls=1 << 24):
        """Fault injection for the bounded pipeline waits (see qstate_debug_set)."""
        _check("qstate_debug_set", lib().qstate_debug_set(self._h, int(drop_from_tile),
                                                          int(wait_polls)))

    # ------------------------------------------------------------ helpers
    def alloc_inputs(self, device="cuda"):
        """Empty q, k, v, gates, out buffers in the step layouts."""
        T = self.tiles
        q = torch.empty((T, self.d_k), dtype=self.qkv_torch_dtype, device=device)
        k = torch.empty_like(q)
        v = torch.empty((T, self.d_v), dtype=self.qkv_torch_dtype, device=device)
        g = (torch.empty((T, self.n_gate), dtype=self.gate_torch_dtype, device=device)
             if self.n_gate else None)
        out = torch.empty((T, self.d_v), dtype=torch.float32, device=device)
        return q, k, v, g, out
