"""CPU oracle of the quantized recurrent-state decode step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product path (``bit_recurrent_state_decode_b200``) never imports it and shares
no code with it.

The arithmetic lives in ``qstate_oracle.c`` (plain scalar C, fp32 with an
explicit operation order, fp64 only for exact products); this module only
builds it and marshals numpy arrays.  It follows "Preserving Updates in
Low-Bit Recurrent State Quantization" (Table 1, Abstract, Figure 4, Table 6)
and "When Dynamic Scaling Fails" (Abstract); the readings of the points those
pages leave open are written next to the C code that implements them.

Every oracle function is pinned in ``tests/test_oracle_*.py`` against closed
forms, invariants, exhaustive enumeration or independent library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qstate_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

RETNET, MAMBA2, GLA, GDN = 0, 1, 2, 3
DYNAMIC, PERSISTENT, YOKED = 0, 1, 2
RTN, BDR = 0, 1
NONE, LOST, MOVED, REVERSED = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC),
                                             os.path.getmtime(SRC[:-2] + ".h"))):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-Wall", "-shared", "-fPIC", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("d_k", ctypes.c_int), ("d_v", ctypes.c_int), ("kind", ctypes.c_int),
                ("group", ctypes.c_int), ("scale_mode", ctypes.c_int),
                ("round_mode", ctypes.c_int), ("scale_f32", ctypes.c_int),
                ("gamma", ctypes.c_float), ("eps_b", ctypes.c_float),
                ("taxonomy", ctypes.c_int), ("rotate", ctypes.c_int)]


class Counts(ctypes.Structure):
    _fields_ = [("nonfinite", ctypes.c_int64), ("saturated", ctypes.c_int64),
                ("lost", ctypes.c_int64), ("moved", ctypes.c_int64),
                ("reversed", ctypes.c_int64), ("bdr_applied", ctypes.c_int64)]

    def as_dict(self):
        return {n: int(getattr(self, n)) for n, _ in self._fields_}


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        _lib.or_f32_to_f16.restype = ctypes.c_uint16
        _lib.or_f32_to_f16.argtypes = [ctypes.c_float]
        _lib.or_f16_to_f32.restype = ctypes.c_float
        _lib.or_f16_to_f32.argtypes = [ctypes.c_uint16]
        _lib.or_bf16_to_f32.restype = ctypes.c_float
        _lib.or_bf16_to_f32.argtypes = [ctypes.c_uint16]
        _lib.or_f32_to_bf16.restype = ctypes.c_uint16
        _lib.or_f32_to_bf16.argtypes = [ctypes.c_float]
        _lib.or_tile_bytes.restype = ctypes.c_int64
        _lib.or_tile_bytes.argtypes = [ctypes.c_int] * 3
        _lib.or_pack.argtypes = [ctypes.c_int] * 3 + [P, P]
        _lib.or_unpack.argtypes = [ctypes.c_int] * 3 + [P, P]
        _lib.or_canon_dot.restype = ctypes.c_float
        _lib.or_canon_dot.argtypes = [ctypes.c_int, P, ctypes.c_int, P]
        _lib.or_round_rtn.restype = ctypes.c_int
        _lib.or_round_rtn.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_int]
        _lib.or_round.restype = ctypes.c_int
        _lib.or_round.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_float, ctypes.c_float,
                                  ctypes.c_float, ctypes.c_int, ctypes.POINTER(Counts)]
        _lib.or_classify.restype = ctypes.c_int
        _lib.or_classify.argtypes = [ctypes.c_float] * 3 + [ctypes.c_int]
        _lib.or_step.restype = ctypes.c_int
        _lib.or_step.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64, P, P, P, P, P,
                                 P, P, P, P, P, P, ctypes.POINTER(Counts)]
        _lib.or_step_trace.restype = ctypes.c_int
        _lib.or_step_trace.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64, P, P, P, P, P,
                                       P, P, P, P, P, P, ctypes.POINTER(Counts), P, P, P]
        _lib.or_n_scales.restype = ctypes.c_int
        _lib.or_n_scales.argtypes = [ctypes.POINTER(_Cfg)]
        _lib.or_dequant.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, P, P, P]
        _lib.or_fwht.argtypes = [ctypes.c_int, P]
        _lib.or_lrb_step.restype = ctypes.c_int
        _lib.or_lrb_step.argtypes = [ctypes.POINTER(_Cfg), ctypes.POINTER(LrbCfg), ctypes.c_int64,
                                     P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                     ctypes.POINTER(Counts), P, P]
        _lib.or_e4m3_to_f32.restype = ctypes.c_float
        _lib.or_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        _lib.or_f32_to_e4m3.restype = ctypes.c_uint8
        _lib.or_f32_to_e4m3.argtypes = [ctypes.c_float]
        _lib.or_pw_step.restype = ctypes.c_int
        _lib.or_pw_step.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_int64,
                                    P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                    ctypes.POINTER(Counts)]
        _lib.or_rc_step.restype = ctypes.c_int
        _lib.or_rc_step.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64, P, P, P, P, P, P, P, P,
                                    P, ctypes.POINTER(Counts)]
        _lib.or_rc_dequant.argtypes = [ctypes.POINTER(_Cfg), P, P, P]
        _lib.or_rank_k.argtypes = [ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, P, P]
        _lib.or_lrb_bits.restype = ctypes.c_double
        _lib.or_lrb_bits.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double]
    return _lib


class LrbCfg(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int), ("m", ctypes.c_int), ("eps_l", ctypes.c_float)]


_pools = {}


def _pool(threads: int):
    """A thread pool kept for the life of the process (the C step releases
    the GIL, so the threads run the scalar code in parallel)."""
    import concurrent.futures
    if threads not in _pools:
        _pools[threads] = concurrent.futures.ThreadPoolExecutor(threads)
    return _pools[threads]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


# ---------------------------------------------------------------- formats
def f32_to_f16_bits(x: float) -> int:
    return int(lib().or_f32_to_f16(float(x)))


def f16_bits_to_f32(h: int) -> float:
    return float(lib().or_f16_to_f32(int(h)))


def bf16_bits_to_f32(h: int) -> float:
    return float(lib().or_bf16_to_f32(int(h)))


def f32_to_bf16_bits(x: float) -> int:
    return int(lib().or_f32_to_bf16(float(x)))


# ---------------------------------------------------------------- layout
def tile_bytes(bits: int, d_k: int, d_v: int) -> int:
    return int(lib().or_tile_bytes(bits, d_k, d_v))


def pack(bits: int, codes: np.ndarray) -> np.ndarray:
    """codes [..., d_k, d_v] int8 -> packed bytes [..., tile_bytes] uint8."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    d_k, d_v = codes.shape[-2:]
    lead = codes.shape[:-2]
    flat = codes.reshape(-1, d_k, d_v)
    nb = tile_bytes(bits, d_k, d_v)
    out = np.zeros((flat.shape[0], nb), dtype=np.uint8)
    for t in range(flat.shape[0]):
        lib().or_pack(bits, d_k, d_v, _ptr(flat[t]), _ptr(out[t]))
    return out.reshape(*lead, nb)


def unpack(bits: int, d_k: int, d_v: int, data: np.ndarray) -> np.ndarray:
    data = np.ascontiguousarray(data, dtype=np.uint8)
    nb = tile_bytes(bits, d_k, d_v)
    lead = data.shape[:-1]
    flat = data.reshape(-1, nb)
    out = np.zeros((flat.shape[0], d_k, d_v), dtype=np.int8)
    for t in range(flat.shape[0]):
        lib().or_unpack(bits, d_k, d_v, _ptr(flat[t]), _ptr(out[t]))
    return out.reshape(*lead, d_k, d_v)


def canon_dot(a: np.ndarray, b: np.ndarray) -> float:
    """Canonical-order sum_i a[i] b[i] (blocks of 8 rows, pairwise tree)."""
    a = _f32(a)
    b = _f32(b)
    return float(lib().or_canon_dot(len(a), _ptr(a), 1, _ptr(b)))


def fwht(x: np.ndarray) -> np.ndarray:
    """H x for the Sylvester Hadamard matrix H (butterfly order of the C code)."""
    y = _f32(x).copy()
    lib().or_fwht(len(y), _ptr(y))
    return y


def round_rtn(x: float, inv: float, qmax: int) -> int:
    return int(lib().or_round_rtn(float(x), float(inv), int(qmax)))


def classify(a: float, x: float, inv: float, qmax: int) -> int:
    return int(lib().or_classify(float(a), float(x), float(inv), int(qmax)))


class Config:
    """Per-tile configuration of the oracle (mirrors the step's parameters)."""

    def __init__(self, d_k, d_v, kind, group, scale_mode=DYNAMIC, round_mode=RTN,
                 scale_f32=False, gamma=1.0 - 2.0 ** -5, eps_b=0.0, taxonomy=False, rotate=0):
        self.c = _Cfg(d_k, d_v, kind, group, scale_mode, round_mode, int(bool(scale_f32)),
                      gamma, eps_b, int(bool(taxonomy)), int(rotate))

    def __getattr__(self, name):
        return getattr(self.__dict__["c"], name)

    @property
    def n_scales(self) -> int:
        return int(lib().or_n_scales(ctypes.byref(self.c)))

    def round(self, a, x, inv, qmax, counts=None) -> int:
        return int(lib().or_round(ctypes.byref(self.c), float(a), float(x), float(inv),
                                  int(qmax), ctypes.byref(counts) if counts else None))


class State:
    """Unpacked oracle state of ``ntiles`` independent tiles.

    codes  [T, d_k, d_v] int8   (quantized tiles)
    S      [T, d_k, d_v] f32    (32-bit tiles)
    scales [T, n_scales] f32    (stored scale values, exactly)
    ref    [T, d_k, d_v] f32    (yoked reference state)
    """

    def __init__(self, cfg: Config, tile_bits):
        self.cfg = cfg
        self.tile_bits = np.ascontiguousarray(tile_bits, dtype=np.int32)
        T = len(self.tile_bits)
        dk, dv = cfg.d_k, cfg.d_v
        self.codes = np.zeros((T, dk, dv), np.int8)
        self.S = np.zeros((T, dk, dv), np.float32)
        self.scales = np.zeros((T, cfg.n_scales), np.float32)
        self.ref = np.zeros((T, dk, dv), np.float32) if cfg.scale_mode == YOKED else None
        self.counts = Counts()

    @property
    def ntiles(self):
        return len(self.tile_bits)

    def step(self, q, k, v, alpha=None, beta=None, threads: int = 1):
        """One step of every tile; ``threads`` > 1 splits the tiles over host
        threads (the tiles are independent; each thread runs the same scalar
        code on its own slice)."""
        return step_many([(self, (q, k, v, alpha, beta))], threads)[0]

    def _jobs(self, q, k, v, alpha, beta, pieces):
        """The step of this state's tiles cut into `pieces` independent jobs;
        returns (jobs, out)."""
        cfg = self.cfg
        T = self.ntiles
        q, k, v = _f32(q).reshape(T, -1), _f32(k).reshape(T, -1), _f32(v).reshape(T, -1)
        if alpha is not None:
            alpha = _f32(alpha).reshape(T, -1)
        if beta is not None:
            beta = _f32(beta).reshape(T)
        out = np.zeros((T, cfg.d_v), np.float32)

        def run(lo, hi):
            cnt = Counts()
            sl = slice(lo, hi)
            rc = lib().or_step(ctypes.byref(cfg.c), hi - lo, _ptr(self.tile_bits[sl]),
                               _ptr(self.codes[sl]), _ptr(self.S[sl]), _ptr(self.scales[sl]),
                               _ptr(None if self.ref is None else self.ref[sl]), _ptr(q[sl]),
                               _ptr(k[sl]), _ptr(v[sl]),
                               _ptr(None if alpha is None else alpha[sl]),
                               _ptr(None if beta is None else beta[sl]), _ptr(out[sl]),
                               ctypes.byref(cnt))
            if rc != 0:
                raise ValueError("oracle rejected the configuration")
            return cnt

        pieces = max(1, min(int(pieces), T))
        bounds = np.linspace(0, T, pieces + 1).astype(int)
        return [(run, int(bounds[i]), int(bounds[i + 1])) for i in range(pieces)], out

    def _add_counts(self, c):
        for name, _ in Counts._fields_:
            setattr(self.counts, name, getattr(self.counts, name) + getattr(c, name))

    def step_trace(self, q, k, v, alpha=None, beta=None):
        """One step of every tile (as ``step``), also returning the decayed
        state a, the updated state before rounding x (both [T, d_k, d_v] f32)
        and each element's rounding class ([T, d_k, d_v] int8: NONE / LOST /
        MOVED / REVERSED)."""
        cfg = self.cfg
        T = self.ntiles
        q, k, v = _f32(q).reshape(T, -1), _f32(k).reshape(T, -1), _f32(v).reshape(T, -1)
        if alpha is not None:
            alpha = _f32(alpha).reshape(T, -1)
        if beta is not None:
            beta = _f32(beta).reshape(T)
        out = np.zeros((T, cfg.d_v), np.float32)
        a = np.zeros((T, cfg.d_k, cfg.d_v), np.float32)
        x = np.zeros_like(a)
        cls = np.zeros((T, cfg.d_k, cfg.d_v), np.int8)
        cnt = Counts()
        rc = lib().or_step_trace(ctypes.byref(cfg.c), T, _ptr(self.tile_bits), _ptr(self.codes),
                                 _ptr(self.S), _ptr(self.scales), _ptr(self.ref), _ptr(q),
                                 _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(out),
                                 ctypes.byref(cnt), _ptr(a), _ptr(x), _ptr(cls))
        if rc != 0:
            raise ValueError("oracle rejected the configuration")
        for name, _ in Counts._fields_:
            setattr(self.counts, name, getattr(self.counts, name) + getattr(cnt, name))
        return out, a, x, cls

    def dequant(self) -> np.ndarray:
        T = self.ntiles
        out = np.zeros((T, self.cfg.d_k, self.cfg.d_v), np.float32)
        for t in range(T):
            if self.tile_bits[t] == 32:
                out[t] = self.S[t]
            else:
                lib().or_dequant(ctypes.byref(self.cfg.c), int(self.tile_bits[t]),
                                 _ptr(self.codes[t]), _ptr(self.scales[t]), _ptr(out[t]))
        return out

    def packed(self, t: int) -> np.ndarray:
        return pack(int(self.tile_bits[t]), self.codes[t])


def rank_k(R: np.ndarray, k: int):
    """Top-k singular values and vectors (s[k], U[k][rows], V[k][cols]) of R."""
    R = np.ascontiguousarray(R, np.float64)
    rows, cols = R.shape
    s = np.zeros(k)
    U = np.zeros((k, rows))
    V = np.zeros((k, cols))
    lib().or_rank_k(rows, cols, _ptr(R), k, _ptr(s), _ptr(U), _ptr(V))
    return s, U, V


def lrb_bits(bits: int, group: int, d_k: int, d_v: int, cols_used: float,
             scale_bits: int = 16) -> float:
    """Storage per state element with `cols_used` bypass columns."""
    return float(lib().or_lrb_bits(bits, group, scale_bits, d_k, d_v, float(cols_used)))


class LrbState(State):
    """A quantized state with a Low-Rank Bypass (readings L1-L7 of the C
    code): codes and scales as State, plus per tile u [k+m][d_k] and
    w [k+m][d_v] (binary16 patterns), g [k+m], the slot counts and the decay
    D since the last merge (GLA: one factor per key row, [d_k])."""

    def __init__(self, cfg: Config, tile_bits, k: int, m: int, eps_l: float,
                 keep_resid: bool = False):
        super().__init__(cfg, tile_bits)
        self.lcfg = LrbCfg(k, m, eps_l)
        T = self.ntiles
        K = k + m
        self.u = np.zeros((T, K, cfg.d_k), np.uint16)
        self.w = np.zeros((T, K, cfg.d_v), np.uint16)
        self.g = np.zeros((T, K), np.float32)
        self.nres = np.zeros(T, np.int32)
        self.nnew = np.zeros(T, np.int32)
        # decay since the last merge (GLA: one per key row)
        self.gla = cfg.c.kind == GLA
        self.D = np.ones((T, cfg.d_k) if self.gla else T, np.float32)
        self.merged = np.zeros(T, np.int32)
        self.peak_cols = 0                  # most columns held at once (before a merge)
        # the unmerged rest of the bypass at each tile's last merge
        self.resid = np.zeros((T, cfg.d_k, cfg.d_v), np.float32) if keep_resid else None

    def step(self, q, k, v, alpha=None, beta=None, threads: int = 1):
        cfg = self.cfg
        T = self.ntiles
        q, k, v = _f32(q).reshape(T, -1), _f32(k).reshape(T, -1), _f32(v).reshape(T, -1)
        if alpha is not None:
            alpha = _f32(alpha).reshape(T, -1)
            alpha = alpha.copy() if self.gla else alpha[:, :1].copy()
        if beta is not None:
            beta = _f32(beta).reshape(T)
        out = np.zeros((T, cfg.d_v), np.float32)
        self.peak_cols = max(self.peak_cols, int(np.max(self.nres + self.nnew)) + 1)
        cnt = Counts()
        rc = lib().or_lrb_step(ctypes.byref(cfg.c), ctypes.byref(self.lcfg), T,
                               _ptr(self.tile_bits), _ptr(self.codes), _ptr(self.scales),
                               _ptr(self.u), _ptr(self.w), _ptr(self.g), _ptr(self.nres),
                               _ptr(self.nnew), _ptr(self.D), _ptr(q), _ptr(k), _ptr(v),
                               _ptr(alpha),
                               _ptr(beta), _ptr(out), ctypes.byref(cnt), _ptr(self.merged),
                               _ptr(self.resid))
        if rc != 0:
            raise ValueError("oracle rejected the LRB configuration")
        self._add_counts(cnt)
        return out

    def cols_used(self) -> np.ndarray:
        """Bypass columns held per tile after the last step."""
        return self.nres + self.nnew

    def _dfac(self, t: int):
        """Tile t's decay since the last merge, as a column to scale rows."""
        return self.D[t].astype(np.float64)[:, None] if self.gla else float(self.D[t])

    def state(self, t: int) -> np.ndarray:
        """The tile's state D * S_hat + P (fp64; GLA: D per key row)."""
        return self._dfac(t) * self.dequant()[t].astype(np.float64) + self.bypass(t)

    def bypass(self, t: int) -> np.ndarray:
        """The bypass matrix P = sum_l g_l u_l w_l^T of tile t (fp64; GLA: the
        key sides read as D * u)."""
        n = int(self.nres[t] + self.nnew[t])
        u = self.u[t, :n].view(np.float16).astype(np.float64)
        if self.gla:
            u = u * self.D[t].astype(np.float64)[None, :]
        w = self.w[t, :n].view(np.float16).astype(np.float64)
        return np.einsum("l,li,lj->ij", self.g[t, :n].astype(np.float64), u, w)


def e4m3_to_f32(b: int) -> float:
    return float(lib().or_e4m3_to_f32(int(b)))


def f32_to_e4m3(x: float) -> int:
    return int(lib().or_f32_to_e4m3(float(x)))


class PwState(State):
    """A Gated DeltaNet state with a pure-write sliding window of W FP8 pairs
    (readings W1-W6 of the C code): the history as State (codes and scales,
    or an fp32 S for 32-bit tiles), plus per tile A [W][d_k] and B [W][d_v]
    (E4M3 bytes), the slot of the oldest pair and the pairs held."""

    def __init__(self, cfg: Config, tile_bits, W: int):
        super().__init__(cfg, tile_bits)
        T = self.ntiles
        self.W = int(W)
        self.A = np.zeros((T, W, cfg.d_k), np.uint8)
        self.B = np.zeros((T, W, cfg.d_v), np.uint8)
        self.head = np.zeros(T, np.int32)
        self.count = np.zeros(T, np.int32)

    def step(self, q, k, v, alpha=None, beta=None, threads: int = 1):
        cfg = self.cfg
        T = self.ntiles
        q, k, v = _f32(q).reshape(T, -1), _f32(k).reshape(T, -1), _f32(v).reshape(T, -1)
        alpha = _f32(alpha).reshape(T, -1)[:, 0].copy()
        beta = _f32(beta).reshape(T)
        out = np.zeros((T, cfg.d_v), np.float32)
        cnt = Counts()
        rc = lib().or_pw_step(ctypes.byref(cfg.c), self.W, T, _ptr(self.tile_bits),
                              _ptr(self.codes), _ptr(self.S), _ptr(self.scales), _ptr(self.A),
                              _ptr(self.B), _ptr(self.head), _ptr(self.count), _ptr(q), _ptr(k),
                              _ptr(v), _ptr(alpha), _ptr(beta), _ptr(out), ctypes.byref(cnt))
        if rc != 0:
            raise ValueError("oracle rejected the PW configuration")
        self._add_counts(cnt)
        return out

    def pairs(self, t: int):
        """(a, b) of tile t's pairs, oldest first, as fp64 [n, d_k], [n, d_v]."""
        dec = np.vectorize(e4m3_to_f32, otypes=[np.float64])
        n, h = int(self.count[t]), int(self.head[t])
        sl = [(h + l) % self.W for l in range(n)]
        return dec(self.A[t, sl]).reshape(n, -1), dec(self.B[t, sl]).reshape(n, -1)

    def history(self, t: int) -> np.ndarray:
        if int(self.tile_bits[t]) == 32:
            return self.S[t].astype(np.float64)
        return self.dequant()[t].astype(np.float64)

    def state(self, t: int) -> np.ndarray:
        """History plus the window's pairs (fp64)."""
        a, b = self.pairs(t)
        return self.history(t) + a.T @ b


class RcState(State):
    """A quantized state with key-row x value-column scales (readings R1-R5
    of the C code): codes as State, scales [T][d_k + d_v] (rho, then
    kappa)."""

    def __init__(self, cfg: Config, tile_bits):
        super().__init__(cfg, tile_bits)
        self.scales = np.zeros((self.ntiles, cfg.d_k + cfg.d_v), np.float32)

    def step(self, q, k, v, alpha=None, beta=None, threads: int = 1):
        cfg = self.cfg
        T = self.ntiles
        q, k, v = _f32(q).reshape(T, -1), _f32(k).reshape(T, -1), _f32(v).reshape(T, -1)
        if alpha is not None:
            alpha = _f32(alpha).reshape(T, -1)
        if beta is not None:
            beta = _f32(beta).reshape(T)
        out = np.zeros((T, cfg.d_v), np.float32)
        cnt = Counts()
        rc = lib().or_rc_step(ctypes.byref(cfg.c), T, _ptr(self.tile_bits), _ptr(self.codes),
                              _ptr(self.scales), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                              _ptr(beta), _ptr(out), ctypes.byref(cnt))
        if rc != 0:
            raise ValueError("oracle rejected the row x column configuration")
        self._add_counts(cnt)
        return out

    def dequant(self) -> np.ndarray:
        T = self.ntiles
        out = np.zeros((T, self.cfg.d_k, self.cfg.d_v), np.float32)
        for t in range(T):
            lib().or_rc_dequant(ctypes.byref(self.cfg.c), _ptr(self.codes[t]),
                                _ptr(self.scales[t]), _ptr(out[t]))
        return out


def step_many(work, threads: int = 1):
    """One step of several independent oracle states at once: ``work`` is a
    list of (state, (q, k, v, alpha, beta)).  The tiles of all states are
    cut into jobs that ``threads`` host threads run together; returns the
    outputs in order."""
    pieces = max(1, int(threads))
    jobs, outs = [], []
    for st, args in work:
        j, out = st._jobs(*args, pieces=pieces)
        jobs.append((st, j))
        outs.append(out)
    flat = [(st, job) for st, js in jobs for job in js]
    if len(flat) == 1 or threads <= 1:
        results = [run(lo, hi) for _, (run, lo, hi) in flat]
    else:
        results = list(_pool(pieces).map(lambda sj: sj[1][0](sj[1][1], sj[1][2]), flat))
    for (st, _), c in zip(flat, results):
        st._add_counts(c)
    return outs


if __name__ == "__main__":  # pragma: no cover
    print(build(force="--force" in sys.argv))
