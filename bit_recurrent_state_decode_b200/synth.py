"""Seeded synthetic decode streams for the five workloads.

This module holds no arithmetic of the decode step: it only draws the step
inputs (q, k, v and the materialised gates) that both the CUDA path and the
CPU oracle consume.  Every value is a pure function of
(workload seed, layer, step, tile, field, element), so any subset of tiles can
be regenerated on its own.

Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
numbers: as easy as 1, 2, 3", SC'11), key = (seed, layer), counter =
(step, tile, field, element // 8).  Each 128-bit output gives eight 16-bit
draws u; a standard normal is the table value Z[u] = Phi^-1((u + 1/2) / 65536)
(fp64, rounded to fp32), so the tails stop at about 4.3 sigma.

Workload recipes (the five decode configurations):
  q, k, v ~ N(0, sigma^2): fp32 Z[u] times fp32 sigma, then cast to the input
  dtype (bf16 round-to-nearest-even).  Gated DeltaNet keys and queries are
  N(0, 1) draws L2-normalised in fp32 (sequential sum of squares, sqrt, divide)
  before the bf16 cast.  Gates are looked up from fp64 tables indexed by the
  same 16-bit draw u (so no transcendental runs at generation time):
    Mamba2  alpha = exp(-softplus(a)) = 1 / (1 + e^a),  a ~ N(0, 1)
    GLA     alpha = sigmoid(g)^(1/16),                   g ~ N(2, 1)
    GDN     alpha = sigmoid(N(3, 1)),  beta = sigmoid(N(0, 1))
"""
from __future__ import annotations

import dataclasses
import functools

import numpy as np

# Philox4x32 constants (multipliers and Weyl key increments), SC'11.
_M0, _M1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
_W0, _W1 = np.uint32(0x9E3779B9), np.uint32(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)

RETNET, MAMBA2, GLA, GDN = 0, 1, 2, 3
DYNAMIC, PERSISTENT, YOKED = 0, 1, 2
RTN, BDR = 0, 1
F32, BF16, F16 = 0, 1, 2

FIELD_Q, FIELD_K, FIELD_V, FIELD_ALPHA, FIELD_BETA = 0, 1, 2, 3, 4


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10.  All arguments uint32 arrays (broadcast)."""
    c0, c1, c2, c3 = (np.asarray(c, np.uint32) for c in (c0, c1, c2, c3))
    k0 = np.asarray(k0, np.uint32).copy()
    k1 = np.asarray(k1, np.uint32).copy()
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    with np.errstate(over="ignore"):
        for r in range(10):
            if r:
                k0 = k0 + _W0
                k1 = k1 + _W1
            p0 = _M0 * c0.astype(np.uint64)
            p1 = _M1 * c2.astype(np.uint64)
            hi0, lo0 = (p0 >> np.uint64(32)).astype(np.uint32), (p0 & _MASK).astype(np.uint32)
            hi1, lo1 = (p1 >> np.uint64(32)).astype(np.uint32), (p1 & _MASK).astype(np.uint32)
            c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


@functools.lru_cache(maxsize=None)
def normal_table() -> np.ndarray:
    """Z[u] = Phi^-1((u + 1/2) / 65536), fp64."""
    from scipy.special import ndtri
    return ndtri((np.arange(65536, dtype=np.float64) + 0.5) / 65536.0)


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


@functools.lru_cache(maxsize=None)
def gate_table(name: str) -> np.ndarray:
    """fp64 gate value for each 16-bit draw."""
    z = normal_table()
    if name == "mamba2_alpha":
        return 1.0 / (1.0 + np.exp(z))                 # exp(-softplus(z))
    if name == "gla_alpha":
        return _sigmoid(2.0 + z) ** (1.0 / 16.0)
    if name == "gdn_alpha":
        return _sigmoid(3.0 + z)
    if name == "gdn_beta":
        return _sigmoid(z)
    raise KeyError(name)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    nan = np.isnan(x)
    rnd = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    with np.errstate(over="ignore"):
        out = ((u + rnd) >> np.uint32(16)).astype(np.uint16)
    out[nan] = ((u[nan] >> np.uint32(16)) | np.uint32(0x40)).astype(np.uint16)
    return out


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------- workloads
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    kind: int
    batch: int
    heads: int
    d_k: int
    d_v: int
    steps: int
    bits: int                    # uniform bits, or 0 when head_bits is used
    group: int                   # 0 = one scale per tile (per-token)
    scale_modes: tuple           # one qstate object per mode, stepped side by side
    round_mode: int
    qkv_dtype: int
    gate_dtype: int
    scale_dtype: int
    layers: int = 1
    eps_b: float = 0.0
    gamma: float = 1.0 - 2.0 ** -5
    q_sigma: float = 0.0         # 0: L2-normalised N(0,1) (GDN)
    k_sigma: float = 0.0
    v_sigma: float = 1.0
    head_bits_multiset: tuple = ()
    description: str = ""
    rotation: int = 0            # 1: Hadamard-rotated state (INT4+Had)
    lrb: tuple = ()              # (k, m, eps_L): Low-Rank Bypass
    pw: int = 0                  # W > 0: pure-write sliding window of W FP8 pairs
    rowcol: bool = False         # key-row x value-column scales

    @property
    def seed(self) -> int:
        return 0x5EED0000 + self.index

    @property
    def tiles_per_layer(self) -> int:
        return self.batch * self.heads

    @property
    def n_gate(self) -> int:
        return {RETNET: 0, MAMBA2: 1, GLA: self.d_k, GDN: 2}[self.kind]

    def head_bits(self):
        if not self.head_bits_multiset:
            return None
        pool = [b for b, n in self.head_bits_multiset for _ in range(n)]
        assert len(pool) == self.heads
        rng = np.random.Generator(np.random.PCG64(self.seed))
        return np.asarray(rng.permutation(pool), np.uint8)

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "retnet_b1_h2_d64_int4g64": Workload(
        "retnet_b1_h2_d64_int4g64", 0, RETNET, 1, 2, 64, 64, 256, 4, 64, (DYNAMIC,), RTN,
        F32, F32, F16, q_sigma=1 / 8, k_sigma=1 / 8,
        description="RetNet gamma=1-2^-5, INT4 g64 fp16 dynamic scale, RTN, fp32 inputs"),
    "mamba2_b64_h32_dk128_dv64_int8tok": Workload(
        "mamba2_b64_h32_dk128_dv64_int8tok", 1, MAMBA2, 64, 32, 128, 64, 1024, 8, 0,
        (DYNAMIC,), RTN, F32, F32, F16, q_sigma=float(np.float32(1 / np.sqrt(128))),
        k_sigma=float(np.float32(1 / np.sqrt(128))),
        description="Mamba2 scalar decay, INT8 per-token dynamic scale, RTN, fp32 inputs"),
    "gla_b128_h16_d128_int4g32_persistent": Workload(
        "gla_b128_h16_d128_int4g32_persistent", 2, GLA, 128, 16, 128, 128, 4096, 4, 32,
        (PERSISTENT,), RTN, BF16, F32, F16, q_sigma=float(np.float32(1 / np.sqrt(128))),
        k_sigma=float(np.float32(1 / np.sqrt(128))),
        description="GLA diagonal decay, INT4 g32 fp16 persistent scale, RTN, bf16 inputs"),
    "gdn_l24_b256_h32_d128_int4g64_bdr": Workload(
        "gdn_l24_b256_h32_d128_int4g64_bdr", 3, GDN, 256, 32, 128, 128, 2048, 4, 64,
        (PERSISTENT,), BDR, BF16, BF16, F16, layers=24,
        description="Gated DeltaNet x24 layers, INT4 g64 fp16 persistent scale, BDR, bf16"),
    "gdn_b32_h16_d128_mixed_3modes": Workload(
        "gdn_b32_h16_d128_mixed_3modes", 4, GDN, 32, 16, 128, 128, 32768, 0, 64,
        (DYNAMIC, PERSISTENT, YOKED), BDR, BF16, BF16, F32,
        head_bits_multiset=((2, 4), (4, 9), (6, 2), (8, 1)),
        description="GDN long horizon, mixed per-head bits {2,4,6,8} (mean 4), g64 fp32 "
                    "scales, dynamic + persistent + yoked side by side, BDR"),
}
BY_INDEX = {w.index: w for w in WORKLOADS.values()}

# Layout variants the pages compare against, on the shapes above (not among
# the five decode configurations).  INT4+Had: Table 2 of "Preserving Updates
# in Low-Bit Recurrent State Quantization", INT4 at 4.50 bits (group 32,
# binary16 scales) with a Hadamard rotation before quantization, on the
# 24-layer Gated DeltaNet decode.
VARIANTS = {
    "gdn_l24_b256_h32_d128_int4g32_had": Workload(
        "gdn_l24_b256_h32_d128_int4g32_had", 5, GDN, 256, 32, 128, 128, 2048, 4, 32,
        (DYNAMIC,), RTN, BF16, BF16, F16, layers=24, rotation=1,
        description="Gated DeltaNet x24 layers, Hadamard-rotated INT4 g32 fp16 dynamic scale "
                    "(INT4+Had), RTN, bf16"),
    # LRB+BDR with the Gated DeltaNet configuration of Table 6 (k = 1,
    # m = 15, eps_L = 0.50, eps_B = 0.30) on INT4 g32 binary16 scales
    "gdn_l24_b256_h32_d128_int4g32_lrb": Workload(
        "gdn_l24_b256_h32_d128_int4g32_lrb", 6, GDN, 256, 32, 128, 128, 2048, 4, 32,
        (PERSISTENT,), BDR, BF16, BF16, F16, layers=24, eps_b=0.3, lrb=(1, 15, 0.5),
        description="Gated DeltaNet x24 layers, INT4 g32 fp16 persistent scale with a Low-Rank "
                    "Bypass (k=1, m=15, eps_L=0.5) and BDR (eps_B=0.3): LRB+BDR of Table 6"),
    # the 24-layer Gated DeltaNet decode with the pure-write window of
    # "Low-Bit GDN Recurrent-State Quantization ..." at 8 pairs (PW-S8)
    "gdn_l24_b256_h32_d128_int4g64_pw8": Workload(
        "gdn_l24_b256_h32_d128_int4g64_pw8", 7, GDN, 256, 32, 128, 128, 2048, 4, 64,
        (PERSISTENT,), BDR, BF16, BF16, F16, layers=24, pw=8,
        description="Gated DeltaNet x24 layers, INT4 g64 fp16 persistent scale, BDR, with a "
                    "pure-write window of 8 FP8 E4M3 pairs (PW-S8)"),
    # the same decode with key-row x value-column scales (STEPQuant's layout,
    # fitted from the state every step): 4.25 bits per element
    "gdn_l24_b256_h32_d128_int4rc": Workload(
        "gdn_l24_b256_h32_d128_int4rc", 8, GDN, 256, 32, 128, 128, 2048, 4, 0,
        (DYNAMIC,), BDR, BF16, BF16, F16, layers=24, rowcol=True,
        description="Gated DeltaNet x24 layers, INT4 with fp16 key-row x value-column scales "
                    "fitted every step, BDR, bf16"),
    # the GLA decode with the same bypass (k = 1, m = 15, eps_L = 0.50): a
    # decay factor per key row instead of one per tile
    "gla_b128_h16_d128_int4g32_lrb": Workload(
        "gla_b128_h16_d128_int4g32_lrb", 9, GLA, 128, 16, 128, 128, 4096, 4, 32,
        (PERSISTENT,), RTN, BF16, F32, F16, q_sigma=float(np.float32(1 / np.sqrt(128))),
        k_sigma=float(np.float32(1 / np.sqrt(128))), lrb=(1, 15, 0.5),
        description="GLA diagonal decay, INT4 g32 fp16 persistent scale, RTN, bf16, with a "
                    "Low-Rank Bypass (k=1, m=15, eps_L=0.5; one decay factor per key row)"),
}


def workload(name: str) -> Workload:
    """A decode configuration or a layout variant, by name."""
    return WORKLOADS[name] if name in WORKLOADS else VARIANTS[name]


def _draw16(seed, layer, step, tiles, field, n):
    """uint16 draws [..., len(tiles), n] for one field; `step` may be an array
    of steps (leading axis)."""
    tiles = np.asarray(tiles, np.uint32)
    steps = np.atleast_1d(np.asarray(step, np.uint32))
    nchunk = (n + 7) // 8
    chunk = np.arange(nchunk, dtype=np.uint32)
    c0 = steps[:, None, None]
    c1 = tiles[None, :, None]
    c2 = np.full((1, 1, 1), field, np.uint32)
    c3 = chunk[None, None, :]
    w = philox4x32_10(c0, c1, c2, c3, np.uint32(seed & 0xFFFFFFFF), np.uint32(layer))
    words = np.stack(w, axis=-1)                      # [S, T, nchunk, 4]
    lo = (words & np.uint32(0xFFFF)).astype(np.uint16)
    hi = (words >> np.uint32(16)).astype(np.uint16)
    draws = np.stack([lo, hi], axis=-1).reshape(len(steps), len(tiles), nchunk * 8)[..., :n]
    return draws if np.ndim(step) else draws[0]


def _normal(seed, layer, step, tiles, field, n, sigma):
    z = normal_table().astype(np.float32)[_draw16(seed, layer, step, tiles, field, n)]
    if sigma == 1.0:
        return z
    return z * np.float32(sigma)


def _l2_normalised(z: np.ndarray) -> np.ndarray:
    """fp32: s = sum of squares in ascending order, then z / sqrt(s)."""
    s = np.zeros(z.shape[:-1], np.float32)
    for i in range(z.shape[-1]):
        s = s + z[..., i] * z[..., i]
    return z / np.sqrt(s)[..., None]


def _cast(x32: np.ndarray, dtype: int) -> np.ndarray:
    if dtype == F32:
        return np.ascontiguousarray(x32, np.float32)
    if dtype == BF16:
        return f32_to_bf16_bits(x32)
    raise ValueError(dtype)


@dataclasses.dataclass
class StepInputs:
    """Inputs of one decode step for a set of tiles, in their storage dtype
    (float32, or bf16 as uint16 bit patterns).  Shapes: q,k [T, d_k], v [T, d_v],
    gates [T, n_gate] (None for RetNet)."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    gates: np.ndarray | None

    def as_f32(self, wl: Workload):
        def f(x, dt):
            if x is None:
                return None
            return bf16_bits_to_f32(x) if dt == BF16 else np.asarray(x, np.float32)
        return (f(self.q, wl.qkv_dtype), f(self.k, wl.qkv_dtype), f(self.v, wl.qkv_dtype),
                f(self.gates, wl.gate_dtype))


def gen_step(wl: Workload, step, layer: int = 0, tiles=None) -> StepInputs:
    """Inputs of decode step ``step`` for the given tiles (default: all tiles
    of one layer, tile = b * heads + h).  With an array of steps every field
    gains a leading step axis (the values are those of the single steps)."""
    if tiles is None:
        tiles = np.arange(wl.tiles_per_layer)
    tiles = np.asarray(tiles)
    s = wl.seed
    if wl.kind == GDN:
        q = _l2_normalised(_normal(s, layer, step, tiles, FIELD_Q, wl.d_k, 1.0))
        k = _l2_normalised(_normal(s, layer, step, tiles, FIELD_K, wl.d_k, 1.0))
    else:
        q = _normal(s, layer, step, tiles, FIELD_Q, wl.d_k, wl.q_sigma)
        k = _normal(s, layer, step, tiles, FIELD_K, wl.d_k, wl.k_sigma)
    v = _normal(s, layer, step, tiles, FIELD_V, wl.d_v, wl.v_sigma)
    gates = None
    if wl.kind == MAMBA2:
        u = _draw16(s, layer, step, tiles, FIELD_ALPHA, 1)
        gates = gate_table("mamba2_alpha")[u].astype(np.float32)
    elif wl.kind == GLA:
        u = _draw16(s, layer, step, tiles, FIELD_ALPHA, wl.d_k)
        gates = gate_table("gla_alpha")[u].astype(np.float32)
    elif wl.kind == GDN:
        ua = _draw16(s, layer, step, tiles, FIELD_ALPHA, 1)
        ub = _draw16(s, layer, step, tiles, FIELD_BETA, 1)
        gates = np.concatenate([gate_table("gdn_alpha")[ua], gate_table("gdn_beta")[ub]],
                               axis=-1).astype(np.float32)
    if gates is not None:
        gates = _cast(gates, wl.gate_dtype)
    return StepInputs(_cast(q, wl.qkv_dtype), _cast(k, wl.qkv_dtype), _cast(v, wl.qkv_dtype),
                      gates)
