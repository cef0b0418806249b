"""Error accounting of a quantized recurrence by its per-step rounding errors
("Preserving Updates in Low-Bit Recurrent State Quantization", Figures 1 and 2;
Table 5 of its appendix).

TEST INFRASTRUCTURE ONLY, like the rest of this package: it steps an oracle
``State`` and never touches the CUDA library.

The pages give these quantities by their captions only.  Readings:

- R_t = S_hat_t - x_t, the error the requantization adds at step t: the
  dequantized new state minus the updated state before rounding (fp64; both
  are binary32 values, so the difference is exact).
- a_{tau:T} = product over s = tau+1 .. T of the decay of step s: gamma
  (RetNet), alpha_s (Mamba2, GDN: its scalar alpha_s; the delta rule's
  projection is not part of the weight), alpha_{s,i} per key row i (GLA).
- E_T = sum_tau a_{tau:T} R_tau, the accumulated error; its diagonal terms
  D_T = sum_tau ||a_{tau:T} R_tau||_F^2; the coherent gain g_T = ||E_T||_F^2 / D_T
  (1 when the per-step errors are mutually orthogonal).
- g^lost_T and g^moved_T: the same with R_tau kept only on the elements whose
  update is lost, or moved to another grid point, at step tau (the oracle's
  rounding classes).
- |b| / Delta_t: the update b = x - a of every element with b != 0 over the new
  scale of its group, pooled over steps and tiles; the lost fraction is the
  share of those elements whose update is lost.

For the rank-1 recurrences (RetNet, Mamba2, GLA) E_T equals S_hat_T - S_T, S_T
the unquantized recurrence on the same inputs, up to the binary32 rounding of
the updates; for Gated DeltaNet it does not (the delta rule feeds the error
back through k).
"""
from __future__ import annotations

import numpy as np

from . import GDN, GLA, LOST, MOVED, RETNET, State

MODES = ("all", "lost", "moved")


def accumulate(E, Drow, R, w):
    """One step of E_t = w * E_{t-1} + R_t and of the per-row diagonal terms
    Drow_t = w^2 * Drow_{t-1} + sum_j R_t^2.  E, R: [..., d_k, d_v] fp64;
    Drow: [..., d_k]; w: the step's decay per row, [..., d_k]."""
    E = w[..., None] * E + R
    Drow = w * w * Drow + np.sum(R * R, axis=-1)
    return E, Drow


def coherent_gain(E, Drow):
    """||E||_F^2 / D, pooled over every leading axis (tiles)."""
    d = float(np.sum(Drow))
    return float(np.sum(E * E)) / d if d > 0 else float("nan")


class ErrorAccount:
    """Steps an oracle state and keeps E_T, D_T (all / lost / moved) and the
    update-to-scale ratios."""

    def __init__(self, state: State, gamma: float | None = None):
        self.state = state
        cfg = state.cfg
        self.kind = cfg.c.kind
        self.gamma = np.float32(cfg.c.gamma if gamma is None else gamma)
        T, dk, dv = state.codes.shape
        self.E = {m: np.zeros((T, dk, dv)) for m in MODES}
        self.Drow = {m: np.zeros((T, dk)) for m in MODES}
        self.ratios = []
        self.n_updates = 0
        self.n_lost = 0
        self.steps = 0

    def _decay(self, alpha):
        T, dk = self.state.codes.shape[:2]
        if self.kind == RETNET:
            return np.full((T, dk), float(self.gamma))
        a = np.asarray(alpha, np.float32).reshape(T, -1).astype(np.float64)
        if self.kind == GLA:
            return a[:, :dk]
        return np.repeat(a[:, :1], dk, axis=1)

    def _scale_per_element(self):
        st = self.state
        cfg = st.cfg
        T, dk, dv = st.codes.shape
        g = cfg.c.group
        if g == 0:
            return np.broadcast_to(st.scales[:, :1, None].astype(np.float64), (T, dk, dv))
        ng = dv // g
        sc = st.scales.reshape(T, dk, ng).astype(np.float64)
        return np.repeat(sc, g, axis=2)

    def step(self, q, k, v, alpha=None, beta=None):
        out, a, x, cls = self.state.step_trace(q, k, v, alpha, beta)
        shat = self.state.dequant().astype(np.float64)
        R = shat - x.astype(np.float64)
        w = self._decay(alpha)
        for m in MODES:
            Rm = R if m == "all" else np.where(cls == (LOST if m == "lost" else MOVED), R, 0.0)
            self.E[m], self.Drow[m] = accumulate(self.E[m], self.Drow[m], Rm, w)
        b = x.astype(np.float64) - a.astype(np.float64)
        delta = self._scale_per_element()
        upd = (b != 0.0) & (delta > 0.0)
        self.ratios.append(np.abs(b[upd]) / delta[upd])
        self.n_updates += int(np.count_nonzero(b != 0.0))
        self.n_lost += int(np.count_nonzero(cls == LOST))
        self.steps += 1
        return out

    def gain(self, mode: str = "all") -> float:
        return coherent_gain(self.E[mode], self.Drow[mode])

    def ratio_quartiles(self):
        r = np.concatenate(self.ratios) if self.ratios else np.zeros(0)
        return tuple(float(v) for v in np.percentile(r, [25, 50, 75])) if r.size else (np.nan,) * 3

    def lost_fraction(self) -> float:
        return self.n_lost / self.n_updates if self.n_updates else float("nan")

    def report(self) -> dict:
        q25, q50, q75 = self.ratio_quartiles()
        gl, gm = self.gain("lost"), self.gain("moved")
        return {"steps": self.steps, "g": self.gain("all"), "g_lost": gl, "g_moved": gm,
                "g_lost_over_g_moved": gl / gm if gm else float("nan"),
                "b_over_delta_q25": q25, "b_over_delta_q50": q50, "b_over_delta_q75": q75,
                "lost_fraction": self.lost_fraction()}


__all__ = ["ErrorAccount", "accumulate", "coherent_gain", "GDN"]
