"""Shared helpers of the parity tests: the error metric and oracle runners.

Error metric for floats, per tensor: err = max_i |a_i - r_i| / max(|r_i|,
rms(r)), where r is the oracle. The rms floor keeps near-zero cancellations
from producing spurious relative errors. Bounds: 1e-5 for fp32 state and y,
2e-2 for bf16 state and y. Slots and conv caches compare bit for bit.
"""

from __future__ import annotations

import numpy as np

import m2synth as S
import oracle as O
from m2synth import workloads as W

TOL = {S.F32: 1e-5, S.BF16: 2e-2}


def rel_err(a, r) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    r = np.asarray(r, dtype=np.float64).ravel()
    if r.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(r * r)))
    denom = np.maximum(np.abs(r), rms if rms > 0 else 1.0)
    return float(np.max(np.abs(a - r) / denom))


def assert_close(a, r, dtype: int, what: str, tol: float | None = None) -> float:
    tol = TOL[dtype] if tol is None else tol
    e = rel_err(a, r)
    assert e <= tol, f"{what}: err {e:.3e} > {tol:.1e}"
    return e


def f64(storage: np.ndarray, dtype: int) -> np.ndarray:
    return S.storage_to_f64(storage, dtype)


class OracleLayer:
    """Oracle view of one workload layer: params as float64 and per-row state.

    Rows are regenerated from the seeded streams on demand (slot states, conv
    caches, per-step inputs), so any sample of a large workload can be checked
    without materialising the whole cache on the host.
    """

    def __init__(self, w: W.Workload, layer: int = 0, orc: O.Oracle | None = None):
        self.w, self.layer = w, layer
        self.orc = orc or O.default()
        p = W.layer_params(w, layer)
        self.conv_w = f64(p.conv_w, w.act_dtype)
        self.conv_b = f64(p.conv_b, w.act_dtype)
        self.A_log = p.A_log.astype(np.float64)
        self.dt_bias = p.dt_bias.astype(np.float64)
        self.D = p.D.astype(np.float64)
        self.slots = W.slot_indices(w, layer)

    def initial_ssm(self, slot: int) -> np.ndarray:
        return np.ascontiguousarray(f64(W.ssm_slot(self.w, slot, self.layer), self.w.state_dtype))

    def initial_conv(self, slot: int) -> np.ndarray:
        return np.ascontiguousarray(f64(W.conv_slot(self.w, slot, self.layer), self.w.act_dtype))

    def inputs(self, step: int, rows) -> dict:
        d = W.step_inputs(self.w, step, self.layer, rows=rows)
        return {k: f64(v, self.w.act_dtype) for k, v in d.items()}

    def decode(self, ssm_rows, conv_rows, inp: dict, with_z: bool = True, activation: int = 1,
               post_conv_round=None, threads=None) -> np.ndarray:
        w = self.w
        return O.decode_rows(self.orc, w.H, w.P, w.N, w.G, O.round_mode_for(w.state_dtype),
                             ssm_rows, conv_rows, inp["xBC"], inp["dt"],
                             inp["z"] if with_z else None, self.conv_w, self.conv_b,
                             self.dt_bias, self.A_log, self.D, activation=activation,
                             post_conv_round=post_conv_round, threads=threads)
