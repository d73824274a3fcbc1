"""Workload tensors on a CUDA device, from the seeded generators.

Small per-layer parameters come from the host generator (exact same bits the
oracle sees); caches and per-step inputs are filled on the device by the
twin generator (bit-identical for the same key and element index). No method
arithmetic lives here.
"""

from __future__ import annotations

import numpy as np
import torch

from . import BF16, F32, T_DT, T_XBC, T_Z
from . import device as dev
from . import workloads as W


def to_torch(a: np.ndarray, dtype: int, device="cuda") -> torch.Tensor:
    """Storage array (float32, or uint16 bf16 bits) -> torch tensor of that dtype."""
    if dtype == F32:
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def to_storage_np(t: torch.Tensor) -> np.ndarray:
    """torch float32 / bfloat16 tensor -> storage numpy array (float32 / uint16 bits)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float16:
        return t.numpy()
    raise TypeError(t.dtype)


def torch_dtype(code: int) -> torch.dtype:
    return torch.float32 if code == F32 else torch.bfloat16


def layer_tensors(w: W.Workload, layer: int = 0, device="cuda") -> dict:
    p = W.layer_params(w, layer)
    return {
        "conv_w": to_torch(p.conv_w, w.act_dtype, device),
        "conv_b": to_torch(p.conv_b, w.act_dtype, device),
        "A_log": torch.from_numpy(p.A_log).to(device),
        "dt_bias": torch.from_numpy(p.dt_bias).to(device),
        "D": torch.from_numpy(p.D).to(device),
        "slots": torch.from_numpy(W.slot_indices(w, layer)).to(device),
    }


def fill_caches(w: W.Workload, ssm: torch.Tensor, conv: torch.Tensor, layer: int = 0) -> None:
    """Initial caches of a layer: SSM ~ N(0, 0.1), conv ~ N(0, 1), all slots."""
    dev.fill_normal(ssm, W.ssm_key(w, layer), 0, 0.0, W.SSM_STD)
    dev.fill_normal(conv, W.conv_key(w, layer), 0, 0.0, W.CONV_STD)


def step_tensors(w: W.Workload, step: int, layer: int = 0, device="cuda", rows: int | None = None,
                 out: dict | None = None) -> dict:
    """xBC (raw) [rows, conv_dim], z [rows, H*P], dt [rows, H] for one step.

    ``rows`` defaults to the batch (decode); for the prefill of workload 4 pass
    batch * seqlen (row = b * seqlen + t) and step 0.
    """
    rows = w.batch if rows is None else rows
    dt_ = torch_dtype(w.act_dtype)
    if out is None:
        out = {
            "xBC": torch.empty((rows, w.conv_dim), dtype=dt_, device=device),
            "z": torch.empty((rows, w.H * w.P), dtype=dt_, device=device),
            "dt": torch.empty((rows, w.H), dtype=dt_, device=device),
        }
    dev.fill_normal(out["xBC"], W.step_key(w, T_XBC, step, layer), 0, 0.0, 1.0)
    dev.fill_normal(out["z"], W.step_key(w, T_Z, step, layer), 0, 0.0, 1.0)
    dev.fill_normal(out["dt"], W.step_key(w, T_DT, step, layer), 0, 0.0, 1.0)
    return out


__all__ = ["to_torch", "to_storage_np", "torch_dtype", "layer_tensors", "fill_caches",
           "step_tensors", "BF16", "F32"]
