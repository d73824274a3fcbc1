"""The synthetic workloads: shapes, dtypes and the recipe for every input tensor.

Five workloads, all synthetic (no trained weights exist for this path):

0. ``small_fp32``: one Mamba-2 mixer on a CPU-checkable size. H=8, P=64, N=128,
   G=1, K=4, conv_dim=768, fp32 state and activations, batch 4 in an 8-slot
   cache, 16 consecutive decode steps.
1. ``nemotron_h_layer``: the Nemotron-H-8B mixer shape (H=128, P=64, N=128,
   G=8, K=4, conv_dim=10240), bf16 state (2 MiB per sequence) and activations,
   batch 64 over a 256-slot cache, one decode step.
2. ``nemotron_h_stack48``: the previous mixer times 48 layers (independent
   weights per layer), 384 sequences in a 384-slot cache, slots permuted per
   layer, one decode token.
3. ``fp32_state_23l``: H=64, P=64, N=128, G=8, K=4, fp32 state (2 MiB per layer
   per sequence), bf16 activations, 23 layers, batch 128 in a 512-slot cache, 64
   decode steps carried in place.
4. ``prefill_then_decode``: Nemotron-H layer shape, 8 sequences of T=2048
   tokens, chunk 128, zero initial state, then 32 decode steps.

Distributions (std is the second parameter of N(.,.)): raw x/B/C (the xBC row),
z and dt_raw ~ N(0,1); D ~ N(0,1); conv weight ~ N(0,0.5), conv bias
~ N(0,0.1); A_log = log(U[1,16]); dt_bias = log(expm1(U[1e-3,0.1])); initial
SSM state ~ N(0,0.1) in the state dtype; initial conv cache ~ N(0,1) in the
activation dtype (every slot, used or not). dt_raw and the conv weight and bias
are stored in the activation dtype; A_log, dt_bias and D in fp32.
"""

from __future__ import annotations

import dataclasses
import numpy as np

from . import (BF16, F32, T_A_LOG, T_CONV, T_CONV_B, T_CONV_W, T_D, T_DT, T_DT_BIAS, T_NORM_W,
               T_SLOTS, T_SSM, T_XBC, T_Z, config_seed, normal, normal_storage, permutation,
               stream_key, to_storage, uniform)


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    H: int
    P: int
    N: int
    G: int
    K: int
    state_dtype: int
    act_dtype: int
    num_slots: int
    batch: int
    layers: int = 1
    steps: int = 1
    seqlen: int = 1          # prefill tokens per sequence (workload 4)
    chunk: int = 128
    decode_after: int = 0    # decode steps after the prefill (workload 4)

    @property
    def conv_dim(self) -> int:
        return self.H * self.P + 2 * self.G * self.N

    @property
    def hpg(self) -> int:
        return self.H // self.G

    def seed(self, layer: int = 0) -> int:
        return config_seed(self.index, layer)

    def shape_dict(self) -> dict:
        return dict(H=self.H, P=self.P, N=self.N, G=self.G, K=self.K)

    def state_bytes_per_slot(self) -> int:
        return self.H * self.P * self.N * (4 if self.state_dtype == F32 else 2)


WORKLOADS = [
    Workload(0, "small_fp32", 8, 64, 128, 1, 4, F32, F32, 8, 4, steps=16),
    Workload(1, "nemotron_h_layer", 128, 64, 128, 8, 4, BF16, BF16, 256, 64),
    Workload(2, "nemotron_h_stack48", 128, 64, 128, 8, 4, BF16, BF16, 384, 384, layers=48),
    Workload(3, "fp32_state_23l", 64, 64, 128, 8, 4, F32, BF16, 512, 128, layers=23, steps=64),
    Workload(4, "prefill_then_decode", 128, 64, 128, 8, 4, BF16, BF16, 8, 8, seqlen=2048,
             chunk=128, decode_after=32),
]


@dataclasses.dataclass
class LayerParams:
    """Per-layer mixer parameters in storage form (numpy)."""
    conv_w: np.ndarray   # [conv_dim, K] act storage
    conv_b: np.ndarray   # [conv_dim] act storage
    A_log: np.ndarray    # [H] float32
    dt_bias: np.ndarray  # [H] float32
    D: np.ndarray        # [H] float32


def layer_params(w: Workload, layer: int = 0) -> LayerParams:
    s = w.seed(layer)
    cd = w.conv_dim
    conv_w = normal_storage(stream_key(s, T_CONV_W), 0, cd * w.K, 0.0, 0.5, w.act_dtype).reshape(cd, w.K)
    conv_b = normal_storage(stream_key(s, T_CONV_B), 0, cd, 0.0, 0.1, w.act_dtype)
    A_log = np.log(uniform(stream_key(s, T_A_LOG), 0, w.H, 1.0, 16.0)).astype(np.float32)
    u = uniform(stream_key(s, T_DT_BIAS), 0, w.H, 1e-3, 0.1)
    dt_bias = np.log(np.expm1(u)).astype(np.float32)
    D = normal(stream_key(s, T_D), 0, w.H, 0.0, 1.0).astype(np.float32)
    return LayerParams(conv_w, conv_b, A_log, dt_bias, D)


def norm_weight(w: Workload, layer: int = 0) -> np.ndarray:
    """Gated RMSNorm weight [H*P] in act storage form, ~N(1, 0.1)."""
    return normal_storage(stream_key(w.seed(layer), T_NORM_W), 0, w.H * w.P, 1.0, 0.1, w.act_dtype)


def slot_indices(w: Workload, layer: int = 0) -> np.ndarray:
    """Batch row -> cache slot (int32), a seeded permutation prefix."""
    perm = permutation(stream_key(w.seed(layer), T_SLOTS), w.num_slots)
    return perm[: w.batch].astype(np.int32)


def slot_sets(w: Workload, layer: int = 0) -> list[np.ndarray]:
    """The same permutation cut into num_slots // batch disjoint batches of
    slots (set 0 is ``slot_indices``): a benchmark that rotates through them
    touches each slot's state once per rotation."""
    perm = permutation(stream_key(w.seed(layer), T_SLOTS), w.num_slots)
    return [perm[i * w.batch:(i + 1) * w.batch].astype(np.int32) for i in range(w.num_slots // w.batch)]


# --- initial caches: element index = flat index in the full cache tensor ----------

def ssm_key(w: Workload, layer: int = 0) -> int:
    return stream_key(w.seed(layer), T_SSM)


def conv_key(w: Workload, layer: int = 0) -> int:
    return stream_key(w.seed(layer), T_CONV)


SSM_STD = 0.1
CONV_STD = 1.0


def ssm_slot(w: Workload, slot: int, layer: int = 0) -> np.ndarray:
    """Initial SSM state of one slot, storage form [H, P, N]."""
    slot = int(slot)  # a numpy int32 slot would overflow the element offset
    n = w.H * w.P * w.N
    return normal_storage(ssm_key(w, layer), slot * n, n, 0.0, SSM_STD, w.state_dtype).reshape(w.H, w.P, w.N)


def conv_slot(w: Workload, slot: int, layer: int = 0) -> np.ndarray:
    """Initial conv cache of one slot, storage form [K-1, conv_dim]."""
    slot = int(slot)
    n = (w.K - 1) * w.conv_dim
    return normal_storage(conv_key(w, layer), slot * n, n, 0.0, CONV_STD, w.act_dtype).reshape(w.K - 1, w.conv_dim)


def ssm_cache(w: Workload, layer: int = 0) -> np.ndarray:
    n = w.num_slots * w.H * w.P * w.N
    return normal_storage(ssm_key(w, layer), 0, n, 0.0, SSM_STD, w.state_dtype).reshape(
        w.num_slots, w.H, w.P, w.N)


def conv_cache(w: Workload, layer: int = 0) -> np.ndarray:
    n = w.num_slots * (w.K - 1) * w.conv_dim
    return normal_storage(conv_key(w, layer), 0, n, 0.0, CONV_STD, w.act_dtype).reshape(
        w.num_slots, w.K - 1, w.conv_dim)


# --- per-step inputs: element index = row * dim + column --------------------------

def step_key(w: Workload, tensor_id: int, step: int, layer: int = 0) -> int:
    return stream_key(w.seed(layer), tensor_id, step)


def step_rows(w: Workload, tensor_id: int, step: int, rows, layer: int = 0) -> np.ndarray:
    """Rows of one per-step input (xBC raw, z or dt_raw) in act storage form.

    ``rows`` are batch rows (decode) or flattened (sequence, token) rows
    (prefill, step 0 of workload 4). Each row is regenerated independently.
    """
    dim = {T_XBC: w.conv_dim, T_Z: w.H * w.P, T_DT: w.H}[tensor_id]
    key = step_key(w, tensor_id, step, layer)
    rows = np.atleast_1d(np.asarray(rows, dtype=np.int64))
    out = np.empty((len(rows), dim), dtype=np.float32 if w.act_dtype == F32 else np.uint16)
    # contiguous runs are generated in one call
    i = 0
    while i < len(rows):
        j = i
        while j + 1 < len(rows) and rows[j + 1] == rows[j] + 1:
            j += 1
        out[i:j + 1] = normal_storage(key, int(rows[i]) * dim, (j - i + 1) * dim, 0.0, 1.0,
                                      w.act_dtype).reshape(j - i + 1, dim)
        i = j + 1
    return out


def step_inputs(w: Workload, step: int, layer: int = 0, rows=None) -> dict:
    """xBC (raw), z and dt_raw for the given rows (default: the whole batch)."""
    if rows is None:
        rows = np.arange(w.batch)
    return {
        "xBC": step_rows(w, T_XBC, step, rows, layer),
        "z": step_rows(w, T_Z, step, rows, layer),
        "dt": step_rows(w, T_DT, step, rows, layer),
    }


def bytes_per_unit(w: Workload) -> int:
    """Algorithmic HBM bytes of one (sequence, layer, decode step) unit.

    State read + write, conv cache read + write of K-1 rows, xBC row in, z row
    in, dt row in, y row out, one slot index.
    """
    s_state = 4 if w.state_dtype == F32 else 2
    s_act = 4 if w.act_dtype == F32 else 2
    hp = w.H * w.P
    return (2 * hp * w.N * s_state + 2 * (w.K - 1) * w.conv_dim * s_act + w.conv_dim * s_act
            + hp * s_act + w.H * s_act + hp * s_act + 4)


def param_bytes_per_launch(w: Workload) -> int:
    """Parameters read once per launch: conv weight and bias, A_log, dt_bias, D."""
    s_act = 4 if w.act_dtype == F32 else 2
    return w.conv_dim * (w.K + 1) * s_act + 3 * w.H * 4
