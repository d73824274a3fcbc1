"""Seeded synthetic inputs for the Mamba-2 recurrent-state workloads.

This module is shared by the tests, the benchmark and the smoke check. It holds
none of the method's arithmetic: it only turns (seed, tensor id, step, element
index) into numbers with the distributions the workloads call for, so that the
oracle and the CUDA path can be fed identical bits.

Generator definition (the device twin in ``fill.cu`` implements the same one):

* ``word(key, i)`` is output ``i`` (0-based) of the SplitMix64 sequence seeded
  with ``key``: ``mix(key + (i + 1) * 0x9E3779B97F4A7C15)`` with the SplitMix64
  finaliser ``mix`` (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014).
* ``normal`` is an Irwin-Hall sum of twelve 32-bit uniforms: element ``i`` takes
  words ``6i .. 6i+5``, adds their high and low 32-bit halves (an exact integer
  below 2**36), subtracts ``6 * 2**32`` and divides by ``2**32``. Every step is
  exact in float64, so host and device agree bit for bit. The result has mean 0,
  variance 1 and support [-6, 6].
* ``mean + std * n`` is evaluated in float64 with one rounding per operation
  (no fused multiply-add), then rounded to float32 (round to nearest even) and,
  for bfloat16 storage, from float32 to bfloat16 (round to nearest even).
* ``uniform(a, b)`` uses the top 53 bits of a word: ``a + (b - a) * u``.

Small per-head parameters that need ``log``/``expm1`` (A_log, dt_bias) are only
ever drawn on the host and copied to the device, so no transcendental function
has to agree between the two sides.
"""

from __future__ import annotations

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK = (1 << 64) - 1

F32 = 0
BF16 = 1
F16 = 2  # IEEE binary16 (only as a post-conv buffer; never drawn by the generator)

# Tensor ids mixed into the per-tensor stream key.
T_SSM = 1
T_CONV = 2
T_CONV_W = 3
T_CONV_B = 4
T_A_LOG = 5
T_DT_BIAS = 6
T_D = 7
T_SLOTS = 8
T_NORM_W = 9
T_XBC = 10
T_Z = 11
T_DT = 12


def mix64(z: int) -> int:
    """SplitMix64 finaliser on a Python int (mod 2**64)."""
    z &= _MASK
    z = ((z ^ (z >> 30)) * _M1) & _MASK
    z = ((z ^ (z >> 27)) * _M2) & _MASK
    return z ^ (z >> 31)


def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= np.uint64(_M1)
    z ^= z >> np.uint64(27)
    z *= np.uint64(_M2)
    z ^= z >> np.uint64(31)
    return z


def config_seed(config: int, layer: int = 0) -> int:
    """Base seed of one workload layer: 0x4D320000 + 1000*config + 10*layer."""
    return 0x4D320000 + 1000 * config + 10 * layer


def stream_key(seed: int, tensor_id: int, step: int = 0) -> int:
    """Key of one tensor's stream; independent of every other (seed, id, step)."""
    k = mix64(seed + tensor_id * GAMMA)
    return mix64(k + (step + 1) * 0xD1B54A32D192ED03)


def words(key: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of the SplitMix64 sequence seeded with key."""
    start, count = int(start), int(count)  # Python ints: no fixed-width overflow
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = np.uint64(key) + i * np.uint64(GAMMA)
        return _mix64_np(z)


def normal(key: int, start: int, count: int, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """Elements start .. start+count-1 of a seeded ~N(mean, std) stream, float64."""
    w = words(key, 6 * start, 6 * count).reshape(count, 6)
    s = ((w >> np.uint64(32)) + (w & np.uint64(0xFFFFFFFF))).sum(axis=1, dtype=np.uint64)
    n = (s.astype(np.float64) - 6.0 * 4294967296.0) / 4294967296.0
    # one rounding per operation, matching the device twin (no FMA)
    return np.float64(mean) + np.float64(std) * n


def uniform(key: int, start: int, count: int, a: float, b: float) -> np.ndarray:
    """Elements of a seeded U[a, b) stream, float64."""
    u = (words(key, start, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return np.float64(a) + (np.float64(b) - np.float64(a)) * u


def permutation(key: int, n: int) -> np.ndarray:
    """Seeded Fisher-Yates permutation of 0..n-1 (int64)."""
    w = words(key, 0, max(n, 1))
    perm = np.arange(n, dtype=np.int64)
    for i in range(n - 1, 0, -1):
        j = int(w[n - 1 - i] % np.uint64(i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return perm


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even, finite inputs."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact)."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def to_storage(x: np.ndarray, dtype: int) -> np.ndarray:
    """float64 -> storage array: float32, or bfloat16 bits as uint16 (via float32)."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    if dtype == F32:
        return x32
    if dtype == BF16:
        return f32_to_bf16_bits(x32)
    raise ValueError(f"unknown storage dtype {dtype}")


def storage_to_f64(a: np.ndarray, dtype: int) -> np.ndarray:
    """Storage array -> float64 (exact)."""
    if dtype == F32:
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == BF16:
        return bf16_bits_to_f64(a)
    if dtype == F16:
        return np.asarray(a, dtype=np.float16).astype(np.float64)
    raise ValueError(f"unknown storage dtype {dtype}")


def normal_storage(key: int, start: int, count: int, mean: float, std: float, dtype: int) -> np.ndarray:
    return to_storage(normal(key, start, count, mean, std), dtype)


def np_storage_dtype(dtype: int):
    return np.float32 if dtype == F32 else np.uint16
