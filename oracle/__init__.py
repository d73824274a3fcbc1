"""CPU oracle for the Mamba-2 recurrent-state path (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package. It wraps ``m2_oracle.c`` (plain C,
IEEE double) with ctypes and converts storage-precision arrays to and from
float64. It never touches the CUDA path and shares nothing with it; inputs come
from ``m2synth`` (seeded generators, no method arithmetic).

Parity of every function here is pinned by ``tests/test_oracle_*.py`` against
closed forms, the quadratic (SSD dual) form, brute force on tiny inputs and
invariants; see the oracle's C header comment for the definitions.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libm2_oracle.so")

ROUND_F32 = 0
ROUND_BF16 = 1
ROUND_NONE = 2
ROUND_F16 = 3

_dp = ctypes.POINTER(ctypes.c_double)


def build(out_path: str = _LIB_PATH, defines=(), force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    if (not force and not defines and os.path.exists(out_path)
            and os.path.getmtime(out_path) >= os.path.getmtime(_SRC)):
        return out_path
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", _SRC, "-o", out_path, "-lm"]
    cmd[1:1] = [f"-D{d}" for d in defines] + (["-Wno-unused-parameter"] if defines else [])
    subprocess.run(cmd, check=True)
    return out_path


class Oracle:
    """One loaded build of the oracle library."""

    def __init__(self, path: str = _LIB_PATH):
        if path == _LIB_PATH:
            build()
        self.lib = ctypes.CDLL(path)
        L = self.lib
        L.m2o_round_f32.restype = ctypes.c_double
        L.m2o_round_f32.argtypes = [ctypes.c_double]
        L.m2o_round_bf16.restype = ctypes.c_double
        L.m2o_round_bf16.argtypes = [ctypes.c_double]
        L.m2o_round_f16.restype = ctypes.c_double
        L.m2o_round_f16.argtypes = [ctypes.c_double]
        L.m2o_softplus.restype = ctypes.c_double
        L.m2o_softplus.argtypes = [ctypes.c_double]
        L.m2o_silu.restype = ctypes.c_double
        L.m2o_silu.argtypes = [ctypes.c_double]
        L.m2o_build_tag.restype = ctypes.c_char_p
        L.m2o_round_array.restype = None
        L.m2o_round_array.argtypes = [_dp, ctypes.c_int64, ctypes.c_int]
        L.m2o_conv1d.restype = None
        L.m2o_conv1d.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp,
                                 ctypes.c_int, _dp]
        L.m2o_ssm_step.restype = None
        L.m2o_ssm_step.argtypes = [ctypes.c_int] * 4 + [_dp, ctypes.c_int] + [_dp] * 7
        L.m2o_ssm_scan.restype = None
        L.m2o_ssm_scan.argtypes = [ctypes.c_int] * 5 + [_dp, ctypes.c_int] + [_dp] * 7
        L.m2o_group_rmsnorm.restype = None
        L.m2o_group_rmsnorm.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, _dp, _dp, _dp]

    @property
    def tag(self) -> str:
        return self.lib.m2o_build_tag().decode()

    # -------------------------------------------------------------- scalars
    def round_f32(self, x: float) -> float:
        return self.lib.m2o_round_f32(float(x))

    def round_bf16(self, x: float) -> float:
        return self.lib.m2o_round_bf16(float(x))

    def round_f16(self, x: float) -> float:
        return self.lib.m2o_round_f16(float(x))

    def round_array(self, x, mode: int) -> np.ndarray:
        """Rounded copy of x (float64) in the given mode."""
        out = np.array(x, dtype=np.float64, copy=True, order="C")
        self.lib.m2o_round_array(out.ctypes.data_as(_dp), out.size, int(mode))
        return out

    def softplus(self, x: float) -> float:
        return self.lib.m2o_softplus(float(x))

    def silu(self, x: float) -> float:
        return self.lib.m2o_silu(float(x))

    # --------------------------------------------------------------- arrays
    @staticmethod
    def _f64(a, shape=None) -> np.ndarray:
        a = np.ascontiguousarray(a, dtype=np.float64)
        if shape is not None:
            a = a.reshape(shape)
        return a

    @staticmethod
    def _p(a):
        return None if a is None else a.ctypes.data_as(_dp)

    def conv1d(self, conv_state: np.ndarray, x_raw: np.ndarray, w: np.ndarray, bias,
               activation: int = 1) -> np.ndarray:
        """Causal depthwise conv over T tokens of one sequence.

        conv_state [K-1, C] float64 is updated in place (rolled); x_raw [T, C];
        w [C, K]; bias [C] or None. Returns out [T, C] float64.
        """
        assert conv_state.dtype == np.float64 and conv_state.flags.c_contiguous
        K = w.shape[1]
        C = w.shape[0]
        x_raw = self._f64(x_raw).reshape(-1, C)
        T = x_raw.shape[0]
        assert conv_state.shape == (K - 1, C)
        w = self._f64(w)
        bias = None if bias is None else self._f64(bias)
        out = np.empty((T, C), dtype=np.float64)
        self.lib.m2o_conv1d(C, K, T, self._p(conv_state), self._p(x_raw), self._p(w),
                            self._p(bias), int(activation), self._p(out))
        return out

    def ssm_step(self, state: np.ndarray, round_mode: int, xbc_post, dt_raw, dt_bias, A_log, D,
                 z, G: int) -> np.ndarray:
        """One decode step of one sequence; state [H, P, N] float64 updated in place."""
        assert state.dtype == np.float64 and state.flags.c_contiguous
        H, P, N = state.shape
        xbc_post = self._f64(xbc_post)
        assert xbc_post.size == H * P + 2 * G * N
        y = np.empty(H * P, dtype=np.float64)
        zz = None if z is None else self._f64(z)
        self.lib.m2o_ssm_step(H, P, N, G, self._p(state), int(round_mode), self._p(xbc_post),
                              self._p(self._f64(dt_raw)), self._p(self._f64(dt_bias)),
                              self._p(self._f64(A_log)), self._p(self._f64(D)), self._p(zz),
                              self._p(y))
        return y

    def ssm_scan(self, state: np.ndarray, round_mode: int, xbc_post, dt_raw, dt_bias, A_log, D,
                 z, G: int) -> np.ndarray:
        """T tokens of one sequence (state in double, rounded once). Returns y [T, H*P]."""
        assert state.dtype == np.float64 and state.flags.c_contiguous
        H, P, N = state.shape
        cd = H * P + 2 * G * N
        xbc_post = self._f64(xbc_post).reshape(-1, cd)
        T = xbc_post.shape[0]
        dt_raw = self._f64(dt_raw).reshape(T, H)
        zz = None if z is None else self._f64(z).reshape(T, H * P)
        y = np.empty((T, H * P), dtype=np.float64)
        self.lib.m2o_ssm_scan(H, P, N, G, T, self._p(state), int(round_mode), self._p(xbc_post),
                              self._p(dt_raw), self._p(self._f64(dt_bias)),
                              self._p(self._f64(A_log)), self._p(self._f64(D)), self._p(zz),
                              self._p(y))
        return y

    def group_rmsnorm(self, v, G: int, eps: float, w) -> np.ndarray:
        """Gated RMSNorm of one row: v [H*P] is the gated y; groups of H*P/G
        consecutive channels; w [H*P] the norm weight. Returns out [H*P]."""
        v = self._f64(v).reshape(-1)
        w = self._f64(w).reshape(-1)
        out = np.empty_like(v)
        self.lib.m2o_group_rmsnorm(int(v.size), int(G), float(eps), self._p(v), self._p(w), self._p(out))
        return out


_DEFAULT: Oracle | None = None


def default() -> Oracle:
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT


def round_mode_for(dtype: int) -> int:
    """Storage dtype code (0 = fp32, 1 = bf16) -> oracle rounding mode."""
    return ROUND_F32 if dtype == 0 else ROUND_BF16


def decode_rows(orc: Oracle, H: int, P: int, N: int, G: int, round_mode: int,
                ssm_rows: list, conv_rows: list, xbc_raw: np.ndarray, dt_raw: np.ndarray,
                z, conv_w, conv_b, dt_bias, A_log, D, activation: int = 1,
                post_conv_round=None, threads: int | None = None) -> np.ndarray:
    """One fused decode step (conv update, then state update) for several rows.

    ssm_rows[i] [H,P,N] and conv_rows[i] [K-1,conv_dim] are float64 arrays
    updated in place. xbc_raw [R, conv_dim], dt_raw [R, H], z [R, H*P] or None.
    post_conv_round: None, or a rounding mode applied to the conv output before
    the state update (used when the conv output is stored in bf16/fp32 between
    two separate operations). Rows run concurrently on ``threads`` threads (the
    C calls release the GIL). Returns y [R, H*P] float64.
    """
    R = len(ssm_rows)
    y = np.empty((R, H * P), dtype=np.float64)

    def one(i: int) -> None:
        xp = orc.conv1d(conv_rows[i], xbc_raw[i:i + 1], conv_w, conv_b, activation)[0]
        if post_conv_round is not None:
            xp = orc.round_array(xp, post_conv_round)
        y[i] = orc.ssm_step(ssm_rows[i], round_mode, xp, dt_raw[i], dt_bias, A_log, D,
                            None if z is None else z[i], G)

    _run(one, R, threads)
    return y


def _run(fn, n: int, threads: int | None) -> None:
    threads = threads or min(n, os.cpu_count() or 1)
    if threads <= 1 or n <= 1:
        for i in range(n):
            fn(i)
        return
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fn, range(n)))
