"""B200-native Mamba-2 recurrent-state kernels: thin Python binding of libm2.

Every step of the computation runs in ``libm2.so`` (hand-written sm_100a CUDA
behind the C ABI of ``include/m2.h``); this module only marshals torch tensors
into pointers, sizes and the current CUDA stream, and raises on a non-OK
status. There is no CPU fallback: without the built library, importing the
functions that compute raises immediately.

Operations (vllm.cpp issue #1311 "NemotronH runs the PREFILL mamba kernels at
decode", section "The divergence"; shapes from the Nemotron-H-8B-Base-8K
record):

* ``state_update``  -- one-token selective_state_update, optionally with the
  causal_conv1d_update tap fused into the same launch, in place at slots.
* ``conv1d_update`` -- causal_conv1d_update over seqlen >= 1 tokens.
* ``chunk_scan``    -- prefill scan landing on the same state as sequential
  updates.
* ``Cache``         -- the fixed-size, slot-indexed state cache.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libm2.so")

M2_F32 = 0
M2_BF16 = 1
M2_F16 = 2  # post-conv xBC buffer only

STATUS = {
    0: "ok",
    -1: "invalid argument",
    -2: "unsupported shape or dtype",
    -3: "CUDA error",
    -4: "out of device memory",
    -5: "slot index out of range",
    -6: "bounded wait timed out",
    -7: "operand outside the fp16 range of the tensor-core scan",
}
M2_OK = 0
M2_ERR_INVALID_ARG = -1
M2_ERR_UNSUPPORTED = -2
M2_ERR_CUDA = -3
M2_ERR_OOM = -4
M2_ERR_BAD_SLOT = -5
M2_ERR_TIMEOUT = -6
M2_ERR_RANGE = -7


class M2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status})")
        self.status = status


class m2_shape(ctypes.Structure):
    _fields_ = [("nheads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("d_state", ctypes.c_int32), ("ngroups", ctypes.c_int32),
                ("d_conv", ctypes.c_int32), ("state_dtype", ctypes.c_int32),
                ("act_dtype", ctypes.c_int32)]


class m2_cache(ctypes.Structure):
    _fields_ = [("ssm", ctypes.c_void_p), ("conv", ctypes.c_void_p),
                ("error", ctypes.c_void_p), ("num_slots", ctypes.c_int64),
                ("shape", m2_shape), ("owned", ctypes.c_int32), ("device", ctypes.c_int32)]


class m2_conv_params(ctypes.Structure):
    _fields_ = [("weight", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("activation", ctypes.c_int32)]


class m2_ssm_params(ctypes.Structure):
    _fields_ = [("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p), ("D", ctypes.c_void_p)]


class m2_norm_params(ctypes.Structure):
    _fields_ = [("weight", ctypes.c_void_p), ("eps", ctypes.c_float)]


class m2_decode_rows(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("xBC", ctypes.c_void_p), ("xBC_row_stride", ctypes.c_int64),
                ("dt", ctypes.c_void_p), ("dt_row_stride", ctypes.c_int64), ("z", ctypes.c_void_p),
                ("z_row_stride", ctypes.c_int64), ("y", ctypes.c_void_p), ("y_row_stride", ctypes.c_int64),
                ("slot_idx", ctypes.c_void_p)]


class m2_prefill_rows(ctypes.Structure):
    _fields_ = [("nseq", ctypes.c_int32), ("cu_seqlens", ctypes.c_void_p), ("total_tokens", ctypes.c_int64),
                ("max_seqlen", ctypes.c_int32), ("xBC", ctypes.c_void_p), ("xBC_row_stride", ctypes.c_int64),
                ("xBC_post", ctypes.c_void_p), ("xBC_post_dtype", ctypes.c_int32),
                ("xBC_post_row_stride", ctypes.c_int64), ("dt", ctypes.c_void_p),
                ("dt_row_stride", ctypes.c_int64), ("z", ctypes.c_void_p), ("z_row_stride", ctypes.c_int64),
                ("y", ctypes.c_void_p), ("y_row_stride", ctypes.c_int64), ("slot_idx", ctypes.c_void_p),
                ("has_initial_state", ctypes.c_void_p)]


# exported symbols and their signatures (mirrors include/m2.h)
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
SIGNATURES = {
    "m2_conv_dim": (_I64, [ctypes.POINTER(m2_shape)]),
    "m2_shape_check": (_I32, [ctypes.POINTER(m2_shape)]),
    "m2_cache_bytes": (_I32, [ctypes.POINTER(m2_shape), _I64, ctypes.POINTER(_I64),
                              ctypes.POINTER(_I64)]),
    "m2_cache_alloc": (_I32, [ctypes.POINTER(m2_shape), _I64, _P, ctypes.POINTER(m2_cache)]),
    "m2_cache_wrap": (_I32, [ctypes.POINTER(m2_shape), _I64, _P, _P, _P,
                             ctypes.POINTER(m2_cache)]),
    "m2_cache_free": (_I32, [ctypes.POINTER(m2_cache), _P]),
    "m2_cache_zero_slots": (_I32, [ctypes.POINTER(m2_cache), _I32, _P, _P]),
    "m2_conv1d_update": (_I32, [ctypes.POINTER(m2_cache), ctypes.POINTER(m2_conv_params), _I32,
                                _I32, _P, _I64, _P, _I32, _I64, _P, _P]),
    "m2_state_update": (_I32, [ctypes.POINTER(m2_cache), ctypes.POINTER(m2_ssm_params),
                               ctypes.POINTER(m2_conv_params), _I32, _P, _I32, _I64, _P, _I64,
                               _P, _I64, _P, _I64, _P, _P]),
    "m2_state_update_norm": (_I32, [ctypes.POINTER(m2_cache), ctypes.POINTER(m2_ssm_params),
                                    ctypes.POINTER(m2_conv_params), ctypes.POINTER(m2_norm_params), _I32,
                                    _P, _I64, _P, _I64, _P, _I64, _P, _I64, _P, _P]),
    "m2_chunk_scan": (_I32, [ctypes.POINTER(m2_cache), ctypes.POINTER(m2_ssm_params), _I32, _I32,
                             _I32, _P, _I32, _I64, _P, _I64, _P, _I64, _P, _I64, _P, _P, _P]),
    "m2_chunk_scan_varlen": (_I32, [ctypes.POINTER(m2_cache), ctypes.POINTER(m2_ssm_params), _I32, _P,
                                    _I64, _I32, _I32, _P, _I32, _I64, _P, _I64, _P, _I64, _P, _I64,
                                    _P, _P, _P]),
    "m2_chunk_scan_varlen_static": (_I32, [ctypes.POINTER(m2_cache), ctypes.POINTER(m2_ssm_params), _I32,
                                           _P, _I64, _I32, _I32, _P, _I32, _I64, _P, _I64, _P, _I64,
                                           _P, _I64, _P, _P, _P]),
    "m2_conv1d_update_varlen": (_I32, [ctypes.POINTER(m2_cache), ctypes.POINTER(m2_conv_params), _I32, _P,
                                       _I64, _I32, _P, _I64, _P, _I32, _I64, _P, _P]),
    "m2_mixed_step": (_I32, [ctypes.POINTER(m2_cache), ctypes.POINTER(m2_ssm_params),
                             ctypes.POINTER(m2_conv_params), ctypes.POINTER(m2_decode_rows),
                             ctypes.POINTER(m2_prefill_rows), _P]),
    "m2_state_update_multi": (_I32, [ctypes.POINTER(m2_cache), ctypes.POINTER(m2_ssm_params),
                                     ctypes.POINTER(m2_conv_params), _I32, _I32, _P, _I64, _P, _I64, _P, _I64,
                                     _P, _I64, _P, _P, _P]),
    "m2_host_stage_create": (_I32, [_I32, _I64, _I64, ctypes.POINTER(_P)]),
    "m2_host_stage_destroy": (_I32, [_P]),
    "m2_state_update_host": (_I32, [_P, ctypes.POINTER(m2_cache), ctypes.POINTER(m2_ssm_params),
                                    ctypes.POINTER(m2_conv_params), _I32, _P, _I64, _I64, _I64, _I64, _I64,
                                    _I64, _P, _I64, _P, _P]),
    "m2_host_stage_join": (_I32, [_P, _P]),
    "m2_get_device_error": (_I32, [ctypes.POINTER(m2_cache), _P, ctypes.POINTER(_I32)]),
    "m2_status_string": (ctypes.c_char_p, [_I32]),
    "m2_version": (ctypes.c_char_p, []),
}

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded libm2 (raises if it has not been built: no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m mamba_recurrent_state_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != M2_OK:
        raise M2Error(status, what)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return M2_F32
    if t == torch.bfloat16:
        return M2_BF16
    if t == torch.float16:
        return M2_F16
    raise TypeError(f"unsupported dtype {t} (float32, bfloat16, or float16 for a post-conv buffer)")


def torch_dtype(code: int) -> torch.dtype:
    return torch.float32 if code == M2_F32 else torch.bfloat16


def _stream_ptr() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _row_stride(t: torch.Tensor) -> int:
    if t.stride(-1) != 1:
        raise ValueError("rows must be contiguous (unit stride in the last dimension)")
    return t.stride(-2) if t.dim() >= 2 else t.shape[-1]


@dataclasses.dataclass(frozen=True)
class Shape:
    H: int
    P: int
    N: int
    G: int
    K: int = 4
    state_dtype: int = M2_BF16
    act_dtype: int = M2_BF16

    @property
    def conv_dim(self) -> int:
        return self.H * self.P + 2 * self.G * self.N

    def c(self) -> m2_shape:
        return m2_shape(self.H, self.P, self.N, self.G, self.K, self.state_dtype, self.act_dtype)


def shape_check(shape: Shape) -> int:
    s = shape.c()
    return lib().m2_shape_check(ctypes.byref(s))


def cache_bytes(shape: Shape, num_slots: int) -> tuple[int, int]:
    s = shape.c()
    a, b = _I64(), _I64()
    _check(lib().m2_cache_bytes(ctypes.byref(s), num_slots, ctypes.byref(a), ctypes.byref(b)),
           "m2_cache_bytes")
    return a.value, b.value


class Cache:
    """A slot-indexed state cache of one mixer layer.

    ``ssm``  [num_slots, H, P, N] state dtype; ``conv`` [num_slots, K-1,
    conv_dim] activation dtype (last K-1 raw inputs, oldest row first);
    ``error`` a one-element int32 device word. The memory is owned by torch
    (this object wraps it with ``m2_cache_wrap``) unless created with
    ``native=True``, in which case ``m2_cache_alloc`` owns it.
    """

    def __init__(self, shape: Shape, num_slots: int, device="cuda", native: bool = False,
                 ssm: Optional[torch.Tensor] = None, conv: Optional[torch.Tensor] = None):
        self.shape = shape
        self.num_slots = num_slots
        self._c = m2_cache()
        s = shape.c()
        self.native = native
        if native:
            _check(lib().m2_cache_alloc(ctypes.byref(s), num_slots, _stream_ptr(),
                                        ctypes.byref(self._c)), "m2_cache_alloc")
            self.ssm = self.conv = self.error = None
            return
        dev = torch.device(device)
        if ssm is None:
            ssm = torch.zeros((num_slots, shape.H, shape.P, shape.N),
                              dtype=torch_dtype(shape.state_dtype), device=dev)
        if conv is None:
            conv = torch.zeros((num_slots, shape.K - 1, shape.conv_dim),
                               dtype=torch_dtype(shape.act_dtype), device=dev)
        assert ssm.is_contiguous() and conv.is_contiguous()
        self.ssm, self.conv = ssm, conv
        self.error = torch.zeros(1, dtype=torch.int32, device=ssm.device)
        _check(lib().m2_cache_wrap(ctypes.byref(s), num_slots, ssm.data_ptr(), conv.data_ptr(),
                                   self.error.data_ptr(), ctypes.byref(self._c)), "m2_cache_wrap")

    @property
    def c(self) -> m2_cache:
        return self._c

    def zero_slots(self, slot_idx: torch.Tensor) -> None:
        _check(lib().m2_cache_zero_slots(ctypes.byref(self._c), slot_idx.numel(),
                                         slot_idx.data_ptr(), _stream_ptr()),
               "m2_cache_zero_slots")

    def device_error(self) -> int:
        """Reads and clears the device error word (synchronises the stream)."""
        code = _I32()
        _check(lib().m2_get_device_error(ctypes.byref(self._c), _stream_ptr(), ctypes.byref(code)),
               "m2_get_device_error")
        return code.value

    def free(self) -> None:
        if self.native and self._c.ssm:
            _check(lib().m2_cache_free(ctypes.byref(self._c), _stream_ptr()), "m2_cache_free")

    def __del__(self):  # native caches only
        try:
            if self.native and self._c.ssm:
                lib().m2_cache_free(ctypes.byref(self._c), None)
        except Exception:
            pass


@dataclasses.dataclass
class SSMParams:
    """Per-head fp32 parameters [H]: A = -exp(A_log), dt_bias, D."""
    A_log: torch.Tensor
    dt_bias: torch.Tensor
    D: torch.Tensor

    def c(self) -> m2_ssm_params:
        for t in (self.A_log, self.dt_bias, self.D):
            if t.dtype != torch.float32 or not t.is_contiguous():
                raise TypeError("SSM parameters must be contiguous float32")
        return m2_ssm_params(self.A_log.data_ptr(), self.dt_bias.data_ptr(), self.D.data_ptr())


@dataclasses.dataclass
class ConvParams:
    """Depthwise conv: weight [conv_dim, K], bias [conv_dim] or None, SiLU on/off."""
    weight: torch.Tensor
    bias: Optional[torch.Tensor] = None
    activation: int = 1

    def c(self) -> m2_conv_params:
        if not self.weight.is_contiguous():
            raise ValueError("conv weight must be contiguous [conv_dim, K]")
        return m2_conv_params(self.weight.data_ptr(), _ptr(self.bias), self.activation)


@dataclasses.dataclass
class NormParams:
    """Gated RMSNorm after the decode step: weight [H*P] (activation dtype), eps."""
    weight: torch.Tensor
    eps: float = 1e-5

    def c(self) -> m2_norm_params:
        if not self.weight.is_contiguous():
            raise ValueError("norm weight must be contiguous [H*P]")
        return m2_norm_params(self.weight.data_ptr(), float(self.eps))


def state_update(cache: Cache, ssm: SSMParams, xBC: torch.Tensor, dt: torch.Tensor,
                 slot_idx: torch.Tensor, z: Optional[torch.Tensor] = None,
                 conv: Optional[ConvParams] = None, y: Optional[torch.Tensor] = None,
                 stream: Optional[int] = None, norm: Optional[NormParams] = None) -> torch.Tensor:
    """One decode step for ``xBC.shape[0]`` rows, in place on ``cache``.

    With ``conv`` given, ``xBC`` is the raw row and the conv tap is fused;
    otherwise ``xBC`` is post-conv (float32 or bfloat16). With ``norm`` given
    (requires ``conv``) the gated RMSNorm is fused too (m2_state_update_norm).
    Returns y [batch, H*P] in the activation dtype.
    """
    sh = cache.shape
    batch = xBC.shape[0]
    if y is None:
        y = torch.empty((batch, sh.H * sh.P), dtype=torch_dtype(sh.act_dtype), device=xBC.device)
    sp = ssm.c()
    cp = conv.c() if conv is not None else None
    if norm is not None:
        if cp is None:
            raise ValueError("the fused gated RMSNorm needs the fused conv (conv=...)")
        npar = norm.c()
        st = lib().m2_state_update_norm(
            ctypes.byref(cache.c), ctypes.byref(sp), ctypes.byref(cp), ctypes.byref(npar), batch,
            xBC.data_ptr(), _row_stride(xBC), dt.data_ptr(), _row_stride(dt), _ptr(z),
            _row_stride(z) if z is not None else 0, y.data_ptr(), _row_stride(y), slot_idx.data_ptr(),
            _stream_ptr() if stream is None else stream)
        _check(st, "m2_state_update_norm")
        return y
    st = lib().m2_state_update(
        ctypes.byref(cache.c), ctypes.byref(sp), ctypes.byref(cp) if cp is not None else None,
        batch, xBC.data_ptr(), _dtype_code(xBC.dtype), _row_stride(xBC), dt.data_ptr(),
        _row_stride(dt), _ptr(z), _row_stride(z) if z is not None else 0, y.data_ptr(),
        _row_stride(y), slot_idx.data_ptr(), _stream_ptr() if stream is None else stream)
    _check(st, "m2_state_update")
    return y


class HostStage:
    """Device staging ring for decode steps whose rows live in pinned host
    memory (m2_host_stage_create): ``depth`` buffers of ``in_bytes`` and
    ``y_bytes``, two copy streams and their events."""

    def __init__(self, depth: int, in_bytes: int, y_bytes: int):
        ptr = ctypes.c_void_p()
        _check(lib().m2_host_stage_create(depth, in_bytes, y_bytes, ctypes.byref(ptr)), "m2_host_stage_create")
        self.ptr = ptr
        self.in_bytes, self.y_bytes = in_bytes, y_bytes

    def join(self, stream: Optional[int] = None) -> None:
        """``stream`` waits for every copy the stage has issued."""
        _check(lib().m2_host_stage_join(self.ptr, _stream_ptr() if stream is None else stream), "m2_host_stage_join")

    def close(self) -> None:
        if self.ptr is not None and self.ptr.value:
            _check(lib().m2_host_stage_destroy(self.ptr), "m2_host_stage_destroy")
        self.ptr = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def state_update_host(stage: HostStage, cache: Cache, ssm: SSMParams, conv: Optional[ConvParams], batch: int,
                      host_in: torch.Tensor, off_xBC: int, xBC_row_stride: int, off_dt: int, dt_row_stride: int,
                      off_z: int, z_row_stride: int, host_y: torch.Tensor, y_row_stride: int,
                      slot_idx: torch.Tensor, stream: Optional[int] = None) -> None:
    """One decode step from pinned host memory (m2_state_update_host): the
    packed rows of ``host_in`` (byte offsets and element strides of xBC, dt and
    z; ``off_z`` < 0 for no gate) are copied in, the step runs, y is copied
    into ``host_y``. Asynchronous: read ``host_y`` after ``stage.join`` and a
    synchronisation."""
    if not host_in.is_pinned() or not host_y.is_pinned():
        raise ValueError("host_in and host_y must be pinned host tensors")
    sp = ssm.c()
    cp = conv.c() if conv is not None else None
    st = lib().m2_state_update_host(
        stage.ptr, ctypes.byref(cache.c), ctypes.byref(sp), ctypes.byref(cp) if cp is not None else None, batch,
        host_in.data_ptr(), off_xBC, xBC_row_stride, off_dt, dt_row_stride, off_z, z_row_stride,
        host_y.data_ptr(), y_row_stride, slot_idx.data_ptr(), _stream_ptr() if stream is None else stream)
    _check(st, "m2_state_update_host")


def conv1d_update(cache: Cache, conv: ConvParams, xBC: torch.Tensor, slot_idx: torch.Tensor,
                  out: Optional[torch.Tensor] = None, out_dtype: Optional[torch.dtype] = None,
                  stream: Optional[int] = None) -> torch.Tensor:
    """causal_conv1d_update over xBC [batch, seqlen, conv_dim] (or [batch, conv_dim])."""
    x3 = xBC if xBC.dim() == 3 else xBC.unsqueeze(1)
    batch, seqlen, cd = x3.shape
    if out is None:
        out = torch.empty((batch, seqlen, cd), dtype=out_dtype or xBC.dtype, device=xBC.device)
    o3 = out if out.dim() == 3 else out.unsqueeze(1)
    cp = conv.c()
    st = lib().m2_conv1d_update(ctypes.byref(cache.c), ctypes.byref(cp), batch, seqlen,
                                x3.data_ptr(), x3.stride(1), o3.data_ptr(), _dtype_code(o3.dtype),
                                o3.stride(1), slot_idx.data_ptr(),
                                _stream_ptr() if stream is None else stream)
    _check(st, "m2_conv1d_update")
    return out


def conv1d_update_varlen(cache: Cache, conv: ConvParams, xBC: torch.Tensor, cu_seqlens: torch.Tensor,
                         slot_idx: torch.Tensor, max_seqlen: int, out: Optional[torch.Tensor] = None,
                         out_dtype: Optional[torch.dtype] = None, stream: Optional[int] = None) -> torch.Tensor:
    """causal_conv1d_update over sequences packed back to back: xBC [total_tokens, conv_dim]."""
    total, cd = xBC.shape
    if out is None:
        out = torch.empty((total, cd), dtype=out_dtype or xBC.dtype, device=xBC.device)
    cp = conv.c()
    st = lib().m2_conv1d_update_varlen(ctypes.byref(cache.c), ctypes.byref(cp), cu_seqlens.numel() - 1,
                                       cu_seqlens.data_ptr(), total, max_seqlen, xBC.data_ptr(), xBC.stride(0),
                                       out.data_ptr(), _dtype_code(out.dtype), out.stride(0),
                                       slot_idx.data_ptr(), _stream_ptr() if stream is None else stream)
    _check(st, "m2_conv1d_update_varlen")
    return out


def state_update_multi(cache: Cache, ssm: SSMParams, conv: ConvParams, xBC: torch.Tensor, dt: torch.Tensor,
                       slot_idx: torch.Tensor, token_slots: torch.Tensor, z: Optional[torch.Tensor] = None,
                       y: Optional[torch.Tensor] = None, stream: Optional[int] = None) -> torch.Tensor:
    """T draft tokens per row (m2_state_update_multi): xBC [batch, T, conv_dim] raw,
    dt [batch, T, H]; the state after token t goes to slot token_slots[b, t].
    Returns y [batch, T, H*P]."""
    sh = cache.shape
    batch, T, _ = xBC.shape
    for t in (xBC, dt) + ((z,) if z is not None else ()):
        if t.stride(0) != t.shape[1] * t.stride(1):
            raise ValueError("token rows of a sequence must be consecutive")
    if y is None:
        y = torch.empty((batch, T, sh.H * sh.P), dtype=torch_dtype(sh.act_dtype), device=xBC.device)
    st = lib().m2_state_update_multi(
        ctypes.byref(cache.c), ctypes.byref(ssm.c()), ctypes.byref(conv.c()), batch, T, xBC.data_ptr(),
        xBC.stride(1), dt.data_ptr(), dt.stride(1), _ptr(z), z.stride(1) if z is not None else 0, y.data_ptr(),
        y.stride(1), slot_idx.data_ptr(), token_slots.data_ptr(), _stream_ptr() if stream is None else stream)
    _check(st, "m2_state_update_multi")
    return y


def mixed_step(cache: Cache, ssm: SSMParams, conv: ConvParams, decode: Optional[dict] = None,
               prefill: Optional[dict] = None, stream: Optional[int] = None) -> None:
    """One mixed step (m2_mixed_step). ``decode``: dict(xBC, dt, z, y, slot_idx) with
    one raw row per sequence; ``prefill``: dict(xBC, xBC_post, dt, z, y, cu_seqlens,
    slot_idx, max_seqlen, has_initial_state) over packed tokens. Outputs are written
    into the given y tensors."""
    d = p = None
    if decode is not None:
        z = decode.get("z")
        d = m2_decode_rows(decode["xBC"].shape[0], decode["xBC"].data_ptr(), decode["xBC"].stride(0),
                           decode["dt"].data_ptr(), decode["dt"].stride(0), _ptr(z),
                           z.stride(0) if z is not None else 0, decode["y"].data_ptr(), decode["y"].stride(0),
                           decode["slot_idx"].data_ptr())
    if prefill is not None:
        z = prefill.get("z")
        xp = prefill["xBC_post"]
        cu = prefill["cu_seqlens"]
        p = m2_prefill_rows(cu.numel() - 1, cu.data_ptr(), prefill["xBC"].shape[0], prefill["max_seqlen"],
                            prefill["xBC"].data_ptr(), prefill["xBC"].stride(0), xp.data_ptr(),
                            _dtype_code(xp.dtype), xp.stride(0), prefill["dt"].data_ptr(),
                            prefill["dt"].stride(0), _ptr(z), z.stride(0) if z is not None else 0,
                            prefill["y"].data_ptr(), prefill["y"].stride(0), prefill["slot_idx"].data_ptr(),
                            _ptr(prefill.get("has_initial_state")))
    st = lib().m2_mixed_step(ctypes.byref(cache.c), ctypes.byref(ssm.c()), ctypes.byref(conv.c()),
                             ctypes.byref(d) if d is not None else None, ctypes.byref(p) if p is not None else None,
                             _stream_ptr() if stream is None else stream)
    _check(st, "m2_mixed_step")


def chunk_scan(cache: Cache, ssm: SSMParams, xBC: torch.Tensor, dt: torch.Tensor,
               slot_idx: torch.Tensor, z: Optional[torch.Tensor] = None, chunk_size: int = 128,
               has_initial_state: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
               stream: Optional[int] = None) -> torch.Tensor:
    """Prefill scan over xBC [batch, seqlen, conv_dim] (post-conv), dt [batch, seqlen, H]."""
    sh = cache.shape
    batch, seqlen, _ = xBC.shape
    for t in (xBC, dt) + ((z,) if z is not None else ()):
        if t.stride(0) != t.shape[1] * t.stride(1):
            raise ValueError("token rows of a sequence must be consecutive")
    if y is None:
        y = torch.empty((batch, seqlen, sh.H * sh.P), dtype=torch_dtype(sh.act_dtype),
                        device=xBC.device)
    sp = ssm.c()
    st = lib().m2_chunk_scan(
        ctypes.byref(cache.c), ctypes.byref(sp), batch, seqlen, chunk_size, xBC.data_ptr(),
        _dtype_code(xBC.dtype), xBC.stride(1), dt.data_ptr(), dt.stride(1), _ptr(z),
        z.stride(1) if z is not None else 0, y.data_ptr(), y.stride(1), slot_idx.data_ptr(),
        _ptr(has_initial_state), _stream_ptr() if stream is None else stream)
    _check(st, "m2_chunk_scan")
    return y


def chunk_scan_varlen(cache: Cache, ssm: SSMParams, xBC: torch.Tensor, dt: torch.Tensor,
                      cu_seqlens: torch.Tensor, slot_idx: torch.Tensor, max_seqlen: Optional[int] = None,
                      z: Optional[torch.Tensor] = None, chunk_size: int = 128,
                      has_initial_state: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                      stream: Optional[int] = None, static_scratch: bool = False) -> torch.Tensor:
    """Prefill scan over sequences packed back to back: xBC [total_tokens, conv_dim]
    (post-conv), dt [total_tokens, H], cu_seqlens [nseq+1] int32 on the device.
    ``max_seqlen`` plans the split of long sequences; when None it is read from
    cu_seqlens (a device-to-host copy). ``static_scratch`` calls
    m2_chunk_scan_varlen_static (no allocation; calls must not overlap)."""
    sh = cache.shape
    total = xBC.shape[0]
    nseq = cu_seqlens.numel() - 1
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if max_seqlen is None:
        max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if nseq > 0 else 0
    if y is None:
        y = torch.empty((total, sh.H * sh.P), dtype=torch_dtype(sh.act_dtype), device=xBC.device)
    sp = ssm.c()
    fn = lib().m2_chunk_scan_varlen_static if static_scratch else lib().m2_chunk_scan_varlen
    st = fn(
        ctypes.byref(cache.c), ctypes.byref(sp), nseq, cu_seqlens.data_ptr(), total, max_seqlen,
        chunk_size, xBC.data_ptr(), _dtype_code(xBC.dtype), xBC.stride(0), dt.data_ptr(), dt.stride(0),
        _ptr(z), z.stride(0) if z is not None else 0, y.data_ptr(), y.stride(0), slot_idx.data_ptr(),
        _ptr(has_initial_state), _stream_ptr() if stream is None else stream)
    _check(st, "m2_chunk_scan_varlen_static" if static_scratch else "m2_chunk_scan_varlen")
    return y
