"""The C ABI library (no GPU): it builds, loads, exports every symbol that
include/*.h declares, and its host-only calls behave as documented. No call
here launches a kernel."""

import ctypes
import glob
import os
import re
import subprocess

import pytest

import mamba_recurrent_state_b200 as m2
from mamba_recurrent_state_b200 import build as m2build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(m2_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    m2build.build()
    return m2.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["m2_cache_alloc", "m2_conv1d_update", "m2_state_update", "m2_chunk_scan",
                     "m2_cache_wrap", "m2_cache_free", "m2_cache_zero_slots",
                     "m2_get_device_error"]:
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", m2.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(m2_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    # and the binding knows the signature of each
    assert set(declared_functions()) <= set(m2.SIGNATURES)


def test_conv_dim_and_cache_bytes(lib):
    nemo = m2.Shape(128, 64, 128, 8, 4, m2.M2_BF16, m2.M2_BF16)
    assert nemo.conv_dim == 10240
    assert lib.m2_conv_dim(ctypes.byref(nemo.c())) == 10240
    ssm_b, conv_b = m2.cache_bytes(nemo, 1)
    assert ssm_b == 2 * 1024 * 1024          # Nemotron-H record: 2 MiB per layer per sequence
    assert conv_b == 3 * 10240 * 2
    f32 = m2.Shape(64, 64, 128, 8, 4, m2.M2_F32, m2.M2_BF16)
    assert m2.cache_bytes(f32, 1)[0] == 2 * 1024 * 1024  # the 2.00 MiB/layer f32 page
    assert lib.m2_conv_dim(None) == -1


def test_shape_check(lib):
    ok = m2.Shape(128, 64, 128, 8, 4)
    assert m2.shape_check(ok) == m2.M2_OK
    assert m2.shape_check(m2.Shape(128, 64, 128, 7, 4)) == m2.M2_ERR_INVALID_ARG   # G does not divide H
    assert m2.shape_check(m2.Shape(128, 64, 96, 8, 4)) == m2.M2_ERR_UNSUPPORTED   # N not implemented
    assert m2.shape_check(m2.Shape(128, 64, 128, 8, 9)) == m2.M2_ERR_UNSUPPORTED  # K > 8
    assert m2.shape_check(m2.Shape(8, 64, 256, 1, 4, m2.M2_F32, m2.M2_F32)) == m2.M2_ERR_UNSUPPORTED
    assert m2.shape_check(m2.Shape(0, 64, 128, 1, 4)) == m2.M2_ERR_INVALID_ARG


def test_status_strings(lib):
    for code, text in m2.STATUS.items():
        assert lib.m2_status_string(code).decode() == text
    assert lib.m2_version().decode().startswith("m2 ")


def test_host_validation_rejects_before_launch(lib):
    # NULL cache / params are argument errors; nothing reaches the GPU
    assert lib.m2_state_update(None, None, None, 1, None, 0, 0, None, 0, None, 0, None, 0, None,
                               None) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_chunk_scan(None, None, 1, 1, 128, None, 0, 0, None, 0, None, 0, None, 0, None,
                             None, None) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_conv1d_update(None, None, 1, 1, None, 0, None, 0, 0, None,
                                None) == m2.M2_ERR_INVALID_ARG
    # a described cache with a misaligned base pointer is refused by wrap
    s = m2.Shape(8, 64, 128, 1, 4, m2.M2_F32, m2.M2_F32).c()
    c = m2.m2_cache()
    assert lib.m2_cache_wrap(ctypes.byref(s), 8, 0x1008, 0x2000, None,
                             ctypes.byref(c)) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_cache_wrap(ctypes.byref(s), 0, 0x1000, 0x2000, None,
                             ctypes.byref(c)) == m2.M2_ERR_INVALID_ARG


def test_no_torch_types_in_the_abi():
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        code = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for banned in ("at::", "c10::", "torch", "Tensor"):
            assert banned not in code, banned


def test_newer_entry_points_validate_on_the_host(lib):
    """The variable-length, norm, multi-token and mixed entry points reject bad
    arguments (or return early on empty work) before touching a GPU: a cache
    wrapped around made-up aligned addresses is never dereferenced here."""
    shape = m2.Shape(128, 64, 128, 8, 4, m2.M2_BF16, m2.M2_BF16).c()
    cache = m2.m2_cache()
    assert lib.m2_cache_wrap(ctypes.byref(shape), 4, 0x100000, 0x200000, None, ctypes.byref(cache)) == m2.M2_OK
    ssm = m2.m2_ssm_params(0x300000, 0x300100, 0x300200)
    conv = m2.m2_conv_params(0x400000, None, 1)
    norm = m2.m2_norm_params(0x500000, 1e-5)
    cd, hp = 10240, 8192
    buf = 0x600000  # aligned made-up buffer address
    # the norm is fused only with the conv
    assert lib.m2_state_update_norm(ctypes.byref(cache), ctypes.byref(ssm), None, ctypes.byref(norm), 1, buf,
                                    cd, buf, 128, buf, hp, buf, hp, buf, None) == m2.M2_ERR_INVALID_ARG
    # multi-token decode: T = 0 is a no-op, T above 16 is not supported, an
    # unaligned row stride is an argument error
    args = (buf, cd, buf, 128, buf, hp, buf, hp, buf, buf, None)
    assert lib.m2_state_update_multi(ctypes.byref(cache), ctypes.byref(ssm), ctypes.byref(conv), 2, 0,
                                     *args) == m2.M2_OK
    assert lib.m2_state_update_multi(ctypes.byref(cache), ctypes.byref(ssm), ctypes.byref(conv), 2, 17,
                                     *args) == m2.M2_ERR_UNSUPPORTED
    assert lib.m2_state_update_multi(ctypes.byref(cache), ctypes.byref(ssm), ctypes.byref(conv), 2, 4,
                                     buf, cd + 1, *args[2:]) == m2.M2_ERR_INVALID_ARG
    # varlen scan and conv: empty batches return OK, oversized or missing offsets are refused
    scan_tail = (128, buf, m2.M2_F16, cd, buf, 128, buf, hp, buf, hp, buf, None, None)
    assert lib.m2_chunk_scan_varlen(ctypes.byref(cache), ctypes.byref(ssm), 0, None, 0, 0, *scan_tail) == m2.M2_OK
    assert lib.m2_chunk_scan_varlen(ctypes.byref(cache), ctypes.byref(ssm), 1, buf, 2**31, 2**31 - 1,
                                    *scan_tail) == m2.M2_ERR_UNSUPPORTED
    assert lib.m2_chunk_scan_varlen(ctypes.byref(cache), ctypes.byref(ssm), 2, None, 100, 50,
                                    *scan_tail) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_chunk_scan_varlen_static(ctypes.byref(cache), ctypes.byref(ssm), 2, None, 100, 50,
                                           *scan_tail) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_conv1d_update_varlen(ctypes.byref(cache), ctypes.byref(conv), 2, None, 100, 50, buf, cd, buf,
                                       m2.M2_F16, cd, buf, None) == m2.M2_ERR_INVALID_ARG
    # the mixed step needs the conv parameters; with nothing to do it returns OK
    assert lib.m2_mixed_step(ctypes.byref(cache), ctypes.byref(ssm), None, None, None,
                             None) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_mixed_step(ctypes.byref(cache), ctypes.byref(ssm), ctypes.byref(conv), None, None,
                             None) == m2.M2_OK


def test_host_stage_validates_on_the_host(lib):
    """The host-staged decode entry points refuse bad arguments before any
    CUDA call: no stage is created for a zero depth or size, and a missing
    stage or host buffer is an argument error."""
    out = ctypes.c_void_p()
    assert lib.m2_host_stage_create(0, 1024, 1024, ctypes.byref(out)) == m2.M2_ERR_INVALID_ARG
    assert out.value is None
    assert lib.m2_host_stage_create(4, 0, 1024, ctypes.byref(out)) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_host_stage_create(4, 1024, -1, ctypes.byref(out)) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_host_stage_create(4, 1024, 1024, None) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_host_stage_destroy(None) == m2.M2_ERR_INVALID_ARG
    assert lib.m2_host_stage_join(None, None) == m2.M2_ERR_INVALID_ARG
    shape = m2.Shape(128, 64, 128, 8, 4, m2.M2_BF16, m2.M2_BF16).c()
    cache = m2.m2_cache()
    assert lib.m2_cache_wrap(ctypes.byref(shape), 4, 0x100000, 0x200000, None, ctypes.byref(cache)) == m2.M2_OK
    ssm = m2.m2_ssm_params(0x300000, 0x300100, 0x300200)
    buf = 0x600000
    assert lib.m2_state_update_host(None, ctypes.byref(cache), ctypes.byref(ssm), None, 1, buf, 0, 10240, 0, 128,
                                    -1, 0, buf, 8192, buf, None) == m2.M2_ERR_INVALID_ARG
