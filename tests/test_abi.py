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
