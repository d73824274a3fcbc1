"""causal_conv1d_update over seqlen tokens (decode and prefill conv) against
the oracle: post-conv output within tolerance, conv cache bit-exact, padding
rows untouched, sequences shorter than the window included."""

import numpy as np
import pytest
import torch

import m2synth as S
import mamba_recurrent_state_b200 as m2
from m2synth import T_XBC
from m2synth import torch_inputs as TI
from m2synth import workloads as W
from parity_util import OracleLayer, assert_close, f64
from test_parity_decode import layer_objs, make_cache

pytestmark = pytest.mark.gpu


def wl(index, sd, ad, K=4, batch=3, slots=6):
    return W.Workload(index, f"conv{index}", 8, 64, 128, 2, K, sd, ad, slots, batch)


@pytest.mark.parametrize("T", [1, 2, 3, 5, 16, 17, 100])
@pytest.mark.parametrize("ad,od", [(S.BF16, torch.float32), (S.BF16, torch.bfloat16),
                                   (S.BF16, torch.float16), (S.F32, torch.float32),
                                   (S.F32, torch.bfloat16), (S.F32, torch.float16)],
                         ids=["bf16->f32", "bf16->bf16", "bf16->f16", "f32->f32", "f32->bf16",
                              "f32->f16"])
def test_conv_seqlen(T, ad, od):
    w = wl(200 + T, S.BF16, ad)
    cache = make_cache(w)
    conv0 = cache.conv.clone()
    t, _, conv = layer_objs(w)
    slots = torch.tensor([4, -1, 1], dtype=torch.int32, device="cuda")
    x = TI.step_tensors(w, 0, rows=w.batch * T)["xBC"].view(w.batch, T, w.conv_dim)
    out = m2.conv1d_update(cache, conv, x, slots, out_dtype=od)
    torch.cuda.synchronize()
    ol = OracleLayer(w)
    out_code = {torch.float32: S.F32, torch.bfloat16: S.BF16, torch.float16: S.F16}[od]
    for b, s in enumerate([4, -1, 1]):
        if s < 0:
            assert torch.count_nonzero(out[b]) == 0
            continue
        state = ol.initial_conv(s)
        xr = f64(W.step_rows(w, T_XBC, 0, np.arange(b * T, (b + 1) * T)), ad)
        ref = ol.orc.conv1d(state, xr, ol.conv_w, ol.conv_b, 1)
        tol = {S.F32: 1e-5, S.BF16: 2e-2, S.F16: 1e-3}[out_code]
        assert_close(f64(TI.to_storage_np(out[b]), out_code), ref, S.F32, f"row {b}", tol=tol)
        assert np.array_equal(TI.to_storage_np(cache.conv[s]), S.to_storage(state, ad))
    keep = [s for s in range(w.num_slots) if s not in (4, 1)]
    assert torch.equal(cache.conv[keep], conv0[keep])


@pytest.mark.parametrize("K", [2, 3])
def test_conv_widths(K):
    w = wl(230 + K, S.BF16, S.BF16, K=K, batch=2, slots=4)
    cache = make_cache(w)
    t, _, conv = layer_objs(w)
    slots = torch.tensor([3, 0], dtype=torch.int32, device="cuda")
    T = 9
    x = TI.step_tensors(w, 0, rows=w.batch * T)["xBC"].view(w.batch, T, w.conv_dim)
    out = m2.conv1d_update(cache, conv, x, slots, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ol = OracleLayer(w)
    for b, s in enumerate([3, 0]):
        state = ol.initial_conv(s)
        xr = f64(W.step_rows(w, T_XBC, 0, np.arange(b * T, (b + 1) * T)), w.act_dtype)
        ref = ol.orc.conv1d(state, xr, ol.conv_w, ol.conv_b, 1)
        assert_close(f64(TI.to_storage_np(out[b]), S.F32), ref, S.F32, f"row {b}")
        assert np.array_equal(TI.to_storage_np(cache.conv[s]), S.to_storage(state, w.act_dtype))


def test_conv_bad_slot():
    w = wl(240, S.BF16, S.BF16, batch=2, slots=4)
    cache = make_cache(w)
    conv0 = cache.conv.clone()
    t, _, conv = layer_objs(w)
    x = TI.step_tensors(w, 0)["xBC"]
    m2.conv1d_update(cache, conv, x, torch.tensor([9, -1], dtype=torch.int32, device="cuda"))
    assert cache.device_error() == m2.M2_ERR_BAD_SLOT
    assert torch.equal(cache.conv, conv0)


def test_conv_fp16_range_error():
    """A post-conv value beyond the fp16 range records M2_ERR_RANGE."""
    w = wl(250, S.BF16, S.BF16, batch=1, slots=2)
    cache = make_cache(w)
    t, _, conv = layer_objs(w)
    x = TI.step_tensors(w, 0)["xBC"].clone()
    x[0, 7] = 3.0e5
    m2.conv1d_update(cache, conv, x, torch.tensor([1], dtype=torch.int32, device="cuda"),
                     out_dtype=torch.float16)
    assert cache.device_error() == m2.M2_ERR_RANGE
