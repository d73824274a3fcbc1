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


def _tile_case(index, K, batch, slots):
    # conv_dim = 10*32 + 2*2*64 = 576: two full 256-channel blocks and a
    # 64-channel partial one
    return W.Workload(index, f"convtile{index}", 10, 32, 64, 2, K, S.BF16, S.BF16, slots, batch)


@pytest.mark.parametrize("K,T,od", [(4, 33000, torch.float16), (2, 4133, torch.bfloat16),
                                    (5, 70, torch.float32)],
                         ids=["K4-ring-f16", "K2-bf16", "K5-short-f32"])
def test_conv_tile_kernel(K, T, od):
    """The shared-memory tile kernel (bf16 input, >= 32 tokens): a partial last
    channel block, a ragged last tile, the first tile staged from the conv
    cache, and -- at 33000 tokens -- several tiles per CTA, so the buffers are
    refilled while the other is computed; the last tile's 2-D box reaches past
    the sequence (into the next row's tokens, or past the buffer)."""
    w = _tile_case(260 + K, K, batch=2, slots=5)
    cache = make_cache(w)
    conv0 = cache.conv.clone()
    _, _, conv = layer_objs(w)
    slot_list = [3, 1]
    slots = torch.tensor(slot_list, dtype=torch.int32, device="cuda")
    x = TI.step_tensors(w, 0, rows=w.batch * T)["xBC"].view(w.batch, T, w.conv_dim)
    out = m2.conv1d_update(cache, conv, x, slots, out_dtype=od)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    ol = OracleLayer(w)
    out_code = {torch.float32: S.F32, torch.bfloat16: S.BF16, torch.float16: S.F16}[od]
    tol = {S.F32: 1e-5, S.BF16: 2e-2, S.F16: 1e-3}[out_code]
    for b, s in enumerate(slot_list):
        state = ol.initial_conv(s)
        xr = f64(W.step_rows(w, T_XBC, 0, np.arange(b * T, (b + 1) * T)), w.act_dtype)
        ref = ol.orc.conv1d(state, xr, ol.conv_w, ol.conv_b, 1)
        assert_close(f64(TI.to_storage_np(out[b]), out_code), ref, S.F32, f"row {b}", tol=tol)
        assert np.array_equal(TI.to_storage_np(cache.conv[s]), S.to_storage(state, w.act_dtype))
    keep = [s for s in range(w.num_slots) if s not in slot_list]
    assert torch.equal(cache.conv[keep], conv0[keep])


def test_conv_tile_kernel_varlen():
    """Packed sequences of 4100, 31 (below one tile), 0 (empty) and 2050
    tokens through the tile kernel: a tile's box may hold rows of the next
    sequence, which are never read; the empty sequence leaves its slot
    untouched."""
    lens = [4100, 31, 0, 2050]
    w = _tile_case(270, 4, batch=len(lens), slots=6)
    cache = make_cache(w)
    conv0 = cache.conv.clone()
    _, _, conv = layer_objs(w)
    slot_list = [5, 0, 2, 4]
    slots = torch.tensor(slot_list, dtype=torch.int32, device="cuda")
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    x = TI.step_tensors(w, 0, rows=total)["xBC"]
    out = m2.conv1d_update_varlen(cache, conv, x, torch.from_numpy(cu).cuda(), slots, max(lens),
                                  out_dtype=torch.float16)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    ol = OracleLayer(w)
    for b, s in enumerate(slot_list):
        if lens[b] == 0:
            assert torch.equal(cache.conv[s], conv0[s])
            continue
        state = ol.initial_conv(s)
        xr = f64(W.step_rows(w, T_XBC, 0, np.arange(cu[b], cu[b + 1])), w.act_dtype)
        ref = ol.orc.conv1d(state, xr, ol.conv_w, ol.conv_b, 1)
        assert_close(f64(TI.to_storage_np(out[cu[b]:cu[b + 1]]), S.F16), ref, S.F32, f"seq {b}", tol=1e-3)
        assert np.array_equal(TI.to_storage_np(cache.conv[s]), S.to_storage(state, w.act_dtype))


def test_conv_tile_kernel_strided_rows():
    """The tile kernel on a column slice of a wider buffer (as when xBC is a
    view of the in_proj output): rows xBC_row_stride apart, the 2-D box reading
    only the conv_dim channels of each row."""
    w = _tile_case(275, 4, batch=2, slots=4)
    cache = make_cache(w)
    _, _, conv = layer_objs(w)
    slot_list = [2, 0]
    slots = torch.tensor(slot_list, dtype=torch.int32, device="cuda")
    T = 1000
    x = TI.step_tensors(w, 0, rows=w.batch * T)["xBC"].view(w.batch, T, w.conv_dim)
    wide = torch.full((w.batch, T, w.conv_dim + 64), 7.0, dtype=x.dtype, device="cuda")
    wide[:, :, 32:32 + w.conv_dim] = x
    xs = wide[:, :, 32:32 + w.conv_dim]
    assert xs.stride(1) == w.conv_dim + 64
    out = m2.conv1d_update(cache, conv, xs, slots, out_dtype=torch.float16)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    ol = OracleLayer(w)
    for b, s in enumerate(slot_list):
        state = ol.initial_conv(s)
        xr = f64(W.step_rows(w, T_XBC, 0, np.arange(b * T, (b + 1) * T)), w.act_dtype)
        ref = ol.orc.conv1d(state, xr, ol.conv_w, ol.conv_b, 1)
        assert_close(f64(TI.to_storage_np(out[b]), S.F16), ref, S.F32, f"row {b}", tol=1e-3)
        assert np.array_equal(TI.to_storage_np(cache.conv[s]), S.to_storage(state, w.act_dtype))
