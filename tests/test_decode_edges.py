"""Decode-step edge cases through the C ABI: padding and out-of-range slots,
empty and ragged batches, odd shapes (group sizes from 1 to 64 heads, N from 64
to 256, K from 2 to 4, P = 16), strided rows, no gate, slot-permutation
invariance, CUDA-graph replay, caches beyond 2^31 elements, host validation,
slot zeroing and the native allocator."""

import dataclasses

import numpy as np
import pytest
import torch

import m2synth as S
import mamba_recurrent_state_b200 as m2
from m2synth import torch_inputs as TI
from m2synth import workloads as W
from parity_util import OracleLayer, assert_close, f64
from test_parity_decode import check_slots, layer_objs, make_cache, shape_of

pytestmark = pytest.mark.gpu

BF, F32 = S.BF16, S.F32


def wl(index, H, P, N, G, K=4, sd=BF, ad=BF, slots=11, batch=5, steps=1):
    return W.Workload(index, f"edge{index}", H, P, N, G, K, sd, ad, slots, batch, steps=steps)


def run_and_check(w, steps=1, with_z=True, activation=1, slots=None):
    cache = make_cache(w)
    ssm0, conv0 = cache.ssm.clone(), cache.conv.clone()
    t, ssm, conv = layer_objs(w)
    conv.activation = activation
    ol = OracleLayer(w)
    if slots is not None:
        ol.slots = np.asarray(slots, dtype=np.int32)
        t["slots"] = torch.as_tensor(ol.slots, device="cuda")
    valid = [i for i, s in enumerate(ol.slots) if 0 <= s < w.num_slots]
    ssm_rows = [ol.initial_ssm(ol.slots[i]) for i in valid]
    conv_rows = [ol.initial_conv(ol.slots[i]) for i in valid]
    for step in range(steps):
        inp = TI.step_tensors(w, step)
        y = m2.state_update(cache, ssm, inp["xBC"], inp["dt"], t["slots"],
                            z=inp["z"] if with_z else None, conv=conv)
        y_ref = ol.decode(ssm_rows, conv_rows, ol.inputs(step, valid), with_z=with_z,
                          activation=activation)
        assert_close(f64(TI.to_storage_np(y[valid]), w.act_dtype), y_ref, w.act_dtype, f"y {step}")
        pad = [i for i, s in enumerate(ol.slots) if s < 0]
        if pad:
            assert torch.count_nonzero(y[pad]) == 0
    check_slots(w, cache, ssm0, conv0, ol.slots[valid], ssm_rows, conv_rows)
    return cache


@pytest.mark.parametrize("w", [
    wl(101, 24, 64, 128, 3),                    # 8 heads per group, cluster of 2
    wl(102, 16, 64, 128, 16),                   # one head per group, no cluster
    wl(103, 4, 32, 64, 1, K=3, sd=F32, ad=F32),  # fp32, N=64, K=3
    wl(104, 8, 64, 256, 2, K=2, sd=BF, ad=F32),  # N=256 bf16 state, fp32 activations
    wl(105, 64, 64, 128, 1, batch=3),           # 64 heads per group: 16-CTA cluster
    wl(106, 8, 16, 64, 4, batch=7),             # P=16
    wl(107, 8, 64, 128, 2, sd=F32, ad=BF, batch=1, steps=3),
    wl(108, 8, 24, 128, 1),                     # P=24: 64-row tiles start inside a head
], ids=lambda w: f"H{w.H}P{w.P}N{w.N}G{w.G}K{w.K}s{w.state_dtype}a{w.act_dtype}b{w.batch}")
def test_shapes(w):
    run_and_check(w, steps=w.steps)


def test_no_gate_no_activation():
    run_and_check(wl(110, 8, 64, 128, 2), with_z=False, activation=0)


def test_padding_rows_are_skipped():
    cache = run_and_check(wl(111, 8, 64, 128, 2, slots=8, batch=6), slots=[3, -1, 5, -7, 0, 7])
    assert cache.device_error() == 0


def test_out_of_range_slot_sets_the_error_word():
    w = wl(112, 8, 64, 128, 2, slots=8, batch=3)
    cache = make_cache(w)
    ssm0, conv0 = cache.ssm.clone(), cache.conv.clone()
    t, ssm, conv = layer_objs(w)
    t["slots"] = torch.tensor([1, 99, 2], dtype=torch.int32, device="cuda")
    inp = TI.step_tensors(w, 0)
    y = torch.full((3, w.H * w.P), 7.0, dtype=torch.bfloat16, device="cuda")
    m2.state_update(cache, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv, y=y)
    assert cache.device_error() == m2.M2_ERR_BAD_SLOT
    assert cache.device_error() == 0  # read clears it
    assert torch.all(y[1] == 7.0)      # nothing written for the bad row
    others = [s for s in range(8) if s not in (1, 2)]
    assert torch.equal(cache.ssm[others], ssm0[others]) and torch.equal(cache.conv[others], conv0[others])
    ol = OracleLayer(w)
    rows = [ol.initial_ssm(1), ol.initial_ssm(2)]
    convs = [ol.initial_conv(1), ol.initial_conv(2)]
    y_ref = ol.decode(rows, convs, ol.inputs(0, [0, 2]))
    assert_close(f64(TI.to_storage_np(y[[0, 2]]), w.act_dtype), y_ref, w.act_dtype, "valid rows")


def test_empty_batch_is_a_no_op():
    w = W.WORKLOADS[1]
    cache = m2.Cache(shape_of(w), 4)
    t, ssm, conv = layer_objs(w)
    x = torch.empty((0, w.conv_dim), dtype=torch.bfloat16, device="cuda")
    dt = torch.empty((0, w.H), dtype=torch.bfloat16, device="cuda")
    y = m2.state_update(cache, ssm, x, dt, t["slots"][:0], conv=conv)
    assert y.shape == (0, w.H * w.P)


def test_strided_rows():
    """xBC, z, dt and y as column slices of wider row buffers (in_proj style)."""
    w = wl(113, 8, 64, 128, 2, batch=4)
    cache = make_cache(w)
    t, ssm, conv = layer_objs(w)
    inp = TI.step_tensors(w, 0)
    hp = w.H * w.P
    wide = torch.zeros((w.batch, hp + w.conv_dim + 64), dtype=torch.bfloat16, device="cuda")
    wide[:, :hp] = inp["z"]
    wide[:, hp:hp + w.conv_dim] = inp["xBC"]
    dtw = torch.zeros((w.batch, 16 + w.H), dtype=torch.bfloat16, device="cuda")
    dtw[:, 16:] = inp["dt"]
    yw = torch.zeros((w.batch, hp + 64), dtype=torch.bfloat16, device="cuda")
    ref = make_cache(w)
    y_ref = m2.state_update(ref, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv)
    m2.state_update(cache, ssm, wide[:, hp:hp + w.conv_dim], dtw[:, 16:], t["slots"],
                    z=wide[:, :hp], conv=conv, y=yw[:, :hp])
    assert torch.equal(yw[:, :hp], y_ref)
    assert torch.equal(cache.ssm, ref.ssm) and torch.equal(cache.conv, ref.conv)


def test_slot_permutation_invariance_bitwise():
    w = wl(114, 8, 64, 128, 2, slots=16, batch=6)
    a = make_cache(w)
    t, ssm, conv = layer_objs(w)
    perm = torch.randperm(16, generator=torch.Generator().manual_seed(5)).to("cuda")
    inv = torch.argsort(perm)
    # cache b holds slot s of a at position inv[s]; rows use slot inv[slot]
    b = m2.Cache(shape_of(w), 16, ssm=a.ssm[perm].contiguous(), conv=a.conv[perm].contiguous())
    inp = TI.step_tensors(w, 0)
    ya = m2.state_update(a, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv)
    slots_b = inv[t["slots"].long()].to(torch.int32)
    yb = m2.state_update(b, ssm, inp["xBC"], inp["dt"], slots_b, z=inp["z"], conv=conv)
    assert torch.equal(ya, yb)
    assert torch.equal(a.ssm[perm], b.ssm) and torch.equal(a.conv[perm], b.conv)


def test_graph_replay_equals_eager():
    """48 decode calls captured in one CUDA graph reproduce eager execution bit for bit."""
    w = wl(115, 16, 64, 128, 4, slots=32, batch=24)
    eager = make_cache(w)
    graphed = m2.Cache(shape_of(w), w.num_slots, ssm=eager.ssm.clone(), conv=eager.conv.clone())
    t, ssm, conv = layer_objs(w)
    inp = TI.step_tensors(w, 0)
    y_e = [m2.state_update(eager, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv)
           for _ in range(48)]
    g = torch.cuda.CUDAGraph()
    y_g = [torch.empty_like(y_e[0]) for _ in range(48)]
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for i in range(48):
            m2.state_update(graphed, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv,
                            y=y_g[i])
    g.replay()
    torch.cuda.synchronize()
    for i in range(48):
        assert torch.equal(y_e[i], y_g[i]), i
    assert torch.equal(eager.ssm, graphed.ssm) and torch.equal(eager.conv, graphed.conv)
    del g


def test_cache_beyond_2_pow_31_elements():
    """2100 slots of the Nemotron-H shape (2.2e9 state elements, 4.4 GB): slots
    near the end address past 2^31 elements."""
    w = dataclasses.replace(W.WORKLOADS[1], index=116, name="big", num_slots=2100, batch=3)
    shape = shape_of(w)
    cache = m2.Cache(shape, w.num_slots)
    slots = [2099, 2050, 3]
    ol = OracleLayer(w)
    for s in slots:
        cache.ssm[s].copy_(TI.to_torch(W.ssm_slot(w, s), w.state_dtype))
        cache.conv[s].copy_(TI.to_torch(W.conv_slot(w, s), w.act_dtype))
    t, ssm, conv = layer_objs(w)
    slot_t = torch.tensor(slots, dtype=torch.int32, device="cuda")
    inp = TI.step_tensors(w, 0)
    y = m2.state_update(cache, ssm, inp["xBC"], inp["dt"], slot_t, z=inp["z"], conv=conv)
    ssm_rows = [ol.initial_ssm(s) for s in slots]
    conv_rows = [ol.initial_conv(s) for s in slots]
    y_ref = ol.decode(ssm_rows, conv_rows, ol.inputs(0, [0, 1, 2]))
    assert_close(f64(TI.to_storage_np(y), w.act_dtype), y_ref, w.act_dtype, "y")
    for i, s in enumerate(slots):
        assert_close(f64(TI.to_storage_np(cache.ssm[s]), w.state_dtype), ssm_rows[i], w.state_dtype,
                     f"slot {s}")
    assert cache.device_error() == 0


def test_validate_mode_rejects_duplicate_slots(monkeypatch):
    w = wl(117, 8, 64, 128, 2, slots=8, batch=3)
    cache = make_cache(w)
    t, ssm, conv = layer_objs(w)
    inp = TI.step_tensors(w, 0)
    dup = torch.tensor([1, 4, 1], dtype=torch.int32, device="cuda")
    monkeypatch.setenv("M2_VALIDATE", "1")
    with pytest.raises(m2.M2Error) as e:
        m2.state_update(cache, ssm, inp["xBC"], inp["dt"], dup, z=inp["z"], conv=conv)
    assert e.value.status == m2.M2_ERR_INVALID_ARG
    ok = torch.tensor([1, 4, -1], dtype=torch.int32, device="cuda")
    m2.state_update(cache, ssm, inp["xBC"], inp["dt"], ok, z=inp["z"], conv=conv)


def test_host_argument_errors():
    w = W.WORKLOADS[1]
    cache = make_cache(w)
    t, ssm, conv = layer_objs(w)
    inp = TI.step_tensors(w, 0)
    base = torch.zeros(w.batch * w.conv_dim + 8, dtype=torch.bfloat16, device="cuda")
    misaligned = base[1:1 + w.batch * w.conv_dim].view(w.batch, w.conv_dim)  # 2-byte offset
    with pytest.raises(m2.M2Error) as e:
        m2.state_update(cache, ssm, misaligned, inp["dt"], t["slots"], conv=conv)
    assert e.value.status == m2.M2_ERR_INVALID_ARG
    with pytest.raises(m2.M2Error) as e:  # raw xBC dtype must be the activation dtype when fused
        m2.state_update(cache, ssm, inp["xBC"].float(), inp["dt"], t["slots"], conv=conv)
    assert e.value.status == m2.M2_ERR_INVALID_ARG
    bad = m2.Shape(8, 64, 96, 1, 4)
    with pytest.raises(m2.M2Error) as e:
        m2.Cache(bad, 4)
    assert e.value.status == m2.M2_ERR_UNSUPPORTED


def test_zero_slots_and_native_allocator():
    w = W.WORKLOADS[1]
    cache = make_cache(w)
    before = cache.ssm.clone()
    idx = torch.tensor([3, -1, 200], dtype=torch.int32, device="cuda")
    cache.zero_slots(idx)
    torch.cuda.synchronize()
    assert torch.count_nonzero(cache.ssm[[3, 200]]) == 0 and torch.count_nonzero(cache.conv[[3, 200]]) == 0
    keep = [s for s in range(w.num_slots) if s not in (3, 200)]
    assert torch.equal(cache.ssm[keep], before[keep])
    cache.zero_slots(torch.tensor([999], dtype=torch.int32, device="cuda"))
    assert cache.device_error() == m2.M2_ERR_BAD_SLOT
    native = m2.Cache(shape_of(w), 8, native=True)
    assert native.c.owned == 1 and native.c.ssm
    t, ssm, conv = layer_objs(w)
    inp = TI.step_tensors(w, 0)
    slots = torch.arange(8, dtype=torch.int32, device="cuda")
    y = m2.state_update(native, ssm, inp["xBC"][:8], inp["dt"][:8], slots, z=inp["z"][:8], conv=conv)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    native.free()
    assert native.c.ssm is None
