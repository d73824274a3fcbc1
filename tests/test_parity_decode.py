"""Decode-step parity: libm2 through the C ABI against the CPU oracle.

Workloads 0 and 1 are compared in full (every y, every touched slot's state
and conv cache); workloads 2 (48 layers x 384 sequences, one token as a CUDA
graph of 48 launches) and 3 (23 layers, fp32 state, 64 steps in place) are run
in full on the GPU and compared on sampled (layer, row) pairs that the oracle
recomputes from the seeded streams. Untouched slots must stay bit-identical.
"""

import numpy as np
import pytest
import torch

import m2synth as S
import mamba_recurrent_state_b200 as m2
import oracle as O
from m2synth import torch_inputs as TI
from m2synth import workloads as W
from parity_util import OracleLayer, TOL, assert_close, f64

pytestmark = pytest.mark.gpu


def shape_of(w: W.Workload) -> m2.Shape:
    return m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype)


def make_cache(w: W.Workload, layer: int = 0) -> m2.Cache:
    cache = m2.Cache(shape_of(w), w.num_slots)
    TI.fill_caches(w, cache.ssm, cache.conv, layer)
    return cache


def layer_objs(w: W.Workload, layer: int = 0):
    t = TI.layer_tensors(w, layer)
    return t, m2.SSMParams(t["A_log"], t["dt_bias"], t["D"]), m2.ConvParams(t["conv_w"], t["conv_b"], 1)


def bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.dtype == np.float32 else a.view(np.uint16)


def check_slots(w, cache, ssm0, conv0, slots, ssm_rows, conv_rows, what=""):
    ssm_gpu = TI.to_storage_np(cache.ssm[torch.as_tensor(slots, dtype=torch.long, device=cache.ssm.device)])
    conv_gpu = TI.to_storage_np(cache.conv[torch.as_tensor(slots, dtype=torch.long, device=cache.conv.device)])
    for i in range(len(slots)):
        assert_close(f64(ssm_gpu[i], w.state_dtype), ssm_rows[i], w.state_dtype, f"{what} state row {i}")
        want = S.to_storage(conv_rows[i], w.act_dtype)  # raw inputs: exact in storage precision
        assert np.array_equal(bits(conv_gpu[i]), bits(want)), f"{what} conv cache row {i}"
    untouched = torch.as_tensor(sorted(set(range(w.num_slots)) - set(int(s) for s in slots)),
                                dtype=torch.long, device=cache.ssm.device)
    if len(untouched):
        assert torch.equal(cache.ssm[untouched], ssm0[untouched]), "untouched SSM slots changed"
        assert torch.equal(cache.conv[untouched], conv0[untouched]), "untouched conv slots changed"


def test_device_fill_matches_host_generator():
    w = W.WORKLOADS[1]
    cache = make_cache(w)
    for slot in (0, 77, 255):
        assert np.array_equal(TI.to_storage_np(cache.ssm[slot]), W.ssm_slot(w, slot))
        assert np.array_equal(TI.to_storage_np(cache.conv[slot]), W.conv_slot(w, slot))
    inp = TI.step_tensors(w, 0)
    host = W.step_inputs(w, 0, rows=[0, 5, 63])
    for k in ("xBC", "z", "dt"):
        assert np.array_equal(TI.to_storage_np(inp[k][[0, 5, 63]]), host[k])


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "conv_then_update"])
def test_workload0_sixteen_steps(fused):
    """fp32 everything, H=8, G=1, batch 4 in 8 slots, 16 consecutive steps."""
    w = W.WORKLOADS[0]
    cache = make_cache(w)
    ssm0, conv0 = cache.ssm.clone(), cache.conv.clone()
    t, ssm, conv = layer_objs(w)
    ol = OracleLayer(w)
    ssm_rows = [ol.initial_ssm(s) for s in ol.slots]
    conv_rows = [ol.initial_conv(s) for s in ol.slots]
    for step in range(w.steps):
        inp = TI.step_tensors(w, step)
        if fused:
            y = m2.state_update(cache, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv)
        else:
            xp = m2.conv1d_update(cache, conv, inp["xBC"], t["slots"], out_dtype=torch.float32)
            y = m2.state_update(cache, ssm, xp, inp["dt"], t["slots"], z=inp["z"])
        y_ref = ol.decode(ssm_rows, conv_rows, ol.inputs(step, np.arange(w.batch)))
        assert_close(f64(TI.to_storage_np(y), w.act_dtype), y_ref, w.act_dtype, f"y step {step}")
    check_slots(w, cache, ssm0, conv0, ol.slots, ssm_rows, conv_rows)
    assert cache.device_error() == 0


def test_workload1_full():
    """Nemotron-H layer, bf16, batch 64 over 256 slots, one fused step: every y,
    every touched state and conv row, untouched slots bit-identical."""
    w = W.WORKLOADS[1]
    cache = make_cache(w)
    ssm0, conv0 = cache.ssm.clone(), cache.conv.clone()
    t, ssm, conv = layer_objs(w)
    inp = TI.step_tensors(w, 0)
    y = m2.state_update(cache, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv)
    torch.cuda.synchronize()
    ol = OracleLayer(w)
    ssm_rows = [ol.initial_ssm(s) for s in ol.slots]
    conv_rows = [ol.initial_conv(s) for s in ol.slots]
    y_ref = ol.decode(ssm_rows, conv_rows, ol.inputs(0, np.arange(w.batch)))
    assert_close(f64(TI.to_storage_np(y), w.act_dtype), y_ref, w.act_dtype, "y")
    check_slots(w, cache, ssm0, conv0, ol.slots, ssm_rows, conv_rows)
    assert cache.device_error() == 0


def test_fused_equals_conv_then_update_bitwise():
    """The fused launch (cluster-ordered B/C conv roll) and the two-launch path
    with an fp32 conv output give identical bits: y, state and conv cache."""
    w = W.WORKLOADS[1]
    a = make_cache(w)
    b = m2.Cache(shape_of(w), w.num_slots, ssm=a.ssm.clone(), conv=a.conv.clone())
    t, ssm, conv = layer_objs(w)
    for step in range(3):
        inp = TI.step_tensors(w, step)
        ya = m2.state_update(a, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv)
        xp = m2.conv1d_update(b, conv, inp["xBC"], t["slots"], out_dtype=torch.float32)
        yb = m2.state_update(b, ssm, xp, inp["dt"], t["slots"], z=inp["z"])
        assert torch.equal(ya, yb), f"y differs at step {step}"
    assert torch.equal(a.conv, b.conv)
    assert torch.equal(a.ssm, b.ssm)


@pytest.mark.parametrize("buf", [torch.bfloat16, torch.float16], ids=["bf16", "f16"])
def test_16bit_conv_output_between_launches(buf):
    """Unfused path with the conv output stored in bf16 or fp16: the oracle
    rounds there too."""
    w = W.WORKLOADS[1]
    cache = make_cache(w)
    t, ssm, conv = layer_objs(w)
    inp = TI.step_tensors(w, 0)
    xp = m2.conv1d_update(cache, conv, inp["xBC"], t["slots"], out_dtype=buf)
    y = m2.state_update(cache, ssm, xp, inp["dt"], t["slots"], z=inp["z"])
    torch.cuda.synchronize()
    ol = OracleLayer(w)
    rows = [0, 17, 63]
    ssm_rows = [ol.initial_ssm(ol.slots[r]) for r in rows]
    conv_rows = [ol.initial_conv(ol.slots[r]) for r in rows]
    rnd = O.ROUND_BF16 if buf == torch.bfloat16 else O.ROUND_F16
    y_ref = ol.decode(ssm_rows, conv_rows, ol.inputs(0, rows), post_conv_round=rnd)
    assert_close(f64(TI.to_storage_np(y[rows]), w.act_dtype), y_ref, w.act_dtype, "y")
    for i, r in enumerate(rows):
        assert_close(f64(TI.to_storage_np(cache.ssm[int(ol.slots[r])]), w.state_dtype), ssm_rows[i],
                     w.state_dtype, f"state row {r}")


def test_workload2_stack48_graph_sampled():
    """48 layers x 384 sequences, one token, captured as one CUDA graph of 48
    launches; sampled (layer, row) pairs against the oracle: five layers, with
    the rows holding slots 0 and 383 in each."""
    w = W.WORKLOADS[2]
    caches, objs, inps = [], [], []
    for layer in range(w.layers):
        caches.append(make_cache(w, layer))
        objs.append(layer_objs(w, layer))
        inps.append(TI.step_tensors(w, 0, layer))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    ys = [None] * w.layers
    with torch.cuda.graph(g):
        for layer in range(w.layers):
            t, ssm, conv = objs[layer]
            ys[layer] = m2.state_update(caches[layer], ssm, inps[layer]["xBC"], inps[layer]["dt"],
                                        t["slots"], z=inps[layer]["z"], conv=conv)
    g.replay()
    torch.cuda.synchronize()
    for layer, rows in ((0, [0, 383]), (11, [17]), (23, [191]), (35, [250]), (47, [5, 300])):
        ol = OracleLayer(w, layer)
        # also the rows whose slots sit at the two ends of the cache
        rows = sorted(set(rows) | {int(np.argmax(ol.slots)), int(np.argmin(ol.slots))})
        assert int(ol.slots[rows].max()) == w.num_slots - 1 and int(ol.slots[rows].min()) == 0
        ssm_rows = [ol.initial_ssm(ol.slots[r]) for r in rows]
        conv_rows = [ol.initial_conv(ol.slots[r]) for r in rows]
        y_ref = ol.decode(ssm_rows, conv_rows, ol.inputs(0, rows))
        assert_close(f64(TI.to_storage_np(ys[layer][rows]), w.act_dtype), y_ref, w.act_dtype,
                     f"layer {layer} y")
        for i, r in enumerate(rows):
            s = int(ol.slots[r])
            assert_close(f64(TI.to_storage_np(caches[layer].ssm[s]), w.state_dtype), ssm_rows[i],
                         w.state_dtype, f"layer {layer} row {r} state")
            want = S.to_storage(conv_rows[i], w.act_dtype)
            assert np.array_equal(TI.to_storage_np(caches[layer].conv[s]), want)
    for c in caches:
        assert c.device_error() == 0
    del g


def test_workload3_fp32_state_64_steps_sampled():
    """23 layers, fp32 state, batch 128 in 512 slots, 64 steps carried in place;
    sampled (layer, row) pairs (five layers, the row with the layer's highest
    slot among them) followed through all 64 steps by the oracle."""
    w = W.WORKLOADS[3]
    samples = {0: [0, 127], 5: [33], 11: [64], 17: [100], 22: [1]}
    caches, objs = [], []
    for layer in range(w.layers):
        caches.append(make_cache(w, layer))
        objs.append(layer_objs(w, layer))
    for layer in samples:  # also the row holding the layer's highest slot
        slots = W.slot_indices(w, layer)
        samples[layer] = sorted(set(samples[layer]) | {int(np.argmax(slots))})
    y_hist = {layer: [] for layer in samples}
    buf = None
    for step in range(w.steps):
        for layer in range(w.layers):
            buf = TI.step_tensors(w, step, layer, out=buf)
            t, ssm, conv = objs[layer]
            y = m2.state_update(caches[layer], ssm, buf["xBC"], buf["dt"], t["slots"], z=buf["z"],
                                conv=conv)
            if layer in samples:
                y_hist[layer].append(y[samples[layer]].clone())
    torch.cuda.synchronize()
    for layer, rows in samples.items():
        ol = OracleLayer(w, layer)
        ssm_rows = [ol.initial_ssm(ol.slots[r]) for r in rows]
        conv_rows = [ol.initial_conv(ol.slots[r]) for r in rows]
        for step in range(w.steps):
            y_ref = ol.decode(ssm_rows, conv_rows, ol.inputs(step, rows))
            assert_close(f64(TI.to_storage_np(y_hist[layer][step]), w.act_dtype), y_ref,
                         w.act_dtype, f"layer {layer} step {step} y")
        for i, r in enumerate(rows):
            s = int(ol.slots[r])
            assert_close(f64(TI.to_storage_np(caches[layer].ssm[s]), w.state_dtype), ssm_rows[i],
                         w.state_dtype, f"layer {layer} row {r} state after 64 steps")
    for c in caches:
        assert c.device_error() == 0
