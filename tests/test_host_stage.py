"""Decode steps from pinned host memory (m2_state_update_host): the staged
copies around the same fused launch give the bits of the device-resident
path, over more steps than the staging ring holds (and with a ring of one
buffer, every step waiting for the last), with and without the gate, and the
first step also against the oracle."""

import numpy as np
import pytest
import torch

import mamba_recurrent_state_b200 as m2
from m2synth import torch_inputs as TI
from m2synth import workloads as W
from parity_util import OracleLayer, assert_close, f64
from test_parity_decode import layer_objs, make_cache, shape_of

pytestmark = pytest.mark.gpu


def pack_steps(w, steps, gate):
    """Each step's xBC | dt | z rows in one pinned buffer (16-byte aligned blocks)."""
    parts = ["xBC", "dt"] + (["z"] if gate else [])
    bufs, offs = [], None
    for step in range(steps):
        inp = TI.step_tensors(w, step)
        blocks = [inp[k].contiguous().view(torch.uint8).view(-1).cpu() for k in parts]
        if offs is None:
            offs, off = {}, 0
            for k, b in zip(parts, blocks):
                offs[k] = off
                off += (b.numel() + 255) // 256 * 256
            size = off
        hb = torch.zeros(size, dtype=torch.uint8).pin_memory()
        for k, b in zip(parts, blocks):
            hb[offs[k]:offs[k] + b.numel()].copy_(b)
        bufs.append(hb)
    return bufs, offs, size


@pytest.mark.parametrize("gate,depth", [(True, 4), (False, 4), (True, 1)], ids=["gate", "no-gate", "depth1"])
def test_host_steps_equal_device_steps_bitwise(gate, depth):
    w = W.WORKLOADS[1]
    steps = 6
    a = make_cache(w)
    b = m2.Cache(shape_of(w), w.num_slots, ssm=a.ssm.clone(), conv=a.conv.clone())
    t, ssm, conv = layer_objs(w)
    hp, cd = w.H * w.P, w.conv_dim
    bufs, offs, size = pack_steps(w, steps, gate)
    ybytes = w.batch * hp * 2
    stage = m2.HostStage(depth, size, ybytes)
    host_y = [torch.empty((w.batch, hp), dtype=torch.bfloat16).pin_memory() for _ in range(steps)]
    for i in range(steps):
        m2.state_update_host(stage, a, ssm, conv, w.batch, bufs[i], offs["xBC"], cd, offs["dt"], w.H,
                             offs["z"] if gate else -1, hp, host_y[i], hp, t["slots"])
    stage.join()
    torch.cuda.synchronize()
    for i in range(steps):
        inp = TI.step_tensors(w, i)
        yd = m2.state_update(b, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"] if gate else None, conv=conv)
        torch.cuda.synchronize()
        assert torch.equal(host_y[i], yd.cpu()), f"y of step {i}"
    assert torch.equal(a.ssm, b.ssm)
    assert torch.equal(a.conv, b.conv)
    assert a.device_error() == 0
    stage.close()


def test_host_step_against_the_oracle():
    w = W.WORKLOADS[1]
    cache = make_cache(w)
    t, ssm, conv = layer_objs(w)
    hp, cd = w.H * w.P, w.conv_dim
    bufs, offs, size = pack_steps(w, 1, True)
    stage = m2.HostStage(2, size, w.batch * hp * 2)
    host_y = torch.empty((w.batch, hp), dtype=torch.bfloat16).pin_memory()
    m2.state_update_host(stage, cache, ssm, conv, w.batch, bufs[0], offs["xBC"], cd, offs["dt"], w.H, offs["z"], hp,
                         host_y, hp, t["slots"])
    stage.join()
    torch.cuda.synchronize()
    ol = OracleLayer(w)
    ssm_rows = [ol.initial_ssm(s) for s in ol.slots]
    conv_rows = [ol.initial_conv(s) for s in ol.slots]
    y_ref = ol.decode(ssm_rows, conv_rows, ol.inputs(0, np.arange(w.batch)))
    assert_close(f64(TI.to_storage_np(host_y), w.act_dtype), y_ref, w.act_dtype, "y")
    assert cache.device_error() == 0
    stage.close()


def test_host_step_refuses_blocks_outside_the_stage():
    w = W.WORKLOADS[1]
    cache = make_cache(w)
    t, ssm, conv = layer_objs(w)
    hp, cd = w.H * w.P, w.conv_dim
    stage = m2.HostStage(2, 4096, 4096)
    hin = torch.zeros(4096, dtype=torch.uint8).pin_memory()
    hy = torch.zeros(4096, dtype=torch.uint8).pin_memory()
    with pytest.raises(m2.M2Error) as e:
        m2.state_update_host(stage, cache, ssm, conv, w.batch, hin, 0, cd, 0, w.H, -1, hp, hy, hp, t["slots"])
    assert e.value.status == m2.M2_ERR_INVALID_ARG
    stage.close()
