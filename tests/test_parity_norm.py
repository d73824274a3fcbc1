"""Decode step with the gated RMSNorm fused (m2_state_update_norm) against the
oracle: the gated y of the decode step, then the group RMSNorm over H*P/G
channels with the norm weight. The state and conv-cache updates must be the
ones of the plain decode step, bit for bit.

Shapes cover clusters of 4 (Nemotron-H), 2, 1 and 16 CTAs per group, fp32
and bf16 storage, no gate, several steps in place, and a large eps.
"""

import numpy as np
import pytest
import torch

import m2synth as S
import mamba_recurrent_state_b200 as m2
from m2synth import torch_inputs as TI
from m2synth import workloads as W
from parity_util import OracleLayer, assert_close, f64
from test_decode_edges import wl
from test_parity_decode import check_slots, layer_objs, make_cache, shape_of

pytestmark = pytest.mark.gpu


def norm_of(w, eps):
    weight = TI.to_torch(W.norm_weight(w), w.act_dtype)
    return m2.NormParams(weight, eps), f64(W.norm_weight(w), w.act_dtype)


def run_norm(w, steps=1, with_z=True, eps=1e-5):
    cache = make_cache(w)
    ssm0, conv0 = cache.ssm.clone(), cache.conv.clone()
    t, ssm, conv = layer_objs(w)
    norm, w_host = norm_of(w, eps)
    ol = OracleLayer(w)
    ssm_rows = [ol.initial_ssm(s) for s in ol.slots]
    conv_rows = [ol.initial_conv(s) for s in ol.slots]
    for step in range(steps):
        inp = TI.step_tensors(w, step)
        y = m2.state_update(cache, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"] if with_z else None,
                            conv=conv, norm=norm)
        v = ol.decode(ssm_rows, conv_rows, ol.inputs(step, np.arange(w.batch)), with_z=with_z)
        y_ref = np.stack([ol.orc.group_rmsnorm(v[i], w.G, eps, w_host) for i in range(w.batch)])
        assert_close(f64(TI.to_storage_np(y), w.act_dtype), y_ref, w.act_dtype, f"normed y, step {step}")
    torch.cuda.synchronize()
    check_slots(w, cache, ssm0, conv0, ol.slots, ssm_rows, conv_rows, "norm")
    assert cache.device_error() == 0


def test_nemotron_h_layer():
    """Workload 1 (H=128, P=64, N=128, G=8: 1024-channel groups, clusters of 4)."""
    run_norm(W.WORKLOADS[1])


@pytest.mark.parametrize("w", [
    wl(121, 24, 64, 128, 3),                     # clusters of 2
    wl(122, 16, 64, 128, 16),                    # one head per group: no cluster
    wl(123, 64, 64, 128, 1, batch=3),            # 64 heads per group: 16-CTA cluster
    wl(124, 8, 64, 128, 2, sd=S.F32, ad=S.BF16, batch=2, steps=4),
    wl(125, 8, 64, 128, 1, sd=S.F32, ad=S.F32, batch=3),
], ids=lambda w: f"H{w.H}G{w.G}s{w.state_dtype}a{w.act_dtype}")
def test_shapes(w):
    run_norm(w, steps=w.steps)


def test_no_gate_and_large_eps():
    w = wl(126, 16, 64, 128, 2)
    run_norm(w, with_z=False)
    run_norm(w, eps=4.0)


def test_state_and_conv_match_the_plain_step_bitwise():
    """The norm changes y only: state and conv cache equal the plain fused
    step's, bit for bit, over three steps."""
    w = W.WORKLOADS[1]
    a = make_cache(w)
    b = m2.Cache(shape_of(w), w.num_slots, ssm=a.ssm.clone(), conv=a.conv.clone())
    t, ssm, conv = layer_objs(w)
    norm, _ = norm_of(w, 1e-5)
    for step in range(3):
        inp = TI.step_tensors(w, step)
        m2.state_update(a, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv, norm=norm)
        m2.state_update(b, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], conv=conv)
    torch.cuda.synchronize()
    assert torch.equal(a.ssm, b.ssm) and torch.equal(a.conv, b.conv)


def test_norm_needs_the_fused_conv():
    w = W.WORKLOADS[1]
    cache = make_cache(w)
    t, ssm, conv = layer_objs(w)
    norm, _ = norm_of(w, 1e-5)
    inp = TI.step_tensors(w, 0)
    with pytest.raises(ValueError):
        m2.state_update(cache, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"], norm=norm)
