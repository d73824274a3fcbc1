"""Multi-token decode for speculative drafts (m2_state_update_multi) against the
oracle: T decode steps in a row (conv tap, state update rounded to the storage
dtype after each, gated y) from the input slot, with the state and conv window
after every token compared with the destination slot the call wrote. The
input slot must stay untouched; a negative destination stores nothing; a
padding row writes y = 0. T = 1 stores the state and conv window of one fused
decode step bit for bit (y agrees within the bf16 tolerance: the row sum runs
in another order).
"""

import numpy as np
import pytest
import torch

import m2synth as S
import mamba_recurrent_state_b200 as m2
from m2synth import T_DT, T_XBC, T_Z
from m2synth import torch_inputs as TI
from m2synth import workloads as W
from parity_util import OracleLayer, assert_close, f64
from test_parity_decode import layer_objs, make_cache, shape_of

pytestmark = pytest.mark.gpu


def bits(a):
    return a.view(np.uint32) if a.dtype == np.float32 else a.view(np.uint16)


def run_multi(w, T, slot_list, dest, with_z=True):
    """dest: [batch][T] destination slots (negative: not stored)."""
    cache = make_cache(w)
    ssm0, conv0 = cache.ssm.clone(), cache.conv.clone()
    _, ssm, conv = layer_objs(w)
    batch = len(slot_list)
    d = TI.step_tensors(w, 0, rows=batch * T)
    x = d["xBC"].view(batch, T, -1)
    dt = d["dt"].view(batch, T, -1)
    z = d["z"].view(batch, T, -1)
    slots = torch.tensor(slot_list, dtype=torch.int32, device="cuda")
    tok = torch.tensor(dest, dtype=torch.int32, device="cuda")
    y = m2.state_update_multi(cache, ssm, conv, x, dt, slots, tok, z=z if with_z else None)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    ol = OracleLayer(w)
    written = set()
    for b, s in enumerate(slot_list):
        if s < 0:
            assert torch.count_nonzero(y[b]) == 0, f"padding row {b}"
            continue
        ssm_rows = [ol.initial_ssm(s)]
        conv_rows = [ol.initial_conv(s)]
        for t in range(T):
            r = [b * T + t]
            inp = {k: f64(W.step_rows(w, tid, 0, r), w.act_dtype) for k, tid in (("xBC", T_XBC), ("dt", T_DT), ("z", T_Z))}
            y_ref = ol.decode(ssm_rows, conv_rows, inp, with_z=with_z)
            assert_close(f64(TI.to_storage_np(y[b, t:t + 1]), w.act_dtype), y_ref, w.act_dtype, f"y row {b} token {t}")
            q = dest[b][t]
            if q >= 0:
                written.add(q)
                assert_close(f64(TI.to_storage_np(cache.ssm[q]), w.state_dtype), ssm_rows[0], w.state_dtype,
                             f"state after row {b} token {t}")
                want = S.to_storage(conv_rows[0], w.act_dtype)
                assert np.array_equal(bits(TI.to_storage_np(cache.conv[q])), bits(want)), f"conv row {b} token {t}"
    keep = torch.as_tensor(sorted(set(range(w.num_slots)) - written), device="cuda")
    assert torch.equal(cache.ssm[keep], ssm0[keep]), "input or unrelated slots changed"
    assert torch.equal(cache.conv[keep], conv0[keep]), "input or unrelated conv slots changed"


def test_small_bf16_four_drafts():
    w = W.Workload(440, "multi", 8, 64, 128, 2, 4, S.BF16, S.BF16, 20, 3)
    run_multi(w, 4, [2, -1, 7], [[10, 11, 12, 13], [14, 15, 16, 17], [18, -1, 19, 0]])


def test_nemotron_h_layer_three_drafts():
    w = W.Workload(441, "multi_nemo", 128, 64, 128, 8, 4, S.BF16, S.BF16, 16, 4)
    run_multi(w, 3, [0, 1, 2, 3], [[4, 5, 6], [7, 8, 9], [10, 11, 12], [13, 14, 15]])


@pytest.mark.parametrize("w", [
    W.Workload(442, "multi_f32", 8, 64, 64, 2, 4, S.F32, S.BF16, 12, 2),
    W.Workload(443, "multi_f32a", 8, 64, 128, 1, 3, S.F32, S.F32, 12, 2),
    W.Workload(444, "multi_n256", 4, 64, 256, 1, 4, S.BF16, S.BF16, 12, 2),
    # P = 24 does not divide the 64-row tiles, so tiles start and end inside a head
    W.Workload(446, "multi_p24", 8, 24, 128, 1, 4, S.BF16, S.BF16, 12, 2),
], ids=lambda w: f"P{w.P}N{w.N}K{w.K}s{w.state_dtype}a{w.act_dtype}")
def test_dtypes_and_shapes(w):
    run_multi(w, 5, [0, 1], [[2, 3, 4, 5, 6], [7, 8, -1, 9, 10]])


def test_without_gate():
    """z = NULL: every token's y is the ungated output."""
    w = W.Workload(445, "multi_nogate", 8, 64, 128, 2, 4, S.BF16, S.BF16, 12, 2)
    run_multi(w, 3, [0, 1], [[2, 3, 4], [5, -1, 6]], with_z=False)


def test_one_token_equals_the_fused_decode_step():
    w = W.WORKLOADS[1]
    a = make_cache(w)
    b = m2.Cache(shape_of(w), w.num_slots, ssm=a.ssm.clone(), conv=a.conv.clone())
    t, ssm, conv = layer_objs(w)
    inp = TI.step_tensors(w, 0)
    slots = t["slots"]
    dest = torch.tensor([[s] for s in range(w.num_slots) if s not in set(slots.tolist())][:w.batch],
                        dtype=torch.int32, device="cuda")
    ym = m2.state_update_multi(a, ssm, conv, inp["xBC"].unsqueeze(1), inp["dt"].unsqueeze(1), slots, dest,
                               z=inp["z"].unsqueeze(1))
    yd = m2.state_update(b, ssm, inp["xBC"], inp["dt"], slots, z=inp["z"], conv=conv)
    torch.cuda.synchronize()
    # the state and conv window follow the same per-element arithmetic: same bits;
    # y sums its row in another order: equal within the bf16 tolerance
    src = slots.long()
    dst = dest[:, 0].long()
    assert torch.equal(a.ssm[dst], b.ssm[src]) and torch.equal(a.conv[dst], b.conv[src])
    assert_close(f64(TI.to_storage_np(ym[:, 0]), w.act_dtype), f64(TI.to_storage_np(yd), w.act_dtype),
                 w.act_dtype, "y")
