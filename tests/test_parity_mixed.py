"""One mixed serving step (m2_mixed_step): prefill sequences (varlen conv into
a post-conv buffer, then the chunk scan) and decode rows (fused decode step)
on one slot-indexed cache, in one graph-capturable call.

Checked against the oracle (decode rows: the decode step; prefill rows: the
conv from the slot's conv cache, rounded to the post-conv buffer's precision,
then the scan from the slot's state or zero), against the separate calls bit
for bit, and as a replayed CUDA graph against the eager call.
"""

import numpy as np
import pytest
import torch

import m2synth as S
import mamba_recurrent_state_b200 as m2
import oracle as O
from m2synth import T_DT, T_XBC, T_Z
from m2synth import torch_inputs as TI
from m2synth import workloads as W
from parity_util import OracleLayer, assert_close, f64
from test_parity_decode import layer_objs, make_cache, shape_of

pytestmark = pytest.mark.gpu

DEC_SLOTS = [0, 3, 5, 7]
PRE_SLOTS = [1, 4, 9]
PRE_LENGTHS = [37, 300, 129]
PRE_INIT = [0, 1, 0]


def setup(w):
    cache = make_cache(w)
    t, ssm, conv = layer_objs(w)
    # fresh prefill sequences start from zeroed slots; the continued one keeps its caches
    fresh = torch.tensor([s for s, i in zip(PRE_SLOTS, PRE_INIT) if not i], dtype=torch.int32, device="cuda")
    cache.zero_slots(fresh)
    total = sum(PRE_LENGTHS)
    pre = TI.step_tensors(w, 0, rows=total)              # packed prefill rows (raw xBC)
    dec = TI.step_tensors(w, 1, rows=len(DEC_SLOTS))      # one raw row per decode sequence
    cu = torch.tensor(np.concatenate([[0], np.cumsum(PRE_LENGTHS)]).astype(np.int32), device="cuda")
    # index tensors made up front (no host copies inside a graph capture)
    pre["slots"] = torch.tensor(PRE_SLOTS, dtype=torch.int32, device="cuda")
    pre["init"] = torch.tensor(PRE_INIT, dtype=torch.uint8, device="cuda")
    dec["slots"] = torch.tensor(DEC_SLOTS, dtype=torch.int32, device="cuda")
    return cache, ssm, conv, pre, dec, cu, total


def mixed(w, cache, ssm, conv, pre, dec, cu, total):
    y_dec = torch.empty((len(DEC_SLOTS), w.H * w.P), dtype=torch.bfloat16, device="cuda")
    y_pre = torch.empty((total, w.H * w.P), dtype=torch.bfloat16, device="cuda")
    xpost = torch.empty((total, w.conv_dim), dtype=torch.float16, device="cuda")
    m2.mixed_step(cache, ssm, conv,
                  decode=dict(xBC=dec["xBC"], dt=dec["dt"], z=dec["z"], y=y_dec, slot_idx=dec["slots"]),
                  prefill=dict(xBC=pre["xBC"], xBC_post=xpost, dt=pre["dt"], z=pre["z"], y=y_pre, cu_seqlens=cu,
                               slot_idx=pre["slots"], max_seqlen=max(PRE_LENGTHS),
                               has_initial_state=pre["init"]))
    return y_dec, y_pre


def small():
    return W.Workload(430, "mixed", 8, 64, 128, 2, 4, S.BF16, S.BF16, 12, len(DEC_SLOTS), chunk=128)


def test_mixed_step_against_oracle():
    w = small()
    cache, ssm, conv, pre, dec, cu, total = setup(w)
    y_dec, y_pre = mixed(w, cache, ssm, conv, pre, dec, cu, total)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    ol = OracleLayer(w)
    # decode rows: one step from the initial caches
    ssm_rows = [ol.initial_ssm(s) for s in DEC_SLOTS]
    conv_rows = [ol.initial_conv(s) for s in DEC_SLOTS]
    inp = {k: f64(W.step_rows(w, tid, 1, np.arange(len(DEC_SLOTS))), w.act_dtype)
           for k, tid in (("xBC", T_XBC), ("dt", T_DT), ("z", T_Z))}
    y_ref = ol.decode(ssm_rows, conv_rows, inp)
    assert_close(f64(TI.to_storage_np(y_dec), w.act_dtype), y_ref, w.act_dtype, "decode y")
    for i, s in enumerate(DEC_SLOTS):
        assert_close(f64(TI.to_storage_np(cache.ssm[s]), w.state_dtype), ssm_rows[i], w.state_dtype, f"decode {i}")
    # prefill sequences: conv from the slot's conv cache (zero when fresh), fp16 buffer, scan
    r0 = 0
    for b, (s, L, init) in enumerate(zip(PRE_SLOTS, PRE_LENGTHS, PRE_INIT)):
        rows = np.arange(r0, r0 + L)
        raw = f64(W.step_rows(w, T_XBC, 0, rows), w.act_dtype)
        conv_state = ol.initial_conv(s) if init else np.zeros((w.K - 1, w.conv_dim))
        post = ol.orc.round_array(ol.orc.conv1d(conv_state, raw, ol.conv_w, ol.conv_b), O.ROUND_F16)
        state = ol.initial_ssm(s) if init else np.zeros((w.H, w.P, w.N))
        y_ref = ol.orc.ssm_scan(state, O.round_mode_for(w.state_dtype), post,
                                f64(W.step_rows(w, T_DT, 0, rows), w.act_dtype), ol.dt_bias, ol.A_log, ol.D,
                                f64(W.step_rows(w, T_Z, 0, rows), w.act_dtype), w.G)
        assert_close(f64(TI.to_storage_np(y_pre[r0:r0 + L]), w.act_dtype), y_ref, w.act_dtype, f"prefill y {b}")
        assert_close(f64(TI.to_storage_np(cache.ssm[s]), w.state_dtype), state, w.state_dtype, f"prefill state {b}")
        want_conv = S.to_storage(conv_state, w.act_dtype)  # the rolled raw inputs, exact
        got_conv = TI.to_storage_np(cache.conv[s])
        assert np.array_equal(got_conv, want_conv), f"prefill conv cache {b}"
        r0 += L


def test_mixed_step_equals_separate_calls_bitwise():
    """Nemotron-H layer shape: the mixed call and the separate calls (varlen
    conv, varlen scan, fused decode) give the same bits for y and both caches."""
    w = W.Workload(431, "mixed_nemo", 128, 64, 128, 8, 4, S.BF16, S.BF16, 12, len(DEC_SLOTS), chunk=128)
    a, ssm, conv, pre, dec, cu, total = setup(w)
    b = m2.Cache(shape_of(w), w.num_slots, ssm=a.ssm.clone(), conv=a.conv.clone())
    ya_dec, ya_pre = mixed(w, a, ssm, conv, pre, dec, cu, total)
    xpost = m2.conv1d_update_varlen(b, conv, pre["xBC"], cu, pre["slots"], max(PRE_LENGTHS),
                                    out_dtype=torch.float16)
    yb_pre = m2.chunk_scan_varlen(b, ssm, xpost, pre["dt"], cu, pre["slots"], max_seqlen=max(PRE_LENGTHS),
                                  z=pre["z"], has_initial_state=pre["init"])
    yb_dec = m2.state_update(b, ssm, dec["xBC"], dec["dt"], dec["slots"], z=dec["z"], conv=conv)
    torch.cuda.synchronize()
    assert torch.equal(ya_dec, yb_dec) and torch.equal(ya_pre, yb_pre)
    assert torch.equal(a.ssm, b.ssm) and torch.equal(a.conv, b.conv)
    assert a.device_error() == 0 and b.device_error() == 0


def test_mixed_step_graph_replay_equals_eager():
    w = small()
    a, ssm, conv, pre, dec, cu, total = setup(w)
    b = m2.Cache(shape_of(w), w.num_slots, ssm=a.ssm.clone(), conv=a.conv.clone())
    ya_dec, ya_pre = mixed(w, a, ssm, conv, pre, dec, cu, total)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s), torch.cuda.graph(g, stream=s):
        yb_dec, yb_pre = mixed(w, b, ssm, conv, pre, dec, cu, total)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(ya_dec, yb_dec) and torch.equal(ya_pre, yb_pre)
    assert torch.equal(a.ssm, b.ssm) and torch.equal(a.conv, b.conv)
    del g


def test_one_part_only():
    w = small()
    cache, ssm, conv, pre, dec, cu, total = setup(w)
    y = torch.empty((len(DEC_SLOTS), w.H * w.P), dtype=torch.bfloat16, device="cuda")
    m2.mixed_step(cache, ssm, conv, decode=dict(xBC=dec["xBC"], dt=dec["dt"], z=dec["z"], y=y,
                  slot_idx=dec["slots"]))
    m2.mixed_step(cache, ssm, conv)  # nothing to do
    torch.cuda.synchronize()
    assert cache.device_error() == 0


def test_varlen_conv_equals_per_sequence_calls():
    """m2_conv1d_update_varlen over ragged sequences (a padding row, an empty
    sequence, lengths below K-1 and across token tiles, a max_seqlen hint below
    the longest so the CTAs loop over tiles) equals one fixed-length call per
    sequence, bit for bit, for the output and the rolled conv cache."""
    w = small()
    lengths = [1, 2, 17, 40, 0, 75]
    slots = [2, -1, 6, 8, 10, 11]
    a = make_cache(w)
    b = m2.Cache(shape_of(w), w.num_slots, ssm=a.ssm.clone(), conv=a.conv.clone())
    _, _, conv = layer_objs(w)
    total = sum(lengths)
    x = TI.step_tensors(w, 0, rows=total)["xBC"]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32), device="cuda")
    out_a = m2.conv1d_update_varlen(a, conv, x, cu, torch.tensor(slots, dtype=torch.int32, device="cuda"),
                                    max_seqlen=20, out_dtype=torch.float32)
    r0 = 0
    for L, s in zip(lengths, slots):
        if L > 0:
            out_b = m2.conv1d_update(b, conv, x[r0:r0 + L].unsqueeze(0),
                                     torch.tensor([s], dtype=torch.int32, device="cuda"), out_dtype=torch.float32)
            assert torch.equal(out_a[r0:r0 + L], out_b[0]), f"sequence of length {L}"
        r0 += L
    torch.cuda.synchronize()
    assert torch.equal(a.conv, b.conv)
    assert a.device_error() == 0 and b.device_error() == 0
