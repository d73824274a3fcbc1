"""Edge cases of the variable-length scan (split and unsplit), the varlen conv
and the multi-token decode: padding rows and out-of-range slots must behave
as in the fixed-length calls (padding: zero output, caches untouched; out of
range: the device error word, nothing written for that row), and the other
rows must still be right.
"""

import numpy as np
import pytest
import torch

import m2synth as S
import mamba_recurrent_state_b200 as m2
from m2synth import torch_inputs as TI
from m2synth import workloads as W
from parity_util import TOL, rel_err
from test_parity_decode import layer_objs, make_cache, shape_of

pytestmark = pytest.mark.gpu


def small(index, batch, slots=10):
    return W.Workload(index, f"edge{index}", 8, 64, 128, 2, 4, S.BF16, S.BF16, slots, batch, chunk=128)


def test_split_scan_padding_and_bad_slot():
    """Three long sequences over 8 heads (split into segments): a padding row,
    an out-of-range slot and a valid row. The valid row agrees with the same row
    scanned alone; the padding row's y is zero; the error word says BAD_SLOT;
    only the valid slot changes."""
    w = small(460, 3)
    lengths = [700, 900, 500]
    cache = make_cache(w)
    ssm0 = cache.ssm.clone()
    _, ssm, _ = layer_objs(w)
    total = sum(lengths)
    d = TI.step_tensors(w, 0, rows=total)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32), device="cuda")
    slots = torch.tensor([-1, w.num_slots + 3, 4], dtype=torch.int32, device="cuda")
    y = m2.chunk_scan_varlen(cache, ssm, d["xBC"], d["dt"], cu, slots, max_seqlen=max(lengths), z=d["z"])
    torch.cuda.synchronize()
    assert cache.device_error() == m2.M2_ERR_BAD_SLOT
    assert torch.count_nonzero(y[:700]) == 0
    # the valid row alone
    ref = m2.Cache(shape_of(w), w.num_slots, ssm=ssm0.clone(), conv=cache.conv.clone())
    cu1 = torch.tensor([0, 500], dtype=torch.int32, device="cuda")
    y1 = m2.chunk_scan_varlen(ref, ssm, d["xBC"][1600:], d["dt"][1600:], cu1,
                              torch.tensor([4], dtype=torch.int32, device="cuda"), max_seqlen=900,
                              z=d["z"][1600:])
    torch.cuda.synchronize()
    # another split plan (one sequence instead of three): equal within the bf16 tolerance
    assert rel_err(y[1600:].float().cpu().numpy(), y1.float().cpu().numpy()) <= TOL[S.BF16]
    assert rel_err(cache.ssm[4].float().cpu().numpy(), ref.ssm[4].float().cpu().numpy()) <= TOL[S.BF16]
    keep = torch.as_tensor([q for q in range(w.num_slots) if q != 4], device="cuda")
    assert torch.equal(cache.ssm[keep], ssm0[keep])


def test_varlen_conv_bad_slot_and_padding():
    w = small(461, 3)
    lengths = [40, 100, 70]
    cache = make_cache(w)
    conv0 = cache.conv.clone()
    _, _, conv = layer_objs(w)
    total = sum(lengths)
    x = TI.step_tensors(w, 0, rows=total)["xBC"]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32), device="cuda")
    slots = torch.tensor([2, -1, w.num_slots], dtype=torch.int32, device="cuda")
    out = m2.conv1d_update_varlen(cache, conv, x, cu, slots, max_seqlen=100, out_dtype=torch.float16)
    torch.cuda.synchronize()
    assert cache.device_error() == m2.M2_ERR_BAD_SLOT
    assert torch.count_nonzero(out[40:140]) == 0
    keep = torch.as_tensor([q for q in range(w.num_slots) if q != 2], device="cuda")
    assert torch.equal(cache.conv[keep], conv0[keep])
    assert not torch.equal(cache.conv[2], conv0[2])


def test_multi_token_bad_destination():
    """A destination slot out of range is a device error; the other tokens'
    states are still stored."""
    w = small(462, 2, slots=12)
    cache = make_cache(w)
    ssm0 = cache.ssm.clone()
    _, ssm, conv = layer_objs(w)
    T = 3
    d = TI.step_tensors(w, 0, rows=2 * T)
    x, dt, z = (d[k].view(2, T, -1) for k in ("xBC", "dt", "z"))
    slots = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    dest = torch.tensor([[2, 3, 4], [5, w.num_slots + 7, 6]], dtype=torch.int32, device="cuda")
    m2.state_update_multi(cache, ssm, conv, x, dt, slots, dest, z=z)
    torch.cuda.synchronize()
    assert cache.device_error() == m2.M2_ERR_BAD_SLOT
    for q in (2, 3, 4, 5, 6):
        assert not torch.equal(cache.ssm[q], ssm0[q]), f"slot {q} was not written"
    for q in (0, 1, 7, 8, 9, 10, 11):
        assert torch.equal(cache.ssm[q], ssm0[q]), f"slot {q} changed"
