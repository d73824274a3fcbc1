"""Variable-length prefill scan (sequences packed back to back, cu_seqlens) and
the split of long sequences across CTAs, against the oracle's definition: each
sequence is its own run of T sequential updates from its slot's state (or
zero), the working state unrounded until the end.

Cases: ragged lengths with a padding row, an empty sequence and mixed initial
states (6 x 8 pairs: split into 3 segments); few long sequences, which the call
splits into segments (first pass, fp32 combine, scan pass); the Nemotron-H
layer with one 4096-token prompt, checked on sampled heads; a sequence longer
than the max_seqlen hint; and the split result against the unsplit
fixed-length scan of the same input.
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
from parity_util import OracleLayer, assert_close, f64, rel_err, TOL
from test_parity_decode import layer_objs, make_cache

pytestmark = pytest.mark.gpu


def wl(index, H=8, G=2, batch=6, slots=8, T=64):
    return W.Workload(index, f"varlen{index}", H, 64, 128, G, 4, S.BF16, S.BF16, slots, batch,
                      seqlen=T, chunk=128)


def packed_inputs(w, total):
    d = TI.step_tensors(w, 0, rows=total)
    return d["xBC"], d["dt"], d["z"]


def gen_cols(w, tid, rows, c0, c1):
    """Columns c0..c1-1 of the given packed rows of one input, host generator."""
    dim = {T_XBC: w.conv_dim, T_Z: w.H * w.P, T_DT: w.H}[tid]
    key = W.step_key(w, tid, 0)
    out = np.empty((len(rows), c1 - c0), dtype=S.np_storage_dtype(w.act_dtype))
    for i, r in enumerate(rows):
        out[i] = S.normal_storage(key, int(r) * dim + c0, c1 - c0, 0.0, 1.0, w.act_dtype)
    return f64(out, w.act_dtype)


def oracle_heads(ol, w, row0, T, state0, heads, with_z=True):
    """The oracle scan of one packed sequence, head by head (a head only sees
    its own x, dt, z and its group's B, C: one-group runs of H = 1)."""
    rows = np.arange(row0, row0 + T)
    P, N, G, HP = w.P, w.N, w.G, w.H * w.P
    hpg = w.H // w.G
    ys, states = {}, {}
    for h in heads:
        g = h // hpg
        sub = np.concatenate([gen_cols(w, T_XBC, rows, h * P, (h + 1) * P),
                              gen_cols(w, T_XBC, rows, HP + g * N, HP + (g + 1) * N),
                              gen_cols(w, T_XBC, rows, HP + G * N + g * N, HP + G * N + (g + 1) * N)],
                             axis=1)
        dt = gen_cols(w, T_DT, rows, h, h + 1)
        z = gen_cols(w, T_Z, rows, h * P, (h + 1) * P) if with_z else None
        st = np.ascontiguousarray(state0[h:h + 1])
        ys[h] = ol.orc.ssm_scan(st, O.round_mode_for(w.state_dtype), sub, dt, ol.dt_bias[h:h + 1],
                                ol.A_log[h:h + 1], ol.D[h:h + 1], z, 1)
        states[h] = st[0]
    return ys, states


def run_case(w, lengths, slot_list, init_list, heads=None, max_seqlen=None, with_z=True):
    cache = make_cache(w)
    ssm0 = cache.ssm.clone()
    t, ssm, _ = layer_objs(w)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    total = int(cu[-1])
    x, dt, z = packed_inputs(w, total)
    cu_d = torch.from_numpy(cu).cuda()
    slots = torch.tensor(slot_list, dtype=torch.int32, device="cuda")
    init = torch.tensor(init_list, dtype=torch.uint8, device="cuda")
    y = m2.chunk_scan_varlen(cache, ssm, x, dt, cu_d, slots, max_seqlen=max_seqlen, z=z if with_z else None,
                             has_initial_state=init)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    ol = OracleLayer(w)
    heads = list(range(w.H)) if heads is None else heads
    cols = np.concatenate([np.arange(h * w.P, (h + 1) * w.P) for h in heads])
    for b, (s, L) in enumerate(zip(slot_list, lengths)):
        r0 = int(cu[b])
        if s < 0:
            assert torch.count_nonzero(y[r0:r0 + L]) == 0, f"padding row {b}"
            continue
        if L == 0:
            assert torch.equal(cache.ssm[s], ssm0[s]), f"empty sequence {b} touched its slot"
            continue
        state0 = ol.initial_ssm(s) if init_list[b] else np.zeros((w.H, w.P, w.N))
        ys, states = oracle_heads(ol, w, r0, L, state0, heads, with_z=with_z)
        y_ref = np.concatenate([ys[h] for h in heads], axis=1)
        y_gpu = f64(TI.to_storage_np(y[r0:r0 + L][:, torch.as_tensor(cols, device="cuda")]), w.act_dtype)
        assert_close(y_gpu, y_ref, w.act_dtype, f"y of sequence {b} (length {L})")
        st_gpu = f64(TI.to_storage_np(cache.ssm[s]), w.state_dtype)
        for h in heads:
            assert_close(st_gpu[h], states[h], w.state_dtype, f"final state of sequence {b}, head {h}")
    keep = [q for q in range(w.num_slots) if q not in slot_list]
    if keep:
        k = torch.as_tensor(keep, device="cuda")
        assert torch.equal(cache.ssm[k], ssm0[k]), "slots outside the batch changed"
    return cache, y


def test_varlen_ragged_mixed():
    """Ragged lengths (1 .. 300, partial and exact chunks), a padding row, an
    empty sequence that must leave its slot alone, and mixed initial states."""
    w = wl(400)
    run_case(w, lengths=[37, 5, 128, 0, 300, 1], slot_list=[5, -1, 2, 7, 0, 3],
             init_list=[1, 0, 0, 1, 1, 0])


def test_varlen_split_long_sequences():
    """Two long sequences over 8 heads: 16 (sequence, head) pairs, so the call
    splits each sequence into segments of three chunks (summary pass, fp32
    combine, scan pass), with and without an initial state."""
    w = wl(401, batch=2)
    run_case(w, lengths=[1000, 2500], slot_list=[6, 1], init_list=[1, 0])


def test_varlen_split_longer_than_hint():
    """max_seqlen underestimates the longest sequence: its last segment runs to
    the end of the sequence, still exact."""
    w = wl(402, batch=2)
    run_case(w, lengths=[700, 1500], slot_list=[3, 4], init_list=[0, 1], max_seqlen=700)


def test_nemotron_h_one_long_prompt_sampled_heads():
    """Nemotron-H layer (H = 128, G = 8), one 4096-token prompt from the slot's
    state through the variable-length call (128 (sequence, head) pairs: one
    CTA per head, no split on a 148-SM GPU); heads 0, 77 and 127 are followed
    by the oracle."""
    w = W.Workload(403, "varlen_nemotron", 128, 64, 128, 8, 4, S.BF16, S.BF16, 4, 1, seqlen=4096,
                   chunk=128)
    run_case(w, lengths=[4096], slot_list=[2], init_list=[1], heads=[0, 77, 127])


def test_varlen_split_without_gate():
    """z = NULL through the split path (summary pass, combine, scan pass) and an
    unsplit short sequence."""
    w = wl(405, batch=3)
    run_case(w, lengths=[1200, 90, 700], slot_list=[2, 5, 7], init_list=[1, 0, 1], with_z=False)


def test_split_matches_fixed_length_scan():
    """The split varlen call and the one-CTA-per-head fixed-length scan of the
    same single sequence agree within the bf16 tolerance (the carry is the
    same linear recurrence, summed in another order)."""
    w = wl(404, batch=1, T=1536)
    a = make_cache(w)
    b = m2.Cache(m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype), w.num_slots,
                 ssm=a.ssm.clone(), conv=a.conv.clone())
    t, ssm, _ = layer_objs(w)
    x, dt, z = packed_inputs(w, w.seqlen)
    slots = torch.tensor([3], dtype=torch.int32, device="cuda")
    init = torch.tensor([1], dtype=torch.uint8, device="cuda")
    cu = torch.tensor([0, w.seqlen], dtype=torch.int32, device="cuda")
    ya = m2.chunk_scan_varlen(a, ssm, x, dt, cu, slots, max_seqlen=w.seqlen, z=z, has_initial_state=init)
    yb = m2.chunk_scan(b, ssm, x.view(1, w.seqlen, -1), dt.view(1, w.seqlen, -1), slots,
                       z=z.view(1, w.seqlen, -1), has_initial_state=init)
    torch.cuda.synchronize()
    assert rel_err(ya.float().cpu().numpy(), yb.view(w.seqlen, -1).float().cpu().numpy()) <= TOL[S.BF16]
    assert rel_err(a.ssm[3].float().cpu().numpy(), b.ssm[3].float().cpu().numpy()) <= TOL[S.BF16]
    assert a.device_error() == 0 and b.device_error() == 0
