"""The allocation-free variable-length scan (m2_chunk_scan_varlen_static: the
split scan's scratch is a fixed device array) against the allocating entry
point (m2_chunk_scan_varlen: stream-ordered scratch) on the same inputs, two
calls in a row on twin caches. Both run the same split plan and the same
kernels, so y and the cache must agree bit for bit, and the second call must
not see anything left over in the fixed array by the first.

This file is collected last, so it also runs after every other test has used
the library in the same process.
"""

import numpy as np
import pytest
import torch

import m2synth as S
import mamba_recurrent_state_b200 as m2
from m2synth import torch_inputs as TI
from m2synth import workloads as W
from test_parity_decode import layer_objs, make_cache

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_allocating_entry_two_calls():
    # 8 heads x 2 sequences: 16 (sequence, head) pairs, so both calls split
    # every sequence into segments and use their scratch
    w = W.Workload(410, "no_alloc", 8, 64, 128, 2, 4, S.BF16, S.BF16, 8, 2, seqlen=2500, chunk=128)
    a = make_cache(w)
    b = m2.Cache(m2.Shape(w.H, w.P, w.N, w.G, w.K, w.state_dtype, w.act_dtype), w.num_slots,
                 ssm=a.ssm.clone(), conv=a.conv.clone())
    _, ssm, _ = layer_objs(w)
    lengths = [1000, 2500]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32), device="cuda")
    total = sum(lengths)
    slots = torch.tensor([6, 1], dtype=torch.int32, device="cuda")
    for call, init_list in enumerate(([1, 0], [1, 1])):  # the second call continues from the first
        d = TI.step_tensors(w, call, rows=total)
        init = torch.tensor(init_list, dtype=torch.uint8, device="cuda")
        ya = m2.chunk_scan_varlen(a, ssm, d["xBC"], d["dt"], cu, slots, max_seqlen=max(lengths), z=d["z"],
                                  has_initial_state=init)
        yb = m2.chunk_scan_varlen(b, ssm, d["xBC"], d["dt"], cu, slots, max_seqlen=max(lengths), z=d["z"],
                                  has_initial_state=init, static_scratch=True)
        torch.cuda.synchronize()
        assert torch.equal(ya, yb), f"y differs on call {call}"
        assert torch.equal(a.ssm, b.ssm), f"cache differs after call {call}"
    assert a.device_error() == 0 and b.device_error() == 0
