"""Chunked prefill scan against the oracle's definition (T sequential updates
with the working state unrounded until the end), the T = 1 equivalence with
the decode step, and the prefill-then-decode workload (8 x 2048 tokens, then
32 decode steps continuing from the scanned state)."""

from concurrent.futures import ThreadPoolExecutor

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
from test_parity_decode import layer_objs, make_cache, shape_of

pytestmark = pytest.mark.gpu


def wl(index, H=8, G=2, sd=S.BF16, ad=S.BF16, N=128, batch=3, slots=6, T=37, chunk=16):
    return W.Workload(index, f"scan{index}", H, 64, N, G, 4, sd, ad, slots, batch, seqlen=T,
                      chunk=chunk)


def prefill_inputs(w, xdtype=None):
    """Post-conv inputs are drawn directly here (the scan takes post-conv xBC)."""
    rows = w.batch * w.seqlen
    d = TI.step_tensors(w, 0, rows=rows)
    x = d["xBC"] if xdtype is None else d["xBC"].to(xdtype)
    return (x.view(w.batch, w.seqlen, -1), d["dt"].view(w.batch, w.seqlen, -1),
            d["z"].view(w.batch, w.seqlen, -1))


def oracle_scan_row(ol, w, b, s, init: bool, x_code, with_z: bool = True):
    rows = np.arange(b * w.seqlen, (b + 1) * w.seqlen)
    xbc = f64(W.step_rows(w, T_XBC, 0, rows), w.act_dtype)
    if x_code != w.act_dtype:  # xBC handed over in another precision
        mode = {S.F32: O.ROUND_F32, S.BF16: O.ROUND_BF16, S.F16: O.ROUND_F16}[x_code]
        xbc = ol.orc.round_array(xbc, mode)
    dt = f64(W.step_rows(w, T_DT, 0, rows), w.act_dtype)
    z = f64(W.step_rows(w, T_Z, 0, rows), w.act_dtype) if with_z else None
    state = ol.initial_ssm(s) if init else np.zeros((w.H, w.P, w.N))
    y = ol.orc.ssm_scan(state, O.round_mode_for(w.state_dtype), xbc, dt, ol.dt_bias, ol.A_log,
                        ol.D, z, w.G)
    return state, y


@pytest.mark.parametrize("w", [
    wl(300),
    wl(301, T=1),
    wl(302, T=200, chunk=64),
    wl(303, sd=S.F32, ad=S.BF16, T=50),
    wl(304, sd=S.F32, ad=S.F32, T=20, N=64),
    wl(305, H=16, G=16, T=33, batch=2),
], ids=lambda w: f"H{w.H}G{w.G}N{w.N}s{w.state_dtype}a{w.act_dtype}T{w.seqlen}")
def test_scan_small(w):
    cache = make_cache(w)
    ssm0 = cache.ssm.clone()
    t, ssm, _ = layer_objs(w)
    slot_list = [5, -1, 2][: w.batch]
    init_list = [1, 0, 0][: w.batch]
    slots = torch.tensor(slot_list, dtype=torch.int32, device="cuda")
    init = torch.tensor(init_list, dtype=torch.uint8, device="cuda")
    x, dt, z = prefill_inputs(w)
    y = m2.chunk_scan(cache, ssm, x, dt, slots, z=z, chunk_size=w.chunk, has_initial_state=init)
    torch.cuda.synchronize()
    ol = OracleLayer(w)
    for b, s in enumerate(slot_list):
        if s < 0:
            assert torch.count_nonzero(y[b]) == 0
            continue
        state, y_ref = oracle_scan_row(ol, w, b, s, bool(init_list[b]), w.act_dtype)
        assert_close(f64(TI.to_storage_np(y[b]), w.act_dtype), y_ref, w.act_dtype, f"y row {b}")
        assert_close(f64(TI.to_storage_np(cache.ssm[s]), w.state_dtype), state, w.state_dtype,
                     f"final state row {b}")
    keep = [q for q in range(w.num_slots) if q not in slot_list]
    assert torch.equal(cache.ssm[keep], ssm0[keep])
    assert cache.device_error() == 0


@pytest.mark.parametrize("xdt,code,T", [(torch.float32, S.F32, 24), (torch.float16, S.F16, 24),
                                       (torch.float16, S.F16, 300)], ids=["f32", "f16", "f16_T300"])
def test_scan_other_xbc_dtypes(xdt, code, T):
    """Post-conv xBC handed over in fp32 (CUDA-core scan) or fp16 (tensor-core
    scan, used as loaded)."""
    w = wl(306 + T, T=T)
    cache = make_cache(w)
    t, ssm, _ = layer_objs(w)
    slots = torch.tensor([0, 3, 4], dtype=torch.int32, device="cuda")
    x, dt, z = prefill_inputs(w, xdtype=xdt)
    y = m2.chunk_scan(cache, ssm, x, dt, slots, z=z)
    torch.cuda.synchronize()
    ol = OracleLayer(w)
    for b, s in enumerate([0, 3, 4]):
        state, y_ref = oracle_scan_row(ol, w, b, s, False, code)
        assert_close(f64(TI.to_storage_np(y[b]), w.act_dtype), y_ref, w.act_dtype, "y")
        assert_close(f64(TI.to_storage_np(cache.ssm[s]), w.state_dtype), state, w.state_dtype, "S")


@pytest.mark.parametrize("xdt,code,T", [(None, S.BF16, 300), (torch.float16, S.F16, 300),
                                       (torch.float32, S.F32, 40)],
                         ids=["bf16_tensor_core", "f16_pipelined", "f32_cuda_core"])
def test_scan_without_gate(xdt, code, T):
    """z = NULL: y is the ungated scan output, on each scan kernel (bf16 input:
    the single-chain tensor-core kernel; fp16: the pipelined one; fp32: the
    CUDA-core scan), with and without an initial state."""
    w = wl(330 + T, T=T)
    cache = make_cache(w)
    t, ssm, _ = layer_objs(w)
    slot_list, init_list = [1, 2, 5], [1, 0, 1]
    slots = torch.tensor(slot_list, dtype=torch.int32, device="cuda")
    init = torch.tensor(init_list, dtype=torch.uint8, device="cuda")
    x, dt, _ = prefill_inputs(w, xdtype=xdt)
    y = m2.chunk_scan(cache, ssm, x, dt, slots, has_initial_state=init)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    ol = OracleLayer(w)
    for b, s in enumerate(slot_list):
        state, y_ref = oracle_scan_row(ol, w, b, s, bool(init_list[b]), code, with_z=False)
        assert_close(f64(TI.to_storage_np(y[b]), w.act_dtype), y_ref, w.act_dtype, f"y row {b}")
        assert_close(f64(TI.to_storage_np(cache.ssm[s]), w.state_dtype), state, w.state_dtype,
                     f"final state row {b}")


@pytest.mark.parametrize("G", [1, 8])
def test_scan_T1_equals_state_update(G):
    """A one-token scan from the cached state equals one decode step on the
    same post-conv input (including n_groups = 8), state and y within the bf16
    tolerance (the scan's tensor-core path forms its state increment from bf16
    MMA operands, the decode step element by element in fp32)."""
    w = W.Workload(310 + G, "t1", 128, 64, 128, G, 4, S.BF16, S.BF16, 16, 8, seqlen=1)
    a = make_cache(w)
    b = m2.Cache(shape_of(w), w.num_slots, ssm=a.ssm.clone(), conv=a.conv.clone())
    t, ssm, _ = layer_objs(w)
    x, dt, z = prefill_inputs(w)
    ones = torch.ones(w.batch, dtype=torch.uint8, device="cuda")
    y_scan = m2.chunk_scan(a, ssm, x, dt, t["slots"], z=z, chunk_size=128, has_initial_state=ones)
    y_dec = m2.state_update(b, ssm, x[:, 0], dt[:, 0], t["slots"], z=z[:, 0])
    torch.cuda.synchronize()
    rows = t["slots"].long()
    es = rel_err(f64(TI.to_storage_np(a.ssm[rows]), S.BF16), f64(TI.to_storage_np(b.ssm[rows]), S.BF16))
    assert es <= TOL[S.BF16], es
    others = [q for q in range(w.num_slots) if q not in rows.tolist()]
    assert torch.equal(a.ssm[others], b.ssm[others])
    e = rel_err(f64(TI.to_storage_np(y_scan[:, 0]), S.BF16), f64(TI.to_storage_np(y_dec), S.BF16))
    assert e <= TOL[S.BF16], e


# Bound of the fully chained workload-4 comparisons: the GPU's prefill and 32
# decode steps against the oracle's own prefill and 32 decode steps, the oracle
# never seeing a GPU value. Two effects put these above the per-kernel bf16
# bound of 2e-2:
#  * the prefill leaves the stored state one bf16 unit in the last place
#    (2^-8..2^-7 of the value) away from the oracle's in places, and those
#    differences are correlated along n (they come from the same fp16 operands
#    of one chunk), so y, a 128-term sum over n, can move by several of its own
#    units;
#  * the recurrence carries an absolute state difference forward (times
#    dA <= 1) while the element itself can shrink under the decode inputs, so
#    the difference reads larger relative to the element at the end than at
#    the start, and both sides keep rounding the state to bf16 at every step.
# Measured on this workload: 3.7e-2 on the decode y and 3.2e-2 on the final
# state; the bound is 5e-2. Measured against the larger of the element's size
# at the start of the decode chain and at its end (rel_err_carried below), which
# removes the second effect, the final state differs by 2.1e-2 (about three
# bf16 units in the last place); that figure is printed, not asserted.
CHAIN_TOL = 5e-2


def rel_err_carried(a, r, r0) -> float:
    """max_i |a_i - r_i| / max(|r_i|, |r0_i|, rms(r)): a difference carried
    from the start of a decode chain (r0) is measured against the element's
    size at the start as well as at the end."""
    a, r, r0 = (np.asarray(v, dtype=np.float64).ravel() for v in (a, r, r0))
    rms = float(np.sqrt(np.mean(r * r)))
    denom = np.maximum(np.maximum(np.abs(r), np.abs(r0)), rms if rms > 0 else 1.0)
    return float(np.max(np.abs(a - r) / denom))


def test_workload4_prefill_then_decode():
    """Zero initial state; prefill conv over 2048 tokens (fp16 post-conv buffer),
    chunk scan, then 32 fused decode steps continuing from the scanned state.
    Every y and the states of all 8 sequences are checked three ways:

    * chained, as the equivalence contract words it: the oracle runs the plain
      definition -- the conv output in double (no fp16 buffer) straight into
      2048 sequential updates, the state rounded once to bf16 at the end, then
      32 decode steps from that state, each rounding the stored state -- and
      never sees a GPU value; the GPU's prefill y and state are held to that
      trajectory at the bf16 bound, its 32 decode y and final state at
      CHAIN_TOL;
    * per kernel, on the kernels' own inputs: the prefill against the oracle
      run on the fp16-rounded conv output the scan actually reads, and each
      decode step against the oracle continued from the state the prefill
      stored (bf16, exact) and the conv cache it left;
    * the conv cache bit for bit."""
    w = W.WORKLOADS[4]
    cache = make_cache(w)
    t, ssm, conv = layer_objs(w)
    cache.zero_slots(t["slots"])
    T = w.seqlen
    d = TI.step_tensors(w, 0, rows=w.batch * T)
    xr = d["xBC"].view(w.batch, T, -1)
    xp = m2.conv1d_update(cache, conv, xr, t["slots"], out_dtype=torch.float16)
    y_pre = m2.chunk_scan(cache, ssm, xp, d["dt"].view(w.batch, T, -1), t["slots"],
                          z=d["z"].view(w.batch, T, -1), chunk_size=w.chunk)
    state_after_prefill = TI.to_storage_np(cache.ssm[t["slots"].long()])
    y_dec = []
    for step in range(1, w.decode_after + 1):
        inp = TI.step_tensors(w, step)
        y_dec.append(m2.state_update(cache, ssm, inp["xBC"], inp["dt"], t["slots"], z=inp["z"],
                                     conv=conv))
    torch.cuda.synchronize()
    y_pre_np = TI.to_storage_np(y_pre)
    y_dec_np = np.stack([TI.to_storage_np(y) for y in y_dec])
    ssm_np = TI.to_storage_np(cache.ssm)
    conv_np = TI.to_storage_np(cache.conv)
    ol = OracleLayer(w)

    def decode_step(state, conv_state, step, b):
        inp = ol.inputs(step, [b])
        return O.decode_rows(ol.orc, w.H, w.P, w.N, w.G, O.ROUND_BF16, [state], [conv_state],
                             inp["xBC"], inp["dt"], inp["z"], ol.conv_w, ol.conv_b, ol.dt_bias,
                             ol.A_log, ol.D, threads=1)

    def one(b):
        s = int(ol.slots[b])
        rows = np.arange(b * T, (b + 1) * T)
        conv_state = np.zeros((w.K - 1, w.conv_dim))
        xraw = f64(W.step_rows(w, T_XBC, 0, rows), w.act_dtype)
        xpost = ol.orc.conv1d(conv_state, xraw, ol.conv_w, ol.conv_b, 1)
        dt = f64(W.step_rows(w, T_DT, 0, rows), w.act_dtype)
        z = f64(W.step_rows(w, T_Z, 0, rows), w.act_dtype)
        # the plain definition: unrounded conv output, 2048 sequential updates
        chained = np.zeros((w.H, w.P, w.N))
        y_plain = ol.orc.ssm_scan(chained, O.ROUND_BF16, xpost, dt, ol.dt_bias, ol.A_log, ol.D, z, w.G)
        # the scan's own input: the fp16 buffer between the two launches
        state16 = np.zeros((w.H, w.P, w.N))
        y16 = ol.orc.ssm_scan(state16, O.ROUND_BF16, ol.orc.round_array(xpost, O.ROUND_F16), dt,
                              ol.dt_bias, ol.A_log, ol.D, z, w.G)
        gpu_pre_state = f64(state_after_prefill[b], w.state_dtype)
        errs = {"prefill_y": rel_err(f64(y_pre_np[b], w.act_dtype), y16),
                "prefill_state": rel_err(gpu_pre_state, state16),
                "plain_prefill_y": rel_err(f64(y_pre_np[b], w.act_dtype), y_plain),
                "plain_prefill_state": rel_err(gpu_pre_state, chained)}
        chain_start = chained.copy()
        dstate = np.ascontiguousarray(gpu_pre_state)  # per kernel: from the stored GPU state
        dconv = conv_state.copy()
        cconv = conv_state.copy()                     # chained: the oracle's own conv cache
        dec, chain = [], []
        for step in range(1, w.decode_after + 1):
            yd = decode_step(dstate, dconv, step, b)
            yc = decode_step(chained, cconv, step, b)
            g = f64(y_dec_np[step - 1][b], w.act_dtype)
            dec.append(rel_err(g, yd))
            chain.append(rel_err(g, yc))
        gpu_final = f64(ssm_np[s], w.state_dtype)
        errs["decode_y"] = max(dec)
        errs["final_state"] = rel_err(gpu_final, dstate)
        errs["chained_decode_y"] = max(chain)
        errs["chained_final_state"] = rel_err(gpu_final, chained)
        errs["chained_final_state_carried"] = rel_err_carried(gpu_final, chained, chain_start)
        errs["conv_exact"] = bool(np.array_equal(conv_np[s], S.to_storage(cconv, w.act_dtype)))
        return errs

    with ThreadPoolExecutor(max_workers=8) as ex:
        results = list(ex.map(one, range(w.batch)))
    keys = [k for k in results[0] if k != "conv_exact"]
    print("workload 4, max over the 8 sequences:",
          {k: float(f"{max(r[k] for r in results):.3e}") for k in keys})
    for b, e in enumerate(results):
        assert e["prefill_y"] <= TOL[S.BF16], (b, e)
        assert e["prefill_state"] <= TOL[S.BF16], (b, e)
        assert e["plain_prefill_y"] <= TOL[S.BF16], (b, e)
        assert e["plain_prefill_state"] <= TOL[S.BF16], (b, e)
        assert e["decode_y"] <= TOL[S.BF16], (b, e)
        assert e["final_state"] <= TOL[S.BF16], (b, e)
        assert e["chained_decode_y"] <= CHAIN_TOL, (b, e)
        assert e["chained_final_state"] <= CHAIN_TOL, (b, e)
        assert e["conv_exact"], (b, e)
    assert cache.device_error() == 0


def test_scan_operand_range_error_is_reported():
    """A value beyond the fp16 range of the tensor-core scan's operands sets
    M2_ERR_RANGE in the error word (the launch itself completes normally)."""
    w = wl(320, H=8, G=2, T=64, batch=1, slots=2)
    cache = make_cache(w)
    t, ssm, _ = layer_objs(w)
    x, dt, z = prefill_inputs(w)
    x = x.clone()
    x[0, 5, 3] = 1.0e5  # an x channel of head 0
    slots = torch.tensor([1], dtype=torch.int32, device="cuda")
    m2.chunk_scan(cache, ssm, x, dt, slots, z=z)
    assert cache.device_error() == m2.M2_ERR_RANGE
    x[0, 5, 3] = 1.0
    m2.chunk_scan(cache, ssm, x, dt, slots, z=z)
    assert cache.device_error() == 0
