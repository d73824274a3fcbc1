"""The seeded input generator: determinism, slice regeneration, distributions,
storage rounding and the workload tables (host side, no GPU)."""

import numpy as np
import pytest

import m2synth as S
from m2synth import workloads as W


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0 (published reference outputs of the generator)
    w = S.words(0, 0, 3)
    assert [int(v) for v in w] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_slices_regenerate_exactly():
    key = S.stream_key(123, S.T_SSM)
    full = S.normal(key, 0, 5000, 0.0, 0.1)
    part = S.normal(key, 1234, 777, 0.0, 0.1)
    assert np.array_equal(full[1234:1234 + 777], part)


def test_normal_moments():
    x = S.normal(S.stream_key(7, 1), 0, 400000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert x.min() >= -6.0 and x.max() <= 6.0


def test_uniform_range():
    u = S.uniform(S.stream_key(8, 1), 0, 100000, 1.0, 16.0)
    assert u.min() >= 1.0 and u.max() < 16.0 and abs(u.mean() - 8.5) < 0.05


def test_streams_independent():
    a = S.normal(S.stream_key(1, S.T_XBC, 0), 0, 1000)
    b = S.normal(S.stream_key(1, S.T_XBC, 1), 0, 1000)
    c = S.normal(S.stream_key(1, S.T_Z, 0), 0, 1000)
    assert abs(np.corrcoef(a, b)[0, 1]) < 0.1 and abs(np.corrcoef(a, c)[0, 1]) < 0.1


def test_bf16_storage_round_to_nearest_even():
    x32 = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-3], dtype=np.float32)
    bits = S.f32_to_bf16_bits(x32)
    back = S.bf16_bits_to_f64(bits)
    # 1 + 2^-8 is a tie -> even (1.0); 1 + 3*2^-8 is a tie -> even (1 + 2^-6)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.015625 and back[3] == -2.5
    assert abs(back[4] - 3.0e-3) <= 2 ** -8 * 3.0e-3


def test_permutation_is_permutation():
    p = S.permutation(S.stream_key(3, S.T_SLOTS), 384)
    assert sorted(p.tolist()) == list(range(384))


@pytest.mark.parametrize("w", W.WORKLOADS, ids=lambda w: w.name)
def test_workload_tables(w):
    assert w.H % w.G == 0
    assert w.conv_dim == w.H * w.P + 2 * w.G * w.N
    slots = W.slot_indices(w)
    assert len(set(slots.tolist())) == w.batch and slots.min() >= 0 and slots.max() < w.num_slots
    p = W.layer_params(w)
    assert p.A_log.dtype == np.float32 and np.all(np.exp(p.A_log.astype(np.float64)) >= 0.999)
    assert np.all(np.exp(p.A_log.astype(np.float64)) <= 16.001)
    assert p.conv_w.shape == (w.conv_dim, w.K)


def test_workload_sizes_match_pages():
    w1 = W.WORKLOADS[1]
    assert w1.state_bytes_per_slot() == 2 * 1024 * 1024
    assert W.WORKLOADS[3].state_bytes_per_slot() == 2 * 1024 * 1024
    assert W.bytes_per_unit(w1) == 4370692 and W.param_bytes_per_launch(w1) == 103936


def test_slot_streams_take_numpy_slot_indices():
    """A slot index taken from a numpy int32 array regenerates the same state as
    a Python int, also where the element offset passes 2^31 (slot 383 of the
    Nemotron-H shape: 6 * 383 * 2^20 words)."""
    from m2synth import workloads as W
    w = W.WORKLOADS[2]
    for slot in (0, 341, 383):
        a = W.ssm_slot(w, np.int32(slot), 11)
        b = W.ssm_slot(w, slot, 11)
        assert np.array_equal(a, b)
        assert np.array_equal(W.conv_slot(w, np.int32(slot), 11), W.conv_slot(w, slot, 11))
    # the last slot is the tail of the whole-cache stream
    n = w.H * w.P * w.N
    tail = S.normal_storage(W.ssm_key(w, 11), 383 * n + n - 4, 4, 0.0, W.SSM_STD, w.state_dtype)
    assert np.array_equal(W.ssm_slot(w, np.int32(383), 11).reshape(-1)[-4:], tail)
