"""Pins of the oracle's loss-free bias update ("GLM-4.5 Group Router", How it works:
b is updated from expert load during training at rate 0.001).  The pages give the
rate, not the rule; the oracle takes the plainest reading (b_e += rate * sign(mean
load - load_e)) and these tests fix each part of that reading: the direction, the
step size, the exact tie at the mean, what counts as load, rate 0 and the
single fp32 rounding.
"""

import numpy as np
import torch

import oracle


def test_hand_example():
    # E = 4, loads (3, 1, 0, 4) over 8 pairs: mean 2 -> signs (-, +, +, -)
    idx = np.array([[0, 1], [0, 3], [0, 3], [3, 3]], dtype=np.int32)
    b = torch.tensor([0.5, -0.25, 0.0, 1.0])
    b_new, loads = oracle.bias_update(idx, 4, 0.001, b)
    np.testing.assert_array_equal(loads, [3, 1, 0, 4])
    expect = np.array([0.5 - 0.001, -0.25 + 0.001, 0.001, 1.0 - 0.001], dtype=np.float32)
    np.testing.assert_array_equal(b_new, expect)


def test_at_the_mean_nothing_moves_and_rate_zero_is_identity():
    idx = np.tile(np.arange(8, dtype=np.int32), (3, 1))      # every expert loaded 3 times
    b = torch.randn(8, generator=torch.Generator().manual_seed(0))
    b_new, _ = oracle.bias_update(idx, 8, 0.001, b)
    np.testing.assert_array_equal(b_new, b.numpy())
    rng = np.random.default_rng(1)
    idx = rng.integers(0, 8, size=(50, 2)).astype(np.int32)
    np.testing.assert_array_equal(oracle.bias_update(idx, 8, 0.0, b)[0], b.numpy())


def test_sentinel_and_out_of_range_ids_carry_no_load():
    idx = np.array([[0, 4], [1, 9], [4, -1]], dtype=np.int32)  # E = 4: ids 4, 9, -1 count for nobody
    _, loads = oracle.bias_update(idx, 4, 0.001, torch.zeros(4))
    np.testing.assert_array_equal(loads, [1, 1, 0, 0])


def test_overloaded_down_underloaded_up_by_exactly_rate():
    rng = np.random.default_rng(2)
    E = 16
    idx = rng.integers(0, E, size=(200, 4)).astype(np.int32)
    b = torch.zeros(E)
    b_new, loads = oracle.bias_update(idx, E, 0.125, b)          # a power of two: exact steps
    mean = loads.sum() / E
    for e in range(E):
        if loads[e] > mean:
            assert b_new[e] == -0.125
        elif loads[e] < mean:
            assert b_new[e] == 0.125
        else:
            assert b_new[e] == 0.0


def test_one_fp32_rounding_of_the_sum():
    # b + rate is not representable in fp32: the result is the fp32 nearest the exact sum
    b = torch.tensor([1.0, 3.0e-8], dtype=torch.float32)
    idx = np.array([[1, 1]], dtype=np.int32)                    # expert 0 underloaded, 1 over
    b_new, _ = oracle.bias_update(idx, 2, 0.001, b)
    r = np.float32(0.001)
    assert b_new[0] == np.float32(np.float64(1.0) + np.float64(r))
    assert b_new[1] == np.float32(np.float64(np.float32(3.0e-8)) - np.float64(r))
