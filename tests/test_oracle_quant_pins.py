"""Pins of the oracle's blockwise quantizer (the fused epilogue on the rotated rows:
HARP technical summary §2.4, a drop-in preprocessing step in front of a blockwise
quantizer): hand-worked codes with ties to even, zero blocks, the block maximum at
+-127, the half-step error bound and invariance under power-of-two scaling."""
import numpy as np
import pytest

from oracle import harp_oracle as O


def test_hand_worked_block_rounds_half_to_even():
    # block maximum 127, so s = 1 and the codes are the values rounded half to even
    y = np.zeros((1, 32))
    y[0, :9] = [127.0, -63.5, 0.5, 1.5, 2.5, -2.5, 126.5, -0.49, 3.51]
    q, s = O.quantize_blocks(y, 32)
    assert s.shape == (1, 1) and s[0, 0] == 1.0
    assert q[0, :9].tolist() == [127, -64, 0, 2, 2, -2, 126, 0, 4]
    assert np.all(q[0, 9:] == 0)


def test_two_blocks_have_their_own_scales():
    y = np.concatenate([np.full(32, 0.5), np.linspace(-3.0, 2.0, 32)])[None, :]
    q, s = O.quantize_blocks(y, 32)
    assert s[0, 0] == 0.5 / 127 and s[0, 1] == 3.0 / 127
    assert np.all(q[0, :32] == 127) and q[0, 32] == -127


def test_zero_block_gives_zero_scale_and_codes():
    y = np.zeros((2, 64))
    y[1, 40] = -1e-30
    q, s = O.quantize_blocks(y, 32)
    assert s[0].tolist() == [0.0, 0.0] and s[1, 0] == 0.0 and s[1, 1] > 0
    assert np.all(q[0] == 0) and q[1, 40] == -127


@pytest.mark.parametrize("qblock", [32, 64, 128, 256])
def test_error_bound_and_extreme_codes(qblock):
    y = np.random.default_rng(qblock).standard_normal((5, 512)) * np.exp(np.linspace(-3, 3, 512))
    q, s = O.quantize_blocks(y, qblock)
    deq = q.reshape(5, -1, qblock) * s[..., None]
    yb = y.reshape(5, -1, qblock)
    assert np.all(np.abs(deq - yb) <= s[..., None] / 2 * (1 + 1e-12))
    assert np.all(np.max(np.abs(q.reshape(5, -1, qblock).astype(int)), axis=2) == 127)


def test_power_of_two_scaling_keeps_the_codes():
    y = np.random.default_rng(3).standard_normal((3, 128))
    q1, s1 = O.quantize_blocks(y, 64)
    q2, s2 = O.quantize_blocks(8.0 * y, 64)
    assert np.array_equal(q1, q2) and np.array_equal(8.0 * s1, s2)
