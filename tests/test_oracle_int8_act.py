"""Pins of the oracle's int8-activation reading (quantize_act_q8, matmul_q8act).

Each run of 32 activations becomes int8 codes with one fp32 scale:
d = amax/127, q = rint(x * (127/amax)).  The pins below fix the scale, the
rounding (half to even), the zero and tiny blocks, the block boundaries and the
final sum, so that a wrong divisor, rounding mode, block size or index fails.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle
from block_quantized_matmul_lwq_b200 import inputs


def test_integers_with_a_127_are_exact():
    # amax = 127: s = 1 and d = 1, so q = x for every integer in [-127, 127]
    g = np.random.default_rng(0)
    x = g.integers(-127, 128, size=(3, 96)).astype(np.float32)
    x[:, ::32] = 127.0
    q, d = oracle.quantize_act_q8(x)
    assert np.array_equal(q.astype(np.float32), x)
    assert np.array_equal(d, np.ones((3, 3), np.float32))


def test_round_half_to_even():
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 127.0
    x[0, 1:7] = [2.5, 3.5, -2.5, -3.5, 0.5, 1.5]
    q, _ = oracle.quantize_act_q8(x)
    assert q[0, 1:7].tolist() == [2, 4, -2, -4, 0, 2]


def test_zero_and_tiny_blocks():
    x = np.zeros((2, 64), np.float32)
    x[1, :32] = np.float32(2.0 ** -101)     # below 2^-100: a zero block
    x[1, 32] = np.float32(2.0 ** -99)       # above: quantized
    q, d = oracle.quantize_act_q8(x)
    assert not q[0].any() and not d[0].any()
    assert not q[1, :32].any() and d[1, 0] == 0
    assert q[1, 32] == 127 and d[1, 1] == np.float32(2.0 ** -99) / np.float32(127)


def test_block_boundaries_and_scales():
    # each block is scaled by its own largest |x|: a large value in block 1 leaves block 0 alone
    x = np.full((1, 64), 1.0, np.float32)
    x[0, 40] = -1000.0
    q, d = oracle.quantize_act_q8(x)
    assert (q[0, :32] == 127).all()
    assert d[0, 0] == np.float32(1) / np.float32(127)
    assert q[0, 40] == -127 and d[0, 1] == np.float32(1000) / np.float32(127)
    assert (q[0, 32:40] == 0).all()          # 1/1000 * 127 = 0.127 rounds to 0


@pytest.mark.parametrize("act", ["f32", "f16", "bf16"])
def test_round_trip_bound_and_extremes(act):
    x = inputs.activations(inputs.rng(3), 4, 1024, act)
    q, d = oracle.quantize_act_q8(x, act=act)
    xf = oracle.activations_f32(x, act).astype(np.float64)
    dq = q.astype(np.float64) * np.repeat(d.astype(np.float64), 32, axis=1)
    # |x - q d| <= d/2 + |x| |1 - s d| + d |fl(x s) - x s|: s and d are correctly rounded
    # quotients and |x| <= 127 d, so the last two terms stay below 2^-14 d
    bound = np.repeat(d.astype(np.float64), 32, axis=1) * (0.5 + 2.0 ** -14)
    assert (np.abs(xf - dq) <= bound).all()
    # the largest |x| of every block maps to +-127
    blk = np.abs(q.reshape(4, 32, 32)).max(axis=2)
    assert (blk == 127).all()


def test_power_of_two_scaling_keeps_codes():
    x = inputs.activations(inputs.rng(4), 2, 256, "f32")
    q1, d1 = oracle.quantize_act_q8(x)
    q2, d2 = oracle.quantize_act_q8((x * np.float32(2.0 ** -7)).astype(np.float32))
    assert np.array_equal(q1, q2) and np.array_equal(d2, d1 * np.float32(2.0 ** -7))


@pytest.mark.parametrize("fmt", ["q4_0", "q8_0", "q4_k"])
def test_matmul_brute_force_one_block(fmt):
    # K = one weight block; sums written out element by element, independent of the matmul primitive
    K = 256 if fmt == "q4_k" else 32
    M, N = 2, 3
    Wq, x = inputs.make_problem(fmt, "f32", M, N, K, seed=9)
    y, den = oracle.matmul_q8act(fmt, Wq, x)
    W = oracle.dequant(fmt, Wq, K)
    q, d = oracle.quantize_act_q8(x)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            ab = 0.0
            for k in range(K):
                v = float(W[n, k]) * int(q[m, k]) * float(d[m, k // 32])
                acc += v
                ab += abs(v)
            assert abs(y[m, n] - acc) <= 1e-12 * max(1.0, ab)
            assert abs(den[m, n] - ab) <= 1e-12 * max(1.0, ab)


def test_matmul_close_to_exact_product():
    # quantizing N(0,1) activations to 8 bits moves the product by far less than 1e-2 of sum |x w|
    Wq, x = inputs.make_problem("q4_0", "f32", 4, 64, 4096, seed=5)
    y8, _ = oracle.matmul_q8act("q4_0", Wq, x)
    y, den = oracle.matmul("q4_0", Wq, x)
    assert oracle.normalised_error(y8, y, den) < 1e-2
