"""Planted mistakes in the oracle's int8-activation reading must each fail a pin.

Each mutant replaces oracle.quantize_act_q8 (or matmul_q8act) with a plausible
wrong version; the pins of test_oracle_int8_act run against it and at least
one must fail.  The mistakes are planted in the oracle, on the CPU.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import test_oracle_int8_act as pins

_real_quantize = oracle.quantize_act_q8


def _quantizer(block=32, div=127.0, rnd=np.rint, tiny=2.0 ** -100, axis_k=True):
    def q(x, act=None):
        xf = oracle.activations_f32(x, act)
        M, K = xf.shape
        blk = xf.reshape(M, K // block, block) if axis_k else xf.T.reshape(K, M // block, block)
        amax = np.max(np.abs(blk), axis=2)
        small = amax < np.float32(tiny)
        safe = np.where(small, np.float32(1), amax)
        d = np.where(small, np.float32(0), amax / np.float32(div)).astype(np.float32)
        s = np.where(small, np.float32(0), np.float32(div) / safe).astype(np.float32)
        with np.errstate(invalid="ignore", over="ignore"):   # a mutant may divide by zero
            qq = np.clip(np.nan_to_num(rnd((blk * s[:, :, None]).astype(np.float32))), -127, 127).astype(np.int8)
        if not axis_k:
            return qq.reshape(K, M).T.copy(), d.T.copy()
        if block != 32:   # report scales per 32 as the real function does (first sub-block's)
            d = d.reshape(M, K // 32, 32 // block)[:, :, 0]
        return qq.reshape(M, K), d
    return q


def _half_away(v):
    return np.sign(v) * np.floor(np.abs(v) + 0.5)


def _matmul_unquantized(fmt, Wq, x, K=None, act=None, lib=None):
    return oracle.matmul(fmt, Wq, x, K=K, act=act)


MUTANTS = {
    "round half away from zero": dict(quantize=_quantizer(rnd=_half_away)),
    "divisor 128": dict(quantize=_quantizer(div=128.0)),
    "blocks of 16": dict(quantize=_quantizer(block=16)),
    "no tiny-block threshold": dict(quantize=_quantizer(tiny=0.0)),
    "truncation": dict(quantize=_quantizer(rnd=np.trunc)),
    "matmul on the unquantized x": dict(matmul=_matmul_unquantized),
}

PINS = [
    pins.test_integers_with_a_127_are_exact,
    pins.test_round_half_to_even,
    pins.test_zero_and_tiny_blocks,
    pins.test_block_boundaries_and_scales,
    lambda: pins.test_round_trip_bound_and_extremes("f32"),
    pins.test_power_of_two_scaling_keeps_codes,
    lambda: pins.test_matmul_brute_force_one_block("q4_0"),
]


@pytest.mark.parametrize("name", list(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    m = MUTANTS[name]
    if "quantize" in m:
        monkeypatch.setattr(oracle, "quantize_act_q8", m["quantize"])
    if "matmul" in m:
        monkeypatch.setattr(oracle, "matmul_q8act", m["matmul"])
    failed = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed.append(pin)
    assert failed, f"no pin caught the mutant: {name}"


def test_pins_pass_on_the_real_oracle():
    assert oracle.quantize_act_q8 is _real_quantize
    for pin in PINS:
        pin()
