"""Pins for the oracle's number formats (bf16 and OCP E4M3).

The oracle's rounding is checked against torch's own dtype conversions (an
independent library routine) and against code points fixed by the OCP FP8
specification (tests/golden/e4m3_ocp_points.txt).
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_ocp_points.txt")


def _torch_bf16_bits(v32):
    return torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_matches_torch_random_and_ties():
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(200000) * np.exp2(rng.integers(-140, 120, 200000))).astype(np.float32)
    # exact ties: halfway between neighbouring bf16 values
    b = rng.integers(0, 0x7F00, 20000).astype(np.uint32)
    ties = ((b << 16) | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, -ties, np.float32([0.0, -0.0, 3.3895314e38, 3.40e38, 1e-45])])
    got = oracle.bf16_bits(v.astype(np.float64))
    assert np.array_equal(got, _torch_bf16_bits(v))


def test_e4m3_matches_torch():
    rng = np.random.default_rng(2)
    v = (rng.uniform(-1, 1, 200000) * np.exp2(rng.integers(-12, 9, 200000))).astype(np.float32)
    v = np.clip(v, -448, 448)
    # exact midpoints between all neighbouring positive codes
    vals = oracle.e4m3_to_f64(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, -mids])
    got = oracle.e4m3_bits(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_ocp_code_points():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    vals = np.array([float(r[0]) for r in rows])
    codes = np.array([int(r[1], 16) for r in rows], np.uint8)
    assert np.array_equal(oracle.e4m3_bits(vals), codes)
    exact = np.abs(vals) <= 448
    back = oracle.e4m3_to_f64(codes)
    assert np.all(np.abs(back[exact]) <= 448)


@pytest.mark.parametrize("planted", ["truncate", "ties_away"])
def test_format_pins_catch_planted_rounding_mistakes(planted):
    """The torch comparison above fails for a plausibly wrong rounding rule."""
    rng = np.random.default_rng(3)
    b = rng.integers(0, 0x7F00, 5000).astype(np.uint32)
    ties = ((b << 16) | 0x8000).view(np.float32)
    bits = ties.view(np.uint32)
    if planted == "truncate":
        wrong = (bits >> 16).astype(np.uint16)
    else:
        wrong = ((bits + 0x8000) >> 16).astype(np.uint16)
    assert not np.array_equal(wrong, _torch_bf16_bits(ties))
