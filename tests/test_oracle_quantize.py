"""Pins for the oracle's block-128 E4M3 quantiser (S2).

Definition ("Supporting MegaKernel for DeepSeek Models", layer table,
bf16_to_fp8_quantize): per block of 128 values an E4M3 code per value and one
power-of-two (ue8m0) scale.  Reading: scale = smallest power of two with
amax/scale <= 448, code = E4M3_RNE_sat(x / scale).
Checked by properties that pin it (power of two, fits, minimal) and by
torch's float8_e4m3fn conversion of x/scale (library routine).
"""
import numpy as np
import torch

import oracle


def _bits(x32):
    return torch.from_numpy(np.asarray(x32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _check(xb):
    q, s = oracle.quantize_fp8_block128(xb)
    x = oracle.bf16_to_f64(xb)
    rows, cols = x.shape
    blocks = x.reshape(rows, cols // 128, 128)
    amax = np.abs(blocks).max(-1)
    s64 = s.astype(np.float64)
    m, e = np.frexp(s64)
    assert np.all(m == 0.5)                                      # power of two
    assert np.all(amax / s64 <= 448)                             # fits
    nz = amax > 0
    assert np.all((amax / (s64 / 2) > 448)[nz & (s64 > 2.0 ** -127)])   # minimal
    assert np.all(s64[~nz] == 1.0)
    ref = torch.from_numpy((blocks / s64[..., None]).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(q.reshape(rows, cols // 128, 128), ref.view(torch.uint8).numpy())
    return q, s


def test_random_rows():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((37, 1024)) * np.exp2(rng.integers(-20, 20, (37, 1)))
    _check(_bits(x))


def test_boundaries():
    blk = np.zeros((6, 128), np.float32)
    blk[0, 5] = 448.0          # s = 1
    blk[1, 0] = 449.0          # bf16(449) = 448 -> s = 1
    blk[2, 0] = 452.0          # s = 2
    blk[3, 7] = 224.0          # s = 0.5
    blk[4, 1] = -225.0         # s = 1
    blk[5, :] = 0.0            # all zero -> s = 1, q = 0
    q, s = _check(_bits(blk.reshape(1, -1)))
    assert list(s[0]) == [1.0, 1.0, 2.0, 0.5, 1.0, 1.0]
    assert q[0, 5] == 0x7E and q[0, 3 * 128 + 7] == 0x7E and q[0, 4 * 128 + 1] == 0xF6
    assert np.all(q[0, 5 * 128:] == 0)


def test_negative_zero_keeps_sign_and_tiny_values():
    x = np.zeros((1, 128), np.float32)
    x[0, 0] = -0.0
    x[0, 1] = 1e-30
    x[0, 2] = -3e-31
    q, s = _check(_bits(x))
    assert q[0, 0] == 0x80


def test_roundtrip_error_bound():
    rng = np.random.default_rng(5)
    xb = _bits(rng.standard_normal((16, 512)))
    q, s = oracle.quantize_fp8_block128(xb)
    x = oracle.bf16_to_f64(xb)
    deq = oracle.e4m3_to_f64(q) * np.repeat(s.astype(np.float64), 128, axis=1)
    # relative error of a normal E4M3 value is at most 2^-4 (3 mantissa bits)
    big = np.abs(deq) >= np.repeat(s, 128, axis=1) * 2.0 ** -6
    assert np.all(np.abs(x - deq)[big] <= np.abs(x[big]) * 2.0 ** -4 + 1e-300)
