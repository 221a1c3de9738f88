"""Pins of the oracle's MXFP4-weight forward (FP8 activations x packed FP4
routed weights: GC MoE issue on the DeepGEMM tracker, DeepGEMM Mega MoE news;
MXFP4 = OCP Microscaling: E2M1 elements, one E8M0 scale per 32):

- dequantisation of every code and scale equals an independent route: each
  E2M1 code is re-encoded bit by bit as the E4M3 code of the same value and
  decoded by torch's float8_e4m3fn, times 2^(scale-127) (numpy ldexp), with
  the block layout of the scales written out as loops;
- the forward equals the already pinned E4M3 forward, bit for bit, on the
  same real weights expressed as E4M3 codes with per-(row,128) power-of-two
  scales (torch's E4M3 conversion, exact by construction);
- planted mistakes (nibbles swapped, scales read in plain row order) are
  caught by that equality;
- the offline MXFP4 quantiser of the input recipe keeps the OCP bound."""
import numpy as np
import torch

import oracle
from mixture_experts_routed_expert_b200 import inputs


def _e2m1_as_e4m3_code(nib):
    """E2M1 code -> the E4M3 code of the same value, by fields: exponent
    e > 0 is 2^(e-1)(1 + m/2) -> E4M3 exponent e - 1 + 7, mantissa m << 2;
    e = 0 is 0.5 m -> 0 or 2^-1 (E4M3 exponent 6)."""
    s, e, m = (nib >> 3) & 1, (nib >> 1) & 3, nib & 1
    if e > 0:
        code = ((e + 6) << 3) | (m << 2)
    else:
        code = (6 << 3) if m else 0
    return (s << 7) | code


def _e2m1_values():
    codes = torch.tensor([_e2m1_as_e4m3_code(n) for n in range(16)], dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _blocked_index(r, c, C):
    blk = (r // 128) * (C // 128) + c // 128
    return blk * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 128) // 32


def _random_mxf4(rng, R, C, exp_lo, exp_hi):
    codes = rng.integers(0, 16, (R, C)).astype(np.uint8)
    plain = rng.integers(exp_lo, exp_hi + 1, (R, C // 32)).astype(np.uint8)   # E8M0 bytes
    blocked = np.empty(R * C // 32, np.uint8)
    for r in range(R):
        for j in range(C // 32):
            blocked[_blocked_index(r, 32 * j, C)] = plain[r, j]
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return codes, plain, blocked, packed


def test_dequant_matches_field_reencoding():
    rng = np.random.default_rng(0)
    R, C = 256, 384
    codes, plain, blocked, packed = _random_mxf4(rng, R, C, 100, 150)
    vals = _e2m1_values()
    expect = vals[codes] * np.ldexp(1.0, plain.astype(np.int64) - 127).repeat(32, axis=1)
    got = oracle.mxf4_dequant(packed, blocked, R, C)
    assert np.array_equal(got, expect)
    # the eight magnitudes of the OCP table, from torch's E4M3 decoding
    assert sorted(set(np.abs(vals).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    # E8M0 255 is NaN
    blocked2 = blocked.copy()
    blocked2[_blocked_index(5, 64, C)] = 255
    d = oracle.mxf4_dequant(packed, blocked2, R, C)
    assert np.isnan(d[5, 64:96]).all() and not np.isnan(d[5, :64]).any()


def _as_fp8(codes, plain, R, C):
    """Same real values as E4M3 codes with a power-of-two scale per (row,128):
    the block's largest E8M0 exponent; sub-blocks at most 8 binades lower stay
    exact in E4M3 (E2M1 magnitudes >= 2^-1 land at >= 2^-9)."""
    vals = _e2m1_values()
    smax = plain.reshape(R, C // 128, 4).max(axis=2).astype(np.int64)           # [R, C/128]
    rel = plain.astype(np.int64) - smax.repeat(4, axis=1)                        # [R, C/32] <= 0
    v = vals[codes] * np.ldexp(1.0, rel).repeat(32, axis=1)
    q = torch.from_numpy(v).to(torch.float8_e4m3fn)
    assert np.array_equal(q.to(torch.float64).numpy(), v)                       # exact
    return q.view(torch.uint8).numpy(), np.ldexp(1.0, smax - 127).astype(np.float32)


def _layer(rng, T, H, F, E, K, planted=None):
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30))))
    x = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    mx = {"w13": [], "w13s": [], "w2": [], "w2s": []}
    f8 = {"w13": [], "w13s": [], "w2": [], "w2s": []}
    for _ in range(E):
        for name, (R, C) in (("w13", (2 * F, H)), ("w2", (H, F))):
            # exponents around 2^-7 (weights ~0.02); a 128-block spans <= 8 binades
            codes, plain, blocked, packed = _random_mxf4(rng, R, C, 116, 124)
            if planted == "nibbles":
                packed = (codes[:, 1::2] | (codes[:, 0::2] << 4)).astype(np.uint8)
            if planted == "plain_scales":
                blocked = plain.reshape(-1).copy()
            mx[name].append(packed)
            mx[name + "s"].append(blocked)
            q, s = _as_fp8(codes, plain, R, C)
            f8[name].append(q)
            f8[name + "s"].append(s)
    idx = rng.integers(-1, E, (T, K)).astype(np.int32)
    w = rng.uniform(0.1, 1.0, (T, K)).astype(np.float32)
    mx = {k: np.stack(v) for k, v in mx.items()}
    f8 = {k: np.stack(v) for k, v in f8.items()}
    return x, mx, f8, idx, w


def test_forward_equals_fp8_forward_on_same_values():
    rng = np.random.default_rng(1)
    x, mx, f8, idx, w = _layer(rng, 5, 256, 256, 3, 2)
    a = oracle.moe_forward_mxf4(x, mx["w13"], mx["w13s"], mx["w2"], mx["w2s"], idx, w)
    b = oracle.moe_forward_fp8(x, f8["w13"], f8["w13s"], f8["w2"], f8["w2s"], idx, w)
    assert np.array_equal(a, b)
    assert np.abs(oracle.bf16_to_f64(a)).max() > 0


def test_planted_mistakes_are_caught():
    for planted in ("nibbles", "plain_scales"):
        rng = np.random.default_rng(2)
        x, mx, f8, idx, w = _layer(rng, 4, 256, 256, 2, 2, planted=planted)
        a = oracle.moe_forward_mxf4(x, mx["w13"], mx["w13s"], mx["w2"], mx["w2s"], idx, w)
        b = oracle.moe_forward_fp8(x, f8["w13"], f8["w13s"], f8["w2"], f8["w2s"], idx, w)
        assert not np.array_equal(a, b), planted


def test_input_quantiser_ocp_bound():
    """Offline MXFP4 quantisation (input recipe): the shared exponent is
    floor(log2 amax) - 2, and every element is the nearest E2M1 value of
    w / 2^X below the saturation point 6."""
    g = torch.Generator().manual_seed(3)
    wf = torch.randn(256, 256, generator=g) * 0.02
    q, sc = inputs.quantize_weight_mxf4(wf)
    d = oracle.mxf4_dequant(q.numpy(), sc.numpy(), 256, 256)
    blk = wf.double().reshape(256, 8, 32)
    X = torch.floor(torch.log2(blk.abs().amax(-1))) - 2
    step = torch.exp2(X).unsqueeze(-1).expand_as(blk)
    err = (torch.from_numpy(d).reshape(256, 8, 32) - blk).abs()
    sat = blk.abs() > 6 * step
    # half the E2M1 spacing: 0.25 below 2, 0.5 in [2, 4), 1 in [4, 6] (units of 2^X)
    a = blk.abs() / step
    half = torch.where(a < 2, 0.25, torch.where(a < 4, 0.5, 1.0)) * step
    assert (err[~sat] <= half[~sat] + 1e-15).all()
    assert (torch.from_numpy(d).reshape(256, 8, 32).abs()[sat] == (6 * step)[sat]).all()
