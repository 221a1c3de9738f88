"""Pins for the oracle's routed-experts forward (bf16 and FP8 variants).

Definition ("deepseek-ocr2-moe-experts" model card, description + "Usage"):
out[t] = sum_k w[t,k] * down_e(SiLU(gate_e x_t) * (up_e x_t)), gate_up_proj
[E,2F,H] with gate rows first, down_proj [E,H,F].  Pinned by: the dense
special case (E=1, K=1) against torch float64 matmuls; invariants I1-I4 from
the definition; out-of-range ids; an independent pure-Python brute force.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import brute

BF = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
F64 = oracle.bf16_to_f64


def _layer(rng, T, H, F, E, K):
    x = BF(rng.standard_normal((T, H)))
    gu = BF(rng.standard_normal((E, 2 * F, H)) * 0.05)
    dn = BF(rng.standard_normal((E, H, F)) * 0.05)
    idx = rng.integers(0, E, (T, K)).astype(np.int32)
    w = rng.uniform(0.05, 1.0, (T, K)).astype(np.float32)
    return x, gu, dn, idx, w


def _dense_ref(x, gu, dn, wscale=1.0, swap=False, no_silu=False, transpose_down=False):
    F = gu.shape[1] // 2
    X = torch.from_numpy(F64(x))
    G = torch.from_numpy(F64(gu[0, :F])); U = torch.from_numpy(F64(gu[0, F:]))
    if swap:
        G, U = U, G
    D = torch.from_numpy(F64(dn[0]))
    if transpose_down:
        D = D.T
    g = X @ G.T; u = X @ U.T
    h = (g if no_silu else torch.nn.functional.silu(g)) * u
    h = torch.from_numpy(F64(oracle.bf16_bits(h.numpy())))
    return oracle.bf16_bits((wscale * (h @ D.T)).numpy())


def _ulps(a, b):
    return np.abs(a.astype(np.int32) - b.astype(np.int32))


def test_dense_special_case_bf16():
    rng = np.random.default_rng(0)
    x, gu, dn, _, _ = _layer(rng, 8, 128, 96, 1, 1)
    for wscale in (1.0, 0.37):
        out = oracle.moe_forward_bf16(x, gu, dn, np.zeros((8, 1), np.int32),
                                      np.full((8, 1), wscale, np.float32))
        ref = _dense_ref(x, gu, dn, wscale)
        d = _ulps(out, ref)
        assert d.max() <= 1 and (d == 0).mean() > 0.99


@pytest.mark.parametrize("mistake", ["swap", "no_silu", "transpose_down"])
def test_dense_pin_catches_planted_mistakes(mistake):
    rng = np.random.default_rng(1)
    x, gu, dn, _, _ = _layer(rng, 4, 64, 64, 1, 1)
    out = oracle.moe_forward_bf16(x, gu, dn, np.zeros((4, 1), np.int32), np.ones((4, 1), np.float32))
    wrong = _dense_ref(x, gu, dn, **{mistake: True})
    assert (_ulps(out, wrong) > 1).mean() > 0.5


def test_invariants_bf16():
    rng = np.random.default_rng(2)
    T, H, F, E, K = 6, 128, 64, 5, 4
    x, gu, dn, idx, w = _layer(rng, T, H, F, E, K)
    base = oracle.moe_forward_bf16(x, gu, dn, idx, w)
    # I1: all K slots on one expert == (sum w) * expert(x)
    one = np.full((T, K), 3, np.int32)
    a = oracle.moe_forward_bf16(x, gu, dn, one, w)
    b = oracle.moe_forward_bf16(x, gu, dn, one[:, :1], w.sum(1, keepdims=True, dtype=np.float64).astype(np.float32))
    assert _ulps(a, b).max() <= 1
    # I2: zero weights -> exactly zero
    z = oracle.moe_forward_bf16(x, gu, dn, idx, np.zeros_like(w))
    assert np.all(z == 0)
    # I3: permuting the K slots (idx and w together)
    p = rng.permutation(K)
    c = oracle.moe_forward_bf16(x, gu, dn, idx[:, p], w[:, p])
    assert _ulps(c, base).max() <= 1
    # I4: linear in w (x2 is exact in bf16; general sums within rounding)
    d2 = oracle.moe_forward_bf16(x, gu, dn, idx, 2 * w)
    assert np.array_equal(F64(d2), 2 * F64(base))
    w1 = rng.uniform(0, 1, w.shape).astype(np.float32)
    s = oracle.moe_forward_bf16(x, gu, dn, idx, w + w1)
    s1 = oracle.moe_forward_bf16(x, gu, dn, idx, w1)
    np.testing.assert_allclose(F64(s), F64(base) + F64(s1), atol=2e-2 * np.abs(F64(s)).max())


def test_out_of_range_ids_contribute_zero():
    rng = np.random.default_rng(3)
    x, gu, dn, idx, w = _layer(rng, 3, 64, 32, 4, 3)
    bad = idx.copy(); bad[:, 1] = [-1, 4, 1000]
    a = oracle.moe_forward_bf16(x, gu, dn, bad, w)
    wz = w.copy(); wz[:, 1] = 0
    b = oracle.moe_forward_bf16(x, gu, dn, idx, wz)
    assert np.array_equal(a, b)


def test_bruteforce_bf16():
    rng = np.random.default_rng(4)
    T, H, F, E, K = 3, 48, 40, 4, 3
    x, gu, dn, idx, w = _layer(rng, T, H, F, E, K)
    idx[1, 2] = idx[1, 0]                     # duplicate expert in one token
    out = oracle.moe_forward_bf16(x, gu, dn, idx, w)
    ref = brute.forward_bf16(F64(x).tolist(), F64(gu).tolist(), F64(dn).tolist(),
                             idx.tolist(), w.astype(np.float64).tolist())
    d = _ulps(out, oracle.bf16_bits(np.array(ref)))
    assert d.max() <= 1 and (d == 0).mean() > 0.97


def _fp8_layer(rng, T, H, F, E, K):
    x = BF(rng.standard_normal((T, H)))
    def wq(shape):
        wf = torch.from_numpy(rng.standard_normal(shape) * 0.02).float()
        blk = wf.reshape(*shape[:-1], shape[-1] // 128, 128)
        sc = blk.abs().amax(-1) / 448 * torch.from_numpy(rng.uniform(1, 3, shape[:-1] + (shape[-1] // 128,))).float()
        q = (blk / sc[..., None]).clamp(-448, 448).to(torch.float8_e4m3fn)
        return q.reshape(shape).view(torch.uint8).numpy(), sc.numpy().astype(np.float32)
    w13, s13 = wq((E, 2 * F, H))
    w2, s2 = wq((E, H, F))
    idx = rng.integers(0, E, (T, K)).astype(np.int32)
    w = rng.uniform(0.1, 1, (T, K)).astype(np.float32)
    return x, w13, s13, w2, s2, idx, w


def test_dense_special_case_fp8():
    rng = np.random.default_rng(5)
    T, H, F = 4, 256, 384
    x, w13, s13, w2, s2, _, _ = _fp8_layer(rng, T, H, F, 1, 1)
    out = oracle.moe_forward_fp8(x, w13, s13, w2, s2, np.zeros((T, 1), np.int32), np.ones((T, 1), np.float32))
    deq = lambda q, s: torch.from_numpy(q).view(torch.float8_e4m3fn).double() * torch.from_numpy(s).double().repeat_interleave(128, -1)
    xq, xs = oracle.quantize_fp8_block128(x)
    X = deq(xq, xs)
    W13 = deq(w13[0], s13[0]); W2 = deq(w2[0], s2[0])
    g = X @ W13[:F].T; u = X @ W13[F:].T
    hb = oracle.bf16_bits((torch.nn.functional.silu(g) * u).numpy())
    hq, hs = oracle.quantize_fp8_block128(hb)
    ref = oracle.bf16_bits((deq(hq, hs) @ W2.T).numpy())
    d = _ulps(out, ref)
    assert d.max() <= 1 and (d == 0).mean() > 0.99
    # planted: weight scales indexed by the wrong axis change the result
    s13_wrong = np.ascontiguousarray(np.flip(s13, axis=-1))
    bad = oracle.moe_forward_fp8(x, w13, s13_wrong, w2, s2, np.zeros((T, 1), np.int32), np.ones((T, 1), np.float32))
    assert (_ulps(bad, ref) > 1).mean() > 0.3


def test_bruteforce_fp8():
    rng = np.random.default_rng(6)
    T, H, F, E, K = 2, 128, 128, 3, 2
    x, w13, s13, w2, s2, idx, w = _fp8_layer(rng, T, H, F, E, K)
    out = oracle.moe_forward_fp8(x, w13, s13, w2, s2, idx, w)
    v = lambda q: oracle.e4m3_to_f64(q).tolist()
    ref = brute.forward_fp8(F64(x).tolist(), v(w13), s13.astype(np.float64).tolist(), v(w2),
                            s2.astype(np.float64).tolist(), idx.tolist(), w.astype(np.float64).tolist())
    d = _ulps(out, oracle.bf16_bits(np.array(ref)))
    assert d.max() <= 2 and (d == 0).mean() > 0.95
