"""Pins of the oracle's routed + shared experts + residual forward
("Supporting MegaKernel for DeepSeek Models": shared expert via
silu_mul_layer, moe_local_reduction = weighted sum over k + residual):
- no shared experts and no residual = the routed forward, bit for bit;
- a shared expert is a routed expert that every token uses with weight 1
  (same summation order, bit for bit), for bf16 and E4M3 weights;
- zero routing weights and zero shared weights leave exactly the residual;
- an independent pure-Python brute force (exact sums) within 1 bf16 ulp;
- a planted mistake (shared experts scaled by a router weight) is caught."""
import numpy as np
import torch

import oracle
from oracle import brute

BF = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
F64 = oracle.bf16_to_f64


def _ulps(a, b):
    ia = a.view(np.int16).astype(np.int32)
    ib = b.view(np.int16).astype(np.int32)
    return np.abs(ia - ib)


def _layer(rng, T, H, F, E, K, S):
    x = BF(rng.standard_normal((T, H)))
    gu = BF(rng.standard_normal((E, 2 * F, H)) * 0.05)
    dn = BF(rng.standard_normal((E, H, F)) * 0.05)
    sgu = BF(rng.standard_normal((S, 2 * F, H)) * 0.05)
    sdn = BF(rng.standard_normal((S, H, F)) * 0.05)
    idx = rng.integers(0, E, (T, K)).astype(np.int32)
    w = rng.uniform(0.05, 1.0, (T, K)).astype(np.float32)
    res = BF(rng.standard_normal((T, H)))
    return x, gu, dn, idx, w, sgu, sdn, res


def _augment(gu, dn, idx, w, sgu, sdn):
    """Shared experts appended as routed experts E..E+S-1, weight 1, every token."""
    E, S, T = gu.shape[0], sgu.shape[0], idx.shape[0]
    gu2 = np.concatenate([gu, sgu])
    dn2 = np.concatenate([dn, sdn])
    idx2 = np.concatenate([idx, np.tile(np.arange(E, E + S, dtype=np.int32), (T, 1))], 1)
    w2 = np.concatenate([w, np.ones((T, S), np.float32)], 1)
    return gu2, dn2, idx2, w2


def test_no_shared_no_residual_is_routed():
    rng = np.random.default_rng(1)
    x, gu, dn, idx, w, sgu, sdn, res = _layer(rng, 5, 64, 48, 6, 3, 0)
    a = oracle.moe_forward_shared_bf16(x, gu, dn, idx, w, sgu, sdn, None)
    assert np.array_equal(a, oracle.moe_forward_bf16(x, gu, dn, idx, w))


def test_shared_is_weight_one_routed_expert_bf16():
    rng = np.random.default_rng(2)
    x, gu, dn, idx, w, sgu, sdn, res = _layer(rng, 6, 64, 40, 5, 2, 2)
    idx[2, 1] = -1                                     # an invalid slot stays skipped
    got = oracle.moe_forward_shared_bf16(x, gu, dn, idx, w, sgu, sdn, None)
    gu2, dn2, idx2, w2 = _augment(gu, dn, idx, w, sgu, sdn)
    assert np.array_equal(got, oracle.moe_forward_bf16(x, gu2, dn2, idx2, w2))


def test_shared_is_weight_one_routed_expert_fp8():
    rng = np.random.default_rng(3)
    T, H, F, E, K, S = 3, 128, 128, 3, 2, 2
    x = BF(rng.standard_normal((T, H)))

    def wq(shape):
        wf = torch.from_numpy(rng.standard_normal(shape) * 0.02).float()
        blk = wf.reshape(*shape[:-1], shape[-1] // 128, 128)
        sc = blk.abs().amax(-1) / 448
        q = (blk / sc[..., None]).to(torch.float8_e4m3fn).reshape(shape)
        return q.view(torch.uint8).numpy(), sc.numpy().astype(np.float32)
    w13, s13 = wq((E, 2 * F, H))
    w2, s2 = wq((E, H, F))
    sw13, ss13 = wq((S, 2 * F, H))
    sw2, ss2 = wq((S, H, F))
    idx = rng.integers(0, E, (T, K)).astype(np.int32)
    w = rng.uniform(0.1, 1.0, (T, K)).astype(np.float32)
    got = oracle.moe_forward_shared_fp8(x, w13, s13, w2, s2, idx, w, sw13, ss13, sw2, ss2)
    idx2 = np.concatenate([idx, np.tile(np.arange(E, E + S, dtype=np.int32), (T, 1))], 1)
    w2_ = np.concatenate([w, np.ones((T, S), np.float32)], 1)
    ref = oracle.moe_forward_fp8(x, np.concatenate([w13, sw13]), np.concatenate([s13, ss13]),
                                 np.concatenate([w2, sw2]), np.concatenate([s2, ss2]), idx2, w2_)
    assert np.array_equal(got, ref)


def test_zero_weights_leave_the_residual():
    rng = np.random.default_rng(4)
    x, gu, dn, idx, w, sgu, sdn, res = _layer(rng, 4, 64, 32, 4, 2, 1)
    got = oracle.moe_forward_shared_bf16(x, gu, dn, idx, np.zeros_like(w), np.zeros_like(sgu), sdn, res)
    assert np.array_equal(got, res)


def test_bruteforce_shared_residual():
    rng = np.random.default_rng(5)
    T, H, F, E, K, S = 3, 32, 24, 3, 2, 2
    x, gu, dn, idx, w, sgu, sdn, res = _layer(rng, T, H, F, E, K, S)
    out = oracle.moe_forward_shared_bf16(x, gu, dn, idx, w, sgu, sdn, res)
    L = lambda a: F64(a).tolist()
    ref = brute.forward_shared_bf16(L(x), L(gu), L(dn), idx.tolist(), w.astype(np.float64).tolist(),
                                    L(sgu), L(sdn), L(res))
    d = _ulps(out, oracle.bf16_bits(np.array(ref)))
    assert d.max() <= 1 and (d == 0).mean() > 0.95


def test_planted_mistake_caught():
    """Scaling the shared experts by the first router weight (a plausible
    wrong reading) changes the result well beyond rounding."""
    rng = np.random.default_rng(6)
    x, gu, dn, idx, w, sgu, sdn, res = _layer(rng, 4, 64, 32, 4, 2, 1)
    good = oracle.moe_forward_shared_bf16(x, gu, dn, idx, w, sgu, sdn, None)
    gu2, dn2, idx2, w2 = _augment(gu, dn, idx, w, sgu, sdn)
    w2[:, -1] = w[:, 0]
    bad = oracle.moe_forward_bf16(x, gu2, dn2, idx2, w2)
    assert _ulps(good, bad).max() > 8
