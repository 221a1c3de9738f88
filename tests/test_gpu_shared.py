"""GPU parity of the routed + shared experts + residual forward
(moe_experts_with_shared) against the oracle ("Supporting MegaKernel for
DeepSeek Models": the shared expert is a SwiGLU MLP every token goes
through; moe_local_reduction adds the residual to the weighted expert sum).

Covered: bf16 (gather-GEMV decode sizes and grouped GEMMs) and E4M3 weights,
S = 0 / 1 / 2 shared experts, residual on and off, ragged tiles, the 16-row
E4M3 tiles of decode-sized calls, routed ids outside [0, E) -- including E
and E+1, which must not reach a shared expert --, bitwise determinism,
argument errors, and sampled tokens of the DeepSeek-V3-like E4M3 layer with
one shared expert."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_matches_oracle
from mixture_experts_routed_expert_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_dev):
    import mixture_experts_routed_expert_b200 as m
    return m


def _bad_ids(idx, E, seed):
    """Overwrite a few routed ids with -1, E, E+1 and a large id."""
    idx = idx.clone()
    g = torch.Generator().manual_seed(seed)
    T, K = idx.shape
    n = max(1, T * K // 10)
    pos = torch.randperm(T * K, generator=g)[:n]
    bad = torch.tensor([-1, E, E + 1, 1 << 20], dtype=torch.int32)
    idx.view(-1)[pos] = bad[torch.arange(n) % 4]
    return idx


def _bf16_case(T, H, F, E, K, S, residual, seed, bad=False):
    lay = inputs.ocr2_layer(T, seed=seed, H=H, F=F, E=E, K=K)
    idx = _bad_ids(lay.idx, E, seed) if bad else lay.idx
    sgu, sdn = inputs.shared_experts_bf16(max(S, 1), H, F, seed)
    sgu, sdn = sgu[:S], sdn[:S]
    res = inputs.residual_bf16(T, H, seed) if residual else None
    return lay, idx, sgu, sdn, res


def _bf16_oracle(lay, idx, sgu, sdn, res):
    return oracle.moe_forward_shared_bf16(
        inputs.bf16_bits(lay.x), inputs.bf16_bits(lay.gate_up), inputs.bf16_bits(lay.down),
        inputs.np32(idx), inputs.np32(lay.w), inputs.bf16_bits(sgu), inputs.bf16_bits(sdn),
        None if res is None else inputs.bf16_bits(res))


def _bf16_gpu(moe, lay, idx, sgu, sdn, res, dev):
    S = sgu.shape[0]
    return moe.moe_experts_with_shared(
        lay.x.to(dev), lay.gate_up.to(dev), lay.down.to(dev), idx.to(dev), lay.w.to(dev),
        idx.shape[1], sgu.to(dev) if S else None, sdn.to(dev) if S else None,
        residual=None if res is None else res.to(dev))


@pytest.mark.parametrize("T,H,F,E,K,S,residual,bad", [
    (40, 256, 256, 8, 2, 1, True, False),      # two k-blocks, one shared expert, residual
    (300, 512, 384, 16, 6, 2, False, True),    # ragged tiles, two shared experts, bad ids
    (257, 1280, 896, 64, 6, 2, True, True),    # OCR-2 widths: ragged token tail, both extras
    (3, 256, 256, 8, 2, 2, True, False),       # tiny T (12 slots: gather-GEMV decode kernels)
    (1, 1280, 896, 64, 6, 2, True, True),      # OCR-2 decode, T=1 (gather-GEMV)
    (2, 1280, 896, 64, 6, 2, False, False),    # OCR-2 decode, T=2 (gather-GEMV, 16 slots)
    (3, 1280, 896, 64, 6, 2, True, False),     # 24 slots: grouped GEMMs
    (64, 256, 256, 8, 4, 0, True, True),       # S = 0: routed + residual only
])
def test_bf16_shared_residual(moe, cuda_dev, T, H, F, E, K, S, residual, bad):
    lay, idx, sgu, sdn, res = _bf16_case(T, H, F, E, K, S, residual, seed=T + 7 * S, bad=bad)
    out = _bf16_gpu(moe, lay, idx, sgu, sdn, res, cuda_dev)
    ref = _bf16_oracle(lay, idx, sgu, sdn, res)
    assert_matches_oracle(out, ref, "bf16 T=%d S=%d res=%s" % (T, S, residual))


def test_bf16_shared_all_ids_invalid(moe, cuda_dev):
    """Every routed id invalid: the output is the shared experts + residual."""
    lay, idx, sgu, sdn, res = _bf16_case(16, 256, 256, 8, 4, 2, True, seed=5)
    idx = torch.full_like(idx, 8)          # = E, the first shared id of the widened set
    out = _bf16_gpu(moe, lay, idx, sgu, sdn, res, cuda_dev)
    assert_matches_oracle(out, _bf16_oracle(lay, idx, sgu, sdn, res), "all invalid")


def test_bf16_shared_deterministic(moe, cuda_dev):
    lay, idx, sgu, sdn, res = _bf16_case(200, 512, 256, 16, 6, 2, True, seed=11)
    a = _bf16_gpu(moe, lay, idx, sgu, sdn, res, cuda_dev)
    b = _bf16_gpu(moe, lay, idx, sgu, sdn, res, cuda_dev)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_shared_argument_errors(moe, cuda_dev):
    lay, idx, sgu, sdn, res = _bf16_case(8, 256, 256, 8, 8, 2, True, seed=3)
    d = cuda_dev
    # K + S > 16
    big = torch.zeros(8, 15, dtype=torch.int32)
    with pytest.raises(moe.MoEError):
        moe.moe_experts_with_shared(lay.x.to(d), lay.gate_up.to(d), lay.down.to(d), big.to(d),
                                    torch.ones(8, 15).to(d), 15, sgu.to(d), sdn.to(d))
    assert moe.moe_experts_shared_workspace_size(8, 256, 256, 8, 15, 2) == 0
    assert moe.moe_experts_shared_workspace_size(8, 256, 256, 8, 8, 2) > 0
    # E4M3 weights without the shared scales
    w13, w13s, w2, w2s = inputs.fp8_weights(0, "cpu", 256, 256, 8)
    s13, s13s, s2, s2s = inputs.shared_experts_fp8(1, 256, 256)
    with pytest.raises(moe.MoEError):
        moe.moe_experts_with_shared(lay.x.to(d), w13.to(d), w2.to(d), idx.to(d), lay.w.to(d), 8,
                                    s13.to(d), s2.to(d), gate_up_scale=w13s.to(d),
                                    down_scale=w2s.to(d))


# ---------------------------------------------------------------- E4M3 ----

def _fp8_oracle(lay, idx, w, sh, res, tokens=None):
    """Oracle for `tokens`; only the routed experts they touch go to the host
    (remapped to 0..n-1; ids outside [0, E) stay invalid)."""
    E = lay.dims["E"]
    x = lay.x
    if tokens is not None:
        x, idx, w = x[tokens], idx[tokens], w[tokens]
        res = None if res is None else res[tokens]
    valid = (idx >= 0) & (idx < E)
    used = torch.unique(idx[valid])
    remap = torch.full((E,), -1, dtype=torch.int32)
    remap[used.long()] = torch.arange(len(used), dtype=torch.int32)
    ridx = torch.where(valid, remap[idx.clamp(0, E - 1).long()], torch.full_like(idx, -1))
    sel = used.long().to(lay.w13.device)
    s13, s13s, s2, s2s = sh
    return oracle.moe_forward_shared_fp8(
        inputs.bf16_bits(x), inputs.u8(lay.w13[sel]), inputs.np32(lay.w13_scale[sel]),
        inputs.u8(lay.w2[sel]), inputs.np32(lay.w2_scale[sel]),
        inputs.np32(ridx.to(torch.int32)), inputs.np32(w), inputs.u8(s13), inputs.np32(s13s),
        inputs.u8(s2), inputs.np32(s2s), None if res is None else inputs.bf16_bits(res))


def _fp8_gpu(moe, lay, idx, w, sh, res, dev):
    s13, s13s, s2, s2s = sh
    return moe.moe_experts_with_shared(
        lay.x.to(dev), lay.w13.to(dev), lay.w2.to(dev), idx.to(dev), w.to(dev), idx.shape[1],
        s13.to(dev), s2.to(dev), residual=None if res is None else res.to(dev),
        gate_up_scale=lay.w13_scale.to(dev), down_scale=lay.w2_scale.to(dev),
        shared_gate_up_scale=s13s.to(dev), shared_down_scale=s2s.to(dev))


def _route(lay, K, groups=8, topk_group=4, scale=2.5):
    idx, w = oracle.route_sigmoid_grouped(inputs.np32(lay.logits), inputs.np32(lay.bias), groups,
                                          topk_group, K, scale)
    return torch.from_numpy(idx), torch.from_numpy(w)


@pytest.mark.parametrize("T,H,F,E,K,S,residual,bad", [
    (40, 256, 256, 8, 2, 1, True, False),      # 64-row tiles (40 * 3 slots)
    (300, 1024, 512, 64, 8, 1, True, True),    # ragged tiles, 8 k-blocks, bad ids
    (4, 512, 256, 16, 8, 2, True, True),       # 40 slots: the 16-row tiles of decode sizes
    (7, 256, 384, 16, 4, 2, False, False),     # 42 slots, no residual
])
def test_fp8_shared_residual(moe, cuda_dev, T, H, F, E, K, S, residual, bad):
    lay = inputs.fp8_layer(T, seed=T + S, H=H, F=F, E=E)
    idx, w = _route(lay, K)
    if bad:
        idx = _bad_ids(idx, E, T)
    sh = inputs.shared_experts_fp8(S, H, F, seed=T)
    res = inputs.residual_bf16(T, H, seed=T) if residual else None
    out = _fp8_gpu(moe, lay, idx, w, sh, res, cuda_dev)
    assert_matches_oracle(out, _fp8_oracle(lay, idx, w, sh, res),
                          "fp8 T=%d S=%d res=%s" % (T, S, residual))


@pytest.fixture(scope="module")
def dsv3_weights(cuda_dev):
    return inputs.fp8_weights(seed=0, device=cuda_dev)


@pytest.mark.parametrize("T", [4, 40])
def test_fp8_shared_dsv3_sampled(moe, cuda_dev, dsv3_weights, T):
    """DeepSeek-V3-like layer (H=7168, F=2048, E=256, K=8) with one shared
    expert and a residual: T=4 takes the 16-row tiles (36 slots), T=40 the
    64-row tiles; a few tokens are checked against the oracle."""
    lay = inputs.fp8_layer(T, seed=100 + T, weights=dsv3_weights)
    idx, w = _route(lay, 8)
    H, F = lay.dims["H"], lay.dims["F"]
    sh = inputs.shared_experts_fp8(1, H, F, seed=1)
    res = inputs.residual_bf16(T, H, seed=T)
    out = _fp8_gpu(moe, lay, idx, w, sh, res, cuda_dev)
    tokens = [0, T - 1] if T <= 4 else [0, 17, T - 1]
    ref = _fp8_oracle(lay, idx, w, sh, res, tokens=tokens)
    assert_matches_oracle(out[tokens], ref, "dsv3 shared T=%d" % T)
