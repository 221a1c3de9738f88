"""GPU parity of the MXFP4-weight routed-experts forward (packed E2M1 with
one E8M0 scale per row and 32 columns, E4M3 activations with power-of-two
block-128 scales; block-scaled tcgen05 MMAs) against the oracle: full
outputs on reduced shapes spanning several k-blocks, tiles and ragged tails,
Zipf-skewed routing with empty experts, all three tile heights (16-row
tiles for few routed rows per expert, 112-row tiles for many, 64-row tiles
between), and sampled tokens of the
DeepSeek-V3-like layer (H=7168, F=2048, E=256, K=8) with MXFP4 weights; the
one-kernel decode form (moe_experts_decode_fused) on the same checks."""
import pytest
import torch

import oracle
from _helpers import assert_matches_oracle, grouped_tile_heights, parity_sample
from mixture_experts_routed_expert_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_dev):
    import mixture_experts_routed_expert_b200 as m
    return m


def _route(lay, K, groups=8, topk_group=4, scale=2.5):
    idx, w = oracle.route_sigmoid_grouped(inputs.np32(lay.logits), inputs.np32(lay.bias), groups,
                                          topk_group, K, scale)
    return torch.from_numpy(idx), torch.from_numpy(w)


def _oracle(x, wts, idx, w, E, tokens=None):
    """Oracle output for `tokens`; only the experts they touch go to the host
    (ids remapped to 0..n-1; ids outside [0, E) stay invalid)."""
    w13, w13s, w2, w2s = wts
    if tokens is not None:
        x, idx, w = x[tokens], idx[tokens], w[tokens]
    valid = (idx >= 0) & (idx < E)
    used = torch.unique(idx[valid])
    remap = torch.full((E,), -1, dtype=torch.int32)
    remap[used.long()] = torch.arange(len(used), dtype=torch.int32)
    ridx = torch.where(valid, remap[idx.clamp(0, E - 1).long()], torch.full_like(idx, -1))
    sel = used.long().to(w13.device)
    return oracle.moe_forward_mxf4(inputs.bf16_bits(x), inputs.u8(w13[sel]), inputs.u8(w13s[sel]),
                                   inputs.u8(w2[sel]), inputs.u8(w2s[sel]),
                                   inputs.np32(ridx.to(torch.int32)), inputs.np32(w))


def _run(moe, x, wts, idx, w, dev, fn="moe_experts_prefill"):
    w13, w13s, w2, w2s = wts
    return getattr(moe, fn)(x.to(dev), w13.to(dev), w2.to(dev), idx.to(dev), w.to(dev),
                            idx.shape[1], gate_up_scale=w13s.to(dev), down_scale=w2s.to(dev),
                            weight_format="mxfp4")


@pytest.mark.parametrize("T,H,F,E,K,skew,fn", [
    (40, 256, 256, 8, 2, None, "moe_experts_prefill"),     # two k-blocks, several tiles
    (300, 1024, 512, 64, 8, None, "moe_experts_prefill"),  # ragged row tiles, 8 k-blocks
    (512, 384, 384, 64, 8, 1.1, "moe_experts_prefill"),    # Zipf skew, empty / hot experts, 112-row tiles
    (100, 512, 384, 32, 4, None, "moe_experts_prefill"),   # 12.5 rows per expert: 64-row tiles
    (3, 512, 256, 16, 4, None, "moe_experts_prefill"),     # tiny T, 16-row tiles
    (3, 512, 256, 16, 4, None, "moe_experts_decode"),      # 12 slots: 16-row tiles
    (8, 640, 384, 32, 8, None, "moe_experts_decode"),      # 64 slots: 16-row tiles, 5 k-blocks
])
def test_mxf4_reduced_shapes(moe, cuda_dev, T, H, F, E, K, skew, fn):
    lay = inputs.fp8_layer(T, seed=T + H, H=H, F=F, E=E, zipf=skew,
                           weights=(None, None, None, None))
    wts = inputs.mxf4_weights(seed=T, H=H, F=F, E=E)
    idx, w = _route(lay, K)
    out = _run(moe, lay.x, wts, idx, w, cuda_dev, fn)
    assert_matches_oracle(out, _oracle(lay.x, wts, idx, w, E), "mxf4 T=%d %s" % (T, fn))


def test_mxf4_invalid_ids_and_duplicates(moe, cuda_dev):
    T, H, F, E, K = 24, 256, 256, 8, 4
    lay = inputs.fp8_layer(T, seed=7, H=H, F=F, E=E, weights=(None, None, None, None))
    wts = inputs.mxf4_weights(seed=7, H=H, F=F, E=E)
    idx, w = _route(lay, K)
    idx[0, :] = 3                       # all slots of a token on one expert
    idx[1, 1] = -1
    idx[2, 2] = E
    idx[3, :] = 1 << 20                 # a token with no valid slot -> 0
    out = _run(moe, lay.x, wts, idx, w, cuda_dev)
    assert_matches_oracle(out, _oracle(lay.x, wts, idx, w, E), "mxf4 invalid ids")
    assert torch.all(out[3] == 0)


def test_mxf4_deterministic(moe, cuda_dev):
    T, H, F, E, K = 200, 512, 256, 16, 8
    lay = inputs.fp8_layer(T, seed=11, H=H, F=F, E=E, weights=(None, None, None, None))
    wts = inputs.mxf4_weights(seed=11, H=H, F=F, E=E)
    idx, w = _route(lay, K)
    a = _run(moe, lay.x, wts, idx, w, cuda_dev)
    b = _run(moe, lay.x, wts, idx, w, cuda_dev)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_mxf4_argument_errors(moe, cuda_dev):
    T, H, F, E, K = 8, 256, 256, 8, 2
    lay = inputs.fp8_layer(T, seed=3, H=H, F=F, E=E, weights=(None, None, None, None))
    w13, w13s, w2, w2s = [t.to(cuda_dev) for t in inputs.mxf4_weights(seed=3, H=H, F=F, E=E)]
    idx, w = _route(lay, K)
    x, idx, w = lay.x.to(cuda_dev), idx.to(cuda_dev), w.to(cuda_dev)
    # packed weights must be 32-byte aligned (TMA reads them in 32-byte units)
    buf = torch.empty(w13.numel() + 16, dtype=torch.uint8, device=cuda_dev)
    w13_off = buf[16:].view(w13.shape)
    w13_off.copy_(w13)
    with pytest.raises(moe.MoEError):
        moe.moe_experts_prefill(x, w13_off, w2, idx, w, K, gate_up_scale=w13s, down_scale=w2s,
                                weight_format="mxfp4")
    # scales are required
    with pytest.raises(moe.MoEError):
        moe.moe_experts_prefill(x, w13, w2, idx, w, K, weight_format="mxfp4")


@pytest.fixture(scope="module")
def dsv3_mxf4(cuda_dev):
    return inputs.mxf4_weights(seed=0, device=cuda_dev)


@pytest.mark.parametrize("T,fn", [(1, "moe_experts_decode"), (8, "moe_experts_decode"),
                                  (128, "moe_experts_prefill"), (384, "moe_experts_prefill"),
                                  (2048, "moe_experts_prefill")])
def test_mxf4_dsv3_sampled(moe, cuda_dev, dsv3_mxf4, T, fn):
    """DeepSeek-V3-like layer with MXFP4 weights: T=1 / 8 / 128 (<= 6 routed
    rows per expert) take the 16-row tiles, T=384 the 64-row tiles, T=2048
    (64 rows per expert) the 112-row tiles; sampled tokens (the hottest
    expert's last row tile, the rarest expert's tokens, >= 16 in all)
    checked against the oracle."""
    D = inputs.DSV3_FP8
    lay = inputs.fp8_layer(T, seed=200 + T, device=cuda_dev, weights=(None, None, None, None))
    idx, w = _route(lay, D["K"])
    out = _run(moe, lay.x, dsv3_mxf4, idx, w, cuda_dev, fn)
    tokens = parity_sample(idx.numpy(), D["E"], grouped_tile_heights(T, D["K"], D["E"], "mxfp4"),
                           seed=T)
    ref = _oracle(lay.x, dsv3_mxf4, idx, w, D["E"], tokens=tokens)
    assert_matches_oracle(out[tokens], ref, "mxf4 dsv3 T=%d" % T)


def test_mxf4_zero_tokens_and_zero_weights(moe, cuda_dev):
    H, F, E, K = 256, 256, 8, 4
    wts = inputs.mxf4_weights(seed=5, H=H, F=F, E=E)
    lay = inputs.fp8_layer(0, seed=5, H=H, F=F, E=E, weights=(None, None, None, None))
    idx, w = _route(lay, K)
    out = _run(moe, lay.x, wts, idx, w, cuda_dev)
    assert out.shape == (0, H)
    lay = inputs.fp8_layer(40, seed=6, H=H, F=F, E=E, weights=(None, None, None, None))
    idx, w = _route(lay, K)
    out = _run(moe, lay.x, wts, idx, torch.zeros_like(w), cuda_dev)
    assert torch.count_nonzero(out.float()) == 0


# ------------------------------------------- one-kernel form (decode sizes) ----

@pytest.mark.parametrize("T,H,F,E,K", [
    (1, 512, 256, 16, 8),        # one token
    (8, 640, 384, 32, 8),        # 64 slots; odd k-block counts (5 and 3)
    (5, 384, 128, 16, 4),        # down with one k-block (one partial accumulator)
    (16, 256, 256, 8, 4),        # 16 tokens, experts with > 16 slots (two row tiles)
])
def test_mxf4_fused_reduced_shapes(moe, cuda_dev, T, H, F, E, K):
    lay = inputs.fp8_layer(T, seed=50 + T, H=H, F=F, E=E, weights=(None, None, None, None))
    wts = inputs.mxf4_weights(seed=T + 1, H=H, F=F, E=E)
    idx, w = _route(lay, K)
    out = _run(moe, lay.x, wts, idx, w, cuda_dev, "moe_experts_decode_fused")
    assert_matches_oracle(out, _oracle(lay.x, wts, idx, w, E), "fused T=%d" % T)


def test_mxf4_fused_invalid_ids_and_empty_tokens(moe, cuda_dev):
    T, H, F, E, K = 6, 256, 256, 8, 4
    lay = inputs.fp8_layer(T, seed=9, H=H, F=F, E=E, weights=(None, None, None, None))
    wts = inputs.mxf4_weights(seed=9, H=H, F=F, E=E)
    idx, w = _route(lay, K)
    idx[0, :] = 2                       # every slot of a token on one expert
    idx[1, 3] = -1
    idx[2, 0] = E
    idx[4, :] = -7                      # a token with no valid slot -> 0
    out = _run(moe, lay.x, wts, idx, w, cuda_dev, "moe_experts_decode_fused")
    assert_matches_oracle(out, _oracle(lay.x, wts, idx, w, E), "fused invalid ids")
    assert torch.all(out[4] == 0)
    # nothing valid at all
    idx_none = torch.full_like(idx, -1)
    out = _run(moe, lay.x, wts, idx_none, w, cuda_dev, "moe_experts_decode_fused")
    assert torch.all(out == 0)


def test_mxf4_fused_deterministic_and_limits(moe, cuda_dev, dsv3_mxf4):
    D = inputs.DSV3_FP8
    lay = inputs.fp8_layer(8, seed=77, device=cuda_dev, weights=(None, None, None, None))
    idx, w = _route(lay, D["K"])
    a = _run(moe, lay.x, dsv3_mxf4, idx, w, cuda_dev, "moe_experts_decode_fused")
    b = _run(moe, lay.x, dsv3_mxf4, idx, w, cuda_dev, "moe_experts_decode_fused")
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    ref = _oracle(lay.x, dsv3_mxf4, idx, w, D["E"], tokens=[0, 7])
    assert_matches_oracle(a[[0, 7]], ref, "fused dsv3 T=8")
    # 17 tokens is outside the one-kernel form
    lay17 = inputs.fp8_layer(17, seed=3, H=256, F=256, E=8, weights=(None, None, None, None))
    wts = inputs.mxf4_weights(seed=3, H=256, F=256, E=8)
    idx17, w17 = _route(lay17, 2)
    with pytest.raises(moe.MoEError):
        _run(moe, lay17.x, wts, idx17, w17, cuda_dev, "moe_experts_decode_fused")
