"""GPU parity of the E4M3 routed-experts forward (per-(row,128) fp32 weight
scales, activations quantised per 128 with power-of-two scales) against the
oracle: full outputs on reduced shapes spanning several k-blocks, tiles and
ragged tails, Zipf-skewed routing with empty experts, and sampled tokens of
the DeepSeek-V3-like layer (H=7168, F=2048, E=256, K=8)."""
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


def _oracle(lay, idx, w, tokens=None):
    """Oracle output for `tokens`; only the experts they touch go to the host
    (their ids are remapped to 0..n-1)."""
    E = lay.dims["E"]
    x = lay.x if tokens is None else lay.x[tokens]
    if tokens is not None:
        idx, w = idx[tokens], w[tokens]
    valid = (idx >= 0) & (idx < E)
    used = torch.unique(idx[valid])
    remap = torch.full((E,), -1, dtype=torch.int32)
    remap[used.long()] = torch.arange(len(used), dtype=torch.int32)
    ridx = torch.where(valid, remap[idx.clamp(0, E - 1).long()], torch.full_like(idx, -1))
    sel = used.long().to(lay.w13.device)
    return oracle.moe_forward_fp8(
        inputs.bf16_bits(x), inputs.u8(lay.w13[sel]), inputs.np32(lay.w13_scale[sel]),
        inputs.u8(lay.w2[sel]), inputs.np32(lay.w2_scale[sel]),
        inputs.np32(ridx.to(torch.int32)), inputs.np32(w))


def _run(moe, lay, idx, w, dev, fn="moe_experts_prefill"):
    return getattr(moe, fn)(lay.x.to(dev), lay.w13.to(dev), lay.w2.to(dev), idx.to(dev), w.to(dev),
                            idx.shape[1], gate_up_scale=lay.w13_scale.to(dev),
                            down_scale=lay.w2_scale.to(dev))


@pytest.mark.parametrize("T,H,F,E,K,skew", [
    (40, 256, 256, 8, 2, None),        # two k-blocks, several tiles
    (300, 1024, 512, 64, 8, None),     # ragged row tiles, 8 k-blocks
    (512, 384, 384, 64, 8, 1.1),       # Zipf skew: empty experts, a hot expert (> 64 rows)
    (3, 512, 256, 16, 4, None),        # tiny T
])
def test_fp8_reduced_shapes(moe, cuda_dev, T, H, F, E, K, skew):
    lay = inputs.fp8_layer(T, seed=T + E, device="cpu", H=H, F=F, E=E, zipf=skew)
    idx, w = _route(lay, K)
    out = _run(moe, lay, idx, w, cuda_dev)
    assert_matches_oracle(out, _oracle(lay, idx, w), "fp8 T=%d H=%d F=%d E=%d" % (T, H, F, E))


@pytest.mark.parametrize("T,H,F,E,K,skew", [
    (2, 512, 256, 32, 8, None),        # two tokens, one invalid slot
    (1, 1024, 512, 64, 8, None),       # one token: one slot per expert
    (12, 384, 384, 4, 4, None),        # every token on all 4 experts: 12 slots each (8 + 4 ragged)
    (16, 256, 640, 8, 4, 1.1),         # skewed: a hot expert with > 8 slots (ragged tile)
    (5, 768, 128, 64, 6, None),        # one k-block of F, ragged token count
])
def test_fp8_decode_entry(moe, cuda_dev, T, H, F, E, K, skew):
    lay = inputs.fp8_layer(T, seed=11 * T + K, device="cpu", H=H, F=F, E=E, zipf=skew)
    idx, w = _route(lay, K, groups=min(8, E // 2), topk_group=min(4, E // 2))
    if T >= 2:
        idx[1, K // 2] = -1
    out = _run(moe, lay, idx, w, cuda_dev, "moe_experts_decode")
    assert_matches_oracle(out, _oracle(lay, idx, w), "fp8 decode T=%d H=%d F=%d E=%d K=%d"
                          % (T, H, F, E, K))
    out2 = _run(moe, lay, idx, w, cuda_dev, "moe_experts_decode")
    assert torch.equal(out, out2), "fp8 decode is not deterministic"


def test_fp8_decode_duplicate_and_empty(moe, cuda_dev):
    """A token listing one expert twice (two slots, one tile column each) and a
    token with no valid slot (its output row is zero)."""
    lay = inputs.fp8_layer(3, seed=3, device="cpu", H=512, F=256, E=16)
    idx = torch.tensor([[4, 4, 9, 1], [-1, 16, -1, -1], [9, 0, 4, 15]], dtype=torch.int32)
    w = torch.rand(3, 4, generator=torch.Generator().manual_seed(0))
    out = _run(moe, lay, idx, w, cuda_dev, "moe_experts_decode")
    assert torch.count_nonzero(out[1]) == 0
    assert_matches_oracle(out, _oracle(lay, idx, w), "fp8 decode duplicates")


@pytest.fixture(scope="module")
def dsv3_weights(cuda_dev):
    return inputs.fp8_weights(seed=0, device=cuda_dev)


@pytest.mark.parametrize("T", [128, 1])
def test_fp8_dsv3_sampled(moe, cuda_dev, dsv3_weights, T):
    lay = inputs.fp8_layer(T, seed=T, device="cpu", weights=dsv3_weights)
    idx, w = _route(lay, 8)
    out = _run(moe, lay, idx, w, cuda_dev)
    tokens = torch.tensor(parity_sample(idx.numpy(), 256, grouped_tile_heights(T, 8, 256, "e4m3"),
                                        seed=T))
    assert_matches_oracle(out[tokens.to(out.device)], _oracle(lay, idx, w, tokens),
                          "fp8 DSV3 T=%d sampled" % T)
    out2 = _run(moe, lay, idx, w, cuda_dev)
    assert torch.equal(out, out2), "fp8 path is not deterministic"


@pytest.mark.parametrize("T", [1, 4, 8])
def test_fp8_dsv3_decode_sampled(moe, cuda_dev, dsv3_weights, T):
    """The decode entry on the DeepSeek-V3-like layer (served by the E4M3
    grouped GEMMs with 16-row activation tiles at these sizes); every token
    checked."""
    lay = inputs.fp8_layer(T, seed=100 + T, device="cpu", weights=dsv3_weights)
    idx, w = _route(lay, 8)
    out = _run(moe, lay, idx, w, cuda_dev, "moe_experts_decode")
    tokens = torch.arange(T)
    assert_matches_oracle(out[tokens.to(out.device)], _oracle(lay, idx, w, tokens),
                          "fp8 DSV3 decode T=%d" % T)


@pytest.mark.parametrize("T", [3, 16])
def test_fp8_few_tokens_invalid_slots(moe, cuda_dev, T):
    """Few tokens on E4M3 weights through both entries, with an all-invalid
    token and an all-invalid call."""
    lay = inputs.fp8_layer(T, seed=300 + T, device="cpu", H=512, F=256, E=16)
    idx, w = _route(lay, 4)
    idx[1, :] = -1
    for fn in ("moe_experts_prefill", "moe_experts_decode"):
        out = _run(moe, lay, idx, w, cuda_dev, fn)
        assert_matches_oracle(out, _oracle(lay, idx, w), "fp8 T=%d %s" % (T, fn))
        assert torch.count_nonzero(out[1].float()) == 0
    idx.fill_(-1)
    out = _run(moe, lay, idx, w, cuda_dev)
    assert torch.count_nonzero(out.float()) == 0
