"""GPU parity of the one-kernel bf16 decode (moe_experts_decode_fused with
bf16 weights, T <= 16, T*K <= 64) against the oracle on routings that exercise
its work split: clusters with no groups (fewer feature groups than
clusters), a touched expert split over several clusters, tokens with more
than 8 slots on one expert, segments wider than one staging slab (64 slots
on one expert), duplicate and invalid ids, tokens with no valid slot, and a
reused workspace (the arrival counters must be zero again after every call,
so repeated calls give bit-identical outputs)."""
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


def _ref(lay):
    return oracle.moe_forward_bf16(inputs.bf16_bits(lay.x), inputs.bf16_bits(lay.gate_up),
                                   inputs.bf16_bits(lay.down), inputs.np32(lay.idx),
                                   inputs.np32(lay.w))


def _decode(moe, lay, dev, ws=None):
    return moe.moe_experts_decode_fused(lay.x.to(dev), lay.gate_up.to(dev), lay.down.to(dev),
                                        lay.idx.to(dev), lay.w.to(dev), lay.idx.shape[1],
                                        workspace=ws)


@pytest.mark.parametrize("T,H,F,E,K", [
    (1, 128, 128, 1, 1),       # 16 feature groups: most clusters and CTAs hold none
    (1, 256, 128, 2, 2),
    (3, 384, 256, 4, 2),       # experts shared by tokens
    (16, 256, 128, 8, 4),      # 64 slots, every expert with many slots
    (10, 1280, 896, 64, 6),    # the OCR-2 shape at 60 slots
    (5, 2048, 2048, 16, 4),    # the largest H and F the kernel takes
])
def test_fused_decode_shapes(moe, cuda_dev, T, H, F, E, K):
    """Full outputs against the oracle; 17 tokens are refused."""
    lay = inputs.ocr2_layer(T, seed=31 * T + H, device="cpu", H=H, F=F, E=E, K=K)
    out = _decode(moe, lay, cuda_dev)
    assert_matches_oracle(out, _ref(lay), "fused decode T=%d H=%d F=%d E=%d K=%d" % (T, H, F, E, K))
    with pytest.raises(moe.MoEError):        # 17 tokens: outside the one-kernel form
        lay17 = inputs.ocr2_layer(17, seed=1, device="cpu", H=H, F=F, E=E, K=1)
        _decode(moe, lay17, cuda_dev)


def test_fused_decode_hot_expert_and_slabs(moe, cuda_dev):
    """Every slot of 16 tokens on one expert (64 slots: eight-slot groups and
    several staging slabs per segment), then 10 tokens sharing two experts."""
    H, F, E, K = 1280, 896, 64, 4
    lay = inputs.ocr2_layer(16, seed=5, device="cpu", H=H, F=F, E=E, K=K)
    lay.idx[:] = 17
    assert_matches_oracle(_decode(moe, lay, cuda_dev), _ref(lay), "64 slots on one expert")
    lay = inputs.ocr2_layer(10, seed=6, device="cpu", H=H, F=F, E=E, K=6)
    lay.idx[:, 0] = 3
    lay.idx[:, 1] = 40
    assert_matches_oracle(_decode(moe, lay, cuda_dev), _ref(lay), "10 slots on two experts")


def test_fused_decode_invalid_and_empty_tokens(moe, cuda_dev):
    lay = inputs.ocr2_layer(6, seed=8, device="cpu")
    lay.idx[0, :] = 9                 # all slots of a token on one expert
    lay.idx[1, 2] = -1
    lay.idx[2, 5] = 64
    lay.idx[3, :] = -3                # no valid slot: output row 0
    lay.idx[4, 1] = lay.idx[4, 0]     # duplicate expert in one token
    out = _decode(moe, lay, cuda_dev)
    assert_matches_oracle(out, _ref(lay), "fused decode invalid ids")
    assert torch.count_nonzero(out[3].float()) == 0
    lay.idx[:] = -1                   # nothing valid at all
    out = torch.full((6, 1280), float("nan"), dtype=torch.bfloat16, device=cuda_dev)
    out = moe.moe_experts_decode_fused(lay.x.to(cuda_dev), lay.gate_up.to(cuda_dev),
                                       lay.down.to(cuda_dev), lay.idx.to(cuda_dev),
                                       lay.w.to(cuda_dev), 6, out=out)
    assert torch.count_nonzero(out.float()) == 0


def test_fused_decode_workspace_reuse_is_deterministic(moe, cuda_dev):
    """One workspace for many calls with different routings: every call
    leaves the header zero, so each result equals a fresh-workspace call bit
    for bit, and the status word stays clear."""
    H, F, E, K = 1280, 896, 64, 6
    base = inputs.ocr2_layer(1, seed=0, device=cuda_dev)
    ws = torch.zeros(moe.moe_experts_workspace_size(8, H, F, E, K, decode=True),
                     dtype=torch.uint8, device=cuda_dev)
    for T, seed in ((1, 1), (4, 2), (8, 3), (1, 4), (2, 5)):
        lay = inputs.ocr2_layer(T, seed=seed, device=cuda_dev, weights_from=base)
        a = moe.moe_experts_decode_fused(lay.x, lay.gate_up, lay.down, lay.idx, lay.w, K,
                                         workspace=ws)
        b = moe.moe_experts_decode_fused(lay.x, lay.gate_up, lay.down, lay.idx, lay.w, K)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), (T, seed)
    torch.cuda.synchronize()
    assert torch.count_nonzero(ws[:moe.WORKSPACE_HEADER_BYTES]) == 0
    assert moe.moe_workspace_status(ws) == 0
