"""GPU parity of the bf16 routed-experts forward (decode and prefill paths)
against the oracle: full outputs at sizes the oracle finishes in seconds
(several tiles plus a ragged tail), sampled tokens at the OCR-2 prefill size,
edge cases (T=0, duplicate and out-of-range expert ids, empty experts,
experts with more rows than one tile), and run-to-run determinism."""
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


@pytest.fixture(scope="module")
def ocr_weights(cuda_dev):
    return inputs.ocr2_layer(16, seed=0, device="cpu")


def _ref(lay, tokens=None):
    x, idx, w = lay.x, lay.idx, lay.w
    if tokens is not None:
        x, idx, w = x[tokens], idx[tokens], w[tokens]
    return oracle.moe_forward_bf16(inputs.bf16_bits(x), inputs.bf16_bits(lay.gate_up),
                                   inputs.bf16_bits(lay.down), inputs.np32(idx), inputs.np32(w))


def _run(moe, lay, dev, fn):
    gu = lay.gate_up.to(dev)
    dn = lay.down.to(dev)
    return getattr(moe, fn)(lay.x.to(dev), gu, dn, lay.idx.to(dev), lay.w.to(dev), lay.idx.shape[1])


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_decode_ocr2(moe, cuda_dev, ocr_weights, T):
    lay = inputs.ocr2_layer(T, seed=100 + T, device="cpu", weights_from=ocr_weights)
    out = _run(moe, lay, cuda_dev, "moe_experts_decode")
    assert_matches_oracle(out, _ref(lay), "decode T=%d" % T)


def test_decode_edge_ids(moe, cuda_dev, ocr_weights):
    lay = inputs.ocr2_layer(4, seed=7, device="cpu", weights_from=ocr_weights)
    lay.idx[0, :] = 5                     # all slots of a token on one expert
    lay.idx[1, 2] = -1                    # out-of-range ids contribute nothing
    lay.idx[2, 4] = 64
    lay.idx[3, 1] = lay.idx[3, 0]         # duplicate expert
    out = _run(moe, lay, cuda_dev, "moe_experts_decode")
    assert_matches_oracle(out, _ref(lay), "decode edge ids")


def test_prefill_ocr2_tiny(moe, cuda_dev, ocr_weights):
    lay = inputs.ocr2_layer(16, seed=0, device="cpu")
    out = _run(moe, lay, cuda_dev, "moe_experts_prefill")
    assert_matches_oracle(out, _ref(lay), "prefill T=16")
    out_d = _run(moe, lay, cuda_dev, "moe_experts_decode")   # served by the prefill kernels
    assert torch.equal(out, out_d)


@pytest.mark.parametrize("T,H,F,E,K,skew", [
    (300, 1280, 896, 64, 6, None),     # ragged tiles on the OCR-2 shape
    (700, 256, 384, 8, 2, None),       # ~175 rows per expert: two gate_up row tiles
    (600, 128, 128, 2, 1, None),       # ~300 rows per expert: two down row tiles
    (512, 384, 256, 64, 6, 1.1),       # Zipf skew: empty experts, one hot expert
    (33, 1280, 896, 64, 6, None),
])
def test_prefill_shapes(moe, cuda_dev, T, H, F, E, K, skew):
    lay = inputs.ocr2_layer(T, seed=T + H, device="cpu", H=H, F=F, E=E, K=K, zipf=skew)
    out = _run(moe, lay, cuda_dev, "moe_experts_prefill")
    assert_matches_oracle(out, _ref(lay), "prefill T=%d H=%d F=%d E=%d" % (T, H, F, E))


def test_prefill_ocr2_full_size_sampled(moe, cuda_dev):
    lay = inputs.ocr2_layer(2048, seed=0, device="cpu")
    lay.idx[11, 3] = -1
    out = _run(moe, lay, cuda_dev, "moe_experts_prefill")
    tokens = parity_sample(lay.idx.numpy(), 64, grouped_tile_heights(2048, 6, 64, "bf16"),
                           n_min=48, seed=0)
    tokens = torch.tensor(sorted(set(tokens) | {11}))
    assert_matches_oracle(out[tokens], _ref(lay, tokens), "prefill T=2048 sampled")
    out2 = _run(moe, lay, cuda_dev, "moe_experts_prefill")
    assert torch.equal(out, out2), "prefill is not deterministic"


def test_prefill_zero_tokens_and_zero_weights(moe, cuda_dev, ocr_weights):
    lay = inputs.ocr2_layer(0, seed=1, device="cpu", weights_from=ocr_weights)
    out = _run(moe, lay, cuda_dev, "moe_experts_prefill")
    assert out.shape == (0, 1280)
    lay = inputs.ocr2_layer(40, seed=2, device="cpu", weights_from=ocr_weights)
    lay.w.zero_()
    out = _run(moe, lay, cuda_dev, "moe_experts_prefill")
    assert torch.count_nonzero(out.float()) == 0


@pytest.mark.parametrize("T", [1, 5, 16, 17])
def test_prefill_few_tokens_invalid_slots(moe, cuda_dev, ocr_weights, T):
    """Few tokens through the grouped GEMMs: a token whose slots are all
    invalid, repeated calls, and a call where no slot is valid (no tiles)."""
    lay = inputs.ocr2_layer(T, seed=90 + T, device="cpu", weights_from=ocr_weights)
    if T > 1:
        lay.idx[1, :] = -1
    out = _run(moe, lay, cuda_dev, "moe_experts_prefill")
    assert_matches_oracle(out, _ref(lay), "prefill T=%d invalid slots" % T)
    if T > 1:
        assert torch.count_nonzero(out[1].float()) == 0
    for _ in range(2):                       # deterministic across calls
        assert torch.equal(_run(moe, lay, cuda_dev, "moe_experts_prefill"), out)
    lay.idx.fill_(-1)
    out0 = torch.full((T, 1280), float("nan"), dtype=torch.bfloat16, device=cuda_dev)
    out0 = moe.moe_experts_prefill(lay.x.to(cuda_dev), lay.gate_up.to(cuda_dev), lay.down.to(cuda_dev),
                                   lay.idx.to(cuda_dev), lay.w.to(cuda_dev), 6, out=out0)
    assert torch.count_nonzero(out0.float()) == 0
