"""GPU parity of every point of the skewed sweep that bench.py times:
Zipf(1.1) expert popularity at T = 1, 8, 64, 512, 2048 and 8192 on the
DeepSeek-V3-like layer with E4M3 weights and with MXFP4 weights, and on the
OCR-2 bf16 layer.  Inputs are drawn exactly as the bench draws them (same
seeds, same device, same entry point: the decode entry where T*K <= 64),
routing by the oracle's group-sigmoid router, which is also checked bit for
bit against the library's router on these logits.  Outputs are compared
with the oracle in full where the oracle is quick (bf16 up to T = 512, the
quantised layers up to T = 8) and otherwise on a sample holding the hottest
expert's last row tile, every token of the rarest non-empty expert and at
least 16 tokens."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_matches_oracle, grouped_tile_heights, parity_sample
from mixture_experts_routed_expert_b200 import inputs

pytestmark = pytest.mark.gpu

SWEEP = (1, 8, 64, 512, 2048, 8192)
ZIPF = 1.1


@pytest.fixture(scope="module")
def moe(cuda_dev):
    import mixture_experts_routed_expert_b200 as m
    return m


def _route_checked(moe, lay, D):
    """Oracle routing of the layer's logits; the library's router must give
    the same ids and weights bit for bit."""
    idx, w = oracle.route_sigmoid_grouped(inputs.np32(lay.logits), inputs.np32(lay.bias),
                                          D["num_groups"], D["topk_group"], D["K"], D["scale"])
    gi, gw = moe.moe_route_sigmoid_grouped(lay.logits, lay.bias, D["num_groups"], D["topk_group"],
                                           D["K"], D["scale"])
    assert np.array_equal(gi.cpu().numpy(), idx)
    assert np.array_equal(gw.cpu().numpy().view(np.uint32), w.view(np.uint32))
    return torch.from_numpy(idx), torch.from_numpy(w)


def _touched(idx, E, tokens):
    """Experts used by `tokens`, and their ids remapped to 0..n-1 (ids
    outside [0, E) stay invalid) so that only those experts go to the host."""
    sub = idx[tokens]
    valid = (sub >= 0) & (sub < E)
    used = torch.unique(sub[valid])
    remap = torch.full((E,), -1, dtype=torch.int32)
    remap[used.long()] = torch.arange(len(used), dtype=torch.int32)
    ridx = torch.where(valid, remap[sub.clamp(0, E - 1).long()], torch.full_like(sub, -1))
    return used.long(), ridx.to(torch.int32)


# ------------------------------------------------------------ OCR-2 bf16 ----

@pytest.fixture(scope="module")
def ocr_base(cuda_dev):
    return inputs.ocr2_layer(1, seed=0, device=cuda_dev)


@pytest.fixture(scope="module")
def ocr_host_weights(ocr_base):
    return inputs.bf16_bits(ocr_base.gate_up), inputs.bf16_bits(ocr_base.down)


@pytest.mark.parametrize("T", SWEEP)
def test_zipf_sweep_bf16(moe, cuda_dev, ocr_base, ocr_host_weights, T):
    H, F, E, K = 1280, 896, 64, 6
    lay = inputs.ocr2_layer(T, seed=T, device=cuda_dev, weights_from=ocr_base, zipf=ZIPF)
    fn = moe.moe_experts_decode if T * K <= 64 else moe.moe_experts_prefill
    out = fn(lay.x, lay.gate_up, lay.down, lay.idx, lay.w, K)
    idx = lay.idx.cpu()
    tokens = list(range(T)) if T <= 512 else parity_sample(
        idx.numpy(), E, grouped_tile_heights(T, K, E, "bf16"), seed=T)
    tk = torch.tensor(tokens)
    gu, dn = ocr_host_weights
    ref = oracle.moe_forward_bf16(inputs.bf16_bits(lay.x.cpu()[tk]), gu, dn,
                                  inputs.np32(idx[tk]), inputs.np32(lay.w.cpu()[tk]))
    assert_matches_oracle(out[tk.to(out.device)], ref, "bf16 zipf T=%d" % T)


# ---------------------------------------------------- DeepSeek-V3-like E4M3 --

@pytest.fixture(scope="module")
def fp8_w(cuda_dev):
    return inputs.fp8_weights(seed=0, device=cuda_dev)


@pytest.mark.parametrize("T", SWEEP)
def test_zipf_sweep_fp8(moe, cuda_dev, fp8_w, T):
    D = inputs.DSV3_FP8
    E, K = D["E"], D["K"]
    lay = inputs.fp8_layer(T, seed=T, device=cuda_dev, weights=fp8_w, zipf=ZIPF)
    idx, w = _route_checked(moe, lay, D)
    if T >= 2048:
        counts = np.bincount(idx.numpy().reshape(-1), minlength=E)
        assert counts.max() > 64 and (counts == 0).any()
    fn = moe.moe_experts_decode if T * K <= 64 else moe.moe_experts_prefill
    out = fn(lay.x, lay.w13, lay.w2, idx.to(cuda_dev), w.to(cuda_dev), K,
             gate_up_scale=lay.w13_scale, down_scale=lay.w2_scale)
    tokens = list(range(T)) if T <= 8 else parity_sample(
        idx.numpy(), E, grouped_tile_heights(T, K, E, "e4m3"), seed=T)
    used, ridx = _touched(idx, E, tokens)
    sel = used.to(cuda_dev)
    tk = torch.tensor(tokens)
    ref = oracle.moe_forward_fp8(inputs.bf16_bits(lay.x.cpu()[tk]), inputs.u8(lay.w13[sel]),
                                 inputs.np32(lay.w13_scale[sel]), inputs.u8(lay.w2[sel]),
                                 inputs.np32(lay.w2_scale[sel]), inputs.np32(ridx),
                                 inputs.np32(w[tk]))
    assert_matches_oracle(out[tk.to(out.device)], ref, "e4m3 zipf T=%d" % T)


# --------------------------------------------------- DeepSeek-V3-like MXFP4 --

@pytest.fixture(scope="module")
def mxf4_w(cuda_dev):
    return inputs.mxf4_weights(seed=0, device=cuda_dev)


@pytest.mark.parametrize("T", SWEEP)
def test_zipf_sweep_mxf4(moe, cuda_dev, mxf4_w, T):
    D = inputs.DSV3_FP8
    E, K = D["E"], D["K"]
    lay = inputs.fp8_layer(T, seed=T, device=cuda_dev, weights=(None, None, None, None),
                           zipf=ZIPF)
    idx, w = _route_checked(moe, lay, D)
    fn = moe.moe_experts_decode if T * K <= 64 else moe.moe_experts_prefill
    w13, w13s, w2, w2s = mxf4_w
    out = fn(lay.x, w13, w2, idx.to(cuda_dev), w.to(cuda_dev), K, gate_up_scale=w13s,
             down_scale=w2s, weight_format="mxfp4")
    tokens = list(range(T)) if T <= 8 else parity_sample(
        idx.numpy(), E, grouped_tile_heights(T, K, E, "mxfp4"), seed=T)
    used, ridx = _touched(idx, E, tokens)
    sel = used.to(cuda_dev)
    tk = torch.tensor(tokens)
    ref = oracle.moe_forward_mxf4(inputs.bf16_bits(lay.x.cpu()[tk]), inputs.u8(w13[sel]),
                                  inputs.u8(w13s[sel]), inputs.u8(w2[sel]), inputs.u8(w2s[sel]),
                                  inputs.np32(ridx), inputs.np32(w[tk]))
    assert_matches_oracle(out[tk.to(out.device)], ref, "mxf4 zipf T=%d" % T)
