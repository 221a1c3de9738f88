"""GPU parity of the side kernels against the oracle, bit-exact:
block-128 E4M3 quantisation (S2), group-aware sigmoid router (S1), expert
histogram / offsets / stable permutation (S3)."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_routed_expert_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_dev):
    import mixture_experts_routed_expert_b200 as m
    return m


@pytest.mark.parametrize("rows,cols", [(1, 128), (7, 7168), (129, 2048), (300, 1280)])
def test_quantize_bit_exact(moe, cuda_dev, rows, cols):
    g = torch.Generator().manual_seed(rows * 7 + cols)
    x = torch.randn(rows, cols, generator=g) * torch.exp2(torch.randint(-30, 30, (rows, 1), generator=g).float())
    x[0, :128] = 0.0                      # all-zero block
    if cols > 256:
        x[0, 128] = -0.0
        x[0, 256:384] = 448.0
    xb = x.to(torch.bfloat16)
    q, s = moe.quantize_fp8_block128(xb.to(cuda_dev))
    rq, rs = oracle.quantize_fp8_block128(inputs.bf16_bits(xb))
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy(), rs)


@pytest.mark.parametrize("T,E,G,TG,K", [(1, 256, 8, 4, 8), (128, 256, 8, 4, 8), (1000, 256, 8, 4, 8),
                                        (300, 64, 1, 1, 6), (64, 1024, 32, 5, 16), (50, 16, 4, 2, 3)])
def test_router_bit_exact(moe, cuda_dev, T, E, G, TG, K):
    lay = inputs.fp8_layer(T, seed=T + E, device="cpu", H=128, F=128, E=E, weights=(None,) * 4)
    lg, bias = lay.logits, lay.bias
    if T >= 50:
        lg[3] = 0.0                       # a token whose scores all tie
        bias[:] = torch.where(torch.arange(E) % 3 == 0, bias, torch.zeros(E))
    idx, w, off = moe.moe_route_sigmoid_grouped(lg.to(cuda_dev), bias.to(cuda_dev), G, TG, K, 2.5,
                                                want_offsets=True)
    ridx, rw = oracle.route_sigmoid_grouped(lg.numpy(), bias.numpy(), G, TG, K, 2.5)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.array_equal(w.cpu().numpy(), rw)
    _, roff, _, _ = oracle.permute(ridx, E)
    assert np.array_equal(off.cpu().numpy(), roff)


@pytest.mark.parametrize("T,K,E,skew", [(1, 6, 64, None), (16, 6, 64, None), (2048, 6, 64, None),
                                        (777, 8, 256, 1.1), (8192, 8, 256, 1.1), (5, 4, 1024, None),
                                        (512, 8, 64, None), (513, 8, 64, None)])   # 4096 / 4104 slots
def test_permute_bit_exact(moe, cuda_dev, T, K, E, skew):
    lay = inputs.ocr2_layer(T, seed=T, device="cpu", H=128, F=128, E=E, K=K, zipf=skew)
    idx = lay.idx.clone()
    if T > 20:
        idx[5, 1] = -1
        idx[7, 0] = E + 3
        idx[9, :] = idx[9, 0]             # duplicate expert inside one token
    counts, offsets, perm, inv = moe.moe_debug_permute(idx.to(cuda_dev), E)
    rc, ro, rp, ri = oracle.permute(idx.numpy(), E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(inv.cpu().numpy(), ri)
