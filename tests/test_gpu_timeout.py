"""Failure detection on the GPU without a fault: the fused bf16 decode
kernel's bounded wait is made to expire (the test-only entry point keeps
CTA 0 from ever issuing one chunk's weight copies, so nothing completes that
wait), the kernel returns, moe_workspace_status reports MOE_ERR_TIMEOUT, and
the same workspace, once cleared, serves a normal call whose output matches
the oracle (the context stays usable)."""
import ctypes

import pytest
import torch

import oracle
from _helpers import assert_matches_oracle
from mixture_experts_routed_expert_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunk", [0, 3])
def test_decode_wait_expires_and_is_reported(cuda_dev, chunk):
    import mixture_experts_routed_expert_b200 as moe
    H, F, E, K = 1280, 896, 64, 6
    lay = inputs.ocr2_layer(1, seed=21 + chunk, device=cuda_dev)
    ws = torch.zeros(moe.moe_experts_workspace_size(1, H, F, E, K, decode=True),
                     dtype=torch.uint8, device=cuda_dev)
    out = torch.empty(1, H, dtype=torch.bfloat16, device=cuda_dev)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = moe.lib.moe_debug_decode_withhold(P(lay.x), P(lay.gate_up), P(lay.down), P(lay.idx),
                                           P(lay.w), K, 1, H, F, E, P(out), P(ws), ws.numel(),
                                           chunk, stream)
    assert rc == 0, moe.STATUS.get(rc, rc)
    assert moe.moe_workspace_status(ws, clear=True) == 5          # MOE_ERR_TIMEOUT
    assert torch.count_nonzero(ws[:moe.WORKSPACE_HEADER_BYTES]) == 0
    assert moe.moe_workspace_status(ws) == 0
    # the device and the cleared workspace still serve a normal call
    out = moe.moe_experts_decode_fused(lay.x, lay.gate_up, lay.down, lay.idx, lay.w, K,
                                       workspace=ws)
    ref = oracle.moe_forward_bf16(inputs.bf16_bits(lay.x), inputs.bf16_bits(lay.gate_up),
                                  inputs.bf16_bits(lay.down), inputs.np32(lay.idx),
                                  inputs.np32(lay.w))
    assert_matches_oracle(out, ref, "decode after a timeout")
    assert moe.moe_workspace_status(ws) == 0
