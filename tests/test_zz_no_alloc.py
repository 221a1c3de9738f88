"""moe_experts_decode_static: the decode entry point for callers that cannot
allocate device memory (graph capture that forbids allocation, fixed-budget
serving or real-time hosts, plugin hosts without an allocator).  Its scratch
is a fixed array inside the library, shared by all calls.

Called through the C ABI (ctypes, no Python-side allocation of a workspace)
and compared with moe_experts_decode, the entry point that takes a
workspace, within the tolerance used by the other parity tests, on two calls
in a row.  Kept in a file pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

REL_L2 = 5e-3


def _rel(a, b):
    a = a.float().cpu().double().numpy()
    b = b.float().cpu().double().numpy()
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30), np.abs(a - b).max()


def test_decode_static_matches_decode(cuda_dev):
    import mixture_experts_routed_expert_b200 as moe
    from mixture_experts_routed_expert_b200 import inputs

    lib = moe.lib
    stream = torch.cuda.current_stream()
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    base = inputs.ocr2_layer(4, seed=3, device=cuda_dev)
    H, F, E, K = 1280, 896, 64, 6
    for T, seed in ((4, 11), (1, 12), (8, 13)):   # gather-GEMV kernels up to 48 slots
        lay = inputs.ocr2_layer(T, seed=seed, device=cuda_dev, weights_from=base)
        ref = moe.moe_experts_decode(lay.x, lay.gate_up, lay.down, lay.idx, lay.w, K)
        outs = []
        for _ in range(2):                       # two calls in a row
            out = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device=cuda_dev)
            rc = lib.moe_experts_decode_static(P(lay.x), P(lay.gate_up), P(lay.down), P(lay.idx),
                                               P(lay.w), K, T, H, F, E, 0, None, None, P(out),
                                               ctypes.c_void_p(stream.cuda_stream))
            assert rc == 0, moe.STATUS.get(rc, rc)
            outs.append(out)
        torch.cuda.synchronize()
        for out in outs:
            rel, mx = _rel(out, ref)
            assert rel <= REL_L2 and mx <= 1e-2 * float(ref.float().abs().max()), (T, rel, mx)


def test_decode_static_rejects_oversize(cuda_dev):
    import mixture_experts_routed_expert_b200 as moe
    lib = moe.lib
    p = ctypes.c_void_p(256)
    # outside the decode range: T*K > 64, and F > 2048 (every size inside the
    # range fits the 1 MiB array, which the library checks at compile time)
    assert lib.moe_experts_decode_static(p, p, p, p, p, 8, 16, 1280, 896, 64, 0, None, None, p, None) == 3
    assert lib.moe_experts_decode_static(p, p, p, p, p, 16, 4, 1280, 16384, 64, 0, None, None, p, None) == 3
    # quantised weights are not served, whatever the sizes
    assert lib.moe_experts_decode_static(p, p, p, p, p, 8, 16, 1280, 896, 64, 1, p, p, p, None) == 2
