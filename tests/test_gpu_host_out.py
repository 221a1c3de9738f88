"""The forward entry points take any device-accessible output pointer: with
out in mapped pinned host memory the kernels store the result directly
(no copy back), bit-identical to a device-memory output."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _mapped(nbytes):
    rt = pytest.importorskip("cuda.bindings.runtime")
    ok = rt.cudaError_t.cudaSuccess
    err, hp = rt.cudaHostAlloc(nbytes, rt.cudaHostAllocMapped | rt.cudaHostAllocPortable)
    if err != ok:
        pytest.skip("no mapped pinned host memory")
    err, dp = rt.cudaHostGetDevicePointer(hp, 0)
    if err != ok or not dp:
        rt.cudaFreeHost(hp)
        pytest.skip("host memory not mapped into the device address space")
    return rt, int(hp), int(dp)


@pytest.mark.parametrize("T,entry", [(1, "moe_experts_decode"), (4, "moe_experts_decode"),
                                     (64, "moe_experts_prefill")])
def test_output_in_mapped_host_memory(cuda_dev, T, entry):
    import mixture_experts_routed_expert_b200 as moe
    from mixture_experts_routed_expert_b200 import inputs

    lay = inputs.ocr2_layer(T, seed=40 + T, device=cuda_dev)
    H, F, E, K = 1280, 896, 64, 6
    ref = getattr(moe, entry)(lay.x, lay.gate_up, lay.down, lay.idx, lay.w, K)
    nbytes = T * H * 2
    rt, hp, dp = _mapped(nbytes)
    try:
        ctypes.memset(hp, 0xFF, nbytes)
        ws = torch.empty(max(moe.moe_experts_workspace_size(T, H, F, E, K, 0, entry.endswith("decode")), 256),
                         dtype=torch.uint8, device=cuda_dev)
        C = ctypes.c_void_p
        rc = getattr(moe.lib, entry)(C(lay.x.data_ptr()), C(lay.gate_up.data_ptr()),
                                     C(lay.down.data_ptr()), C(lay.idx.data_ptr()),
                                     C(lay.w.data_ptr()), K, T, H, F, E, 0, None, None, C(dp),
                                     C(ws.data_ptr()), ws.numel(),
                                     C(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, moe.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        got = np.frombuffer(ctypes.string_at(hp, nbytes), dtype=np.uint16)
        want = ref.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
        assert np.array_equal(got, want)
    finally:
        rt.cudaFreeHost(hp)
