"""The forward entry points take any device-accessible output pointer: with
out in mapped pinned host memory the kernels store the result directly
(no copy back), bit-identical to a device-memory output.  moe_stage_inputs
moves a step's inputs from mapped pinned host memory to the device with one
kernel, seeing host writes made between steps."""
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


def test_stage_inputs_from_mapped_host_memory(cuda_dev):
    import mixture_experts_routed_expert_b200 as moe
    from mixture_experts_routed_expert_b200 import inputs

    H, F, E, K = 1280, 896, 64, 6
    base = inputs.ocr2_layer(1, seed=0, device=cuda_dev)
    # x [1,H] bf16, ids [1,K] int32, weights [1,K] fp32 packed at 256-byte offsets
    offs, nbytes = (0, 2 * H, 2 * H + 256), 2 * H + 512
    rt, hp, dp = _mapped(nbytes)
    try:
        dbuf = torch.empty(nbytes, dtype=torch.uint8, device=cuda_dev)
        x = dbuf[0:2 * H].view(torch.bfloat16).view(1, H)
        idx = dbuf[offs[1]:offs[1] + 4 * K].view(torch.int32).view(1, K)
        w = dbuf[offs[2]:offs[2] + 4 * K].view(torch.float32).view(1, K)
        for step in range(3):   # new host inputs before every step
            lay = inputs.ocr2_layer(1, seed=70 + step, device=cuda_dev, weights_from=base)
            for t, o in zip((lay.x, lay.idx, lay.w), offs):
                b = t.cpu().contiguous().view(-1).view(torch.uint8).numpy().tobytes()
                ctypes.memmove(hp + o, b, len(b))
            moe.moe_stage_inputs(dp, dbuf)
            out = moe.moe_experts_decode(x, lay.gate_up, lay.down, idx, w, K)
            ref = moe.moe_experts_decode(lay.x, lay.gate_up, lay.down, lay.idx, lay.w, K)
            torch.cuda.synchronize()
            assert torch.equal(dbuf[0:2 * H].view(torch.bfloat16).view(1, H), lay.x)
            assert torch.equal(out, ref), "step %d" % step
        # several sizes (multiples of 16 bytes) land byte for byte, nothing beyond
        pattern = np.random.default_rng(1).integers(0, 256, nbytes, dtype=np.uint8)
        ctypes.memmove(hp, pattern.tobytes(), nbytes)
        for n in (16, 48, 2560, nbytes):
            dst = torch.zeros(nbytes, dtype=torch.uint8, device=cuda_dev)
            moe.moe_stage_inputs(dp, dst, n)
            torch.cuda.synchronize()
            got = dst.cpu().numpy()
            assert np.array_equal(got[:n], pattern[:n]) and not got[n:].any()
        with pytest.raises(moe.MoEError):
            moe.moe_stage_inputs(dp, dbuf, 24)          # not a multiple of 16
    finally:
        rt.cudaFreeHost(hp)
