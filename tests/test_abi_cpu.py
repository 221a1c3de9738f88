"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host (no GPU needed: validation happens before
any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def mod():
    import mixture_experts_routed_expert_b200 as m
    return m


def test_input_recipe_loads_no_library():
    """The seeded input recipe imports without loading libmoe_b200.so (the
    oracle-only reference arm uses it), while the entry points load it."""
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from mixture_experts_routed_expert_b200 import inputs\n"
            "inputs.ocr2_layer(2, seed=0, H=128, F=128, E=4, K=2)\n"
            "maps = open('/proc/self/maps').read()\n"
            "assert 'libmoe_b200' not in maps, 'library mapped by the input recipe'\n"
            "import mixture_experts_routed_expert_b200 as m\n"
            "m.lib.moe_abi_version()\n"
            "assert 'libmoe_b200' in open('/proc/self/maps').read()\n" % ROOT)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]


def test_exports_match_header(mod):
    decl = set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", open(HEADER).read()))
    assert decl == set(mod.EXPORTS)
    for name in decl:
        assert hasattr(mod.lib, name), name
    assert mod.lib.moe_abi_version() == 1
    assert mod.lib.moe_status_string(3) == b"MOE_ERR_WORKSPACE"


def test_workspace_sizes(mod):
    ws = mod.moe_experts_workspace_size
    assert ws(2048, 1280, 896, 64, 6) > 2048 * 6 * (1280 * 2 + 896 * 2 + 1280 * 4)
    # bf16 decode: the fused kernel's header, h (bf16) and y (fp32) by slot,
    # and at least what the fallback kernels need
    for T in (1, 2, 4, 8, 10):
        d = ws(T, 1280, 896, 64, 6, decode=True)
        assert d >= 8192 + T * 6 * (896 * 2 + 1280 * 4)
    assert ws(11, 1280, 896, 64, 6, decode=True) == ws(11, 1280, 896, 64, 6)   # 66 slots
    # E4M3 weights run the grouped GEMMs and need the prefill workspace
    assert ws(1, 7168, 2048, 256, 8, 1, decode=True) == ws(1, 7168, 2048, 256, 8, 1)
    # E4M3: codes, fp32 scales and their E8M0 bytes (rows padded to 16 bytes)
    # for x and h, and the fp32 y rows
    N, H, F = 2048 * 8, 7168, 2048
    need = N * (H + F + 4 * (H // 128 + F // 128) + 64 + 16 + 4 * H)
    assert ws(2048, H, F, 256, 8, 1) >= 8192 + need
    # every workspace starts with the 8 KiB header
    assert ws(16, 256, 256, 8, 2) > mod.WORKSPACE_HEADER_BYTES == 8192
    assert ws(16, 100, 896, 64, 6) == 0          # H % 128 != 0
    assert ws(16, 1280, 896, 0, 6) == 0          # E == 0
    assert ws(16, 1280, 896, 64, 17) == 0        # K > 16


def test_host_validation_without_gpu(mod):
    L = mod.lib
    N = None
    # T == 0 is a valid no-op
    assert L.moe_experts_prefill(N, N, N, N, N, 6, 0, 1280, 896, 64, 0, N, N, N, N, 0, N) == 0
    # bad sizes
    assert L.moe_experts_prefill(N, N, N, N, N, 6, 4, 1000, 896, 64, 0, N, N, N, N, 0, N) == 1
    assert L.moe_experts_decode(N, N, N, N, N, 0, 4, 1280, 896, 64, 0, N, N, N, N, 0, N) == 1
    # null tensors
    assert L.moe_experts_prefill(N, N, N, N, N, 6, 4, 1280, 896, 64, 0, N, N, N, N, 0, N) == 1
    # misaligned pointer
    p = ctypes.c_void_p(0x1000)
    q = ctypes.c_void_p(0x1001)
    assert L.moe_experts_prefill(q, p, p, p, p, 6, 4, 1280, 896, 64, 0, N, N, p, p, 1 << 30, N) == 1
    # FP8 without scales
    assert L.moe_experts_prefill(p, p, p, p, p, 6, 4, 1280, 896, 64, 1, N, N, p, p, 1 << 30, N) == 1
    # workspace too small / missing
    assert L.moe_experts_prefill(p, p, p, p, p, 6, 4, 1280, 896, 64, 0, N, N, p, p, 16, N) == 3
    assert L.moe_experts_prefill(p, p, p, p, p, 6, 4, 1280, 896, 64, 0, N, N, p, N, 0, N) == 3
    # router limits
    assert L.moe_route_sigmoid_grouped(p, p, 4, 256, 7, 4, 8, 2.5, p, p, N, N) == 1
    assert L.moe_route_sigmoid_grouped(p, p, 4, 256, 8, 9, 8, 2.5, p, p, N, N) == 1
    assert L.moe_route_sigmoid_grouped(p, p, 0, 256, 8, 4, 8, 2.5, p, p, N, N) == 0
    # quantiser limits
    assert L.quantize_fp8_block128(p, 4, 100, p, p, N) == 1
    assert L.quantize_fp8_block128(p, 0, 128, p, p, N) == 0
    # workspace header helpers
    assert L.moe_workspace_init(N, 4096, N) == 1
    assert L.moe_workspace_init(p, 4096, N) == 1
    assert L.moe_workspace_status(N, 0, N) == 1
    assert L.moe_workspace_status(q, 0, N) == 1
    assert L.moe_debug_decode_withhold(p, p, p, p, p, 6, 1, 1280, 896, 64, p, p, 1 << 30, -1, N) == 1
    # input staging: sizes in 16-byte units, aligned pointers
    assert L.moe_stage_inputs(N, N, 0, N) == 0
    assert L.moe_stage_inputs(p, p, 24, N) == 1
    assert L.moe_stage_inputs(q, p, 32, N) == 1
    assert L.moe_stage_inputs(p, N, 32, N) == 1


def test_shared_entry_host_checks(mod):
    """moe_experts_with_shared: sizes, workspace and pointer checks on the host."""
    ws = mod.moe_experts_shared_workspace_size
    # widened to E+S experts and K+S slots, plus the widened routing
    assert ws(64, 1280, 896, 64, 6, 2) > mod.moe_experts_workspace_size(64, 1280, 896, 66, 8)
    assert ws(64, 1280, 896, 64, 6, 0) > mod.moe_experts_workspace_size(64, 1280, 896, 64, 6)
    assert ws(64, 1280, 896, 64, 6, 11) == 0       # K + S > 16
    assert ws(64, 1280, 896, 1020, 6, 5) == 0      # E + S > 1024
    assert ws(64, 1280, 896, 64, 6, -1) == 0
    L = mod.lib
    N = None
    p = ctypes.c_void_p(0x1000)
    q = ctypes.c_void_p(0x1001)
    big = 1 << 34
    f = L.moe_experts_with_shared
    # T == 0 no-op; bad S
    assert f(N, N, N, N, N, 6, 0, 1280, 896, 64, 0, N, N, N, N, N, N, 2, N, N, N, 0, N) == 0
    assert f(p, p, p, p, p, 6, 4, 1280, 896, 64, 0, N, N, p, p, N, N, 11, N, p, p, big, N) == 1
    # shared weights missing or misaligned; residual misaligned
    assert f(p, p, p, p, p, 6, 4, 1280, 896, 64, 0, N, N, N, p, N, N, 2, N, p, p, big, N) == 1
    assert f(p, p, p, p, p, 6, 4, 1280, 896, 64, 0, N, N, q, p, N, N, 2, N, p, p, big, N) == 1
    assert f(p, p, p, p, p, 6, 4, 1280, 896, 64, 0, N, N, p, p, N, N, 2, q, p, p, big, N) == 1
    # E4M3 without the shared scales
    assert f(p, p, p, p, p, 6, 4, 1280, 896, 64, 1, p, p, p, p, N, N, 2, N, p, p, big, N) == 1
    # workspace too small
    assert f(p, p, p, p, p, 6, 4, 1280, 896, 64, 0, N, N, p, p, N, N, 2, N, p, p, 4096, N) == 3


def test_mxfp4_host_checks(mod):
    """MXFP4 weights: scales required, weights 32-byte aligned; workspace
    holds E8M0 scale bytes; no shared-expert or static-scratch form."""
    L = mod.lib
    N = None
    p = ctypes.c_void_p(0x1000)
    p16 = ctypes.c_void_p(0x1010)            # 16- but not 32-byte aligned
    big = 1 << 34
    W = mod.MOE_W_MXFP4
    assert W == 2
    assert L.moe_experts_prefill(p, p, p, p, p, 8, 4, 7168, 2048, 256, W, N, N, p, p, big, N) == 1
    assert L.moe_experts_prefill(p, p16, p, p, p, 8, 4, 7168, 2048, 256, W, p, p, p, p, big, N) == 1
    assert L.moe_experts_prefill(p, p, p, p, p, 8, 4, 7168, 2048, 256, W, p, p, p, p, 64, N) == 3
    ws = mod.moe_experts_workspace_size
    assert 0 < ws(64, 7168, 2048, 256, 8, W) < ws(64, 7168, 2048, 256, 8, mod.MOE_W_FP8_E4M3)
    assert ws(4, 7168, 2048, 256, 8, W, decode=True) == ws(4, 7168, 2048, 256, 8, W)
    f = L.moe_experts_with_shared
    assert f(p, p, p, p, p, 8, 4, 7168, 2048, 256, W, p, p, p, p, N, N, 1, N, p, p, big, N) == 2
    assert L.moe_experts_decode_static(p, p, p, p, p, 6, 1, 1280, 896, 64, W, p, p, p, N) == 2


def test_binding_argument_checks(mod):
    """The Python binding rejects wrong shapes, dtypes and devices before any
    C call, and maps weight dtypes (and weight_format) to the C weight type."""
    import torch
    T, H, F, E, K = 4, 256, 128, 8, 2
    x = torch.zeros(T, H, dtype=torch.bfloat16)
    gu = torch.zeros(E, 2 * F, H, dtype=torch.bfloat16)
    dn = torch.zeros(E, H, F, dtype=torch.bfloat16)
    idx = torch.zeros(T, K, dtype=torch.int32)
    w = torch.zeros(T, K, dtype=torch.float32)
    fwd = mod.moe_experts_prefill
    with pytest.raises(ValueError, match="shape mismatch"):
        fwd(x[:, :128], gu, dn, idx, w, K)
    with pytest.raises(ValueError, match="shape mismatch"):
        fwd(x, gu, dn[:, :, :64], idx, w, K)
    with pytest.raises(ValueError, match="top_k"):
        fwd(x, gu, dn, idx[:, :1], w, K)
    with pytest.raises(TypeError, match="int32"):
        fwd(x, gu, dn, idx.long(), w, K)
    with pytest.raises(TypeError, match="bf16"):
        fwd(x.float(), gu, dn, idx, w, K)
    with pytest.raises(ValueError, match="CUDA"):       # host tensors never reach the library
        fwd(x, gu, dn, idx, w, K)
    # packed MXFP4 shapes: gate_up [E][2F][H/2], down [E][H][F/2]
    gu4 = torch.zeros(E, 2 * F, H // 2, dtype=torch.uint8)
    dn4 = torch.zeros(E, H, F // 2, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):
        fwd(x, gu4, dn4, idx, w, K, weight_format="mxfp4")
    with pytest.raises(ValueError, match="shape mismatch"):
        fwd(x, gu4, dn4, idx, w, K)                     # read as E4M3: H/2 columns
    # the static-scratch decode entry runs the same checks before its C call
    st = mod.moe_experts_decode_static
    with pytest.raises(ValueError, match="shape mismatch"):
        st(x, gu, dn[:, :, :64], idx, w, K)
    with pytest.raises(TypeError, match="int32"):
        st(x, gu, dn, idx.long(), w, K)
    with pytest.raises(TypeError, match="bf16"):
        st(x.float(), gu, dn, idx, w, K)
    with pytest.raises(ValueError, match="CUDA"):
        st(x, gu, dn, idx, w, K)
    with pytest.raises(ValueError, match="out must be"):
        st(x, gu, dn, idx, w, K, out=torch.zeros(T, H + 128, dtype=torch.bfloat16))
    wt = mod._wtype
    assert wt(gu) == mod.MOE_W_BF16
    assert wt(gu4) == mod.MOE_W_FP8_E4M3
    assert wt(gu4.view(torch.float8_e4m3fn)) == mod.MOE_W_FP8_E4M3
    assert wt(gu4, "mxfp4") == mod.MOE_W_MXFP4
    with pytest.raises(TypeError):
        wt(gu, "mxfp4")
    with pytest.raises(TypeError):
        wt(gu.float())
