"""B200 (sm_100a) routed-experts MoE forward.

Thin Python binding of ``libmoe_b200.so`` (C ABI in ``include/moe_b200.h``).
Every function here only marshals arguments -- shapes, dtypes, device
pointers, the current CUDA stream -- and calls the C entry point of the same
name; all arithmetic runs in the library's CUDA kernels.  torch is used for
device memory (outputs, workspaces) and streams only.

The library must be built (``python mixture_experts_routed_expert_b200/build.py``
or ``__graft_entry__.build()``).  It is loaded on first use -- the first
call of an entry point or the first access to ``lib`` -- so that the input
recipe (``mixture_experts_routed_expert_b200.inputs``) imports without it;
every entry point raises ImportError when it is missing.  There is no CPU
fallback.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_W_BF16 = 0
MOE_W_FP8_E4M3 = 1
MOE_W_MXFP4 = 2
WORKSPACE_HEADER_BYTES = 8192   # zero before a workspace's first use (include/moe_b200.h)
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT"}

EXPORTS = ("moe_abi_version", "moe_status_string", "moe_experts_workspace_size",
           "moe_experts_prefill", "moe_experts_decode", "moe_route_sigmoid_grouped",
           "quantize_fp8_block128", "moe_debug_permute", "moe_experts_decode_static",
           "moe_experts_shared_workspace_size", "moe_experts_with_shared",
           "moe_experts_decode_fused", "moe_stage_inputs", "moe_workspace_init",
           "moe_workspace_status", "moe_debug_decode_withhold", "moe_experts_rows",
           "moe_combine_rows")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libmoe_b200.so is not built (run __graft_entry__.build() or "
                          "python -m mixture_experts_routed_expert_b200.build)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    L.moe_abi_version.restype = I
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [I]
    L.moe_experts_workspace_size.restype = Z
    L.moe_experts_workspace_size.argtypes = [I, I, I, I, I, I, I]
    fwd = [P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, Z, P]
    L.moe_experts_prefill.argtypes = fwd
    L.moe_experts_decode.argtypes = fwd
    L.moe_experts_decode_fused.argtypes = fwd
    L.moe_route_sigmoid_grouped.argtypes = [P, P, I, I, I, I, I, F, P, P, P, P]
    L.quantize_fp8_block128.argtypes = [P, I, I, P, P, P]
    L.moe_debug_permute.argtypes = [P, I, I, I, P, P, P, P, P, Z, P]
    L.moe_experts_shared_workspace_size.restype = Z
    L.moe_experts_shared_workspace_size.argtypes = [I, I, I, I, I, I, I]
    L.moe_experts_with_shared.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P,
                                          P, P, P, P, I, P, P, P, Z, P]
    L.moe_stage_inputs.argtypes = [P, P, Z, P]
    L.moe_workspace_init.argtypes = [P, Z, P]
    L.moe_workspace_status.argtypes = [P, I, P]
    L.moe_debug_decode_withhold.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, Z, I, P]
    L.moe_experts_rows.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P, P, Z, P, P]
    L.moe_combine_rows.argtypes = [P, P, I, I, I, I, P, P]
    for n in ("moe_experts_prefill", "moe_experts_decode", "moe_route_sigmoid_grouped",
              "quantize_fp8_block128", "moe_debug_permute", "moe_experts_decode_static",
              "moe_experts_with_shared", "moe_experts_decode_fused", "moe_stage_inputs",
              "moe_workspace_init", "moe_workspace_status", "moe_debug_decode_withhold",
              "moe_experts_rows", "moe_combine_rows"):
        getattr(L, n).restype = I
    return L


_LIB = None


def _lib():
    """The loaded library (loaded on the first call; raises ImportError when
    libmoe_b200.so is not built)."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "lib":
        return _lib()
    raise AttributeError("module %r has no attribute %r" % (__name__, name))


class MoEError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise MoEError("%s failed: %s" % (what, STATUS.get(rc, rc)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _wtype(gate_up_proj, weight_format=None):
    """bf16 -> MOE_W_BF16; float8_e4m3fn or uint8 -> MOE_W_FP8_E4M3, unless
    weight_format == "mxfp4" (uint8 bytes of packed E2M1 codes)."""
    if weight_format == "mxfp4":
        if gate_up_proj.dtype != torch.uint8:
            raise TypeError("MXFP4 weights are passed as uint8 bytes (two E2M1 codes each)")
        return MOE_W_MXFP4
    if gate_up_proj.dtype == torch.bfloat16:
        return MOE_W_BF16
    if gate_up_proj.dtype in (torch.uint8, torch.float8_e4m3fn):
        return MOE_W_FP8_E4M3
    raise TypeError("expert weights must be bf16, e4m3 (uint8 / float8_e4m3fn) or mxfp4 bytes")


def moe_experts_workspace_size(T, H, F, E, K, wtype=MOE_W_BF16, decode=False):
    return int(_lib().moe_experts_workspace_size(T, H, F, E, K, wtype, int(bool(decode))))


def _check_forward_args(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights,
                        top_k, gate_up_scale=None, down_scale=None, out=None, weight_format=None):
    """Shape, dtype and device checks of the forward entry points, made before
    any C call (the library sees only raw pointers and cannot detect a host
    tensor, a non-contiguous view or a wrong integer width).  Returns
    (T, H, F, E, weight type)."""
    T, H = hidden_states.shape
    E, F2, H2 = gate_up_proj.shape
    packed = weight_format == "mxfp4"          # two codes per byte along the reduction
    if packed:
        H2 *= 2
    if H2 != H or down_proj.shape != (E, H, F2 // 2 // (2 if packed else 1)):
        raise ValueError("shape mismatch: hidden %s gate_up %s down %s" % (
            tuple(hidden_states.shape), tuple(gate_up_proj.shape), tuple(down_proj.shape)))
    if tuple(top_k_index.shape) != (T, top_k) or tuple(top_k_weights.shape) != (T, top_k):
        raise ValueError("top_k_index / top_k_weights must be [T, top_k]")
    if top_k_index.dtype != torch.int32 or top_k_weights.dtype != torch.float32:
        raise TypeError("top_k_index must be int32 and top_k_weights float32")
    if hidden_states.dtype != torch.bfloat16:
        raise TypeError("hidden_states must be bf16")
    if out is not None and (tuple(out.shape) != (T, H) or out.dtype != torch.bfloat16):
        raise ValueError("out must be [T, H] bf16")
    for t in (hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, gate_up_scale,
              down_scale, out):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("all tensors must be contiguous CUDA tensors")
    return T, H, F2 // 2, E, _wtype(gate_up_proj, weight_format)


def _forward(name, hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, top_k,
             gate_up_scale=None, down_scale=None, out=None, workspace=None, stream=None,
             weight_format=None):
    T, H, F, E, wt = _check_forward_args(hidden_states, gate_up_proj, down_proj, top_k_index,
                                         top_k_weights, top_k, gate_up_scale, down_scale, out,
                                         weight_format)
    F2 = 2 * F
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=hidden_states.device)
    decode = name in ("moe_experts_decode", "moe_experts_decode_fused")
    need = moe_experts_workspace_size(T, H, F2 // 2, E, top_k, wt, decode)
    if workspace is None:   # zero-filled: the header must be zero before first use
        workspace = torch.zeros(max(need, WORKSPACE_HEADER_BYTES), dtype=torch.uint8, device=hidden_states.device)
    rc = getattr(_lib(), name)(_ptr(hidden_states), _ptr(gate_up_proj), _ptr(down_proj),
                            _ptr(top_k_index), _ptr(top_k_weights), top_k, T, H, F2 // 2, E, wt,
                            _ptr(gate_up_scale), _ptr(down_scale), _ptr(out), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, name)
    return out


def moe_experts_prefill(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, top_k,
                        gate_up_scale=None, down_scale=None, out=None, workspace=None, stream=None,
                        weight_format=None):
    """Routed-experts forward, grouped-GEMM form.  Returns out [T,H] bf16.
    weight_format="mxfp4": gate_up_proj [E,2F,H/2] / down_proj [E,H,F/2] uint8
    packed E2M1 with E8M0 scales (uint8) in the block layout."""
    return _forward("moe_experts_prefill", hidden_states, gate_up_proj, down_proj, top_k_index,
                    top_k_weights, top_k, gate_up_scale, down_scale, out, workspace, stream,
                    weight_format)


def moe_experts_decode(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, top_k,
                       gate_up_scale=None, down_scale=None, out=None, workspace=None, stream=None,
                       weight_format=None):
    """Routed-experts forward, decode form for a few tokens."""
    return _forward("moe_experts_decode", hidden_states, gate_up_proj, down_proj, top_k_index,
                    top_k_weights, top_k, gate_up_scale, down_scale, out, workspace, stream,
                    weight_format)


def moe_experts_shared_workspace_size(T, H, F, E, K, S, wtype=MOE_W_BF16):
    return int(_lib().moe_experts_shared_workspace_size(T, H, F, E, K, S, wtype))


def moe_experts_with_shared(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights,
                            top_k, shared_gate_up_proj, shared_down_proj, residual=None,
                            gate_up_scale=None, down_scale=None, shared_gate_up_scale=None,
                            shared_down_scale=None, out=None, workspace=None, stream=None):
    """Routed experts + S shared experts (weight 1) + optional residual, summed
    in that order and rounded once.  shared_* [S,2F,H] / [S,H,F] (S may be 0
    when both are None).  Returns out [T,H] bf16."""
    T, H = hidden_states.shape
    E, F2, _ = gate_up_proj.shape
    F = F2 // 2
    if shared_gate_up_proj is None:
        S = 0
    else:
        S = shared_gate_up_proj.shape[0]
        if tuple(shared_gate_up_proj.shape) != (S, F2, H) or \
                tuple(shared_down_proj.shape) != (S, H, F) or \
                shared_gate_up_proj.dtype != gate_up_proj.dtype:
            raise ValueError("shared experts must be [S,2F,H] / [S,H,F] of the routed dtype")
    if residual is not None and tuple(residual.shape) != (T, H):
        raise ValueError("residual must be [T,H]")
    for t in (hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, gate_up_scale,
              down_scale, shared_gate_up_proj, shared_down_proj, shared_gate_up_scale,
              shared_down_scale, residual):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("all tensors must be contiguous CUDA tensors")
    wt = _wtype(gate_up_proj)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=hidden_states.device)
    need = moe_experts_shared_workspace_size(T, H, F, E, top_k, S, wt)
    if workspace is None:   # zero-filled: the header must be zero before first use
        workspace = torch.zeros(max(need, WORKSPACE_HEADER_BYTES), dtype=torch.uint8, device=hidden_states.device)
    rc = _lib().moe_experts_with_shared(
        _ptr(hidden_states), _ptr(gate_up_proj), _ptr(down_proj), _ptr(top_k_index),
        _ptr(top_k_weights), top_k, T, H, F, E, wt, _ptr(gate_up_scale), _ptr(down_scale),
        _ptr(shared_gate_up_proj), _ptr(shared_down_proj), _ptr(shared_gate_up_scale),
        _ptr(shared_down_scale), S, _ptr(residual), _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "moe_experts_with_shared")
    return out


def moe_experts_decode_fused(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights,
                             top_k, gate_up_scale=None, down_scale=None, out=None, workspace=None,
                             stream=None, weight_format=None):
    """Decode form as one kernel launch: bf16 weights (T <= 16, T*K <= 64,
    H, F <= 2048) or MXFP4 weights (T <= 16, T*K <= 64, one persistent
    kernel after the permutation)."""
    return _forward("moe_experts_decode_fused", hidden_states, gate_up_proj, down_proj,
                    top_k_index, top_k_weights, top_k, gate_up_scale, down_scale, out, workspace,
                    stream, weight_format)


def moe_experts_decode_static(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights,
                              top_k, gate_up_scale=None, down_scale=None, out=None, stream=None):
    """Decode form without a workspace: scratch comes from a fixed 1 MiB array
    inside the library (for callers that cannot allocate device memory; calls
    that overlap on the GPU race on that array).  The same argument checks as
    moe_experts_decode run first."""
    T, H, F, E, wt = _check_forward_args(hidden_states, gate_up_proj, down_proj, top_k_index,
                                         top_k_weights, top_k, gate_up_scale, down_scale, out)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=hidden_states.device)
    rc = _lib().moe_experts_decode_static(_ptr(hidden_states), _ptr(gate_up_proj), _ptr(down_proj),
                                          _ptr(top_k_index), _ptr(top_k_weights), top_k, T, H, F,
                                          E, wt, _ptr(gate_up_scale), _ptr(down_scale), _ptr(out),
                                          _stream(stream))
    _check(rc, "moe_experts_decode_static")
    return out


def moe_experts_rows(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, top_k,
                     gate_up_scale=None, down_scale=None, workspace=None, stream=None,
                     weight_format=None):
    """Weighted expert rows y [T*K, H] fp32, y[t*K+k] = w[t,k] * expert_e(x_t)
    (the grouped path without its combine).  Returns a view into the
    workspace, valid until the workspace's next use."""
    T, H, F, E, wt = _check_forward_args(hidden_states, gate_up_proj, down_proj, top_k_index,
                                         top_k_weights, top_k, gate_up_scale, down_scale, None,
                                         weight_format)
    need = moe_experts_workspace_size(T, H, F, E, top_k, wt, False)
    if workspace is None:
        workspace = torch.zeros(max(need, WORKSPACE_HEADER_BYTES), dtype=torch.uint8,
                                device=hidden_states.device)
    off = ctypes.c_size_t(0)
    rc = _lib().moe_experts_rows(_ptr(hidden_states), _ptr(gate_up_proj), _ptr(down_proj),
                                 _ptr(top_k_index), _ptr(top_k_weights), top_k, T, H, F, E, wt,
                                 _ptr(gate_up_scale), _ptr(down_scale), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), ctypes.byref(off),
                                 _stream(stream))
    _check(rc, "moe_experts_rows")
    n = T * top_k * H * 4
    return workspace[off.value:off.value + n].view(torch.float32).view(T * top_k, H)


def moe_combine_rows(y, top_k_index, E, out=None, stream=None):
    """out [T, H] bf16 = bf16(sum over valid k, ascending, of y[t*K+k])."""
    T, K = top_k_index.shape
    H = y.shape[1]
    if tuple(y.shape) != (T * K, H) or y.dtype != torch.float32 or top_k_index.dtype != torch.int32:
        raise ValueError("y must be [T*K, H] float32 and top_k_index [T, K] int32")
    for t in (y, top_k_index):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("all tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=y.device)
    rc = _lib().moe_combine_rows(_ptr(y), _ptr(top_k_index), K, T, H, E, _ptr(out), _stream(stream))
    _check(rc, "moe_combine_rows")
    return out


def moe_workspace_init(workspace, stream=None):
    """Zero the workspace's 8 KiB header (needed once before first use unless
    the workspace was allocated zero-filled)."""
    rc = _lib().moe_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check(rc, "moe_workspace_init")
    return workspace


def moe_workspace_status(workspace, clear=False, stream=None):
    """Status code of the calls that used `workspace` (waits for the stream):
    MOE_OK (0) or MOE_ERR_TIMEOUT (5); clear=True also zeroes the header."""
    rc = _lib().moe_workspace_status(_ptr(workspace), int(bool(clear)), _stream(stream))
    if rc not in (0, 5):
        _check(rc, "moe_workspace_status")
    return rc


def moe_stage_inputs(src_ptr, dst, nbytes=None, stream=None):
    """Copy `nbytes` (default: all of dst) from the device-readable address
    `src_ptr` (an int, e.g. the device pointer of mapped pinned host memory)
    into the device tensor `dst` with one kernel on the stream."""
    nbytes = dst.numel() * dst.element_size() if nbytes is None else nbytes
    rc = _lib().moe_stage_inputs(ctypes.c_void_p(src_ptr), _ptr(dst), nbytes, _stream(stream))
    _check(rc, "moe_stage_inputs")
    return dst


def moe_route_sigmoid_grouped(logits, bias, num_groups, topk_group, top_k, routed_scaling_factor,
                              top_k_index=None, top_k_weights=None, expert_offsets=None,
                              want_offsets=False, stream=None):
    """Group-aware sigmoid top-k routing.  Returns (top_k_index, top_k_weights[, offsets])."""
    T, E = logits.shape
    dev = logits.device
    if top_k_index is None:
        top_k_index = torch.empty(T, top_k, dtype=torch.int32, device=dev)
    if top_k_weights is None:
        top_k_weights = torch.empty(T, top_k, dtype=torch.float32, device=dev)
    if want_offsets and expert_offsets is None:
        expert_offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    rc = _lib().moe_route_sigmoid_grouped(_ptr(logits), _ptr(bias), T, E, num_groups, topk_group,
                                       top_k, float(routed_scaling_factor), _ptr(top_k_index),
                                       _ptr(top_k_weights), _ptr(expert_offsets), _stream(stream))
    _check(rc, "moe_route_sigmoid_grouped")
    if expert_offsets is not None:
        return top_k_index, top_k_weights, expert_offsets
    return top_k_index, top_k_weights


def quantize_fp8_block128(x, xq=None, scale=None, stream=None):
    """x [rows, cols] bf16 -> (xq [rows, cols] uint8 E4M3 codes, scale [rows, cols/128] f32)."""
    rows, cols = x.shape
    if xq is None:
        xq = torch.empty(rows, cols, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(rows, cols // 128, dtype=torch.float32, device=x.device)
    rc = _lib().quantize_fp8_block128(_ptr(x), rows, cols, _ptr(xq), _ptr(scale), _stream(stream))
    _check(rc, "quantize_fp8_block128")
    return xq, scale


def moe_debug_permute(top_k_index, E, workspace=None, stream=None):
    """Expert counts, offsets, permutation and inverse of the routing slots."""
    T, K = top_k_index.shape
    dev = top_k_index.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(T * K, 1), dtype=torch.int32, device=dev)
    inv = torch.empty(max(T * K, 1), dtype=torch.int32, device=dev)
    need = moe_experts_workspace_size(T, 128, 128, E, K, MOE_W_BF16, False)
    if workspace is None:
        workspace = torch.zeros(max(need, WORKSPACE_HEADER_BYTES), dtype=torch.uint8, device=dev)
    rc = _lib().moe_debug_permute(_ptr(top_k_index), T, K, E, _ptr(counts), _ptr(offsets), _ptr(perm),
                               _ptr(inv), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "moe_debug_permute")
    return counts, offsets, perm[:T * K], inv[:T * K]
