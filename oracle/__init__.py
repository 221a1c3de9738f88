"""CPU oracle for the routed-experts MoE forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the cpu-baseline / reference
leg of ``bench.py`` may import this package.  The product library never calls
it, and it shares no code with the CUDA path.

All arrays are numpy arrays on the host:
  bf16 tensors as ``uint16`` bit patterns, E4M3 tensors as ``uint8`` codes,
  indices ``int32``, weights / scales / logits ``float32``.

Each wrapper calls one function of ``moe_oracle.c`` (plain C, fp64
accumulation, ascending-index summation order).  Definitions follow the
"deepseek-ocr2-moe-experts" model card (description and "Usage": the forward
formula, weight layouts, argument order) and the "Supporting MegaKernel for
DeepSeek Models" layer table (sigmoid group routing, block-128 E4M3
quantisation, FP8 expert layers with per-(row,128) weight scales).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
        L.oracle_bf16_from_f64.argtypes = [P, i64, P]
        L.oracle_e4m3_from_f64.argtypes = [P, i64, P]
        L.oracle_e4m3_to_f64.argtypes = [P, i64, P]
        L.oracle_quantize_fp8_block128.argtypes = [P, i64, i64, P, P]
        L.oracle_route_sigmoid_grouped.argtypes = [P, P, i64, i32, i32, i32, i32, f32, P, P]
        L.oracle_permute.argtypes = [P, i64, i32, P, P, P, P]
        L.oracle_moe_forward_bf16.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i32, P]
        L.oracle_moe_forward_fp8.argtypes = [P, P, P, P, P, P, P, i64, i32, i32, i32, i32, P]
        L.oracle_moe_forward_shared_bf16.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i32, P, P,
                                                     i32, P, P]
        L.oracle_moe_forward_shared_fp8.argtypes = [P, P, P, P, P, P, P, i64, i32, i32, i32, i32, P,
                                                    P, P, P, i32, P, P]
        L.oracle_mxf4_dequant.argtypes = [P, P, i64, i64, P]
        L.oracle_moe_forward_mxf4.argtypes = [P, P, P, P, P, P, P, i64, i32, i32, i32, i32, P]
        L.oracle_num_threads.restype = ctypes.c_int
        for fn in ("oracle_bf16_from_f64", "oracle_e4m3_from_f64", "oracle_e4m3_to_f64",
                   "oracle_quantize_fp8_block128", "oracle_route_sigmoid_grouped",
                   "oracle_permute", "oracle_moe_forward_bf16", "oracle_moe_forward_fp8",
                   "oracle_mxf4_dequant", "oracle_moe_forward_mxf4"):
            getattr(L, fn).restype = None
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# --- number formats -------------------------------------------------------

def bf16_bits(v) -> np.ndarray:
    """Round float64 values to bf16 (RNE, overflow -> inf); returns uint16 bits."""
    v, pv = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().oracle_bf16_from_f64(pv, v.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


def bf16_to_f64(bits) -> np.ndarray:
    bits = np.ascontiguousarray(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_bits(v) -> np.ndarray:
    """Round float64 values to OCP E4M3 (RNE, saturate to +-448); uint8 codes."""
    v, pv = _c(v, np.float64)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e4m3_from_f64(pv, v.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


def e4m3_to_f64(codes) -> np.ndarray:
    c, pc = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().oracle_e4m3_to_f64(pc, c.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


# --- S2 -------------------------------------------------------------------

def quantize_fp8_block128(x_bits):
    """x [rows, cols] bf16 bits -> (q [rows, cols] uint8, scale [rows, cols/128] f32)."""
    x, px = _c(x_bits, np.uint16)
    rows, cols = x.shape
    assert cols % 128 == 0
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, cols // 128), np.float32)
    lib().oracle_quantize_fp8_block128(px, rows, cols, q.ctypes.data_as(ctypes.c_void_p),
                                       s.ctypes.data_as(ctypes.c_void_p))
    return q, s


# --- S1 -------------------------------------------------------------------

def route_sigmoid_grouped(logits, bias, num_groups, topk_group, top_k, scale):
    lg, pl = _c(logits, np.float32)
    b, pb = _c(bias, np.float32)
    T, E = lg.shape
    assert E % num_groups == 0 and topk_group <= num_groups
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float32)
    lib().oracle_route_sigmoid_grouped(pl, pb, T, E, num_groups, topk_group, top_k,
                                       float(scale), idx.ctypes.data_as(ctypes.c_void_p),
                                       w.ctypes.data_as(ctypes.c_void_p))
    return idx, w


# --- S3 -------------------------------------------------------------------

def permute(idx, E):
    """idx [T,K] -> (counts [E], offsets [E+1], perm [T*K], inv [T*K]), int32."""
    i, pi = _c(idx, np.int32)
    n = i.size
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(n, np.int32)
    inv = np.empty(n, np.int32)
    V = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    lib().oracle_permute(pi, n, E, V(counts), V(offsets), V(perm), V(inv))
    return counts, offsets, perm, inv


# --- forward --------------------------------------------------------------

def moe_forward_bf16(x, gate_up, down, idx, w):
    """bf16 bits: x [T,H], gate_up [E,2F,H], down [E,H,F]; idx/w [T,K] -> out [T,H] bf16 bits."""
    x, px = _c(x, np.uint16)
    gu, pg = _c(gate_up, np.uint16)
    dn, pd = _c(down, np.uint16)
    ix, pi = _c(idx, np.int32)
    ww, pw = _c(w, np.float32)
    T, H = x.shape
    E, F2, H2 = gu.shape
    assert H2 == H and dn.shape == (E, H, F2 // 2) and ix.shape == ww.shape and ix.shape[0] == T
    out = np.empty((T, H), np.uint16)
    lib().oracle_moe_forward_bf16(px, pg, pd, pi, pw, T, H, F2 // 2, E, ix.shape[1],
                                  out.ctypes.data_as(ctypes.c_void_p))
    return out


def moe_forward_fp8(x, w13, w13_scale, w2, w2_scale, idx, w):
    """x [T,H] bf16 bits; w13 [E,2F,H] E4M3 + [E,2F,H/128] f32; w2 [E,H,F] + [E,H,F/128]."""
    x, px = _c(x, np.uint16)
    a, pa = _c(w13, np.uint8)
    sa, psa = _c(w13_scale, np.float32)
    b, pb = _c(w2, np.uint8)
    sb, psb = _c(w2_scale, np.float32)
    ix, pi = _c(idx, np.int32)
    ww, pw = _c(w, np.float32)
    T, H = x.shape
    E, F2, H2 = a.shape
    F = F2 // 2
    assert H2 == H and b.shape == (E, H, F) and H % 128 == 0 and F % 128 == 0
    assert sa.shape == (E, F2, H // 128) and sb.shape == (E, H, F // 128)
    out = np.empty((T, H), np.uint16)
    lib().oracle_moe_forward_fp8(px, pa, psa, pb, psb, pi, pw, T, H, F, E, ix.shape[1],
                                 out.ctypes.data_as(ctypes.c_void_p))
    return out


def moe_forward_shared_bf16(x, gate_up, down, idx, w, shared_gate_up, shared_down, residual=None):
    """Routed + shared experts + residual, bf16 weights: shared_gate_up
    [S,2F,H], shared_down [S,H,F], residual [T,H] (bf16 bits) or None."""
    x, px = _c(x, np.uint16)
    gu, pg = _c(gate_up, np.uint16)
    dn, pd = _c(down, np.uint16)
    ix, pi = _c(idx, np.int32)
    ww, pw = _c(w, np.float32)
    sg, psg = _c(shared_gate_up, np.uint16)
    sd, psd = _c(shared_down, np.uint16)
    T, H = x.shape
    E, F2, _ = gu.shape
    S = sg.shape[0]
    assert sg.shape[1:] == (F2, H) and sd.shape == (S, H, F2 // 2)
    pr = None
    if residual is not None:
        r, pr = _c(residual, np.uint16)
        assert r.shape == (T, H)
    out = np.empty((T, H), np.uint16)
    lib().oracle_moe_forward_shared_bf16(px, pg, pd, pi, pw, T, H, F2 // 2, E, ix.shape[1], psg, psd,
                                         S, pr, out.ctypes.data_as(ctypes.c_void_p))
    return out


def moe_forward_shared_fp8(x, w13, w13_scale, w2, w2_scale, idx, w, sw13, sw13_scale, sw2,
                           sw2_scale, residual=None):
    """Routed + shared experts + residual, E4M3 weights with per-(row,128) scales."""
    x, px = _c(x, np.uint16)
    a, pa = _c(w13, np.uint8)
    sa, psa = _c(w13_scale, np.float32)
    b, pb = _c(w2, np.uint8)
    sb, psb = _c(w2_scale, np.float32)
    ix, pi = _c(idx, np.int32)
    ww, pw = _c(w, np.float32)
    c, pc = _c(sw13, np.uint8)
    sc, psc = _c(sw13_scale, np.float32)
    d, pdd = _c(sw2, np.uint8)
    sd, psd = _c(sw2_scale, np.float32)
    T, H = x.shape
    E, F2, _ = a.shape
    S = c.shape[0]
    assert c.shape[1:] == (F2, H) and d.shape == (S, H, F2 // 2)
    pr = None
    if residual is not None:
        r, pr = _c(residual, np.uint16)
        assert r.shape == (T, H)
    out = np.empty((T, H), np.uint16)
    lib().oracle_moe_forward_shared_fp8(px, pa, psa, pb, psb, pi, pw, T, H, F2 // 2, E, ix.shape[1],
                                        pc, psc, pdd, psd, S, pr, out.ctypes.data_as(ctypes.c_void_p))
    return out


def mxf4_dequant(q, sc, R, C):
    """Packed MXFP4 matrix -> fp64 [R, C]: q [R, C/2] bytes (even column in the
    low nibble), sc the E8M0 scales in the tensor-core block layout (one
    512-byte block per 128 x 128, byte (r%32)*16 + ((r%128)//32)*4 + (c%128)//32)."""
    q, pq = _c(q, np.uint8)
    sc, ps = _c(sc, np.uint8)
    assert q.size == R * C // 2 and sc.size == R * C // 32
    out = np.empty((R, C), np.float64)
    lib().oracle_mxf4_dequant(pq, ps, R, C, out.ctypes.data_as(ctypes.c_void_p))
    return out


def moe_forward_mxf4(x, w13, w13_sc, w2, w2_sc, idx, w):
    """MXFP4 routed weights (w13 [E,2F,H/2], w2 [E,H,F/2] packed E2M1; scales
    E8M0 in the block layout, 2F*H/32 and H*F/32 bytes per expert), FP8
    activations (block-128 E4M3 rule).  Returns out [T,H] bf16 bits."""
    x, px = _c(x, np.uint16)
    a, pa = _c(w13, np.uint8)
    sa, psa = _c(w13_sc, np.uint8)
    b, pb = _c(w2, np.uint8)
    sb, psb = _c(w2_sc, np.uint8)
    ix, pi = _c(idx, np.int32)
    ww, pw = _c(w, np.float32)
    T, H = x.shape
    E, F2 = a.shape[0], a.shape[1]
    F = F2 // 2
    assert a.shape == (E, F2, H // 2) and b.shape == (E, H, F // 2)
    assert sa.size == E * F2 * H // 32 and sb.size == E * H * F // 32
    out = np.empty((T, H), np.uint16)
    lib().oracle_moe_forward_mxf4(px, pa, psa, pb, psb, pi, pw, T, H, F, E, ix.shape[1],
                                  out.ctypes.data_as(ctypes.c_void_p))
    return out
