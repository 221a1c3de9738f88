"""Seeded synthetic inputs for the routed-experts MoE layer.

This module holds only the input recipe (random draws, their distributions
and the routing that the model runs *outside* the op); none of the op's own
arithmetic lives here.  It is the one module that both the CUDA path (tests,
bench) and the CPU oracle (tests) take their inputs from.

Recipes
-------
OCR-2 shape ("deepseek-ocr2-moe-experts" model card: hidden 1280, per-expert
intermediate 896, 64 experts, top-6):
  hidden ~ N(0,1); gate_up [E,2F,H] and down [E,H,F] ~ N(0, 0.02^2); all
  drawn in fp32 in that order and rounded to bf16 (RNE).  Router logits
  [T,E] ~ N(0,1) fp32 drawn after the weights; routing = fp32 softmax, greedy
  top-K (stable: equal probabilities keep the lower expert first), weights =
  probability * routed_scaling_factor (1.0).  The model card places this
  router outside the op, so here it is part of the input recipe.

DeepSeek-V3-like FP8 layer ("Supporting MegaKernel for DeepSeek Models",
layer table: hidden 7168, moe_inter 2048, 256 experts, top-8):
  weights drawn fp32 ~ N(0, 0.02^2) expert by expert, then quantised offline
  per (row, 128-column block): scale = amax / 448, code = E4M3(w / scale)
  (torch's float8_e4m3fn conversion, inputs clamped to +-448);
  hidden bf16 ~ N(0,1); logits fp32 ~ N(0,1) rounded through bf16 (the table
  gives bf16 router logits); bias fp32 ~ N(0, 0.1^2) rounded through bf16.

Skew: expert popularity Zipf(s): a seeded permutation gives each expert a
rank r (1-based); logit_e += ln(r_e^-s) - mean_e ln(r_e^-s).
"""
from dataclasses import dataclass, field
from typing import Optional

import torch

OCR2 = dict(H=1280, F=896, E=64, K=6)
DSV3_FP8 = dict(H=7168, F=2048, E=256, K=8, num_groups=8, topk_group=4, scale=2.5)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zipf_logit_shift(E: int, s: float, gen: torch.Generator, device) -> torch.Tensor:
    rank = torch.randperm(E, generator=gen, device=device).to(torch.float64) + 1.0
    lp = -s * torch.log(rank)
    return (lp - lp.mean()).to(torch.float32)


def softmax_topk_route(logits: torch.Tensor, K: int, routed_scaling_factor: float = 1.0):
    """The model-side router of the OCR-2 model (outside the op): fp32 softmax,
    greedy top-K with a stable order, weights = p * routed_scaling_factor."""
    p = torch.softmax(logits.float(), dim=-1)
    order = torch.sort(p, dim=-1, descending=True, stable=True).indices[:, :K]
    w = torch.gather(p, 1, order) * routed_scaling_factor
    return order.to(torch.int32).contiguous(), w.to(torch.float32).contiguous()


@dataclass
class Bf16Layer:
    x: torch.Tensor            # [T,H] bf16
    gate_up: torch.Tensor      # [E,2F,H] bf16
    down: torch.Tensor         # [E,H,F] bf16
    idx: torch.Tensor          # [T,K] int32
    w: torch.Tensor            # [T,K] fp32
    logits: torch.Tensor       # [T,E] fp32
    dims: dict = field(default_factory=dict)


def ocr2_layer(T: int, seed: int = 0, device="cpu", zipf: Optional[float] = None,
               H=None, F=None, E=None, K=None, weights_from: Optional[Bf16Layer] = None) -> Bf16Layer:
    """OCR-2-shaped bf16 layer.  Smaller H/F/E/K may be given for tests.
    `weights_from` reuses another layer's weights (only x / routing redrawn)."""
    H = H or OCR2["H"]; F = F or OCR2["F"]; E = E or OCR2["E"]; K = K or OCR2["K"]
    g = _gen(seed, device)
    x = torch.randn(T, H, generator=g, device=device).to(torch.bfloat16)
    if weights_from is None:
        gate_up = (torch.randn(E, 2 * F, H, generator=g, device=device) * 0.02).to(torch.bfloat16)
        down = (torch.randn(E, H, F, generator=g, device=device) * 0.02).to(torch.bfloat16)
    else:
        gate_up, down = weights_from.gate_up, weights_from.down
    logits = torch.randn(T, E, generator=g, device=device)
    if zipf is not None:
        logits = logits + zipf_logit_shift(E, zipf, g, device)
    idx, w = softmax_topk_route(logits, K, 1.0)
    return Bf16Layer(x, gate_up, down, idx, w, logits, dict(T=T, H=H, F=F, E=E, K=K))


def quantize_weight_rows_fp8(wf: torch.Tensor):
    """Offline weight quantisation: per (row, 128-column block) scale = amax/448
    (1 for an all-zero block), codes = E4M3(w/scale).  Returns (uint8 codes, f32 scales)."""
    R, C = wf.shape[-2], wf.shape[-1]
    blk = wf.reshape(*wf.shape[:-1], C // 128, 128)
    amax = blk.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (blk / scale.unsqueeze(-1)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.reshape(wf.shape).view(torch.uint8), scale.to(torch.float32)


@dataclass
class Fp8Layer:
    x: torch.Tensor            # [T,H] bf16
    w13: torch.Tensor          # [E,2F,H] uint8 (E4M3 codes)
    w13_scale: torch.Tensor    # [E,2F,H/128] f32
    w2: torch.Tensor           # [E,H,F] uint8
    w2_scale: torch.Tensor     # [E,H,F/128] f32
    logits: torch.Tensor       # [T,E] f32
    bias: torch.Tensor         # [E] f32
    dims: dict = field(default_factory=dict)


def fp8_weights(seed: int = 0, device="cpu", H=None, F=None, E=None):
    H = H or DSV3_FP8["H"]; F = F or DSV3_FP8["F"]; E = E or DSV3_FP8["E"]
    g = _gen(seed + 1000003, device)
    w13 = torch.empty(E, 2 * F, H, dtype=torch.uint8, device=device)
    w13s = torch.empty(E, 2 * F, H // 128, dtype=torch.float32, device=device)
    w2 = torch.empty(E, H, F, dtype=torch.uint8, device=device)
    w2s = torch.empty(E, H, F // 128, dtype=torch.float32, device=device)
    for e in range(E):
        q, s = quantize_weight_rows_fp8(torch.randn(2 * F, H, generator=g, device=device) * 0.02)
        w13[e].copy_(q); w13s[e].copy_(s)
        q, s = quantize_weight_rows_fp8(torch.randn(H, F, generator=g, device=device) * 0.02)
        w2[e].copy_(q); w2s[e].copy_(s)
    return w13, w13s, w2, w2s


def fp8_layer(T: int, seed: int = 0, device="cpu", zipf: Optional[float] = None,
              H=None, F=None, E=None, weights=None) -> Fp8Layer:
    """DeepSeek-V3-like FP8 layer; `weights` = a previous fp8_weights() tuple to reuse."""
    H = H or DSV3_FP8["H"]; F = F or DSV3_FP8["F"]; E = E or DSV3_FP8["E"]
    if weights is None:
        weights = fp8_weights(seed, device, H, F, E)
    g = _gen(seed, device)
    x = torch.randn(T, H, generator=g, device=device).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=g, device=device)
    bias = (torch.randn(E, generator=g, device=device) * 0.1)
    if zipf is not None:
        logits = logits + zipf_logit_shift(E, zipf, g, device)
    logits = logits.to(torch.bfloat16).float().contiguous()
    bias = bias.to(torch.bfloat16).float().contiguous()
    w13, w13s, w2, w2s = weights
    return Fp8Layer(x, w13, w13s, w2, w2s, logits, bias, dict(T=T, H=H, F=F, E=E))


# --- MXFP4 routed weights (offline weight preparation) ----------------------

E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)   # codes 0..7; bit 3 = sign


def e2m1_codes(v: torch.Tensor) -> torch.Tensor:
    """Nearest E2M1 code of each value (ties to the even code, i.e. the even
    mantissa), magnitudes above 6 saturate to 6.  Returns uint8 codes 0..15."""
    a = v.abs()
    # midpoints between neighbouring magnitudes; a tie goes to the even code
    mids = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)
    code = torch.zeros_like(a, dtype=torch.uint8)
    for i, m in enumerate(mids):
        upper_even = (i + 1) % 2 == 0          # code i+1 has an even mantissa
        code = code + ((a > m) | ((a == m) & upper_even)).to(torch.uint8)
    return code | ((v < 0).to(torch.uint8) << 3)


def pack_e2m1(codes: torch.Tensor) -> torch.Tensor:
    """[..., C] codes -> [..., C/2] bytes, even column in the low nibble."""
    return codes[..., 0::2] | (codes[..., 1::2] << 4)


def block_scale_layout(sc: torch.Tensor) -> torch.Tensor:
    """E8M0 scales [..., R, C/32] -> the tensor-core block layout, flattened
    over (R, C/32): one 512-byte block per 128 rows x 128 columns, blocks in
    [R/128][C/128] order, scale (r, c) at byte (r%32)*16 + ((r%128)//32)*4 +
    (c%128)//32 of its block."""
    *lead, R, C32 = sc.shape
    t = sc.reshape(*lead, R // 128, 4, 32, C32 // 4, 4)       # (rb, m1, m0, cb, j)
    n = len(lead)
    perm = list(range(n)) + [n, n + 3, n + 2, n + 1, n + 4]    # (rb, cb, m0, m1, j)
    return t.permute(*perm).contiguous().reshape(*lead, R * C32)


def quantize_weight_mxf4(wf: torch.Tensor):
    """Offline MXFP4 quantisation of [..., R, C] fp32 weights (OCP
    Microscaling): per (row, 32 columns) the shared exponent
    X = floor(log2(amax)) - 2 (E2M1's largest exponent), clamped to
    [-127, 127] (-127 for an all-zero block), elements E2M1(w / 2^X).
    Returns (packed codes [..., R, C/2] uint8, E8M0 scales in the block
    layout [..., R*C/32] uint8)."""
    *lead, R, C = wf.shape
    blk = wf.reshape(*lead, R, C // 32, 32)
    amax = blk.abs().amax(dim=-1)
    X = torch.where(amax > 0, torch.floor(torch.log2(torch.where(amax > 0, amax, torch.ones_like(amax)))) - 2,
                    torch.full_like(amax, -127.0)).clamp(-127, 127)
    codes = e2m1_codes(blk / torch.exp2(X).unsqueeze(-1)).reshape(*lead, R, C)
    return pack_e2m1(codes), block_scale_layout((X + 127).to(torch.uint8))


def mxf4_weights(seed: int = 0, device="cpu", H=None, F=None, E=None):
    """DeepSeek-V3-like experts with MXFP4 weights: (w13 [E,2F,H/2],
    w13_sc [E,2F*H/32], w2 [E,H,F/2], w2_sc [E,H*F/32]), weights drawn fp32
    ~ N(0, 0.02^2) expert by expert, as for the E4M3 layer."""
    H = H or DSV3_FP8["H"]; F = F or DSV3_FP8["F"]; E = E or DSV3_FP8["E"]
    g = _gen(seed + 5000011, device)
    w13 = torch.empty(E, 2 * F, H // 2, dtype=torch.uint8, device=device)
    w13s = torch.empty(E, 2 * F * H // 32, dtype=torch.uint8, device=device)
    w2 = torch.empty(E, H, F // 2, dtype=torch.uint8, device=device)
    w2s = torch.empty(E, H * F // 32, dtype=torch.uint8, device=device)
    for e in range(E):
        q, sc = quantize_weight_mxf4(torch.randn(2 * F, H, generator=g, device=device) * 0.02)
        w13[e].copy_(q); w13s[e].copy_(sc)
        q, sc = quantize_weight_mxf4(torch.randn(H, F, generator=g, device=device) * 0.02)
        w2[e].copy_(q); w2s[e].copy_(sc)
    return w13, w13s, w2, w2s


def shared_experts_bf16(S: int, H: int, F: int, seed: int = 0, device="cpu"):
    """S always-active experts: (gate_up [S,2F,H], down [S,H,F]) bf16, same
    init scale as the routed experts."""
    g = _gen(seed + 2000003, device)
    gu = (torch.randn(S, 2 * F, H, generator=g, device=device) * 0.02).to(torch.bfloat16)
    dn = (torch.randn(S, H, F, generator=g, device=device) * 0.02).to(torch.bfloat16)
    return gu, dn


def shared_experts_fp8(S: int, H: int, F: int, seed: int = 0, device="cpu"):
    """S always-active E4M3 experts: (w13, w13_scale, w2, w2_scale)."""
    return fp8_weights(seed + 3000017, device, H, F, S)


def residual_bf16(T: int, H: int, seed: int = 0, device="cpu"):
    g = _gen(seed + 4000037, device)
    return torch.randn(T, H, generator=g, device=device).to(torch.bfloat16)


# --- host views for the oracle (numpy bit patterns) -------------------------

def bf16_bits(t: torch.Tensor):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def u8(t: torch.Tensor):
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def np32(t: torch.Tensor):
    return t.detach().cpu().contiguous().numpy()
