"""Pure-Python brute force of the routed-experts forward -- TEST INFRASTRUCTURE.

A second, independent statement of the definition in ``moe_oracle.c``, for
tiny shapes only (T <= 4, H, F <= 256, E <= 8).  It shares no code with the C
oracle: rounding is done with exact rationals (``fractions.Fraction`` and
Python's round-half-even ``round``), dot products with ``math.fsum`` (exactly
rounded sums), and the E4M3 grid is enumerated from the format definition.

Definition ("deepseek-ocr2-moe-experts" model card, description + "Usage"):
  out[t] = sum_k w[t,k] * down_e( SiLU(gate_e x_t) * (up_e x_t) ),
  e = top_k_index[t,k]; gate rows [0,F) and up rows [F,2F) of gate_up_proj.
FP8 variant ("Supporting MegaKernel for DeepSeek Models", layer table:
bf16_to_fp8_quantize, moe_w13_fp8_layer, moe_silu_mul_layer,
moe_w2_fp8_layer): activations quantised per 128 with a power-of-two scale,
weights dequantised with their per-(row, 128-col) scales.
"""
import math
from fractions import Fraction


def _round_fraction(x: Fraction, sig_bits: int, emin: int) -> Fraction:
    if x == 0:
        return Fraction(0)
    ax = abs(x)
    # exponent of the leading bit: largest L with 2^L <= ax
    L = ax.numerator.bit_length() - ax.denominator.bit_length()
    if Fraction(2) ** L > ax:
        L -= 1
    elif Fraction(2) ** (L + 1) <= ax:
        L += 1
    L = max(L, emin)
    q = Fraction(2) ** (L - sig_bits + 1)
    return round(x / q) * q            # Fraction.__round__: ties to even


def bf16_round(v: float) -> float:
    r = _round_fraction(Fraction(v), 8, -126)
    if abs(r) > Fraction(255) * Fraction(2) ** 120:
        return math.copysign(math.inf, v)
    return float(r)


def _e4m3_grid():
    vals = []
    for ex in range(16):
        for m in range(8):
            if ex == 15 and m == 7:
                continue                    # NaN
            vals.append(Fraction(m, 8) * Fraction(2) ** -6 if ex == 0
                        else (1 + Fraction(m, 8)) * Fraction(2) ** (ex - 7))
    return vals


E4M3_POS = _e4m3_grid()                     # 0 .. 448, ascending


def e4m3_round(v: Fraction) -> Fraction:
    """Nearest E4M3 value, ties to the code with even mantissa, saturating."""
    a = abs(Fraction(v))
    if a >= 448:
        r = Fraction(448)
    else:
        best = None
        for i, g in enumerate(E4M3_POS):
            d = abs(g - a)
            if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
                best = (d, i, g)
        r = best[2]
    return -r if v < 0 else r


def block_quantize(vals):
    """One block of 128 exact values -> (dequantised values, scale).
    scale = smallest power of two with max|v| / scale <= 448 (1 when all zero)."""
    amax = max(abs(Fraction(v)) for v in vals)
    if amax == 0:
        return [Fraction(0)] * len(vals), Fraction(1)
    k = -200
    while amax / Fraction(2) ** k > 448:
        k += 1
    while k > -127 and amax / Fraction(2) ** (k - 1) <= 448:
        k -= 1
    k = max(k, -127)
    s = Fraction(2) ** k
    return [e4m3_round(Fraction(v) / s) * s for v in vals], s


def silu(g: float) -> float:
    return g / (1.0 + math.exp(-g))


def forward_bf16(x, gate_up, down, idx, w):
    """Nested lists of Python floats (exact bf16 values). Returns out [T][H] floats."""
    T, H = len(x), len(x[0])
    E = len(gate_up)
    F = len(gate_up[0]) // 2
    out = []
    for t in range(T):
        acc = [0.0] * H
        terms = [[] for _ in range(H)]
        for k in range(len(idx[t])):
            e = idx[t][k]
            if not (0 <= e < E):
                continue
            hvec = []
            for f in range(F):
                g = math.fsum(gate_up[e][f][i] * x[t][i] for i in range(H))
                u = math.fsum(gate_up[e][F + f][i] * x[t][i] for i in range(H))
                hvec.append(bf16_round(silu(g) * u))
            for j in range(H):
                y = math.fsum(down[e][j][f] * hvec[f] for f in range(F))
                terms[j].append(w[t][k] * y)
        out.append([bf16_round(math.fsum(terms[j])) for j in range(H)])
    return out


def forward_fp8(x, w13, w13_scale, w2, w2_scale, idx, w):
    """x: bf16 values; w13/w2: E4M3 values (floats); scales per (row, 128 block)."""
    T, H = len(x), len(x[0])
    E = len(w13)
    F = len(w13[0]) // 2
    out = []
    for t in range(T):
        xd = []
        for b in range(H // 128):
            d, _ = block_quantize(x[t][b * 128:(b + 1) * 128])
            xd += [float(v) for v in d]
        terms = [[] for _ in range(H)]
        for k in range(len(idx[t])):
            e = idx[t][k]
            if not (0 <= e < E):
                continue
            hv = []
            for f in range(F):
                g = math.fsum(w13[e][f][i] * w13_scale[e][f][i // 128] * xd[i] for i in range(H))
                u = math.fsum(w13[e][F + f][i] * w13_scale[e][F + f][i // 128] * xd[i]
                              for i in range(H))
                hv.append(bf16_round(silu(g) * u))
            hd = []
            for b in range(F // 128):
                d, _ = block_quantize(hv[b * 128:(b + 1) * 128])
                hd += [float(v) for v in d]
            for j in range(H):
                y = math.fsum(w2[e][j][f] * w2_scale[e][j][f // 128] * hd[f] for f in range(F))
                terms[j].append(w[t][k] * y)
        out.append([bf16_round(math.fsum(terms[j])) for j in range(H)])
    return out


def forward_shared_bf16(x, gate_up, down, idx, w, shared_gate_up, shared_down, residual):
    """Routed + shared experts (weight 1, every token) + residual, bf16
    weights; one exact sum per output (math.fsum), rounded to bf16 once."""
    T, H = len(x), len(x[0])
    E = len(gate_up)
    F = len(gate_up[0]) // 2

    def expert_terms(G, D, t, wk):
        hvec = []
        for f in range(F):
            g = math.fsum(G[f][i] * x[t][i] for i in range(H))
            u = math.fsum(G[F + f][i] * x[t][i] for i in range(H))
            hvec.append(bf16_round(silu(g) * u))
        return [wk * math.fsum(D[j][f] * hvec[f] for f in range(F)) for j in range(H)]

    out = []
    for t in range(T):
        terms = [[] for _ in range(H)]
        for k in range(len(idx[t])):
            e = idx[t][k]
            if 0 <= e < E:
                for j, v in enumerate(expert_terms(gate_up[e], down[e], t, w[t][k])):
                    terms[j].append(v)
        for s in range(len(shared_gate_up)):
            for j, v in enumerate(expert_terms(shared_gate_up[s], shared_down[s], t, 1.0)):
                terms[j].append(v)
        if residual is not None:
            for j in range(H):
                terms[j].append(residual[t][j])
        out.append([bf16_round(math.fsum(terms[j])) for j in range(H)])
    return out
