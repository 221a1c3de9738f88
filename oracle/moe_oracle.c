/*
 * moe_oracle.c -- plain, slow CPU oracle for the routed-experts MoE forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library under
 * mixture_experts_routed_expert_b200/, and the CUDA library never calls it.
 *
 * Arithmetic: every dot product and every sum is accumulated in fp64 in
 * ascending index order, on the exact values of the bf16 / E4M3 operands
 * (E4M3 operands dequantised with their fp32 scales first).  Rounding to
 * bf16 / E4M3 happens only where the method stores a value in that format.
 *
 * Sources (web pages, cited by title and section):
 *  - "deepseek-ocr2-moe-experts" model card, description + "Usage":
 *    out[t] = sum_k w[t,k] * down_e(SiLU(gate_e x_t) * up_e x_t), weight
 *    layout gate_up_proj [E,2F,H], down_proj [E,H,F], top_k_index [T,K] int32,
 *    top_k_weights [T,K] fp32; routing happens outside the op.
 *  - "[Feature Request] - Supporting MegaKernel for DeepSeek Models",
 *    "Layer Tensor Details": moe_topk_sigmoid_routing_layer (group-aware
 *    sigmoid routing, num_groups=8, topk_group=4, routed_scaling_factor=2.5),
 *    bf16_to_fp8_quantize (block 128, E4M3 + power-of-two scale),
 *    moe_w13_fp8_layer / moe_w2_fp8_layer (per (row,128-col) fp32 weight
 *    scales), moe_silu_mul_layer, moe_local_reduction (weighted sum over k).
 *  - GC MoE issue on the DeepGEMM tracker (FP8 activations with packed FP4
 *    routed weights), the DeepGEMM Mega MoE news page (FP8 x FP4) and the
 *    sgl-deep-gemm commit list ("MXF4 kind"): the MXFP4 weight format of
 *    the OCP Microscaling spec (E2M1 elements, one E8M0 scale per 32).
 *
 * Parity pins: every exported function is pinned by tests under tests/
 * (test_oracle_*.py) against library routines, closed forms, invariants and
 * brute force; none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* Round v to the nearest number that has `p` significant bits and whose
 * exponent is at least emin (below 2^emin the spacing stays 2^(emin-p+1),
 * i.e. gradual underflow).  Ties go to the even neighbour: nearbyint() in the
 * default rounding mode.  v/quantum is exact (power-of-two scaling). */
static double round_sig(double v, int p, int emin) {
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    (void)frexp(fabs(v), &e);          /* |v| = m 2^e, m in [0.5,1) */
    int lead = e - 1;                  /* exponent of the leading bit */
    if (lead < emin) lead = emin;
    double quantum = ldexp(1.0, lead - (p - 1));
    return nearbyint(v / quantum) * quantum;
}

/* bf16: 8 significant bits, normal exponents from -126, largest finite
 * (2 - 2^-7) 2^127.  Overflow after rounding gives infinity (IEEE RNE). */
static double bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static uint16_t bf16_from_double(double v) {
    if (isnan(v)) return 0x7FC0;
    double r = round_sig(v, 8, -126);
    const double maxf = ldexp(255.0, 120);         /* (2-2^-7) 2^127 */
    if (fabs(r) > maxf) r = copysign(INFINITY, r);
    float f = (float)r;                            /* exact */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* OCP 8-bit floating point, E4M3 ("fn" variant): 1 sign, 4 exponent bits
 * (bias 7), 3 mantissa bits, no infinities, S.1111.111 = NaN, largest finite
 * S.1111.110 = 448, smallest normal 2^-6, subnormal spacing 2^-9.
 * The conversion is round-to-nearest-even with saturation of finite values
 * to +-448. */
static double e4m3_value(uint8_t c) {
    int s = c >> 7, ex = (c >> 3) & 15, m = c & 7;
    double mag;
    if (ex == 15 && m == 7) return NAN;
    if (ex == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, ex - 7);
    return s ? -mag : mag;
}

static uint8_t e4m3_from_double(double v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double r = fabs(round_sig(v, 4, -6));
    if (r > 448.0) r = 448.0;                      /* satfinite */
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -6)) {                      /* subnormal: m * 2^-9 */
        int m = (int)ldexp(r, 9);
        return (uint8_t)(sign | m);
    }
    int e;
    double fr = frexp(r, &e);                      /* r = fr 2^e */
    int lead = e - 1;
    int m = (int)((ldexp(fr, 1) - 1.0) * 8.0);     /* r/2^lead = 1 + m/8 */
    return (uint8_t)(sign | ((lead + 7) << 3) | m);
}

/* Exported format helpers (pinned against torch's own conversions). */
void oracle_bf16_from_f64(const double *v, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_from_double(v[i]);
}
void oracle_e4m3_from_f64(const double *v, int64_t n, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_from_double(v[i]);
}
void oracle_e4m3_to_f64(const uint8_t *c, int64_t n, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(c[i]);
}

/* ------------------------------------------------------------------------ */
/* S2: block-128 activation quantisation                                     */
/* (MegaKernel DeepSeek layer table, bf16_to_fp8_quantize)                   */
/* ------------------------------------------------------------------------ */

/* Scale of one block: the smallest power of two s = 2^k with amax/s <= 448,
 * with k clamped to [-127, 127] so that s is an unsigned-exponent (ue8m0)
 * value; amax == 0 gives s = 1.  With amax = m 2^e, m in [0.5,1) and
 * 448 = 0.875 2^9:  k = e - 9 when m <= 0.875, else e - 8. */
static int block_scale_exp(double amax) {
    if (amax == 0.0) return 0;
    int e;
    double m = frexp(amax, &e);
    int k = (m <= 0.875) ? e - 9 : e - 8;
    if (k < -127) k = -127;
    if (k > 127) k = 127;
    return k;
}

/* Quantise n_blocks consecutive blocks of 128 values (given as doubles that
 * are exact bf16 values).  q = E4M3(v / s) elementwise, scale = s (fp32). */
static void quantize_blocks(const double *v, int n_blocks, uint8_t *q, float *scale) {
    for (int b = 0; b < n_blocks; ++b) {
        const double *vb = v + (int64_t)b * 128;
        double amax = 0.0;
        for (int i = 0; i < 128; ++i) amax = fmax(amax, fabs(vb[i]));
        int k = block_scale_exp(amax);
        for (int i = 0; i < 128; ++i) q[(int64_t)b * 128 + i] = e4m3_from_double(ldexp(vb[i], -k));
        scale[b] = (float)ldexp(1.0, k);
    }
}

/* x: [rows, cols] bf16 bits, cols % 128 == 0 -> xq [rows, cols] E4M3 bits,
 * scale [rows, cols/128] fp32. */
void oracle_quantize_fp8_block128(const uint16_t *x, int64_t rows, int64_t cols,
                                  uint8_t *xq, float *scale) {
    int nb = (int)(cols / 128);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double *tmp = (double *)malloc(sizeof(double) * cols);
        for (int64_t c = 0; c < cols; ++c) tmp[c] = bf16_value(x[r * cols + c]);
        quantize_blocks(tmp, nb, xq + r * cols, scale + r * nb);
        free(tmp);
    }
}

/* ------------------------------------------------------------------------ */
/* S1: group-aware sigmoid top-k routing                                     */
/* (MegaKernel DeepSeek layer table, moe_topk_sigmoid_routing_layer)         */
/* ------------------------------------------------------------------------ */

/* "a ranks before b": larger score first, lower index on equal scores. */
static int ranks_before(float sa, int ia, float sb, int ib) {
    return sa > sb || (sa == sb && ia < ib);
}

/* logits [T,E] fp32, bias [E] fp32.  Per token:
 *   s_e = sigmoid(logit_e), computed in double and rounded to fp32;
 *   c_e = s_e + bias_e (fp32 add);
 *   group score = top1 + top2 of c inside each of num_groups equal groups
 *                 (just top1 when a group holds one expert);
 *   keep the topk_group best groups; choose the top_k best c among experts
 *   of kept groups (ties: lower index);  w_k = (s_k / sum_j s_j) * scale,
 *   sum_j in selection order, all fp32.
 * Outputs top_k_index [T,K] int32 (selection order), top_k_weights [T,K]. */
void oracle_route_sigmoid_grouped(const float *logits, const float *bias, int64_t T, int E,
                                  int num_groups, int topk_group, int top_k, float scale,
                                  int32_t *top_k_index, float *top_k_weights) {
    int gsize = E / num_groups;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        float *s = (float *)malloc(sizeof(float) * E);
        float *c = (float *)malloc(sizeof(float) * E);
        float *gs = (float *)malloc(sizeof(float) * num_groups);
        char *gkeep = (char *)calloc(num_groups, 1);
        char *taken = (char *)calloc(E, 1);
        for (int e = 0; e < E; ++e) {
            double x = (double)logits[t * E + e];
            s[e] = (float)(1.0 / (1.0 + exp(-x)));
            c[e] = s[e] + bias[e];
        }
        for (int g = 0; g < num_groups; ++g) {
            int b1 = -1, b2 = -1;
            for (int e = g * gsize; e < (g + 1) * gsize; ++e) {
                if (b1 < 0 || ranks_before(c[e], e, c[b1], b1)) { b2 = b1; b1 = e; }
                else if (b2 < 0 || ranks_before(c[e], e, c[b2], b2)) { b2 = e; }
            }
            gs[g] = (b2 >= 0) ? c[b1] + c[b2] : c[b1];
        }
        for (int r = 0; r < topk_group; ++r) {
            int best = -1;
            for (int g = 0; g < num_groups; ++g)
                if (!gkeep[g] && (best < 0 || ranks_before(gs[g], g, gs[best], best))) best = g;
            gkeep[best] = 1;
        }
        for (int k = 0; k < top_k; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (gkeep[e / gsize] && !taken[e] && (best < 0 || ranks_before(c[e], e, c[best], best)))
                    best = e;
            taken[best] = 1;
            top_k_index[t * top_k + k] = best;
        }
        float sum = 0.0f;
        for (int k = 0; k < top_k; ++k) sum += s[top_k_index[t * top_k + k]];
        for (int k = 0; k < top_k; ++k) {
            float q = s[top_k_index[t * top_k + k]] / sum;
            top_k_weights[t * top_k + k] = q * scale;
        }
        free(s); free(c); free(gs); free(gkeep); free(taken);
    }
}

/* ------------------------------------------------------------------------ */
/* S3: expert histogram, offsets and stable permutation                      */
/* ------------------------------------------------------------------------ */

/* idx [T*K] (slot = t*K + k).  counts[e] = slots routed to e;
 * offsets = exclusive prefix of counts (E+1 entries);
 * perm[p] = slot at permuted position p, positions grouped by expert and in
 * ascending slot order inside an expert (p >= offsets[E] -> -1);
 * inv[slot] = its position, -1 for expert ids outside [0,E). */
void oracle_permute(const int32_t *idx, int64_t n_slots, int E, int32_t *counts,
                    int32_t *offsets, int32_t *perm, int32_t *inv) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < n_slots; ++i)
        if (idx[i] >= 0 && idx[i] < E) counts[idx[i]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (E > 0 ? E : 1));
    for (int e = 0; e < E; ++e) next[e] = offsets[e];
    for (int64_t p = 0; p < n_slots; ++p) perm[p] = -1;
    for (int64_t i = 0; i < n_slots; ++i) {
        int e = idx[i];
        if (e >= 0 && e < E) { perm[next[e]] = (int32_t)i; inv[i] = next[e]++; }
        else inv[i] = -1;
    }
    free(next);
}

/* ------------------------------------------------------------------------ */
/* Routed-experts forward (S3..S6 / S7 collapsed into the definition)        */
/* ------------------------------------------------------------------------ */

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* One expert's contribution for one token, bf16 weights: gate rows G [F,H],
 * up rows U [F,H], down D [H,F]; xt = x_t (exact bf16 values).
 * h_f = bf16(SiLU(g_f) u_f); acc_j += wk * sum_f D[j,f] h_f (fp64, ascending
 * indices).  hb: scratch [F]. */
static void contrib_bf16(const double *xt, const uint16_t *G, const uint16_t *U, const uint16_t *D,
                         int H, int F, double wk, double *hb, double *acc) {
    for (int f = 0; f < F; ++f) {
        double g = 0.0, u = 0.0;
        for (int i = 0; i < H; ++i) {
            g += bf16_value(G[(int64_t)f * H + i]) * xt[i];
            u += bf16_value(U[(int64_t)f * H + i]) * xt[i];
        }
        hb[f] = bf16_value(bf16_from_double(silu(g) * u));
    }
    for (int j = 0; j < H; ++j) {
        double y = 0.0;
        for (int f = 0; f < F; ++f) y += bf16_value(D[(int64_t)j * F + f]) * hb[f];
        acc[j] += wk * y;
    }
}

/* Routed experts plus S shared experts and a residual, bf16 weights.
 *   out[t] = bf16( sum_k w[t,k] E_{idx[t,k]}(x_t) + sum_s Shared_s(x_t) + residual[t] )
 * summed in fp64 in that order (k ascending, then s ascending, then the
 * residual), rounded once.  Each shared expert is a SwiGLU MLP of width F
 * applied to every token with weight 1 ("Supporting MegaKernel for DeepSeek
 * Models": shared expert through silu_mul_layer; moe_local_reduction adds the
 * residual to the weighted sum).  shared_gate_up [S,2F,H], shared_down
 * [S,H,F]; residual [T,H] bf16 or NULL; S = 0 and NULL give the routed
 * forward alone. */
void oracle_moe_forward_shared_bf16(const uint16_t *x, const uint16_t *gate_up, const uint16_t *down,
                                    const int32_t *idx, const float *w, int64_t T, int H, int F,
                                    int E, int K, const uint16_t *shared_gate_up,
                                    const uint16_t *shared_down, int S, const uint16_t *residual,
                                    uint16_t *out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        double *xt = (double *)malloc(sizeof(double) * H);
        double *acc = (double *)calloc(H, sizeof(double));
        double *hb = (double *)malloc(sizeof(double) * F);
        for (int i = 0; i < H; ++i) xt[i] = bf16_value(x[t * H + i]);
        for (int k = 0; k < K; ++k) {
            int e = idx[t * K + k];
            if (e < 0 || e >= E) continue;
            const uint16_t *G = gate_up + (int64_t)e * 2 * F * H;
            contrib_bf16(xt, G, G + (int64_t)F * H, down + (int64_t)e * H * F, H, F,
                         (double)w[t * K + k], hb, acc);
        }
        for (int s = 0; s < S; ++s) {
            const uint16_t *G = shared_gate_up + (int64_t)s * 2 * F * H;
            contrib_bf16(xt, G, G + (int64_t)F * H, shared_down + (int64_t)s * H * F, H, F, 1.0, hb,
                         acc);
        }
        if (residual)
            for (int j = 0; j < H; ++j) acc[j] += bf16_value(residual[t * H + j]);
        for (int j = 0; j < H; ++j) out[t * H + j] = bf16_from_double(acc[j]);
        free(xt); free(acc); free(hb);
    }
}

/* bf16 weights.  x [T,H], gate_up [E,2F,H] (rows [0,F) gate, [F,2F) up),
 * down [E,H,F], idx/w [T,K]; out [T,H] bf16.
 * h is rounded to bf16 (the intermediate activation is stored in the
 * activation dtype); y is not rounded; out = bf16(sum_k w y). */
void oracle_moe_forward_bf16(const uint16_t *x, const uint16_t *gate_up, const uint16_t *down,
                             const int32_t *idx, const float *w, int64_t T, int H, int F, int E,
                             int K, uint16_t *out) {
    oracle_moe_forward_shared_bf16(x, gate_up, down, idx, w, T, H, F, E, K, NULL, NULL, 0, NULL, out);
}

/* One expert's contribution for one token, E4M3 weights with fp32 scales per
 * (row, 128 columns): W13 [2F,H] + S13 [2F,H/128], W2 [H,F] + S2 [H,F/128];
 * xd = the token's quantised-dequantised activations.  h = bf16(SiLU(g) u)
 * is quantised per 128 features by the S2 rule and dequantised before the
 * down projection.  Scratch: hv, hd [F], hq [F], hs [F/128]. */
static void contrib_fp8(const double *xd, const double *lut, const uint8_t *W13, const float *S13,
                        const uint8_t *W2, const float *S2, int H, int F, double wk, double *hv,
                        double *hd, uint8_t *hq, float *hs, double *acc) {
    int hb_n = H / 128, fb_n = F / 128;
    for (int f = 0; f < F; ++f) {
        int64_t rg = f, ru = (int64_t)F + f;
        double g = 0.0, u = 0.0;
        for (int i = 0; i < H; ++i) {
            g += lut[W13[rg * H + i]] * (double)S13[rg * hb_n + i / 128] * xd[i];
            u += lut[W13[ru * H + i]] * (double)S13[ru * hb_n + i / 128] * xd[i];
        }
        hv[f] = bf16_value(bf16_from_double(silu(g) * u));
    }
    quantize_blocks(hv, fb_n, hq, hs);
    for (int f = 0; f < F; ++f) hd[f] = e4m3_value(hq[f]) * (double)hs[f / 128];
    for (int j = 0; j < H; ++j) {
        double y = 0.0;
        for (int f = 0; f < F; ++f)
            y += lut[W2[(int64_t)j * F + f]] * (double)S2[(int64_t)j * fb_n + f / 128] * hd[f];
        acc[j] += wk * y;
    }
}

/* Routed experts plus S shared experts and a residual, E4M3 weights (same
 * order and rounding points as oracle_moe_forward_shared_bf16; every E4M3
 * operand dequantised before the fp64 dot products). */
void oracle_moe_forward_shared_fp8(const uint16_t *x, const uint8_t *w13, const float *w13_scale,
                                   const uint8_t *w2, const float *w2_scale, const int32_t *idx,
                                   const float *w, int64_t T, int H, int F, int E, int K,
                                   const uint8_t *sw13, const float *sw13_scale, const uint8_t *sw2,
                                   const float *sw2_scale, int S, const uint16_t *residual,
                                   uint16_t *out) {
    int hb_n = H / 128, fb_n = F / 128;
    double lut[256];                               /* value of every E4M3 code */
    for (int c = 0; c < 256; ++c) lut[c] = e4m3_value((uint8_t)c);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        double *xt = (double *)malloc(sizeof(double) * H);
        double *xd = (double *)malloc(sizeof(double) * H);
        uint8_t *xq = (uint8_t *)malloc(H);
        float *xs = (float *)malloc(sizeof(float) * hb_n);
        double *acc = (double *)calloc(H, sizeof(double));
        double *hv = (double *)malloc(sizeof(double) * F);
        double *hd = (double *)malloc(sizeof(double) * F);
        uint8_t *hq = (uint8_t *)malloc(F);
        float *hs = (float *)malloc(sizeof(float) * fb_n);
        for (int i = 0; i < H; ++i) xt[i] = bf16_value(x[t * H + i]);
        quantize_blocks(xt, hb_n, xq, xs);
        for (int i = 0; i < H; ++i) xd[i] = e4m3_value(xq[i]) * (double)xs[i / 128];
        for (int k = 0; k < K; ++k) {
            int e = idx[t * K + k];
            if (e < 0 || e >= E) continue;
            contrib_fp8(xd, lut, w13 + (int64_t)e * 2 * F * H, w13_scale + (int64_t)e * 2 * F * hb_n,
                        w2 + (int64_t)e * H * F, w2_scale + (int64_t)e * H * fb_n, H, F,
                        (double)w[t * K + k], hv, hd, hq, hs, acc);
        }
        for (int s = 0; s < S; ++s)
            contrib_fp8(xd, lut, sw13 + (int64_t)s * 2 * F * H, sw13_scale + (int64_t)s * 2 * F * hb_n,
                        sw2 + (int64_t)s * H * F, sw2_scale + (int64_t)s * H * fb_n, H, F, 1.0, hv, hd,
                        hq, hs, acc);
        if (residual)
            for (int j = 0; j < H; ++j) acc[j] += bf16_value(residual[t * H + j]);
        for (int j = 0; j < H; ++j) out[t * H + j] = bf16_from_double(acc[j]);
        free(xt); free(xd); free(xq); free(xs); free(acc); free(hv); free(hd); free(hq); free(hs);
    }
}

/* FP8 E4M3 weights with fp32 scales per (row, 128-column block):
 * w13 [E,2F,H] + w13_scale [E,2F,H/128], w2 [E,H,F] + w2_scale [E,H,F/128].
 * x (bf16) is quantised per 128 columns by the S2 rule; h = bf16(SiLU(g) u)
 * is quantised per 128 features by the same rule; every E4M3 operand is
 * dequantised (code value * its block scale) before the fp64 dot products;
 * out = bf16(sum_k w y). */
void oracle_moe_forward_fp8(const uint16_t *x, const uint8_t *w13, const float *w13_scale,
                            const uint8_t *w2, const float *w2_scale, const int32_t *idx,
                            const float *w, int64_t T, int H, int F, int E, int K, uint16_t *out) {
    oracle_moe_forward_shared_fp8(x, w13, w13_scale, w2, w2_scale, idx, w, T, H, F, E, K, NULL, NULL,
                                  NULL, NULL, 0, NULL, out);
}

/* ------------------------------------------------------------------------ */
/* FP4 (MXFP4) routed weights with FP8 activations                          */
/* ("Supporting MegaKernel ..." / GC MoE issue: FP8 activations x packed FP4 */
/* routed weights; DeepGEMM Mega MoE news: FP8 x FP4; sgl-deep-gemm commit    */
/* list: "MXF4 kind")                                                        */
/* ------------------------------------------------------------------------ */

/* OCP Microscaling FP4, E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 * mantissa.  Exponent field 0 is subnormal: 0.5 * mantissa; otherwise
 * 2^(e-1) * (1 + mantissa/2).  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static double e2m1_value(unsigned nib) {
    unsigned e = (nib >> 1) & 3u, m = nib & 1u;
    double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, (int)e - 1);
    return (nib & 8u) ? -mag : mag;
}

/* OCP E8M0 block scale: 2^(b - 127); b = 255 encodes NaN. */
static double e8m0_value(uint8_t b) { return b == 255 ? NAN : ldexp(1.0, (int)b - 127); }

/* Element (r, c) of a packed MXFP4 matrix with R rows and C columns
 * (C % 128 == 0, R % 128 == 0):
 *   q  [R][C/2] bytes: element c of a row in byte c/2, even c in the low
 *      nibble, odd c in the high nibble;
 *   sc block-scale bytes (E8M0, one per row and 32 columns) in the tensor
 *      core's block layout: one 512-byte block per (128 rows, 128 columns),
 *      blocks ordered [R/128][C/128], and inside a block the scale of
 *      (r, c) at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 128) / 32.
 * Value = e2m1(code) * 2^(scale - 127). */
static int64_t mxf4_scale_index(int64_t r, int64_t c, int64_t C) {
    int64_t blk = (r / 128) * (C / 128) + c / 128;
    return blk * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 128) / 32;
}
static double mxf4_element(const uint8_t *q, const uint8_t *sc, int64_t C, int64_t r, int64_t c) {
    uint8_t byte = q[r * (C / 2) + c / 2];
    unsigned nib = (c & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 15u);
    return e2m1_value(nib) * e8m0_value(sc[mxf4_scale_index(r, c, C)]);
}

/* Dequantise a packed MXFP4 matrix (layout above) to fp64 [R][C]. */
void oracle_mxf4_dequant(const uint8_t *q, const uint8_t *sc, int64_t R, int64_t C, double *out) {
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c) out[r * C + c] = mxf4_element(q, sc, C, r, c);
}

/* One expert's contribution for one token with MXFP4 weights:
 * W13 [2F][H/2] + S13 (blocks of the [2F, H] matrix), W2 [H][F/2] + S2
 * (blocks of [H, F]); xd = the token's block-128 E4M3 activations,
 * dequantised.  h = bf16(SiLU(g) u) is quantised per 128 features by the
 * block-128 E4M3 rule and dequantised before the down projection (the same
 * activation path as the FP8 layers).  Scratch: wr [max(H,F)], hv, hd [F],
 * hq [F], hs [F/128]. */
static void contrib_mxf4(const double *xd, const uint8_t *W13, const uint8_t *S13, const uint8_t *W2,
                         const uint8_t *S2, int H, int F, double wk, double *wr, double *hv,
                         double *hd, uint8_t *hq, float *hs, double *acc) {
    int fb_n = F / 128;
    for (int f = 0; f < F; ++f) {
        double g = 0.0, u = 0.0;
        for (int i = 0; i < H; ++i) wr[i] = mxf4_element(W13, S13, H, f, i);
        for (int i = 0; i < H; ++i) g += wr[i] * xd[i];
        for (int i = 0; i < H; ++i) wr[i] = mxf4_element(W13, S13, H, (int64_t)F + f, i);
        for (int i = 0; i < H; ++i) u += wr[i] * xd[i];
        hv[f] = bf16_value(bf16_from_double(silu(g) * u));
    }
    quantize_blocks(hv, fb_n, hq, hs);
    for (int f = 0; f < F; ++f) hd[f] = e4m3_value(hq[f]) * (double)hs[f / 128];
    for (int j = 0; j < H; ++j) {
        double y = 0.0;
        for (int f = 0; f < F; ++f) wr[f] = mxf4_element(W2, S2, F, j, f);
        for (int f = 0; f < F; ++f) y += wr[f] * hd[f];
        acc[j] += wk * y;
    }
}

/* MXFP4 routed weights, FP8 activations:
 *   w13 [E][2F][H/2] packed E2M1 + w13_sc (E8M0 blocks of each expert's
 *   [2F, H] matrix, 2F*H/32 bytes per expert), w2 [E][H][F/2] + w2_sc
 *   (H*F/32 bytes per expert), layouts as for mxf4_element.
 * x (bf16) is quantised per 128 columns by the block-128 E4M3 rule; every
 * operand is dequantised before the fp64 dot products; out = bf16(sum_k w y). */
void oracle_moe_forward_mxf4(const uint16_t *x, const uint8_t *w13, const uint8_t *w13_sc,
                             const uint8_t *w2, const uint8_t *w2_sc, const int32_t *idx,
                             const float *w, int64_t T, int H, int F, int E, int K, uint16_t *out) {
    int hb_n = H / 128, fb_n = F / 128;
    int64_t gu_bytes = (int64_t)2 * F * H / 2, gu_sc = (int64_t)2 * F * H / 32;
    int64_t dn_bytes = (int64_t)H * F / 2, dn_sc = (int64_t)H * F / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        double *xt = (double *)malloc(sizeof(double) * H);
        double *xd = (double *)malloc(sizeof(double) * H);
        uint8_t *xq = (uint8_t *)malloc(H);
        float *xs = (float *)malloc(sizeof(float) * hb_n);
        double *acc = (double *)calloc(H, sizeof(double));
        double *wr = (double *)malloc(sizeof(double) * (H > F ? H : F));
        double *hv = (double *)malloc(sizeof(double) * F);
        double *hd = (double *)malloc(sizeof(double) * F);
        uint8_t *hq = (uint8_t *)malloc(F);
        float *hs = (float *)malloc(sizeof(float) * fb_n);
        for (int i = 0; i < H; ++i) xt[i] = bf16_value(x[t * H + i]);
        quantize_blocks(xt, hb_n, xq, xs);
        for (int i = 0; i < H; ++i) xd[i] = e4m3_value(xq[i]) * (double)xs[i / 128];
        for (int k = 0; k < K; ++k) {
            int e = idx[t * K + k];
            if (e < 0 || e >= E) continue;
            contrib_mxf4(xd, w13 + e * gu_bytes, w13_sc + e * gu_sc, w2 + e * dn_bytes,
                         w2_sc + e * dn_sc, H, F, (double)w[t * K + k], wr, hv, hd, hq, hs, acc);
        }
        for (int j = 0; j < H; ++j) out[t * H + j] = bf16_from_double(acc[j]);
        free(xt); free(xd); free(xq); free(xs); free(acc); free(wr); free(hv); free(hd); free(hq);
        free(hs);
    }
}

#ifdef _OPENMP
#include <omp.h>
#endif
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
