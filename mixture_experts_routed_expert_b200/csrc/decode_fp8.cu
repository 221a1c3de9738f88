// decode_fp8.cu -- S7 for E4M3 expert weights: the decode form of the
// routed-experts forward for a few tokens ("deepseek-ocr2-moe-experts" model
// card: fused gather-GEMV, two persistent-shape kernels, no device-to-host
// synchronisation) with the E4M3 layers of "Supporting MegaKernel for
// DeepSeek Models" (moe_w13_fp8_layer, moe_silu_mul_layer,
// bf16_to_fp8_quantize, moe_w2_fp8_layer).
//
// Decode streams the touched experts' E4M3 weights once from HBM.  Weights go
// straight into registers with 16-byte loads; warp-level m16n8k32 E4M3 MMAs
// (fp32 accumulate) reduce 16 rows x 8 slots per 32 columns.  The k index is
// permuted: thread (g, c) owns physical columns [16c, 16c+16) of every
// 64-column chunk, of the weight rows and of the activation row alike.  Each
// 128-column block is reduced on its own and promoted with its scales:
//     acc += (w_scale[row, kb] * a_scale[slot, kb]) * partial_kb.
//   D1: x quantised per 128 (power-of-two scale, E4M3) into shared memory;
//       unit = (touched expert, 8 features, 8 slots), MMA rows 0-7 = gate,
//       8-15 = up; h = bf16(SiLU(g) * u) stored by slot position.
//   D2 (programmatic dependent of D1): quantises h per 128 features into
//       shared memory, then hidden-row groups of the CTA's rows per touched
//       expert; out[t, j] = bf16( sum_{k in order} w[t,k] * y[t*K+k, j] ).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kWarps8 = 16;
constexpr int kThreads8d = 32 * kWarps8;

struct Touched {
    int n;
    int expert[kDecodeMaxSlots];
    int start[kDecodeMaxSlots + 1];
    int slot[kDecodeMaxSlots];       // slots in expert order
    int pos[kDecodeMaxSlots];        // position of each slot in that order (-1: invalid id)
    int e_of[kDecodeMaxSlots];
    int u_of[kDecodeMaxSlots];
    int is_first[kDecodeMaxSlots];
    int nt_start[kDecodeMaxSlots + 1];   // prefix of 8-slot tiles per touched expert
};

// Distinct experts of the T*K slots in order of first appearance, with the
// slots of each in ascending order; built by the first T*K+1 threads.  Every
// thread of the block must call it.
__device__ void build_touched(const int32_t *__restrict__ idx, int TK, int E, Touched &u) {
    const int s = threadIdx.x;
    if (s < TK) {
        const int e = __ldg(idx + s);
        u.e_of[s] = (e >= 0 && e < E) ? e : -1;
    }
    __syncthreads();
    int e = -1, first = -1;
    if (s < TK) {
        e = u.e_of[s];
        if (e >= 0) {
            first = s;
            for (int q = 0; q < s; ++q)
                if (u.e_of[q] == e) { first = q; break; }
        }
        u.is_first[s] = (e >= 0 && first == s);
    }
    __syncthreads();
    if (s < TK && e >= 0 && first == s) {
        int rank = 0;
        for (int q = 0; q < s; ++q) rank += u.is_first[q];
        u.u_of[s] = rank;
        u.expert[rank] = e;
    }
    __syncthreads();
    if (s < TK && e >= 0 && first != s) u.u_of[s] = u.u_of[first];
    __syncthreads();
    if (s <= TK) {
        int c = 0;
        for (int q = 0; q < TK; ++q) c += (u.e_of[q] >= 0 && u.u_of[q] < s);
        u.start[s] = c;
        if (s == 0) {
            int n = 0;
            for (int q = 0; q < TK; ++q) n += u.is_first[q];
            u.n = n;
        }
    }
    __syncthreads();
    if (s < TK) {
        int p = -1;
        if (e >= 0) {
            p = u.start[u.u_of[s]];
            for (int q = 0; q < s; ++q) p += (u.e_of[q] == e);
            u.slot[p] = s;
        }
        u.pos[s] = p;
    }
    if (s == 0) {
        int c = 0;
        for (int v = 0; v < u.n; ++v) {
            u.nt_start[v] = c;
            c += (u.start[v + 1] - u.start[v] + 7) / 8;
        }
        u.nt_start[u.n] = c;
    }
    __syncthreads();
}

// Weight stream: read once, not kept in L1, first out of L2.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p, uint64_t pol) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p), "l"(pol));
    return r;
}
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ uint4 ld_cg(const uint4 *p) {
    uint4 r;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Touched expert v of 8-slot tile `tile` (tiles are numbered expert by expert).
__device__ __forceinline__ int tile_expert(const Touched &tu, int tile) {
    int v = 0;
    while (tu.nt_start[v + 1] <= tile) ++v;
    return v;
}


// D (16x8 fp32) += A (16x32 e4m3, row) * B (32x8 e4m3, col).
__device__ __forceinline__ void mma_16832_e4m3(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 64-column chunk: lo / hi = 16 bytes of rows g and g+8, b = 16 bytes of
// this thread's B column; two k-steps of 32.
__device__ __forceinline__ void mma_chunk8(float (&d)[4], const uint4 lo, const uint4 hi,
                                           const uint4 b) {
    mma_16832_e4m3(d, lo.x, hi.x, lo.y, hi.y, b.x, b.y);
    mma_16832_e4m3(d, lo.z, hi.z, lo.w, hi.w, b.z, b.w);
}

struct Dec8Args {
    const uint8_t *w13;       // [E][2F][H] e4m3
    const float *w13s;        // [E][2F][H/128]
    const uint8_t *w2;        // [E][H][F] e4m3
    const float *w2s;         // [E][H][F/128]
    const uint4 *x;           // [T][H] bf16
    const int32_t *idx;       // [T][K]
    const float *w;           // [T][K]
    int T, H, F, E, K;
    __nv_bfloat16 *h;         // [T*K][F] bf16, rows in expert order
    __nv_bfloat16 *out;       // [T][H]
    int64_t pf_bytes;         // D2 L2 prefetch budget per (CTA, touched expert)
};

// Block-128 E4M3 quantisation of `rows` bf16 rows of `cols` columns into
// shared memory (row pitch `pitch` bytes) with scales [rows][cols/128].
// A half-warp takes one block of 128; each warp issues the loads of up to
// four passes before converting any.  CG reads through L2 only (data written
// by the previous kernel).  Every thread of the block calls it.
template <bool CG>
__device__ void quantize_rows_smem(const uint4 *src, int rows, int cols, uint8_t *q, int pitch,
                                   float *scales, int warp, int nwarps, int lane) {
    constexpr int kDepth = 4;
    const int nb = cols / 128;
    const int total = rows * nb;
    const int step = 2 * nwarps;
    for (int pb = 2 * warp; pb < total; pb += kDepth * step) {   // uniform per warp
        uint4 raw[kDepth];
#pragma unroll
        for (int d = 0; d < kDepth; ++d) {
            const int b = pb + d * step + (lane >> 4);
            raw[d] = make_uint4(0, 0, 0, 0);
            if (b < total) {
                const int r = b / nb, kb = b - r * nb;
                const uint4 *p = src + (size_t)(r * cols + kb * 128) / 8 + (lane & 15);
                raw[d] = CG ? ld_cg(p) : __ldg(p);
            }
        }
#pragma unroll
        for (int d = 0; d < kDepth; ++d) {
            if (pb + d * step >= total) break;                    // uniform per warp
            const int b = pb + d * step + (lane >> 4);
            float f[8];
            unpack_bf16x8(raw[d], f);
            float sc;
            const uint2 code = quant8_e4m3(f, sc);
            if (b < total) {
                const int r = b / nb, kb = b - r * nb;
                *reinterpret_cast<uint2 *>(q + (size_t)r * pitch + kb * 128 + (lane & 15) * 8) = code;
                if ((lane & 15) == 0) scales[r * nb + kb] = sc;
            }
        }
    }
}

// ---- the shared GEMV engine of D1 and D2 ------------------------------------
//
// A unit is 16 weight rows (A) x 8 activation rows (B, in shared memory) over
// nkb blocks of 128 columns.  A CTA's units are split evenly over its warps in
// block steps ("pieces" where a warp's range meets a unit); each piece's 16x8
// fp32 result goes to shared memory at index (unit - first unit) + warp, and
// the pieces of a unit are later summed in warp order (fixed order, no atomics).

constexpr int kPieces1 = 128;          // D1 piece slots (units per round + 16)
constexpr int kPieces2 = 96;           // D2 piece slots

// This lane's view of one unit: row g of A (row g+8 lies `hi_off` further),
// its scale row, the B row of column g and the B scale rows of columns 2c, 2c+1.
struct UnitView {
    const uint4 *a;
    const float *s;
    int b_row, s_col0, s_col1;
};

struct Blk2 {
    uint4 lo[2][2], hi[2][2];
    float sl[2], sh[2];
};

// Warp w of 16 owns block steps [total*w/16, total*(w+1)/16); the owner of q.
__device__ __forceinline__ int owner_warp(int q, int total) { return (kWarps8 * q + kWarps8 - 1) / total; }

template <class ViewFn>
__device__ __forceinline__ void gemv_pieces(int qa, int qb, int nkb, int64_t hi_vec, int64_t hi_sc,
                                            ViewFn view, const uint8_t *bq, int bpitch,
                                            const float *bs, float4 *part, int warp, int lane,
                                            uint64_t pol) {
    const int c = lane & 3;
    int lu = -1, cu = -1;
    UnitView lv = {}, cv = {};
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    auto load2 = [&](Blk2 &r, int q) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int qq = q + j;
            if (qq < qb) {
                const int u = qq / nkb, kb = qq - u * nkb;
                if (u != lu) { lv = view(u); lu = u; }
                const uint4 *a = lv.a + kb * 8 + c;
                r.lo[j][0] = ld_stream(a, pol);
                r.lo[j][1] = ld_stream(a + 4, pol);
                r.hi[j][0] = ld_stream(a + hi_vec, pol);
                r.hi[j][1] = ld_stream(a + hi_vec + 4, pol);
                r.sl[j] = __ldg(lv.s + kb);
                r.sh[j] = __ldg(lv.s + hi_sc + kb);
            }
        }
    };
    auto comp2 = [&](const Blk2 &r, int q) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int qq = q + j;
            if (qq < qb) {
                const int u = qq / nkb, kb = qq - u * nkb;
                if (u != cu) { cv = view(u); cu = u; }
                const uint8_t *brow = bq + cv.b_row * bpitch + kb * 128 + 16 * c;
                const uint4 b0 = *reinterpret_cast<const uint4 *>(brow);
                const uint4 b1 = *reinterpret_cast<const uint4 *>(brow + 64);
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                mma_chunk8(d, r.lo[j][0], r.hi[j][0], b0);
                mma_chunk8(d, r.lo[j][1], r.hi[j][1], b1);
                const float sx0 = bs[cv.s_col0 * nkb + kb], sx1 = bs[cv.s_col1 * nkb + kb];
                acc[0] = fmaf(r.sl[j] * sx0, d[0], acc[0]);
                acc[1] = fmaf(r.sl[j] * sx1, d[1], acc[1]);
                acc[2] = fmaf(r.sh[j] * sx0, d[2], acc[2]);
                acc[3] = fmaf(r.sh[j] * sx1, d[3], acc[3]);
                if (kb == nkb - 1 || qq == qb - 1) {
                    part[(u + warp) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
                }
            }
        }
    };
    Blk2 ra, rb;
    int q = qa;
    if (q < qb) load2(ra, q);
    for (; q < qb; q += 4) {
        if (q + 2 < qb) load2(rb, q + 2);
        comp2(ra, q);
        if (q + 4 < qb) load2(ra, q + 4);
        if (q + 2 < qb) comp2(rb, q + 2);
    }
}

// Sum of the pieces of local unit i (in warp order) for this lane; warps with
// an empty range between the first and the last owner wrote nothing.
__device__ __forceinline__ float4 sum_pieces(const float4 *part, int i, int nkb, int total, int lane) {
    const int wf = owner_warp(i * nkb, total), wl = owner_warp((i + 1) * nkb - 1, total);
    float4 a = part[(i + wf) * 32 + lane];
    for (int w = wf + 1; w <= wl; ++w) {
        if (total * w / kWarps8 == total * (w + 1) / kWarps8) continue;
        const float4 b = part[(i + w) * 32 + lane];
        a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    return a;
}

// Position of the first slot of 8-slot tile `tile` (of touched expert v) in
// expert order, and the number of slots it holds.
__device__ __forceinline__ void tile_slots(const Touched &tu, int tile, int v, int &p0, int &nval) {
    p0 = tu.start[v] + 8 * (tile - tu.nt_start[v]);
    nval = min(8, tu.start[v + 1] - p0);
}

// D1: units = (tile, 8 features); A rows 0-7 = gate rows f0..f0+7, rows 8-15 =
// the matching up rows; B = the quantised x rows of the tile's tokens.
__global__ void __launch_bounds__(kThreads8d, 1) decode_up_fp8(Dec8Args a) {
    __shared__ Touched tu;
    extern __shared__ __align__(16) uint8_t smem8[];
    float4 *part = reinterpret_cast<float4 *>(smem8);
    const int nkb = a.H / 128;
    const int xpitch = a.H + 64;
    uint8_t *xq = smem8 + sizeof(float4) * 32 * kPieces1;
    float *xs = reinterpret_cast<float *>(xq + (size_t)a.T * xpitch);
    build_touched(a.idx, a.T * a.K, a.E, tu);
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int g = lane >> 2, c = lane & 3;
    const uint64_t pol = policy_evict_first();
    const int fg_n = a.F / 8;
    const int U = tu.nt_start[tu.n] * fg_n;
    const int u0 = (int)((int64_t)U * blockIdx.x / gridDim.x);
    const int u1 = (int)((int64_t)U * (blockIdx.x + 1) / gridDim.x);
    const int64_t hi_vec = (int64_t)a.F * a.H / 16, hi_sc = (int64_t)a.F * nkb;
    const int R = kPieces1 - kWarps8;
    if (u0 >= u1) return;
    for (int r0 = u0; r0 < u1; r0 += R) {
        const int nu = min(R, u1 - r0);
        const int total = nu * nkb;
        auto view = [&](int ul) {
            const int unit = r0 + ul;
            const int tile = unit / fg_n, fg = unit - tile * fg_n;
            const int v = tile_expert(tu, tile);
            int p0, nval;
            tile_slots(tu, tile, v, p0, nval);
            const int64_t row = (int64_t)tu.expert[v] * 2 * a.F + fg * 8 + g;
            UnitView uv;
            uv.a = reinterpret_cast<const uint4 *>(a.w13) + row * (a.H / 16);
            uv.s = a.w13s + row * nkb;
            uv.b_row = tu.slot[p0 + (g < nval ? g : 0)] / a.K;
            uv.s_col0 = tu.slot[p0 + (2 * c < nval ? 2 * c : 0)] / a.K;
            uv.s_col1 = tu.slot[p0 + (2 * c + 1 < nval ? 2 * c + 1 : 0)] / a.K;
            return uv;
        };
        const int qa = total * warp / kWarps8, qb = total * (warp + 1) / kWarps8;
        if (r0 == u0) {
            // Start this warp's first two weight blocks towards L2, then
            // quantise x into shared memory (every CTA, every token).
            if (qa + (c >> 1) < qb) {
                const int qq = qa + (c >> 1), ul = qq / nkb;
                const UnitView uv = view(ul);
                prefetch_l2(uv.a + (qq - ul * nkb) * 8 + ((c & 1) ? hi_vec : 0));
            }
            quantize_rows_smem<false>(a.x, a.T, a.H, xq, xpitch, xs, warp, kWarps8, lane);
            __syncthreads();
        }
        gemv_pieces(qa, qb, nkb, hi_vec, hi_sc, view, xq, xpitch, xs, part, warp, lane, pol);
        __syncthreads();
        for (int i = warp; i < nu; i += kWarps8) {
            const float4 p = sum_pieces(part, i, nkb, total, lane);
            const int unit = r0 + i;
            const int tile = unit / fg_n, fg = unit - tile * fg_n;
            const int v = tile_expert(tu, tile);
            int p0, nval;
            tile_slots(tu, tile, v, p0, nval);
            const int f = fg * 8 + g;
            if (2 * c < nval)
                a.h[(int64_t)(p0 + 2 * c) * a.F + f] = __float2bfloat16_rn(silu_f(p.x) * p.z);
            if (2 * c + 1 < nval)
                a.h[(int64_t)(p0 + 2 * c + 1) * a.F + f] = __float2bfloat16_rn(silu_f(p.y) * p.w);
        }
        __syncthreads();
    }
}

// D2: CTA b owns 16-row groups [rg0, rg1) of the hidden dimension; units =
// (tile, row group); A = 16 consecutive down-projection rows of the tile's
// expert, B = the quantised h rows of the tile's slots.  The per-slot results
// y land in shared memory; then out[t, j] = bf16( sum_{k in order} w[t,k] *
// y[t*K+k, j] ).
__global__ void __launch_bounds__(kThreads8d, 1) decode_down_fp8(Dec8Args a) {
    __shared__ Touched tu;
    extern __shared__ __align__(16) uint8_t smem8[];
    const int TK = a.T * a.K;
    const int nkb = a.F / 128;
    const int hpitch = a.F + 64;
    const int nrg = a.H / 16;
    const int rg0 = (int)((int64_t)nrg * blockIdx.x / gridDim.x);
    const int rg1 = (int)((int64_t)nrg * (blockIdx.x + 1) / gridDim.x);
    const int nrl = rg1 - rg0;
    float4 *part = reinterpret_cast<float4 *>(smem8);
    uint8_t *hq = smem8 + sizeof(float4) * 32 * kPieces2;
    float *hs = reinterpret_cast<float *>(hq + (size_t)TK * hpitch);
    float *ys = hs + (size_t)TK * nkb;                     // [16 * nrl][TK]
    build_touched(a.idx, TK, a.E, tu);
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int g = lane >> 2, c = lane & 3;
    // While D1 runs: start this CTA's down-projection rows towards L2, up to a
    // budget of pf_bytes per touched expert.
    if (threadIdx.x < tu.n && nrl > 0) {
        const uint8_t *base = a.w2 + ((int64_t)tu.expert[threadIdx.x] * a.H + rg0 * 16) * a.F;
        const int64_t rows_bytes = (int64_t)nrl * 16 * a.F;
        const uint32_t bytes = (uint32_t)(rows_bytes < a.pf_bytes ? rows_bytes : a.pf_bytes);
        for (uint32_t off = 0; off < bytes; off += 32768)
            prefetch_l2_bulk(base + off, min(32768u, bytes - off));
    }
    pdl_wait();
    const int nslots = tu.start[tu.n];
    quantize_rows_smem<true>(reinterpret_cast<const uint4 *>(a.h), nslots, a.F, hq, hpitch, hs,
                             warp, kWarps8, lane);
    __syncthreads();
    const uint64_t pol = policy_evict_first();
    const int U = tu.nt_start[tu.n] * nrl;
    const int64_t hi_vec = (int64_t)8 * a.F / 16, hi_sc = (int64_t)8 * nkb;
    const int R = kPieces2 - kWarps8;
    for (int r0 = 0; r0 < U; r0 += R) {
        const int nu = min(R, U - r0);
        const int total = nu * nkb;
        auto view = [&](int ul) {
            const int unit = r0 + ul;
            const int tile = unit / nrl, rgl = unit - tile * nrl;
            const int v = tile_expert(tu, tile);
            int p0, nval;
            tile_slots(tu, tile, v, p0, nval);
            const int64_t row = (int64_t)tu.expert[v] * a.H + (rg0 + rgl) * 16 + g;
            UnitView uv;
            uv.a = reinterpret_cast<const uint4 *>(a.w2) + row * (a.F / 16);
            uv.s = a.w2s + row * nkb;
            uv.b_row = p0 + (g < nval ? g : 0);
            uv.s_col0 = p0 + (2 * c < nval ? 2 * c : 0);
            uv.s_col1 = p0 + (2 * c + 1 < nval ? 2 * c + 1 : 0);
            return uv;
        };
        const int qa = total * warp / kWarps8, qb = total * (warp + 1) / kWarps8;
        gemv_pieces(qa, qb, nkb, hi_vec, hi_sc, view, hq, hpitch, hs, part, warp, lane, pol);
        __syncthreads();
        for (int i = warp; i < nu; i += kWarps8) {
            const float4 p = sum_pieces(part, i, nkb, total, lane);
            const int unit = r0 + i;
            const int tile = unit / nrl, rgl = unit - tile * nrl;
            const int v = tile_expert(tu, tile);
            int p0, nval;
            tile_slots(tu, tile, v, p0, nval);
            const int jl = rgl * 16 + g;
            if (2 * c < nval) {
                ys[jl * TK + p0 + 2 * c] = p.x;
                ys[(jl + 8) * TK + p0 + 2 * c] = p.z;
            }
            if (2 * c + 1 < nval) {
                ys[jl * TK + p0 + 2 * c + 1] = p.y;
                ys[(jl + 8) * TK + p0 + 2 * c + 1] = p.w;
            }
        }
        __syncthreads();
    }
    for (int q = threadIdx.x; q < nrl * 16 * a.T; q += blockDim.x) {
        const int t = q / (nrl * 16), jl = q - t * (nrl * 16);
        float acc = 0.f;
        for (int k = 0; k < a.K; ++k) {
            const int s = t * a.K + k;
            const int p = tu.pos[s];
            if (p < 0) continue;
            acc = fmaf(a.w[s], ys[jl * TK + p], acc);
        }
        a.out[(int64_t)t * a.H + rg0 * 16 + jl] = __float2bfloat16_rn(acc);
    }
}

}  // namespace

namespace {

constexpr size_t kSmemLimit8 = 227 * 1024 - sizeof(Touched) - 1024;
constexpr int64_t kPrefetchBudget8 = 48ll << 20;   // bytes of D2 rows started during D1

size_t d1_smem(int T, int H) {
    return sizeof(float4) * 32 * kPieces1 + (size_t)T * (H + 64) + sizeof(float) * T * (H / 128);
}
size_t d2_smem(int T, int K, int H, int F, int grid) {
    const int TK = T * K, nrl_max = (H / 16 + grid - 1) / grid;
    return sizeof(float4) * 32 * kPieces2 + (size_t)TK * (F + 64) +
           sizeof(float) * TK * (F / 128) + sizeof(float) * 16 * nrl_max * TK;
}

}  // namespace

bool decode_fp8_fits(int T, int K, int H, int F) {
    if (T < 1 || T > kDecodeMaxT || T * K > kDecodeMaxSlots || H % 128 || F % 128) return false;
    return d1_smem(T, H) <= kSmemLimit8 && d2_smem(T, K, H, F, num_sms()) <= kSmemLimit8;
}

cudaError_t launch_decode_fp8(const void *x, const void *w13, const float *w13s, const void *w2,
                              const float *w2s, const int32_t *idx, const float *w, int T, int H,
                              int F, int E, int K, uint8_t *ws, const DecodeWorkspace &L, void *out,
                              cudaStream_t st) {
    static bool attr_set[64] = {};    // per device; both kernels get the full limit once
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(decode_up_fp8, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemLimit8);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_down_fp8, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kSmemLimit8);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int grid = num_sms();
    Dec8Args a;
    a.w13 = static_cast<const uint8_t *>(w13);
    a.w13s = w13s;
    a.w2 = static_cast<const uint8_t *>(w2);
    a.w2s = w2s;
    a.x = static_cast<const uint4 *>(x);
    a.idx = idx;
    a.w = w;
    a.T = T; a.H = H; a.F = F; a.E = E; a.K = K;
    a.h = reinterpret_cast<__nv_bfloat16 *>(ws + L.h);
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.pf_bytes = kPrefetchBudget8 / ((int64_t)grid * std::max(1, std::min(T * K, E))) / 16 * 16;
    cudaError_t e = launch_k(decode_up_fp8, dim3(grid), dim3(kThreads8d), d1_smem(T, H), st, false, a);
    if (e != cudaSuccess) return e;
    return launch_k(decode_down_fp8, dim3(grid), dim3(kThreads8d), d2_smem(T, K, H, F, grid), st,
                    true, a);
}

}  // namespace moe
