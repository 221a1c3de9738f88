// decode.cu -- S7: the decode form of the routed-experts forward for a few
// tokens ("deepseek-ocr2-moe-experts" model card: fused gather-GEMV for
// n_tokens ~ 1-4, two persistent-shape kernels, no per-expert library loop,
// no device-to-host synchronisation).
//
//   D1 (up):   for every distinct expert e touched by the T*K slots and every
//              feature f, stream gate row f and up row f of e once and apply
//              them to every slot routed to e:  h[s, f] = bf16(SiLU(g) * u).
//   D2 (down): output-stationary over the hidden dimension: for a row j,
//              stream row j of every touched down projection once, y_s =
//              D_e[j] . h[s] for the slots of e, then
//              out[t, j] = bf16( sum_{k in order} w[t,k] * y_{t*K+k} ).
// D2 is launched as a programmatic dependent of D1: before waiting for D1 it
// prefetches its own down-projection rows into L2, so both kernels stream
// weights from HBM at the same time.  No atomics; fixed summation order.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kUpWarps = 16;
constexpr int kDownWarps = 16;
constexpr int kSlotGroup = 4;   // slots of one expert handled per weight pass
constexpr int kChunkVec = 4;    // 16-byte vectors per lane kept in flight per row

// Distinct experts of the T*K slots, in order of first appearance, with the
// slots of each in ascending order.  Built by one thread.
struct Touched {
    int n;
    int expert[kDecodeMaxSlots];
    int start[kDecodeMaxSlots + 1];
    int slot[kDecodeMaxSlots];
};

__device__ void build_touched(const int32_t *__restrict__ idx, int TK, int E, Touched &u) {
    int n = 0, m = 0;
    for (int s = 0; s < TK; ++s) {
        const int e = idx[s];
        if (e < 0 || e >= E) continue;
        bool seen = false;
        for (int i = 0; i < n; ++i) seen |= (u.expert[i] == e);
        if (!seen) u.expert[n++] = e;
    }
    for (int i = 0; i < n; ++i) {
        u.start[i] = m;
        for (int s = 0; s < TK; ++s)
            if (idx[s] == u.expert[i]) u.slot[m++] = s;
    }
    u.start[n] = m;
    u.n = n;
}

__device__ __forceinline__ float dot8_bf16(const uint4 a, const uint4 b, float acc) {
    acc = fmaf(bf16_lo(a.x), bf16_lo(b.x), acc);
    acc = fmaf(bf16_hi(a.x), bf16_hi(b.x), acc);
    acc = fmaf(bf16_lo(a.y), bf16_lo(b.y), acc);
    acc = fmaf(bf16_hi(a.y), bf16_hi(b.y), acc);
    acc = fmaf(bf16_lo(a.z), bf16_lo(b.z), acc);
    acc = fmaf(bf16_hi(a.z), bf16_hi(b.z), acc);
    acc = fmaf(bf16_lo(a.w), bf16_lo(b.w), acc);
    acc = fmaf(bf16_hi(a.w), bf16_hi(b.w), acc);
    return acc;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// D1.  One item = (touched expert, feature); items split evenly over blocks.
__global__ void __launch_bounds__(kUpWarps * 32) decode_up_bf16(
    const uint4 *__restrict__ x, const uint4 *__restrict__ gate_up, const int32_t *__restrict__ idx,
    int T, int H, int F, int E, int K, __nv_bfloat16 *__restrict__ h) {
    __shared__ Touched tu;
    if (threadIdx.x == 0) build_touched(idx, T * K, E, tu);
    __syncthreads();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int nv = H / 8;
    const int64_t items = (int64_t)tu.n * F;
    const int64_t i0 = items * blockIdx.x / gridDim.x, i1 = items * (blockIdx.x + 1) / gridDim.x;
    for (int64_t it = i0 + warp; it < i1; it += kUpWarps) {
        const int ui = (int)(it / F), f = (int)(it - (int64_t)ui * F);
        const int e = tu.expert[ui];
        const uint4 *grow = gate_up + ((int64_t)e * 2 * F + f) * nv;
        const uint4 *urow = grow + (int64_t)F * nv;
        for (int g0 = tu.start[ui]; g0 < tu.start[ui + 1]; g0 += kSlotGroup) {
            const int ns = min(kSlotGroup, tu.start[ui + 1] - g0);
            float ga[kSlotGroup] = {}, ua[kSlotGroup] = {};
            for (int v0 = 0; v0 < nv; v0 += 32 * kChunkVec) {
                uint4 wg[kChunkVec], wu[kChunkVec];
#pragma unroll
                for (int c = 0; c < kChunkVec; ++c) {
                    const int v = v0 + c * 32 + lane;
                    wg[c] = v < nv ? ld_stream(grow + v) : make_uint4(0, 0, 0, 0);
                    wu[c] = v < nv ? ld_stream(urow + v) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int si = 0; si < kSlotGroup; ++si) {
                    if (si < ns) {
                        const uint4 *xr = x + (int64_t)(tu.slot[g0 + si] / K) * nv;
#pragma unroll
                        for (int c = 0; c < kChunkVec; ++c) {
                            const int v = v0 + c * 32 + lane;
                            if (v < nv) {
                                const uint4 xv = __ldg(xr + v);
                                ga[si] = dot8_bf16(wg[c], xv, ga[si]);
                                ua[si] = dot8_bf16(wu[c], xv, ua[si]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int si = 0; si < kSlotGroup; ++si) {
                if (si < ns) {
                    const float g = warp_sum(ga[si]);
                    const float u = warp_sum(ua[si]);
                    if (lane == 0)
                        h[(int64_t)tu.slot[g0 + si] * F + f] = __float2bfloat16_rn(silu_f(g) * u);
                }
            }
        }
    }
}

// D2.  One item = hidden row j; rows split evenly over blocks.
__global__ void __launch_bounds__(kDownWarps * 32) decode_down_bf16(
    const uint4 *__restrict__ down, const uint4 *__restrict__ h, const int32_t *__restrict__ idx,
    const float *__restrict__ w, int T, int H, int F, int E, int K, __nv_bfloat16 *__restrict__ out) {
    __shared__ Touched tu;
    __shared__ float ys[kDownWarps][kDecodeMaxSlots];
    if (threadIdx.x == 0) build_touched(idx, T * K, E, tu);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int nv = F / 8;
    const int j0 = (int)((int64_t)H * blockIdx.x / gridDim.x);
    const int j1 = (int)((int64_t)H * (blockIdx.x + 1) / gridDim.x);
    // Stream this block's down rows into L2 while D1 is still running.
    if (j1 > j0 && threadIdx.x < tu.n)
        prefetch_l2_bulk(down + ((int64_t)tu.expert[threadIdx.x] * H + j0) * nv,
                         (uint32_t)((j1 - j0) * F * 2));
    pdl_wait();
    for (int j = j0 + warp; j < j1; j += kDownWarps) {
        for (int ui = 0; ui < tu.n; ++ui) {
            const uint4 *drow = down + ((int64_t)tu.expert[ui] * H + j) * nv;
            for (int g0 = tu.start[ui]; g0 < tu.start[ui + 1]; g0 += kSlotGroup) {
                const int ns = min(kSlotGroup, tu.start[ui + 1] - g0);
                float ya[kSlotGroup] = {};
                for (int v0 = 0; v0 < nv; v0 += 32 * kChunkVec) {
                    uint4 wd[kChunkVec];
#pragma unroll
                    for (int c = 0; c < kChunkVec; ++c) {
                        const int v = v0 + c * 32 + lane;
                        wd[c] = v < nv ? __ldg(drow + v) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int si = 0; si < kSlotGroup; ++si) {
                        if (si < ns) {
                            const uint4 *hr = h + (int64_t)tu.slot[g0 + si] * nv;
#pragma unroll
                            for (int c = 0; c < kChunkVec; ++c) {
                                const int v = v0 + c * 32 + lane;
                                if (v < nv) ya[si] = dot8_bf16(wd[c], __ldg(hr + v), ya[si]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int si = 0; si < kSlotGroup; ++si) {
                    if (si < ns) {
                        const float y = warp_sum(ya[si]);
                        if (lane == 0) ys[warp][tu.slot[g0 + si]] = y;
                    }
                }
            }
        }
        __syncwarp();
        if (lane < T) {
            float acc = 0.f;
            for (int k = 0; k < K; ++k) {
                const int s = lane * K + k;
                const int e = idx[s];
                if (e < 0 || e >= E) continue;
                acc = fmaf(w[s], ys[warp][s], acc);
            }
            out[(int64_t)lane * H + j] = __float2bfloat16_rn(acc);
        }
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_decode_bf16(const void *x, const void *gate_up, const void *down,
                               const int32_t *idx, const float *w, int T, int H, int F, int E,
                               int K, uint8_t *ws, const DecodeWorkspace &L, void *out,
                               cudaStream_t st) {
    const int sms = num_sms();
    __nv_bfloat16 *h = (__nv_bfloat16 *)(ws + L.h);
    cudaError_t err = launch_k(decode_up_bf16, dim3(sms), dim3(kUpWarps * 32), 0, st, false,
                               (const uint4 *)x, (const uint4 *)gate_up, idx, T, H, F, E, K, h);
    if (err != cudaSuccess) return err;
    return launch_k(decode_down_bf16, dim3(sms), dim3(kDownWarps * 32), 0, st, true,
                    (const uint4 *)down, (const uint4 *)h, idx, w, T, H, F, E, K,
                    (__nv_bfloat16 *)out);
}

}  // namespace moe
