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
// Optional shared experts (S of them, weight 1) take slots K..K+S-1 of every
// token after its K routed slots, with their own weight tensors, and an
// optional residual is added after the slot sum.
// D1 is launched as a programmatic dependent of the previous kernel on the
// stream (its blocks are placed while that kernel drains; it waits before
// reading any input).
// D2 is launched as a programmatic dependent of D1: before waiting for D1 it
// prefetches its own down-projection rows into L2, so both kernels stream
// weights from HBM at the same time.  No atomics; fixed summation order.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kUpWarps = 16;
constexpr int kDownWarps = 16;
constexpr int kSlotGroup = 1;   // slots of one expert handled per pass over the loaded rows

// Distinct experts of the T*(K+S) slots, in order of first appearance, with
// the slots of each in ascending order.  Slot t*(K+S)+k holds routed id
// idx[t,k] for k < K (-1 when outside [0, E)) and shared expert E+(k-K)
// after that.  Built cooperatively by the first kDecodeMaxSlots threads of the
// block (one slot each); every thread must call it (it contains
// __syncthreads).
struct Touched {
    int n;
    int expert[kDecodeMaxSlots];
    int start[kDecodeMaxSlots + 1];
    int slot[kDecodeMaxSlots];
    int e_of[kDecodeMaxSlots];     // expert id of each slot (-1 when out of range)
    int u_of[kDecodeMaxSlots];     // touched index of each slot
};

__device__ void build_touched(const int32_t *__restrict__ idx, int T, int K, int S, int E,
                              Touched &u) {
    __shared__ int is_first[kDecodeMaxSlots];
    const int K2 = K + S;
    const int TK = T * K2;
    const int s = threadIdx.x;
    if (s < TK) {
        const int t = s / K2, k = s - t * K2;
        if (k < K) {
            const int e = __ldg(idx + t * K + k);
            u.e_of[s] = (e >= 0 && e < E) ? e : -1;
        } else {
            u.e_of[s] = E + (k - K);
        }
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
        is_first[s] = (e >= 0 && first == s);
    }
    __syncthreads();
    if (s < TK && e >= 0 && first == s) {   // rank among the distinct experts
        int rank = 0;
        for (int q = 0; q < s; ++q) rank += is_first[q];
        u.u_of[s] = rank;
        u.expert[rank] = e;
    }
    __syncthreads();
    if (s < TK && e >= 0 && first != s) u.u_of[s] = u.u_of[first];
    __syncthreads();
    if (s <= TK) {                            // start[v]: slots of earlier experts
        int c = 0;
        for (int q = 0; q < TK; ++q) c += (u.e_of[q] >= 0 && u.u_of[q] < s);
        u.start[s] = c;
        if (s == 0) {
            int n = 0;
            for (int q = 0; q < TK; ++q) n += is_first[q];
            u.n = n;
        }
    }
    __syncthreads();
    if (s < TK && e >= 0) {
        int pos = u.start[u.u_of[s]];
        for (int q = 0; q < s; ++q) pos += (u.e_of[q] == e);
        u.slot[pos] = s;
    }
    __syncthreads();
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

// D1.  One item = (touched expert, feature f): gate row f and up row f are
// loaded whole (VPL 16-byte vectors per lane each) before any use, and the
// next item's rows are requested before the current one is reduced, so every
// warp keeps up to 4*VPL*512 bytes in flight.  Items are split evenly over
// blocks.
template <int VPL>
struct UpRows {
    uint4 g[VPL], u[VPL];
};

template <int VPL, bool EXTRA>
__device__ __forceinline__ void up_load(UpRows<VPL> &r, const uint4 *__restrict__ gate_up,
                                        const uint4 *__restrict__ gate_up2, int E,
                                        const Touched &tu, int64_t it, int F, int nv, int lane) {
    const int ui = (int)(it / F), f = (int)(it - (int64_t)ui * F);
    const int e = tu.expert[ui];
    const uint4 *grow = (!EXTRA || e < E ? gate_up + (int64_t)e * 2 * F * nv
                                         : gate_up2 + (int64_t)(e - E) * 2 * F * nv) +
                        (int64_t)f * nv;
    const uint4 *urow = grow + (int64_t)F * nv;
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
        const int v = c * 32 + lane;
        r.g[c] = v < nv ? ld_stream(grow + v) : make_uint4(0, 0, 0, 0);
        r.u[c] = v < nv ? ld_stream(urow + v) : make_uint4(0, 0, 0, 0);
    }
}

template <int VPL>
__device__ __forceinline__ void up_compute(const UpRows<VPL> &r, const uint4 *__restrict__ x,
                                           const Touched &tu, int64_t it, int F, int K, int nv,
                                           int lane, __nv_bfloat16 *__restrict__ h) {
    const int ui = (int)(it / F), f = (int)(it - (int64_t)ui * F);
    for (int q = tu.start[ui]; q < tu.start[ui + 1]; ++q) {
        const int slot = tu.slot[q];
        const uint4 *xr = x + (int64_t)(slot / K) * nv;
        float ga = 0.f, ua = 0.f;
#pragma unroll
        for (int c = 0; c < VPL; ++c) {
            const int v = c * 32 + lane;
            if (v < nv) {
                const uint4 xv = __ldg(xr + v);
                ga = dot8_bf16(r.g[c], xv, ga);
                ua = dot8_bf16(r.u[c], xv, ua);
            }
        }
        const float g = warp_sum(ga);
        const float u = warp_sum(ua);
        if (lane == 0) h[(int64_t)slot * F + f] = __float2bfloat16_rn(silu_f(g) * u);
    }
}

template <int VPL, bool EXTRA>
__global__ void __launch_bounds__(kUpWarps * 32, 1) decode_up_bf16(
    const uint4 *__restrict__ x, const uint4 *__restrict__ gate_up,
    const uint4 *__restrict__ gate_up2, const int32_t *__restrict__ idx, int T, int H, int F, int E,
    int K, int S_arg, __nv_bfloat16 *__restrict__ h) {
    __shared__ Touched tu;
    const int S = EXTRA ? S_arg : 0;   // EXTRA = false: the routed-only form
    // Launched as a programmatic dependent of whatever precedes it on the
    // stream: every input may come from that kernel.
    pdl_wait();
    build_touched(idx, T, K, S, E, tu);
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int nv = H / 8;
    const int64_t items = (int64_t)tu.n * F;
    const int64_t i0 = items * blockIdx.x / gridDim.x, i1 = items * (blockIdx.x + 1) / gridDim.x;
    UpRows<VPL> ra, rb;
    int64_t it = i0 + warp;
    const int K2 = K + S;
    if (it < i1) up_load<VPL, EXTRA>(ra, gate_up, gate_up2, E, tu, it, F, nv, lane);
    for (; it < i1; it += 2 * kUpWarps) {
        const int64_t nb = it + kUpWarps, na = it + 2 * kUpWarps;
        if (nb < i1) up_load<VPL, EXTRA>(rb, gate_up, gate_up2, E, tu, nb, F, nv, lane);
        up_compute(ra, x, tu, it, F, K2, nv, lane, h);
        if (na < i1) up_load<VPL, EXTRA>(ra, gate_up, gate_up2, E, tu, na, F, nv, lane);
        if (nb < i1) up_compute(rb, x, tu, nb, F, K2, nv, lane, h);
    }
}

// D2.  Block b owns hidden rows [j0, j1).  One item = (row j, touched expert
// u); a warp loads the down rows of two items before using either.  The
// per-slot results y_s land in shared memory; after a block barrier,
// out[t, j] = bf16( sum_{k in order} w[t,k] * y_{t*K+k} [+ residual[t, j]] )
// with weight 1 for the shared slots.  EXTRA = false compiles the routed-only
// form (S = 0, no residual), whose registers fit the two-blocks-per-SM bound.
template <int VPL, bool EXTRA>
__global__ void __launch_bounds__(kDownWarps * 32, VPL <= 4 ? 2 : 1) decode_down_bf16(
    const uint4 *__restrict__ down, const uint4 *__restrict__ down2, const uint4 *__restrict__ h,
    const int32_t *__restrict__ idx, const float *__restrict__ w, int T, int H, int F, int E, int K,
    int S_arg, const __nv_bfloat16 *__restrict__ residual, __nv_bfloat16 *__restrict__ out) {
    __shared__ Touched tu;
    __shared__ const uint4 *dbase[kDecodeMaxSlots];   // row j0 of each touched down projection
    extern __shared__ float ys[];     // [rows of this block][T*(K+S)]
    const int S = EXTRA ? S_arg : 0;
    build_touched(idx, T, K, S, E, tu);
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int nv = F / 8;
    const int K2 = K + S;
    const int TK = T * K2;
    const int j0 = (int)((int64_t)H * blockIdx.x / gridDim.x);
    const int j1 = (int)((int64_t)H * (blockIdx.x + 1) / gridDim.x);
    // Stream this block's down rows into L2 while D1 is still running.
    if (threadIdx.x < tu.n) {
        const int e = tu.expert[threadIdx.x];
        const uint4 *b = (!EXTRA || e < E ? down + (int64_t)e * H * nv
                                          : down2 + (int64_t)(e - E) * H * nv) +
                         (int64_t)j0 * nv;
        if (EXTRA) dbase[threadIdx.x] = b;
        if (j1 > j0) prefetch_l2_bulk(b, (uint32_t)((j1 - j0) * F * 2));
    }
    if (EXTRA) __syncthreads();
    pdl_wait();
    const int items = (j1 - j0) * tu.n;
    for (int i = 2 * warp; i < items; i += 2 * kDownWarps) {
        uint4 wd[2][VPL];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int it = i + p;
            const int jl = it / max(tu.n, 1), ui = it - jl * tu.n;
            const int ue = it < items ? ui : 0;
            const uint4 *drow = EXTRA ? dbase[ue] + (int64_t)jl * nv
                                      : down + ((int64_t)tu.expert[ue] * H + j0 + jl) * nv;
#pragma unroll
            for (int c = 0; c < VPL; ++c) {
                const int v = c * 32 + lane;
                wd[p][c] = (it < items && v < nv) ? __ldg(drow + v) : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int it = i + p;
            if (it >= items) break;
            const int jl = it / tu.n, ui = it - jl * tu.n;
            for (int g0 = tu.start[ui]; g0 < tu.start[ui + 1]; g0 += kSlotGroup) {
                const int ns = min(kSlotGroup, tu.start[ui + 1] - g0);
                float ya[kSlotGroup] = {};
#pragma unroll
                for (int si = 0; si < kSlotGroup; ++si) {
                    if (si < ns) {
                        const uint4 *hr = h + (int64_t)tu.slot[g0 + si] * nv;
#pragma unroll
                        for (int c = 0; c < VPL; ++c) {
                            const int v = c * 32 + lane;
                            if (v < nv) ya[si] = dot8_bf16(wd[p][c], __ldg(hr + v), ya[si]);
                        }
                    }
                }
#pragma unroll
                for (int si = 0; si < kSlotGroup; ++si) {
                    if (si < ns) {
                        const float y = warp_sum(ya[si]);
                        if (lane == 0) ys[jl * TK + tu.slot[g0 + si]] = y;
                    }
                }
            }
        }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < (j1 - j0) * T; q += blockDim.x) {
        const int jl = q / T, t = q - jl * T;
        float acc = 0.f;
        for (int k = 0; k < K2; ++k) {
            const int s = t * K2 + k;
            if (tu.e_of[s] < 0) continue;
            if (!EXTRA || k < K)
                acc = fmaf(w[t * K + k], ys[jl * TK + s], acc);
            else
                acc += ys[jl * TK + s];
        }
        if (EXTRA && residual != nullptr)
            acc += __bfloat162float(residual[(int64_t)t * H + j0 + jl]);
        out[(int64_t)t * H + j0 + jl] = __float2bfloat16_rn(acc);
    }
}

}  // namespace

cudaError_t launch_decode_bf16(const void *x, const void *gate_up, const void *down,
                               const int32_t *idx, const float *w, int T, int H, int F, int E,
                               int K, uint8_t *ws, const DecodeWorkspace &L, void *out,
                               cudaStream_t st, const SharedSet &sh, const void *residual) {
    __nv_bfloat16 *h = (__nv_bfloat16 *)(ws + L.h);
    const int S = sh.S;
    const uint4 *gu2 = (const uint4 *)(S > 0 ? sh.gate_up : gate_up);
    const uint4 *dn2 = (const uint4 *)(S > 0 ? sh.down : down);
    const int vpl_up = (H / 8 + 31) / 32, vpl_dn = (F / 8 + 31) / 32;
    int grid = num_sms();
    const dim3 blk(kUpWarps * 32);
    cudaError_t err;
    const bool extra = S > 0 || residual != nullptr;
#define MOE_UP(V)                                                                                 \
    launch_k(extra ? decode_up_bf16<V, true> : decode_up_bf16<V, false>, dim3(grid), blk, 0, st, \
             true, (const uint4 *)x, (const uint4 *)gate_up, gu2, idx, T, H, F, E, K, S, h)
    switch (vpl_up) {
        case 1: err = MOE_UP(1); break;
        case 2: err = MOE_UP(2); break;
        case 3: err = MOE_UP(3); break;
        case 4: err = MOE_UP(4); break;
        case 5: err = MOE_UP(5); break;
        case 6: err = MOE_UP(6); break;
        case 7: err = MOE_UP(7); break;
        case 8: err = MOE_UP(8); break;
        default: return cudaErrorInvalidValue;
    }
#undef MOE_UP
    if (err != cudaSuccess) return err;
    grid = (vpl_dn <= 4 ? 2 : 1) * num_sms();
    const size_t smem = sizeof(float) * ((H + grid - 1) / grid + 1) * T * (K + S);
#define MOE_DN(V)                                                                                \
    launch_k(extra ? decode_down_bf16<V, true> : decode_down_bf16<V, false>, dim3(grid),           \
             dim3(kDownWarps * 32), smem, st, true, (const uint4 *)down, dn2, (const uint4 *)h, idx, \
             w, T, H, F, E, K, S, (const __nv_bfloat16 *)residual, (__nv_bfloat16 *)out)
    switch (vpl_dn) {
        case 1: return MOE_DN(1);
        case 2: return MOE_DN(2);
        case 3: return MOE_DN(3);
        case 4: return MOE_DN(4);
        case 5: return MOE_DN(5);
        case 6: return MOE_DN(6);
        case 7: return MOE_DN(7);
        case 8: return MOE_DN(8);
        default: return cudaErrorInvalidValue;
    }
#undef MOE_DN
}

}  // namespace moe

namespace moe {

// The decode kernels keep every intermediate in registers and small shared
// arrays; the only shape limit is the per-lane vector count of one row.
bool decode_shape_ok(int H, int F) { return H / 8 <= 32 * 8 && F / 8 <= 32 * 8; }

}  // namespace moe
