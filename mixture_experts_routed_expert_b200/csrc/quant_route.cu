// quant_route.cu -- S2 (block-128 E4M3 activation quantisation) and S1
// (group-aware sigmoid top-k routing), the two side kernels of the FP8 layer
// ("Supporting MegaKernel for DeepSeek Models", layer table:
// bf16_to_fp8_quantize and moe_topk_sigmoid_routing_layer).
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

// One thread per 8 values; 16 threads per block of 128.
__global__ void __launch_bounds__(256) quantize_kernel(const uint4 *__restrict__ x, int64_t n_vec,
                                                       uint2 *__restrict__ xq,
                                                       float *__restrict__ scale) {
    const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool on = v < n_vec;
    float f[8];
    unpack_bf16x8(on ? __ldg(x + v) : make_uint4(0, 0, 0, 0), f);
    float sc;
    const uint2 q = quant8_e4m3(f, sc);   // every lane of the warp takes part
    if (on) {
        xq[v] = q;
        if ((threadIdx.x & 15) == 0) scale[v / 16] = sc;
    }
}

constexpr int kRouteWarps = 4;

// "a ranks before b": larger score first, lower index on equal scores.
__device__ __forceinline__ bool ranks_before(float sa, int ia, float sb, int ib) {
    return sa > sb || (sa == sb && ia < ib);
}

// One warp per token.  smem per warp: s[E] and c[E].
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(
    const float *__restrict__ logits, const float *__restrict__ bias, int64_t T, int E, int G,
    int topk_group, int top_k, float scale, int32_t *__restrict__ idx, float *__restrict__ wout) {
    extern __shared__ float rsm[];
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int64_t t = (int64_t)blockIdx.x * kRouteWarps + warp;
    if (t >= T) return;
    float *s = rsm + (size_t)warp * 2 * E;
    float *c = s + E;
    for (int e = lane; e < E; e += 32) {
        const double lg = (double)__ldg(logits + t * E + e);
        const float se = (float)(1.0 / (1.0 + exp(-lg)));
        s[e] = se;
        c[e] = se + __ldg(bias + e);
    }
    __syncwarp();
    // group scores: sum of the two best c in each group (lane g owns group g)
    const int gsize = E / G;
    float gs = -INFINITY;
    if (lane < G) {
        int b1 = -1, b2 = -1;
        for (int e = lane * gsize; e < (lane + 1) * gsize; ++e) {
            if (b1 < 0 || ranks_before(c[e], e, c[b1], b1)) { b2 = b1; b1 = e; }
            else if (b2 < 0 || ranks_before(c[e], e, c[b2], b2)) { b2 = e; }
        }
        gs = (b2 >= 0) ? c[b1] + c[b2] : c[b1];
    }
    // keep the topk_group best groups
    unsigned keep = 0;
    for (int r = 0; r < topk_group; ++r) {
        float bv = (lane < G && !((keep >> lane) & 1u)) ? gs : -INFINITY;
        int bi = (lane < G && !((keep >> lane) & 1u)) ? lane : 0x7FFFFFFF;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
            if (oi != 0x7FFFFFFF && (bi == 0x7FFFFFFF || ranks_before(ov, oi, bv, bi))) { bv = ov; bi = oi; }
        }
        keep |= 1u << bi;
    }
    // top_k experts among the kept groups
    unsigned taken = 0;  // bit i: expert lane + 32 i already chosen
    int chosen = -1;     // lane k keeps the k-th choice
    for (int k = 0; k < top_k; ++k) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
        for (int i = 0, e = lane; e < E; ++i, e += 32) {
            if (((keep >> (e / gsize)) & 1u) && !((taken >> i) & 1u) &&
                (bi == 0x7FFFFFFF || ranks_before(c[e], e, bv, bi))) {
                bv = c[e];
                bi = e;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
            if (oi != 0x7FFFFFFF && (bi == 0x7FFFFFFF || ranks_before(ov, oi, bv, bi))) { bv = ov; bi = oi; }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == k) chosen = bi;
    }
    // weights: unbiased scores normalised over the choices, in choice order
    const float sk = (lane < top_k) ? s[chosen] : 0.f;
    float sum = 0.f;
    for (int k = 0; k < top_k; ++k) sum += __shfl_sync(0xFFFFFFFFu, sk, k);
    if (lane < top_k) {
        const float q = sk / sum;
        idx[t * top_k + lane] = chosen;
        wout[t * top_k + lane] = q * scale;
    }
}

// Expert offsets of the routing result (optional output of the router):
// one block, integer shared-memory counters, exclusive scan over experts.
__global__ void __launch_bounds__(1024) route_offsets_kernel(const int32_t *__restrict__ idx,
                                                             int64_t n, int E,
                                                             int32_t *__restrict__ offsets) {
    __shared__ int cnt[1024];
    __shared__ int warp_sums[32];
    pdl_wait();
    for (int e = threadIdx.x; e < 1024; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
        const int e = idx[i];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    const int v = cnt[threadIdx.x];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int ws = warp_sums[lane];
        int wi = ws;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, wi, o);
            if (lane >= o) wi += y;
        }
        warp_sums[lane] = wi - ws;
    }
    __syncthreads();
    const int excl = warp_sums[warp] + incl - v;
    if ((int)threadIdx.x <= E) offsets[threadIdx.x] = excl;
    if (E == 1024 && threadIdx.x == 1023) offsets[1024] = excl + v;
}

}  // namespace

cudaError_t launch_quantize(const void *x, int64_t rows, int cols, void *xq, float *scale,
                            cudaStream_t st) {
    const int64_t n_vec = rows * cols / 8;
    return launch_k(quantize_kernel, dim3((unsigned)((n_vec + 255) / 256)), dim3(256), 0, st, false,
                    (const uint4 *)x, n_vec, (uint2 *)xq, scale);
}

cudaError_t launch_route(const float *logits, const float *bias, int64_t T, int E, int num_groups,
                         int topk_group, int top_k, float scale, int32_t *idx, float *w,
                         int32_t *offsets, cudaStream_t st) {
    const size_t smem = sizeof(float) * 2 * E * kRouteWarps;
    static int attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_done[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(sizeof(float) * 2 * 1024 * kRouteWarps));
        if (e != cudaSuccess) return e;
        attr_done[dev & 63] = 1;
    }
    cudaError_t err = launch_k(route_kernel, dim3((unsigned)((T + kRouteWarps - 1) / kRouteWarps)),
                               dim3(kRouteWarps * 32), smem, st, false, logits, bias, T, E,
                               num_groups, topk_group, top_k, scale, idx, w);
    if (err != cudaSuccess || offsets == nullptr) return err;
    return launch_k(route_offsets_kernel, dim3(1), dim3(1024), 0, st, true, (const int32_t *)idx,
                    T * top_k, E, offsets);
}

}  // namespace moe
