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

constexpr int kRouteThreads = 256;

// "a ranks before b": larger score first, lower index on equal scores.
__device__ __forceinline__ bool ranks_before(float sa, int ia, float sb, int ib) {
    return sa > sb || (sa == sb && ia < ib);
}

// Best two of a group held as (value, index) pairs: merge (b1, b2) into (a1, a2).
__device__ __forceinline__ void top2_merge(float &a1, int &i1, float &a2, int &j2, float b1, int k1,
                                           float b2, int k2) {
    if (k1 >= 0 && (i1 < 0 || ranks_before(b1, k1, a1, i1))) {
        // b1 is the new best; the second is the better of a1 and b1's partner
        if (i1 >= 0 && (k2 < 0 || ranks_before(a1, i1, b2, k2))) { a2 = a1; j2 = i1; }
        else { a2 = b2; j2 = k2; }
        a1 = b1; i1 = k1;
    } else if (k1 >= 0 && (j2 < 0 || ranks_before(b1, k1, a2, j2))) {
        a2 = b1; j2 = k1;
    }
}

// One block per token.  s[e] = sigmoid(logit) (double, rounded to fp32),
// c[e] = s[e] + bias[e] (selection score).  Groups are scored by the sum of
// their two best c, the topk_group best groups are kept, and the top_k
// experts of the kept groups are chosen; every selection uses the order
// (score desc, index asc), so each candidate's position is the number of
// candidates ranking before it.  Weights: s of the chosen experts divided by
// their sum (summed in choice order), times the scaling factor.
__global__ void __launch_bounds__(kRouteThreads) route_kernel(
    const float *__restrict__ logits, const float *__restrict__ bias, int64_t T, int E, int G,
    int topk_group, int top_k, float scale, int32_t *__restrict__ idx, float *__restrict__ wout) {
    extern __shared__ float rsm[];
    float *s = rsm;              // [E]
    float *c = s + E;            // [E]
    __shared__ float gsc[32];
    __shared__ unsigned keep_s;
    __shared__ float sel_s[16];
    __shared__ float sum_s;
    const int64_t t = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = lane_id();
    for (int e = tid; e < E; e += kRouteThreads) {
        const double lg = (double)__ldg(logits + t * E + e);
        const float se = (float)(1.0 / (1.0 + exp(-lg)));
        s[e] = se;
        c[e] = se + __ldg(bias + e);
    }
    __syncthreads();
    // group scores: one warp per group (lanes stride over the group)
    const int gsize = E / G;
    for (int g = warp; g < G; g += kRouteThreads / 32) {
        float a1 = 0.f, a2 = 0.f;
        int i1 = -1, j2 = -1;
        for (int e = g * gsize + lane; e < (g + 1) * gsize; e += 32) top2_merge(a1, i1, a2, j2, c[e], e, 0.f, -1);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float b1 = __shfl_xor_sync(0xFFFFFFFFu, a1, o), b2 = __shfl_xor_sync(0xFFFFFFFFu, a2, o);
            const int k1 = __shfl_xor_sync(0xFFFFFFFFu, i1, o), k2 = __shfl_xor_sync(0xFFFFFFFFu, j2, o);
            top2_merge(a1, i1, a2, j2, b1, k1, b2, k2);
        }
        if (lane == 0) gsc[g] = (j2 >= 0) ? c[i1] + c[j2] : c[i1];
    }
    __syncthreads();
    // kept groups: rank of each group score among all G
    if (warp == 0) {
        bool kept = false;
        if (lane < G) {
            const float v = gsc[lane];
            int r = 0;
            for (int g = 0; g < G; ++g) r += ranks_before(gsc[g], g, v, lane);
            kept = r < topk_group;
        }
        const unsigned m = __ballot_sync(0xFFFFFFFFu, kept);
        if (lane == 0) keep_s = m;
    }
    __syncthreads();
    const unsigned keep = keep_s;
    // chosen experts: rank of each kept candidate among the kept candidates
    for (int e = tid; e < E; e += kRouteThreads) {
        if (!((keep >> (e / gsize)) & 1u)) continue;
        const float v = c[e];
        int r = 0;
        for (int g = 0; g < G; ++g) {
            if (!((keep >> g) & 1u)) continue;
            for (int q = g * gsize; q < (g + 1) * gsize; ++q) r += ranks_before(c[q], q, v, e);
        }
        if (r < top_k) {
            idx[t * top_k + r] = e;
            sel_s[r] = s[e];
        }
    }
    __syncthreads();
    if (tid == 0) {
        float sum = 0.f;
        for (int k = 0; k < top_k; ++k) sum += sel_s[k];
        sum_s = sum;
    }
    __syncthreads();
    if (tid < top_k) {
        const float q = sel_s[tid] / sum_s;
        wout[t * top_k + tid] = q * scale;
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
    const size_t smem = sizeof(float) * 2 * E;            // <= 8 KB for E <= 1024
    cudaError_t err = launch_k(route_kernel, dim3((unsigned)T), dim3(kRouteThreads), smem, st, false,
                               logits, bias, T, E, num_groups, topk_group, top_k, scale, idx, w);
    if (err != cudaSuccess || offsets == nullptr) return err;
    return launch_k(route_offsets_kernel, dim3(1), dim3(1024), 0, st, true, (const int32_t *)idx,
                    T * top_k, E, offsets);
}

}  // namespace moe
