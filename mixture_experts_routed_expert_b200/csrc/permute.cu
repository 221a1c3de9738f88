// permute.cu -- S3 (expert histogram, prefix scan, stable permutation of the
// routing slots, gather of the routed activation rows) and S6 (fixed-order
// top-K combine) for the prefill path.
//
// The model card ("deepseek-ocr2-moe-experts", description) computes the
// routed experts as a grouped GEMM followed by a router-weight scale and a
// scatter-add; here the scatter-add becomes a gather (slots are grouped by
// expert before the GEMMs) and a deterministic per-token sum in k order.
//
// Slot s = t*K + k.  Slots of one expert are placed in ascending slot order,
// so every integer output is unique and bit-exact.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kHistWarps = 8;                       // 256 threads per histogram block
constexpr int kSlotsPerWarp = kChunk / kHistWarps;  // 256 consecutive slots per warp

// Block c handles slots [c*kChunk, (c+1)*kChunk).  Each warp walks its 256
// slots in order, 32 at a time; lanes routed to the same expert find each
// other with match.any and take consecutive ranks.  Output: per-block expert
// counts and, per slot, its rank among the block's earlier slots of the same
// expert.  smem: kHistWarps x E counters.
__global__ void __launch_bounds__(256) hist_kernel(const int32_t *__restrict__ idx, int64_t n_slots,
                                                   int E, int32_t *__restrict__ chunk_hist,
                                                   int32_t *__restrict__ slot_rank,
                                                   int32_t *__restrict__ status) {
    extern __shared__ int32_t wcnt[];  // [kHistWarps][E]
    const int warp = threadIdx.x >> 5, lane = lane_id();
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    for (int i = threadIdx.x; i < kHistWarps * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kChunk + (int64_t)warp * kSlotsPerWarp;
    int local[kSlotsPerWarp / 32];
    int ex[kSlotsPerWarp / 32];
    const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int r = 0; r < kSlotsPerWarp / 32; ++r) {
        const int64_t s = base + r * 32 + lane;
        int e = (s < n_slots) ? __ldg(idx + s) : -1;
        const bool valid = (e >= 0 && e < E);
        if (!valid) e = -1;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
        const int rank = __popc(peers & lt_mask);
        const int prior = valid ? wcnt[warp * E + e] : 0;
        __syncwarp();
        if (valid && rank == 0) wcnt[warp * E + e] = prior + __popc(peers);
        __syncwarp();
        local[r] = prior + rank;
        ex[r] = e;
    }
    __syncthreads();
    // exclusive scan over the warps of each expert; block totals to global
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kHistWarps; ++w) {
            const int v = wcnt[w * E + e];
            wcnt[w * E + e] = run;
            run += v;
        }
        chunk_hist[(int64_t)blockIdx.x * E + e] = run;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kSlotsPerWarp / 32; ++r) {
        const int64_t s = base + r * 32 + lane;
        if (ex[r] >= 0) slot_rank[s] = wcnt[warp * E + ex[r]] + local[r];
    }
    pdl_launch_dependents();
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024);
// `total` receives the sum over the block.
__device__ int block_exclusive_scan(int v, int &total) {
    __shared__ int warp_sums[32];
    __shared__ int block_total;
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int ws = warp_sums[lane];
        int wincl = ws;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xFFFFFFFFu, wincl, o);
            if (lane >= o) wincl += n;
        }
        warp_sums[lane] = wincl - ws;
        if (lane == 31) block_total = wincl;
    }
    __syncthreads();
    const int r = warp_sums[warp] + incl - v;
    total = block_total;
    __syncthreads();
    return r;
}

// One block of 1024 threads, one expert per thread (E <= 1024):
// per-chunk counts -> per-chunk exclusive bases (in place), expert counts,
// expert offsets, and prefix sums of row tiles for both grouped GEMMs.
__global__ void __launch_bounds__(1024) scan_kernel(int32_t *__restrict__ chunk_hist, int n_chunks,
                                                    int E, int32_t *__restrict__ counts,
                                                    int32_t *__restrict__ offsets,
                                                    int32_t *__restrict__ tiles_g,
                                                    int32_t *__restrict__ tiles_d, int bn_g,
                                                    int bn_d) {
    int total = 0;
    pdl_wait();
    const int e = threadIdx.x;
    int run = 0;
    if (e < E) {
        for (int c = 0; c < n_chunks; ++c) {
            const int v = chunk_hist[(int64_t)c * E + e];
            chunk_hist[(int64_t)c * E + e] = run;
            run += v;
        }
        counts[e] = run;
    }
    const int n = (e < E) ? run : 0;
    const int off = block_exclusive_scan(n, total);
    if (e < E) offsets[e] = off;
    if (e == 0) offsets[E] = total;
    const int tg = (n + bn_g - 1) / bn_g;
    const int tgo = block_exclusive_scan(tg, total);
    if (e < E) tiles_g[e] = tgo;
    if (e == 0) tiles_g[E] = total;
    const int td = (n + bn_d - 1) / bn_d;
    const int tdo = block_exclusive_scan(td, total);
    if (e < E) tiles_d[e] = tdo;
    if (e == 0) tiles_d[E] = total;
    pdl_launch_dependents();
}

// Whole permutation in one block of 1024 threads, for up to
// kSmallSlots slots: warp w takes slots [w*R, (w+1)*R), R = 32*rounds, and
// ranks them as hist_kernel does; then per-expert bases over the warps,
// expert counts / offsets / tile prefixes, and the final positions.
// smem: 32 x E counters + E+1 offsets.
constexpr int kSmallRounds = 16;
constexpr int kSmallSlots = 1024 * kSmallRounds;

__global__ void __launch_bounds__(1024) permute_small_kernel(
    const int32_t *__restrict__ idx, int n_slots, int E, int32_t *__restrict__ counts,
    int32_t *__restrict__ offsets, int32_t *__restrict__ tiles_g, int32_t *__restrict__ tiles_d,
    int32_t *__restrict__ perm, int32_t *__restrict__ inv, int32_t *__restrict__ status, int bn_g,
    int bn_d) {
    extern __shared__ int32_t sm[];
    int32_t *wcnt = sm;                 // [32][E]
    int32_t *s_off = sm + 32 * E;       // [E+1]
    const int warp = threadIdx.x >> 5, lane = lane_id();
    if (threadIdx.x == 0) *status = 0;
    for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) wcnt[i] = 0;
    const int rounds = (n_slots + 1023) / 1024;
    const int base = warp * rounds * 32;
    int loc[kSmallRounds], ex[kSmallRounds];
#pragma unroll
    for (int r = 0; r < kSmallRounds; ++r) {
        ex[r] = -1;
        const int s = base + r * 32 + lane;
        if (r < rounds && s < n_slots) {
            const int e = __ldg(idx + s);
            if (e >= 0 && e < E) ex[r] = e;
        }
    }
    __syncthreads();
    const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int r = 0; r < kSmallRounds; ++r) {
        if (r < rounds) {
            const int e = ex[r];
            const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
            const int rank = __popc(peers & lt_mask);
            const int prior = (e >= 0) ? wcnt[warp * E + e] : 0;
            __syncwarp();
            if (e >= 0 && rank == 0) wcnt[warp * E + e] = prior + __popc(peers);
            __syncwarp();
            loc[r] = prior + rank;
        }
    }
    __syncthreads();
    int n = 0;
    const int e = threadIdx.x;
    if (e < E) {
        for (int w = 0; w < 32; ++w) {
            const int v = wcnt[w * E + e];
            wcnt[w * E + e] = n;
            n += v;
        }
        counts[e] = n;
    }
    int total = 0;
    const int off = block_exclusive_scan(n, total);
    if (e < E) { offsets[e] = off; s_off[e] = off; }
    if (e == 0) { offsets[E] = total; s_off[E] = total; }
    const int tgo = block_exclusive_scan((n + bn_g - 1) / bn_g, total);
    if (e < E) tiles_g[e] = tgo;
    if (e == 0) tiles_g[E] = total;
    const int tdo = block_exclusive_scan((n + bn_d - 1) / bn_d, total);
    if (e < E) tiles_d[e] = tdo;
    if (e == 0) tiles_d[E] = total;
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kSmallRounds; ++r) {
        const int s = base + r * 32 + lane;
        if (r < rounds && s < n_slots) {
            if (ex[r] >= 0) {
                const int pos = s_off[ex[r]] + wcnt[warp * E + ex[r]] + loc[r];
                perm[pos] = s;
                inv[s] = pos;
            } else {
                inv[s] = -1;
            }
        }
    }
    for (int p = s_off[E] + threadIdx.x; p < n_slots; p += blockDim.x) perm[p] = -1;
    pdl_launch_dependents();
}

// Final slot positions.  One thread per slot; also fills perm entries past
// offsets[E] (slots whose expert id is out of range) with -1.
__global__ void __launch_bounds__(256) scatter_kernel(
    const int32_t *__restrict__ idx, int64_t n_slots, int E, const int32_t *__restrict__ chunk_hist,
    const int32_t *__restrict__ slot_rank, const int32_t *__restrict__ offsets,
    int32_t *__restrict__ perm, int32_t *__restrict__ inv) {
    pdl_wait();
    const int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= n_slots) return;
    const int e = __ldg(idx + s);
    if (e >= 0 && e < E) {
        const int pos = offsets[e] + chunk_hist[(s / kChunk) * E + e] + slot_rank[s];
        perm[pos] = (int32_t)s;
        inv[s] = pos;
    } else {
        inv[s] = -1;
    }
    if (s >= offsets[E]) perm[s] = -1;
    pdl_launch_dependents();
}

// Gather of routed activation rows into expert order: xperm[inv[s]] = x[s/K].
// One warp per slot, 16-byte vectors.
__global__ void __launch_bounds__(256) gather_bf16_kernel(const uint4 *__restrict__ x,
                                                          const int32_t *__restrict__ inv,
                                                          int64_t n_slots, int K, int H,
                                                          uint4 *__restrict__ xperm) {
    pdl_wait();
    const int64_t s = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (s >= n_slots) return;
    const int pos = inv[s];
    if (pos < 0) return;
    const int nv = H / 8;
    const uint4 *src = x + (s / K) * nv;
    uint4 *dst = xperm + (int64_t)pos * nv;
    for (int v = lane_id(); v < nv; v += 32) dst[v] = __ldg(src + v);
    pdl_launch_dependents();
}

// Gather + block-128 E4M3 quantisation of the routed activation rows
// (the rule of quantize_fp8_block128).  One warp per slot; 16 lanes cover a
// block of 128 values (8 per lane).
__global__ void __launch_bounds__(256) gather_fp8_kernel(const uint4 *__restrict__ x,
                                                         const int32_t *__restrict__ inv,
                                                         int64_t n_slots, int K, int H,
                                                         uint2 *__restrict__ xq,
                                                         float *__restrict__ xs) {
    pdl_wait();
    const int64_t s = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (s >= n_slots) return;
    const int pos = inv[s];
    if (pos < 0) return;
    const int lane = lane_id();
    const int nv = H / 8;
    const uint4 *src = x + (s / K) * nv;
    for (int v0 = 0; v0 < nv; v0 += 32) {
        const int v = v0 + lane;
        const bool on = v < nv;
        float f[8];
        unpack_bf16x8(on ? __ldg(src + v) : make_uint4(0, 0, 0, 0), f);
        float sc;
        const uint2 q = quant8_e4m3(f, sc);
        if (on) {
            xq[(int64_t)pos * nv + v] = q;
            if ((lane & 15) == 0) xs[(int64_t)pos * (H / 128) + v / 16] = sc;
        }
    }
    pdl_launch_dependents();
}

// S6: out[t, j] = bf16( sum_{k in order} y[t*K + k, j] ) over slots with a
// valid expert id (y already holds w[t,k] * down_e(h)).  4 columns per thread.
__global__ void __launch_bounds__(256) combine_kernel(const float4 *__restrict__ y,
                                                      const int32_t *__restrict__ idx, int64_t T,
                                                      int H, int E, int K, uint2 *__restrict__ out) {
    pdl_wait();
    const int nv = H / 4;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * nv) return;
    const int64_t t = i / nv;
    const int v = (int)(i - t * nv);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < K; ++k) {
        const int e = __ldg(idx + t * K + k);
        if (e < 0 || e >= E) continue;
        const float4 a = __ldcs(y + (t * K + k) * nv + v);
        acc.x += a.x; acc.y += a.y; acc.z += a.z; acc.w += a.w;
    }
    uint2 o;
    o.x = pack_bf16x2(acc.x, acc.y);
    o.y = pack_bf16x2(acc.z, acc.w);
    out[t * nv + v] = o;
}

}  // namespace

cudaError_t launch_permute(const int32_t *idx, int64_t n_slots, int E, int bn_g, int bn_d,
                           uint8_t *ws, const Workspace &L, cudaStream_t st) {
    if (n_slots <= kSmallSlots) {
        const size_t smem = sizeof(int32_t) * (33 * (size_t)E + 1);
        static int attr_done[64] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        if (!attr_done[dev & 63]) {
            cudaError_t e = cudaFuncSetAttribute(permute_small_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)(sizeof(int32_t) * (33 * 1024 + 1)));
            if (e != cudaSuccess) return e;
            attr_done[dev & 63] = 1;
        }
        return launch_k(permute_small_kernel, dim3(1), dim3(1024), smem, st, false, idx,
                        (int)n_slots, E, (int32_t *)(ws + L.counts), (int32_t *)(ws + L.offsets),
                        (int32_t *)(ws + L.tiles_g), (int32_t *)(ws + L.tiles_d),
                        (int32_t *)(ws + L.perm), (int32_t *)(ws + L.inv),
                        (int32_t *)(ws + L.status), bn_g, bn_d);
    }
    const int n_chunks = (int)((n_slots + kChunk - 1) / kChunk);
    int32_t *status = (int32_t *)(ws + L.status);
    int32_t *chunk_hist = (int32_t *)(ws + L.chunk_hist);
    int32_t *slot_rank = (int32_t *)(ws + L.slot_rank);
    const size_t hsmem = sizeof(int32_t) * kHistWarps * E;
    cudaError_t err = launch_k(hist_kernel, dim3(n_chunks), dim3(256), hsmem, st, false, idx,
                               n_slots, E, chunk_hist, slot_rank, status);
    if (err != cudaSuccess) return err;
    err = launch_k(scan_kernel, dim3(1), dim3(1024), 0, st, true, chunk_hist, n_chunks, E,
                   (int32_t *)(ws + L.counts), (int32_t *)(ws + L.offsets),
                   (int32_t *)(ws + L.tiles_g), (int32_t *)(ws + L.tiles_d), bn_g, bn_d);
    if (err != cudaSuccess) return err;
    return launch_k(scatter_kernel, dim3((unsigned)((n_slots + 255) / 256)), dim3(256), 0, st, true,
                    idx, n_slots, E, (const int32_t *)chunk_hist, (const int32_t *)slot_rank,
                    (const int32_t *)(ws + L.offsets), (int32_t *)(ws + L.perm),
                    (int32_t *)(ws + L.inv));
}

cudaError_t launch_gather(const void *x, const int32_t *idx, int64_t n_slots, int K, int H, int E,
                          moe_wtype_t wt, uint8_t *ws, const Workspace &L, cudaStream_t st) {
    (void)idx;
    (void)E;
    const dim3 grid((unsigned)((n_slots + 7) / 8));
    if (wt == MOE_W_BF16)
        return launch_k(gather_bf16_kernel, grid, dim3(256), 0, st, true, (const uint4 *)x,
                        (const int32_t *)(ws + L.inv), n_slots, K, H, (uint4 *)(ws + L.xperm));
    return launch_k(gather_fp8_kernel, grid, dim3(256), 0, st, true, (const uint4 *)x,
                    (const int32_t *)(ws + L.inv), n_slots, K, H, (uint2 *)(ws + L.xperm),
                    (float *)(ws + L.xscale));
}

cudaError_t launch_debug_outputs(const int32_t *idx, int64_t n_slots, int E, const uint8_t *ws,
                                 const Workspace &L, int32_t *counts, int32_t *offsets,
                                 int32_t *perm, int32_t *inv, cudaStream_t st) {
    (void)idx;
    cudaError_t err;
    if ((err = cudaMemcpyAsync(counts, ws + L.counts, sizeof(int32_t) * E, cudaMemcpyDeviceToDevice, st)))
        return err;
    if ((err = cudaMemcpyAsync(offsets, ws + L.offsets, sizeof(int32_t) * (E + 1),
                               cudaMemcpyDeviceToDevice, st)))
        return err;
    if (n_slots == 0) return cudaSuccess;
    if ((err = cudaMemcpyAsync(perm, ws + L.perm, sizeof(int32_t) * n_slots, cudaMemcpyDeviceToDevice, st)))
        return err;
    return cudaMemcpyAsync(inv, ws + L.inv, sizeof(int32_t) * n_slots, cudaMemcpyDeviceToDevice, st);
}

cudaError_t launch_combine(const int32_t *idx, int64_t T, int H, int E, int K, const uint8_t *ws,
                           const Workspace &L, void *out, cudaStream_t st) {
    const int64_t n = T * (H / 4);
    return launch_k(combine_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true,
                    (const float4 *)(ws + L.y), idx, T, H, E, K, (uint2 *)out);
}

}  // namespace moe
