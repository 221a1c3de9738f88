// permute.cu -- S3 (expert histogram, offsets, stable permutation of the
// routing slots and gather of the routed activation rows, E4M3-quantised on
// the way for the FP8 path) and S6 (fixed-order top-K combine) of the prefill
// path.
//
// The model card ("deepseek-ocr2-moe-experts", description) computes the
// routed experts as a grouped GEMM followed by a router-weight scale and a
// scatter-add; here the scatter-add becomes a gather (slots are grouped by
// expert before the GEMMs) and a deterministic per-token sum in k order.
//
// Slot s = t*K + k.  Slots of one expert are placed in ascending slot order,
// so every integer output is unique and bit-exact.
//
// One kernel does S3 without any inter-block communication: every block
// recounts the whole routing (T*K int32, read from L2) to get the expert
// offsets and the number of earlier slots of each expert before its own chunk,
// ranks its chunk's slots stably, writes perm / inv and gathers its rows.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kPThreads = 256;
constexpr int kPWarps = kPThreads / 32;

// Exclusive scan of n ints in place (n <= 4096) by one block of kPThreads
// threads; returns the total.  Each thread scans a contiguous run.
__device__ int block_scan_inplace(int32_t *v, int n) {
    __shared__ int warp_tot[kPWarps];
    __shared__ int grand;
    const int t = threadIdx.x, lane = lane_id(), warp = t >> 5;
    const int per = (n + kPThreads - 1) / kPThreads;
    const int b = min(n, t * per), e = min(n, b + per);
    int local = 0;
    for (int i = b; i < e; ++i) local += v[i];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (t == 0) {
        int run = 0;
        for (int w = 0; w < kPWarps; ++w) {
            const int x = warp_tot[w];
            warp_tot[w] = run;
            run += x;
        }
        grand = run;
    }
    __syncthreads();
    int run = warp_tot[warp] + incl - local;
    for (int i = b; i < e; ++i) {
        const int x = v[i];
        v[i] = run;
        run += x;
    }
    const int total = grand;
    __syncthreads();
    return total;
}

// MODE 0: permutation only; 1: + bf16 row gather; 2: + gather with block-128
// E4M3 quantisation (the rule of quantize_fp8_block128), fp32 scales [N][H/128];
// 3: as 2, scales stored as E8M0 bytes in rows of round16(H/128) bytes.
// Block (b, c) handles slots [b*chunk, (b+1)*chunk), chunk <= kPThreads, and
// gathers column slice c of their rows (gridDim.y slices of whole 128-column
// blocks, so that a few slots still spread over many blocks); only blocks
// with c = 0 write the permutation.
// Dynamic shared memory: cnt_all[E+1], cnt_before[E], wc[kPWarps][E], tiles[E+1].
template <int MODE>
__global__ void __launch_bounds__(kPThreads) permute_gather_kernel(
    const int32_t *__restrict__ idx, int n_slots, int E, int K, int H, int chunk, int bn_g,
    int bn_d, const uint4 *__restrict__ x, void *__restrict__ xperm, float *__restrict__ xscale,
    int32_t *__restrict__ counts, int32_t *__restrict__ offsets, int32_t *__restrict__ tiles_g,
    int32_t *__restrict__ tiles_d, int32_t *__restrict__ perm, int32_t *__restrict__ inv,
    int32_t *__restrict__ status, int32_t *__restrict__ zero, int nzero,
    uint8_t *__restrict__ xsb) {
    extern __shared__ int32_t psm[];
    int32_t *cnt_all = psm;                 // [E+1] -> exclusive offsets
    int32_t *cnt_bef = cnt_all + (E + 1);   // [E] slots of e before this chunk
    int32_t *wc = cnt_bef + E;              // [kPWarps][E] per-warp counts in the chunk
    int32_t *tl = wc + kPWarps * E;         // [E+1] tile counts (block 0)
    __shared__ int32_t pos_s[kPThreads];
    const int t = threadIdx.x, lane = lane_id(), warp = t >> 5;
    const int c0 = blockIdx.x * chunk;
    for (int i = t; i < (2 + kPWarps) * E + 1; i += kPThreads) psm[i] = 0;
    __syncthreads();
    // 1. global counts and counts before this chunk (integer smem atomics);
    //    16-byte index loads, eight in flight per thread
    const int n4 = (reinterpret_cast<uintptr_t>(idx) & 15) == 0 ? n_slots / 4 : 0;
    const int4 *idx4 = reinterpret_cast<const int4 *>(idx);
    for (int q0 = 0; q0 < n4; q0 += 8 * kPThreads) {
        int4 ev[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * kPThreads + t;
            ev[u] = q < n4 ? __ldg(idx4 + q) : make_int4(-1, -1, -1, -1);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int s4 = 4 * (q0 + u * kPThreads + t);
            const int ee[4] = {ev[u].x, ev[u].y, ev[u].z, ev[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (ee[j] >= 0 && ee[j] < E) {
                    atomicAdd(&cnt_all[ee[j]], 1);
                    if (s4 + j < c0) atomicAdd(&cnt_bef[ee[j]], 1);
                }
            }
        }
    }
    for (int s = 4 * n4 + t; s < n_slots; s += kPThreads) {   // tail (n_slots % 4)
        const int e = __ldg(idx + s);
        if (e >= 0 && e < E) {
            atomicAdd(&cnt_all[e], 1);
            if (s < c0) atomicAdd(&cnt_bef[e], 1);
        }
    }
    __syncthreads();
    const bool lead = blockIdx.x == 0 && blockIdx.y == 0;   // writes counts, offsets, tiles
    if (lead)
        for (int i = t; i < E; i += kPThreads) {
            counts[i] = cnt_all[i];
            tl[i] = cnt_all[i];
        }
    const int total = block_scan_inplace(cnt_all, E);   // cnt_all -> offsets
    // 2. stable rank of each slot of the chunk among the chunk's slots of its expert
    const int s = c0 + t;
    const bool mine = t < chunk && s < n_slots;
    int e = mine ? __ldg(idx + s) : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rank_w == 0) wc[warp * E + e] = __popc(peers);
    __syncthreads();
    int pos = -1;
    if (e >= 0) {
        int r = rank_w;
        for (int w = 0; w < warp; ++w) r += wc[w * E + e];
        pos = cnt_all[e] + cnt_bef[e] + r;
        if (blockIdx.y == 0) perm[pos] = s;
    }
    if (mine && blockIdx.y == 0) inv[s] = pos;
    pos_s[t] = mine ? pos : -1;
    if (lead) {
        if (t == 0) {
            *status = 0;
            offsets[E] = total;
        }
        for (int i = t; i < nzero; i += kPThreads) zero[i] = 0;   // consumers' work counters
        for (int i = t; i < E; i += kPThreads) offsets[i] = cnt_all[i];
        for (int p = total + t; p < n_slots; p += kPThreads) perm[p] = -1;
        // row-tile prefixes for both GEMMs
        __syncthreads();
        for (int i = t; i < E; i += kPThreads) tl[i] = (tl[i] + bn_g - 1) / bn_g;
        __syncthreads();
        const int tg = block_scan_inplace(tl, E);
        for (int i = t; i < E; i += kPThreads) tiles_g[i] = tl[i];
        if (t == 0) tiles_g[E] = tg;
        __syncthreads();
        for (int i = t; i < E; i += kPThreads) tl[i] = (counts[i] + bn_d - 1) / bn_d;
        __syncthreads();
        const int td = block_scan_inplace(tl, E);
        for (int i = t; i < E; i += kPThreads) tiles_d[i] = tl[i];
        if (t == 0) tiles_d[E] = td;
    }
    __syncthreads();
    if (MODE == 0) return;
    // 3. gather the chunk's rows (this block's column slice): one warp per
    //    row, 16-byte vectors
    const int nv = H / 8;
    const int nb16 = (nv + 15) / 16;                       // 128-column blocks
    const int vs0 = 16 * (int)((int64_t)nb16 * blockIdx.y / gridDim.y);
    const int vs1 = min(nv, 16 * (int)((int64_t)nb16 * (blockIdx.y + 1) / gridDim.y));
    for (int r = warp; r < chunk; r += kPWarps) {
        const int p = pos_s[r];
        if (p < 0) continue;
        const uint4 *src = x + (size_t)((c0 + r) / K) * nv;
        if (MODE == 1) {
            uint4 *dst = reinterpret_cast<uint4 *>(xperm) + (size_t)p * nv;
            for (int v = vs0 + lane; v < vs1; v += 32) dst[v] = __ldg(src + v);
        } else {
            uint2 *dst = reinterpret_cast<uint2 *>(xperm) + (size_t)p * nv;
            for (int v0 = vs0; v0 < vs1; v0 += 32) {
                const int v = v0 + lane;
                const bool on = v < vs1;
                float f[8];
                unpack_bf16x8(on ? __ldg(src + v) : make_uint4(0, 0, 0, 0), f);
                float sc;
                const uint2 q = quant8_e4m3(f, sc);   // every lane takes part
                if (on) {
                    dst[v] = q;
                    if ((lane & 15) == 0) {
                        if (MODE == 2) {
                            xscale[(size_t)p * (H / 128) + v / 16] = sc;
                            // the scale's E8M0 byte (its exponent field) in rows of
                            // round16(H/128) bytes, for the block-scaled MMA
                            if (xsb != nullptr)
                                xsb[(size_t)p * ((H / 128 + 15) & ~15) + v / 16] =
                                    (uint8_t)((__float_as_uint(sc) >> 23) & 0xFF);
                        } else {   // E8M0 byte of the power-of-two scale, rows of KBp bytes
                            const int kbp = (H / 128 + 15) & ~15;
                            reinterpret_cast<uint8_t *>(xscale)[(size_t)p * kbp + v / 16] =
                                (uint8_t)((__float_as_uint(sc) >> 23) & 0xFF);
                        }
                    }
                }
            }
        }
    }
}

// Shared experts as extra slots: row t of the widened routing holds the K
// routed ids (ids outside [0, E) become -1 so they can never name a shared
// expert) followed by the S shared ids E..E+S-1 with weight 1.
__global__ void __launch_bounds__(256) widen_routing_kernel(const int32_t *__restrict__ idx,
                                                            const float *__restrict__ w, int64_t T,
                                                            int E, int K, int S,
                                                            int32_t *__restrict__ idx2,
                                                            float *__restrict__ w2) {
    pdl_wait();
    const int K2 = K + S;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * K2) return;
    const int64_t t = i / K2;
    const int k = (int)(i - t * K2);
    if (k < K) {
        const int e = idx[t * K + k];
        idx2[i] = e >= 0 && e < E ? e : -1;
        w2[i] = w[t * K + k];
    } else {
        idx2[i] = E + (k - K);
        w2[i] = 1.0f;
    }
    pdl_launch_dependents();
}

// S6: out[t, j] = bf16( sum_{k in order} y[t*K + k, j] [+ residual[t, j]] )
// over slots with a valid expert id (y already holds w[t,k] * down_e(h)); the
// residual, when given, is added after the slot sum.  4 columns per thread.
__global__ void __launch_bounds__(256) combine_kernel(const float4 *__restrict__ y,
                                                      const int32_t *__restrict__ idx, int64_t T,
                                                      int H, int E, int K,
                                                      const uint2 *__restrict__ residual,
                                                      uint2 *__restrict__ out) {
    pdl_wait();
    const int nv = H / 4;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * nv) return;
    const int64_t t = i / nv;
    const int v = (int)(i - t * nv);
    // ids first (one mask), then the row loads four at a time, summed in k order
    unsigned valid = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        if (k < K) {
            const int e = __ldg(idx + t * K + k);
            if (e >= 0 && e < E) valid |= 1u << k;
        }
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < K; k0 += 4) {       // four row loads in flight, then their sum
        float4 a[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            a[i] = (valid >> (k0 + i)) & 1u ? __ldcs(y + (t * K + k0 + i) * nv + v)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if ((valid >> (k0 + i)) & 1u) {
                acc.x += a[i].x; acc.y += a[i].y; acc.z += a[i].z; acc.w += a[i].w;
            }
        }
    }
    if (residual != nullptr) {
        const uint2 r = __ldg(residual + t * nv + v);
        acc.x += bf16_lo(r.x); acc.y += bf16_hi(r.x); acc.z += bf16_lo(r.y); acc.w += bf16_hi(r.y);
    }
    uint2 o;
    o.x = pack_bf16x2(acc.x, acc.y);
    o.y = pack_bf16x2(acc.z, acc.w);
    out[t * nv + v] = o;
}

template <int MODE>
cudaError_t launch_pg(const void *x, const int32_t *idx, int64_t n_slots, int K, int H, int E,
                      int bn_g, int bn_d, uint8_t *ws, const Workspace &L, cudaStream_t st,
                      int32_t *zero = nullptr, int nzero = 0) {
    const size_t smem = sizeof(int32_t) * ((3 + kPWarps) * (size_t)E + 2);
    static std::atomic<int> attr_done[64];
    const cudaError_t e = enable_max_dyn_smem((const void *)permute_gather_kernel<MODE>, attr_done);
    if (e != cudaSuccess) return e;
    // about two blocks per SM for the gather; at least 128 slots per block
    // once the redundant recount of all slots becomes the larger cost
    int chunk = kPThreads;
    const int64_t floor_chunk = n_slots > 32768 ? 128 : 8;
    while (chunk > floor_chunk && n_slots / chunk < 2 * num_sms()) chunk /= 2;
    const unsigned blocks = (unsigned)((n_slots + chunk - 1) / chunk);
    // column slices: enough blocks for about two per SM when there are few slots
    const int nb16 = (H / 8 + 15) / 16;
    const unsigned slices = MODE == 0 ? 1u
                                      : (unsigned)std::max<int64_t>(
                                            1, std::min<int64_t>(nb16, (2 * num_sms() + blocks - 1) / blocks));
    return launch_k(permute_gather_kernel<MODE>, dim3(blocks, slices), dim3(kPThreads), smem, st, false,
                    idx, (int)n_slots, E, K, H, chunk, bn_g, bn_d, (const uint4 *)x,
                    (void *)(ws + L.xperm), (float *)(ws + L.xscale), (int32_t *)(ws + L.counts),
                    (int32_t *)(ws + L.offsets), (int32_t *)(ws + L.tiles_g),
                    (int32_t *)(ws + L.tiles_d), (int32_t *)(ws + L.perm), (int32_t *)(ws + L.inv),
                    (int32_t *)(ws + L.status), zero, nzero,
                    MODE == 2 ? (uint8_t *)(ws + L.xsb) : (uint8_t *)nullptr);   // E4M3 layouts hold xsb
}

}  // namespace

cudaError_t launch_permute(const int32_t *idx, int64_t n_slots, int E, int bn_g, int bn_d,
                           uint8_t *ws, const Workspace &L, cudaStream_t st) {
    return launch_pg<0>(nullptr, idx, n_slots, 1, 128, E, bn_g, bn_d, ws, L, st);
}

cudaError_t launch_permute_gather(const void *x, const int32_t *idx, int64_t n_slots, int K, int H,
                                  int E, int bn_g, int bn_d, moe_wtype_t wt, uint8_t *ws,
                                  const Workspace &L, cudaStream_t st, int32_t *zero, int nzero) {
    if (wt == MOE_W_BF16) return launch_pg<1>(x, idx, n_slots, K, H, E, bn_g, bn_d, ws, L, st);
    if (wt == MOE_W_MXFP4)
        return launch_pg<3>(x, idx, n_slots, K, H, E, bn_g, bn_d, ws, L, st, zero, nzero);
    return launch_pg<2>(x, idx, n_slots, K, H, E, bn_g, bn_d, ws, L, st);
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
                           const Workspace &L, void *out, cudaStream_t st, const void *residual) {
    const int64_t n = T * (H / 4);
    return launch_k(combine_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true,
                    (const float4 *)(ws + L.y), idx, T, H, E, K, (const uint2 *)residual,
                    (uint2 *)out);
}

cudaError_t launch_combine_rows(const float *y, const int32_t *idx, int64_t T, int H, int E, int K,
                                void *out, cudaStream_t st) {
    const int64_t n = T * (H / 4);
    return launch_k(combine_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true,
                    (const float4 *)y, idx, T, H, E, K, (const uint2 *)nullptr, (uint2 *)out);
}

cudaError_t launch_widen_routing(const int32_t *idx, const float *w, int64_t T, int E, int K,
                                 int S, int32_t *idx2, float *w2, cudaStream_t st) {
    const int64_t n = T * (K + S);
    return launch_k(widen_routing_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true,
                    idx, w, T, E, K, S, idx2, w2);
}

}  // namespace moe
