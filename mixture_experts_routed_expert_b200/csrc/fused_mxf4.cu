// fused_mxf4.cu -- the MXFP4 routed-experts forward of a decode-sized call
// (T <= 16 tokens, T*K <= 64 slots): gate_up (+SiLU, h quantisation), down
// (+router weight) and the top-K combine as ONE persistent kernel, after the
// permutation kernel (which gathers and quantises x); no kernel boundary
// between the GEMMs and the combine, no host synchronisation (DeepGEMM Mega
// MoE news page: the MoE steps fused into a single kernel so that the
// intermediate round trips disappear; there with FP8 x FP4, as here).
//
//   - Every CTA derives the expert-sorted slot order of the permutation kernel
//     (experts ascending, slots ascending) from top_k_index in shared memory
//     (at most 64 slots).
//   - Work units: all gate_up tiles (touched expert, 16-row tile, 128
//     features), then all down tiles (touched expert, 16-row tile, 128 hidden
//     rows); CTA b takes units b, b + grid, ...  gate_up tiles never wait, so
//     a down tile's wait always ends.
//   - gate_up's activations are the permutation kernel's E4M3 rows (TMA)
//     with their E8M0 scale bytes expanded into the block layout.
//   - A gate_up tile publishes its h rows (E4M3 + E8M0 scale bytes) to global
//     memory and then counts itself done for its (expert, row tile); the down
//     tiles of that row tile load h only after all F/128 of them have (bounded
//     wait).  The weights of a down tile stream from the start.
//   - A down tile writes its rows y = w * down(h) (fp32, by slot) and counts
//     itself done for each of its tokens' (token, 128-row block); the CTA
//     that completes a block sums its token's K rows in k order and writes
//     out: fixed order, no floating-point atomics.
// The arithmetic per tile is the one of the grouped MXFP4 GEMMs
// (tcgen05.mma.kind::mxf8f6f4.block_scale, two producer and two MMA warps,
// eight epilogue warps).  Every wait is bounded; on expiry the kernel sets
// the status word and returns.
#include "common.cuh"
#include "gemm_common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kFE = 8;                         // epilogue warps (2..9)
constexpr int kFMma1 = 2 + kFE, kFProd1 = 3 + kFE;   // warps 10 and 11
constexpr int kFThreads = 32 * (kFProd1 + 1);
constexpr int kFBN = 16;                       // routed rows per tile
// k-blocks per stage: gate_up 2 (two weight tiles), down 3 (one weight tile),
// so that both fill the same stage: [weights 64 KB][activations 6 KB]
// [weight scales 2 KB][activation scales 1.5 KB]
constexpr int kFKPBg = 2, kFKPBd = 3;
constexpr int kFMaxStages = 8;
constexpr int kFA_KB = kBM * 128;              // one weight tile, one k-block (E2M1 in 16-byte slots)
constexpr int kFB_KB = kFBN * 128;             // activations, one k-block
constexpr int kFBOff = 4 * kFA_KB;             // activations after 4 weight k-block slots
constexpr int kFSfA = kFBOff + kFKPBd * kFB_KB;            // weight scale blocks
constexpr int kFSfB = kFSfA + 4 * 512;                     // activation scale blocks
constexpr int kFStage = (kFSfB + kFKPBd * 512 + 1023) / 1024 * 1024;
constexpr int kFBarBytes = 256;                // mbarriers + TMEM slot + abort flag
constexpr int kFAcc = 2 * kFBN;                // TMEM columns of one accumulator set
constexpr int kFSfCol = 2 * kFAcc;             // scale columns: 8 per MMA warp
constexpr int kFTmemCols = 128;

struct FusedArgs {
    const uint8_t *xsf;          // [N][KBp] E8M0 scales of the permuted E4M3 activations
    int KBp;
    const int32_t *idx;
    const float *w;
    int T, K, H, F, E;
    const uint8_t *w13sf, *w2sf; // E8M0 weight scales, block layout
    uint8_t *h;                  // [N][F] e4m3, rows in expert-sorted slot order
    uint8_t *hsf;                // [N][FBp] E8M0
    int FBp;
    float *y;                    // [T*K][H] fp32, by slot
    __nv_bfloat16 *out;          // [T][H]
    int32_t *gu_done;            // [kFusedMaxSlots] gate_up tiles done per row tile
    int32_t *blk_done;           // [T][H/128] down tiles done per (token, 128-row block)
    int32_t *status;
    int stages;
};

// The expert-sorted order of the valid slots, built by every CTA.
struct Routing {
    int nt;                           // touched experts
    int texp[kFusedMaxSlots];         // expert id of touched expert u (ascending)
    int tstart[kFusedMaxSlots];       // first sorted position of u
    int tcnt[kFusedMaxSlots];         // slots of u
    int pos_slot[kFusedMaxSlots];     // sorted position -> slot
    int nvalid[kFusedMaxT];           // valid slots of each token
    int gu_pre[kFusedMaxSlots + 1];   // prefix of gate_up units over u
    int dn_pre[kFusedMaxSlots + 1];   // prefix of down units over u
};

struct FTile {
    bool gu;
    int u, e, rt, m, row0, nrows;
};

__device__ FTile f_decode(int w, const Routing &R, int MTg, int MTh) {
    FTile t;
    t.gu = w < R.gu_pre[R.nt];
    const int *pre = t.gu ? R.gu_pre : R.dn_pre;
    const int ww = t.gu ? w : w - R.gu_pre[R.nt];
    int u = 0;
    while (pre[u + 1] <= ww) ++u;
    const int MT = t.gu ? MTg : MTh;
    const int local = ww - pre[u];
    t.rt = local / MT;
    t.m = local - t.rt * MT;
    t.u = u;
    t.e = R.texp[u];
    t.row0 = R.tstart[u] + kFBN * t.rt;
    t.nrows = min(kFBN, R.tcnt[u] - kFBN * t.rt);
    return t;
}

// Built by the first kFusedMaxSlots threads (O(T*K) work each); every thread
// must call it (it contains __syncthreads).
__device__ void build_routing(const int32_t *__restrict__ idx, int T, int K, int E, int MTg, int MTh,
                              Routing &R) {
    __shared__ int s_e[kFusedMaxSlots];
    __shared__ int s_first[kFusedMaxSlots];     // slot is the first of its expert
    const int N = T * K;
    const int s = threadIdx.x;
    if (s < N) {
        const int e = __ldg(idx + s);
        s_e[s] = (e >= 0 && e < E) ? e : -1;
    }
    __syncthreads();
    if (s < N) {
        const int e = s_e[s];
        int first = e >= 0;
        for (int q = 0; q < s && first; ++q) first = s_e[q] != e;
        s_first[s] = first;
    }
    __syncthreads();
    if (s < N && s_e[s] >= 0) {
        const int e = s_e[s];
        int before = 0, same = 0, distinct_before = 0;
        for (int q = 0; q < N; ++q) {
            const int f = s_e[q];
            if (f < 0) continue;
            before += (f < e) || (f == e && q < s);
            same += (f == e);
            distinct_before += (f < e) && s_first[q];
        }
        R.pos_slot[before] = s;
        if (s_first[s]) {
            R.texp[distinct_before] = e;
            R.tstart[distinct_before] = before;       // no equal slot before the first one
            R.tcnt[distinct_before] = same;
        }
    }
    if (s < T) {
        int nv = 0;
        for (int k = 0; k < K; ++k) {
            const int e = __ldg(idx + s * K + k);
            nv += (e >= 0 && e < E);
        }
        R.nvalid[s] = nv;
    }
    __syncthreads();
    if (s == 0) {
        int nt = 0;
        for (int q = 0; q < N; ++q) nt += s_first[q];
        R.nt = nt;
        R.gu_pre[0] = R.dn_pre[0] = 0;
        for (int u = 0; u < nt; ++u) {
            const int nrt = (R.tcnt[u] + kFBN - 1) / kFBN;
            R.gu_pre[u + 1] = R.gu_pre[u] + nrt * MTg;
            R.dn_pre[u + 1] = R.dn_pre[u] + nrt * MTh;
        }
    }
    __syncthreads();
}

__device__ __forceinline__ void cp_async16f(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void epi_sync_fused() {
    asm volatile("bar.sync 3, %0;" ::"n"(32 * kFE) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int32_t *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__global__ void __launch_bounds__(kFThreads, 1)
    fused_moe_mxf4(const __grid_constant__ CUtensorMap tm13, const __grid_constant__ CUtensorMap tm2,
                   const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmH,
                   const FusedArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    const int NST = args.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)NST * kFStage);
    uint64_t *empty = full + kFMaxStages;
    uint64_t *afull = empty + kFMaxStages;
    uint64_t *aempty = afull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(aempty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int SXP = max(args.KBp, args.FBp);                             // row stride of sxs
    uint8_t *sxs = smem + (size_t)NST * kFStage + kFBarBytes;           // [16][SXP] activation scale bytes
    float *amax_s = reinterpret_cast<float *>(sxs + kFBN * SXP);        // [4][16]
    float *scale_s = amax_s + 4 * kFBN;                                  // [16]
    int *last_t = reinterpret_cast<int *>(scale_s + kFBN);               // [16] tokens to combine
    int *n_last = last_t + kFBN;
    Routing &R = *reinterpret_cast<Routing *>(n_last + 4);

    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int KBg = args.H / 128, KBd = args.F / 128;
    const int MTg = args.F / kBM, MTh = args.H / kBM;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 2);
            mbar_init(&empty[s], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&afull[b], 2);
            mbar_init(&aempty[b], 32 * kFE);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if ((warp == 0 || warp == kFProd1) && lane == 0) {
        prefetch_tmap(&tm13);
        prefetch_tmap(&tm2);
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmH);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kFTmemCols);
        tmem_relinquish();
    }
    pdl_wait();
    build_routing(args.idx, args.T, args.K, args.E, MTg, MTh, R);   // contains __syncthreads
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = R.gu_pre[R.nt] + R.dn_pre[R.nt];
    pdl_launch_dependents();
    // tokens with no valid slot: out = 0
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < args.T * args.H; i += blockDim.x)
            if (R.nvalid[i / args.H] == 0) args.out[i] = __float2bfloat16_rn(0.f);

    if (warp == 0 || warp == kFProd1) {
        // ------------------------------------------------ TMA producers ----
        // gate_up: producer 0 quantises the activations into the B tile and
        // loads the gate weights, producer 1 the up weights.  down: producer
        // 0 the weights, producer 1 (after the tile's gate_up work is done)
        // the h rows and their scales.
        const int p = warp == 0 ? 0 : 1;
        const uint64_t pol_once = policy_evict_first();
        const uint64_t pol_x = policy_evict_last();
        int stage = 0, armed[kFMaxStages];
        uint32_t phase = 0;
        for (int s = 0; s < kFMaxStages; ++s) armed[s] = -1;
        bool ok = true;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            const FTile t = f_decode(w, R, MTg, MTh);
            const int KB = t.gu ? KBg : KBd;
            const bool do_a = t.gu || p == 0;
            const bool do_b = t.gu ? p == 0 : p == 1;
            if (do_b) {
              if (!t.gu) {
                // h rows of this row tile: wait for its F/128 gate_up tiles
                if (lane == 0) {
                    const int32_t *flag = args.gu_done + R.gu_pre[t.u] / MTg + t.rt;
                    const long long t0 = clock64();
                    while (ld_acquire(flag) < MTg) {
                        if (*abort_flag || clock64() - t0 > kWaitLimitCycles) { ok = false; break; }
                        __nanosleep(64);
                    }
                    fence_proxy_async_global();
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
              }
                // the tile's activation-scale bytes (x's or h's), row n -> sxs[n]
                const int rs = t.gu ? args.KBp : args.FBp;
                const uint8_t *src = t.gu ? args.xsf : args.hsf;
                const int nch = rs / 16;
                for (int i = lane; i < t.nrows * nch; i += 32) {
                    const int n = i / nch, c = i - n * nch;
                    cp_async16f(sxs + n * SXP + 16 * c, src + (size_t)(t.row0 + n) * rs + 16 * c);
                }
                cp_async_commit();
                cp_async_wait<0>();
                __syncwarp();
            }
            const uint64_t pol_w = pol_once;
            const int rows_e = t.gu ? 2 * args.F : args.H;
            const int arow = t.e * rows_e + t.m * kBM + (t.gu ? p * args.F : 0);
            const uint8_t *sfa = (t.gu ? args.w13sf : args.w2sf) + (size_t)t.e * rows_e * KB * 4 +
                                 ((size_t)t.m + (t.gu ? (size_t)p * MTg : 0)) * KB * 512;
            const CUtensorMap *mA = t.gu ? &tm13 : &tm2;
            const int kpb = t.gu ? kFKPBg : kFKPBd;
            for (int kb0 = 0; kb0 < KB; kb0 += kpb) {
                const int nkb = min(kpb, KB - kb0);
                if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1, abort_flag);
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
                uint8_t *sA = ring + stage * kFStage;
                uint8_t *sB = sA + kFBOff;
                uint32_t *sfb = reinterpret_cast<uint32_t *>(sA + kFSfB);
                if (do_b) {
                    // activation scales in the block layout: row n at word 4n
                    // of its k-block's block, the byte repeated for the slices
                    for (int i = lane; i < kpb * kFBN; i += 32) {
                        const int n = i & 15, j = i >> 4;
                        const uint32_t b = (n < t.nrows && j < nkb) ? (uint32_t)sxs[n * SXP + kb0 + j] : 127u;
                        sfb[j * 128 + n * 4] = b * 0x01010101u;
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    // E2M1 loads count their packed bytes; boxes past the last
                    // k-block are zero-filled and still counted
                    const uint32_t bytes =
                        (do_a ? kpb * kFA_KB / 2 + nkb * 512 : 0) + (do_b ? kpb * kFB_KB : 0);
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    armed[stage] = (int)phase;
                    if (do_a) {
                        tma_load_3d(sA + p * kpb * kFA_KB, mA, &full[stage], 0, arow, kb0, pol_w);
                        bulk_load(sA + kFSfA + p * kpb * 512, sfa + (size_t)kb0 * 512, nkb * 512,
                                  &full[stage], pol_w);
                    }
                    if (do_b) tma_load_3d(sB, t.gu ? &tmX : &tmH, &full[stage], 0, t.row0, kb0, pol_x);
                }
                if (++stage == NST) { stage = 0; phase ^= 1; }
            }
        }
        if (lane == 0) {
            if (!ok) {
                *abort_flag = 1;
                atomicOr(args.status, DEV_TIMEOUT);
            }
            volatile int never = 0;
            for (int s = 0; s < NST; ++s)
                if (armed[s] >= 0 && !mbar_wait(&full[s], (uint32_t)armed[s], &never))
                    atomicOr(args.status, DEV_TIMEOUT);
        }
    } else if (warp == 1 || warp == kFMma1) {
        // ------------------------------------------------ MMA issue (role r) ----
        // gate_up: weight tile r (gate, up), every k-block; down: the k-blocks
        // j == r of each stage into partial accumulator r
        const int r = warp == 1 ? 0 : 1;
        if (lane == 0) {
            int stage = 0, ab = 0;
            uint32_t phase = 0, aphase = 0;
            bool ok = true;
            const uint32_t tsfa = tmem_base + kFSfCol + 8 * r;
            const uint32_t tsfb = tsfa + 4;
            const uint32_t idesc = idesc_mxf4_e4m3(kBM, kFBN);
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
                const FTile t = f_decode(w, R, MTg, MTh);
                const int KB = t.gu ? KBg : KBd;
                const int op = t.gu ? r : 0;
                if (!mbar_wait(&aempty[ab], aphase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + ab * kFAcc + r * kFBN;
                const int kpb = t.gu ? kFKPBg : kFKPBd;
                for (int kb0 = 0; kb0 < KB; kb0 += kpb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + stage * kFStage);
                    for (int j = 0; j < kpb && kb0 + j < KB; ++j) {
                        if (!t.gu && (j & 1) != r) continue;   // down: alternate k-blocks per warp
                        tmem_cp_32x128b_x4(tsfa, sdesc_rows16(sa + kFSfA + (op * kpb + j) * 512));
                        tmem_cp_32x128b_x4(tsfb, sdesc_rows16(sa + kFSfB + j * 512));
                        const uint64_t da = sdesc_sw128(sa + (op * kpb + j) * kFA_KB);
                        const uint64_t db = sdesc_sw128(sa + kFBOff + j * kFB_KB);
                        const int first = t.gu ? 0 : r;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t sel = (uint32_t)k << 30;
                            mma_mxf4_ss(d, da + 2 * k, db + 2 * k, idesc | idesc_sf_ids(k, k),
                                        tsfa | sel, tsfb | sel, (kb0 + j > first || k > 0) ? 1u : 0u);
                        }
                    }
                    mma_commit(&empty[stage]);
                    if (++stage == NST) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&afull[ab]);
                if (++ab == 2) { ab = 0; aphase ^= 1; }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(args.status, DEV_TIMEOUT);
            }
        }
    } else {
        // ---------------------------------------------------- epilogue ----
        constexpr int NC = kFBN / 2;
        const int ew = warp - 2, et = threadIdx.x - 64;
        const int eg = warp & 3;                 // TMEM lanes [32*eg, 32*eg+32)
        const int half = ew >> 2;                // columns [NC*half, NC*half+NC)
        const int row = eg * 32 + lane;
        int ab = 0;
        uint32_t aphase = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const FTile t = f_decode(w, R, MTg, MTh);
            const int live = t.nrows - half * NC;
            if (ok && !mbar_wait(&afull[ab], aphase, abort_flag)) {
                ok = false;
                *abort_flag = 1;
                atomicOr(args.status, DEV_TIMEOUT);
            }
            tc_fence_after();
            const uint32_t ta = tmem_base + ((uint32_t)(eg * 32) << 16) + ab * kFAcc + half * NC;
            float ag[NC], au[NC];
            {
                uint32_t r0[NC], r1[NC];
                tmem_ld8(ta, r0);
                tmem_ld8(ta + kFBN, r1);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < NC; ++j) {
                    ag[j] = __uint_as_float(r0[j]);
                    au[j] = __uint_as_float(r1[j]);
                }
            }
            tc_fence_before();
            mbar_arrive(&aempty[ab]);
            if (++ab == 2) { ab = 0; aphase ^= 1; }
            if (t.gu) {
                // h = bf16(SiLU(g) * u), quantised per 128 features (this tile)
#pragma unroll
                for (int j = 0; j < NC; ++j)
                    ag[j] = __bfloat162float(__float2bfloat16_rn(silu_f(ag[j]) * au[j]));
                // column max of |h| over this warp's 32 rows (lane l ends with column l)
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = j < NC ? fabsf(ag[j]) : 0.f;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
                    for (int i = 0; i < o; ++i) {
                        const bool upper = (lane & o) != 0;
                        const float send = upper ? v[i] : v[i + o];
                        const float keep = upper ? v[i + o] : v[i];
                        v[i] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, send, o));
                    }
                }
                if (lane < NC) amax_s[eg * kFBN + half * NC + lane] = v[0];
                epi_sync_fused();
                if (et < kFBN) {
                    const float m = fmaxf(fmaxf(amax_s[et], amax_s[kFBN + et]),
                                          fmaxf(amax_s[2 * kFBN + et], amax_s[3 * kFBN + et]));
                    const int k = fp8_block_exp(m);
                    scale_s[et] = pow2f(-k);
                    if (et < t.nrows) args.hsf[(size_t)(t.row0 + et) * args.FBp + t.m] = (uint8_t)(k + 127);
                }
                epi_sync_fused();
                uint8_t *hp = args.h + (size_t)(t.row0 + half * NC) * args.F + t.m * kBM + row;
#pragma unroll
                for (int j = 0; j < NC; ++j)
                    if (j < live)
                        hp[(size_t)j * args.F] = (uint8_t)(e4m3x2(ag[j] * scale_s[half * NC + j], 0.f) & 0xFF);
                __threadfence();
                epi_sync_fused();                // every h store of the tile is out
                if (et == 0) atomicAdd(args.gu_done + R.gu_pre[t.u] / MTg + t.rt, 1);
            } else {
                // the two partial accumulators, times the router weight, by slot
                const int c0 = half * NC;
                for (int j = 0; j < NC; ++j) {
                    if (j < live) {
                        const int slot = R.pos_slot[t.row0 + c0 + j];
                        args.y[(size_t)slot * args.H + t.m * kBM + row] =
                            __ldg(args.w + slot) * (KBd > 1 ? ag[j] + au[j] : ag[j]);
                    }
                }
                __threadfence();
                if (et == 0) *n_last = 0;
                epi_sync_fused();                // the tile's y rows are out
                if (et < t.nrows) {
                    const int slot = R.pos_slot[t.row0 + et];
                    const int tok = slot / args.K;
                    const int old = atomicAdd(args.blk_done + tok * MTh + t.m, 1);
                    if (old + 1 == R.nvalid[tok]) {  // every slot of this token's block is in
                        __threadfence();
                        last_t[atomicAdd(n_last, 1)] = tok;
                    }
                }
                epi_sync_fused();
                const int nl = *n_last;
                for (int i = et; i < nl * kBM; i += 32 * kFE) {
                    const int tok = last_t[i / kBM], jr = t.m * kBM + i % kBM;
                    // all K rows requested at once, then summed in k order
                    float v[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        v[k] = 0.f;
                        if (k < args.K) {
                            const int e = __ldg(args.idx + tok * args.K + k);
                            if (e >= 0 && e < args.E)
                                v[k] = __ldcg(args.y + (size_t)(tok * args.K + k) * args.H + jr);
                        }
                    }
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        if (k < args.K) acc += v[k];
                    args.out[(size_t)tok * args.H + jr] = __float2bfloat16_rn(acc);
                }
                epi_sync_fused();                // last_t / n_last are reused by the next tile
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kFTmemCols);
    }
}

}  // namespace

bool fused_mxf4_fits(int T, int K) { return T <= kFusedMaxT && T * K <= kFusedMaxSlots; }

cudaError_t launch_fused_mxf4(const void *x, const void *w13, const uint8_t *w13sf, const void *w2,
                              const uint8_t *w2sf, const int32_t *idx, const float *w, int T, int H,
                              int F, int E, int K, uint8_t *ws, const Workspace &L, void *out,
                              cudaStream_t st) {
    if (!fused_mxf4_fits(T, K) || L.ctr_bytes == 0) return cudaErrorInvalidValue;
    const uint64_t N = (uint64_t)T * K;
    CUtensorMap t13, t2, tx, th;
    if (!make_tmap_e2m1(&t13, w13, (uint64_t)E * 2 * F, H, kFKPBg) ||
        !make_tmap_e2m1(&t2, w2, (uint64_t)E * H, F, kFKPBd) ||
        !make_tmap_e4m3_kb(&tx, ws + L.xperm, N, H, kFBN, kFKPBg) ||
        !make_tmap_e4m3_kb(&th, ws + L.h, N, F, kFBN, kFKPBd))
        return cudaErrorInvalidValue;
    // S3 (permutation, E4M3 gather of x with E8M0 scale bytes) stays its own
    // kernel: it needs every slot of the call; it also clears the status
    // word and the work counters that the fused kernel starts from
    cudaError_t err = launch_permute_gather(x, idx, (int64_t)N, K, H, E, kFBN, kFBN, MOE_W_MXFP4, ws, L, st,
                                            (int32_t *)(ws + L.ctr), (int)(L.ctr_bytes / sizeof(int32_t)));
    if (err != cudaSuccess) return err;
    FusedArgs a = {};
    a.xsf = ws + L.xscale;
    a.KBp = (int)align_up(H / 128, 16);
    a.idx = idx;
    a.w = w;
    a.T = T; a.K = K; a.H = H; a.F = F; a.E = E;
    a.w13sf = w13sf;
    a.w2sf = w2sf;
    a.h = ws + L.h;
    a.hsf = ws + L.hscale;
    a.FBp = (int)align_up(F / 128, 16);
    a.y = (float *)(ws + L.y);
    a.out = (__nv_bfloat16 *)out;
    a.gu_done = (int32_t *)(ws + L.ctr);
    a.blk_done = a.gu_done + kFusedMaxSlots;
    a.status = (int32_t *)(ws + L.status);
    auto smem_for = [&](int stages) {
        return (size_t)1024 + (size_t)stages * kFStage + kFBarBytes + (size_t)kFBN * (a.KBp > a.FBp ? a.KBp : a.FBp) +
               sizeof(float) * 5 * kFBN + sizeof(int) * (kFBN + 4) + sizeof(Routing) + 64;
    };
    constexpr size_t kSmemMax = 227 * 1024;
    a.stages = kFMaxStages;
    while (a.stages > 2 && smem_for(a.stages) > kSmemMax) --a.stages;
    const size_t need = smem_for(a.stages);
    if (need > kSmemMax) return cudaErrorInvalidValue;
    static std::atomic<int> attr_done[64];
    err = enable_max_dyn_smem((const void *)fused_moe_mxf4, attr_done);
    if (err != cudaSuccess) return err;
    return launch_k(fused_moe_mxf4, dim3(num_sms()), dim3(kFThreads), need, st, true, t13, t2, tx, th, a);
}

}  // namespace moe
