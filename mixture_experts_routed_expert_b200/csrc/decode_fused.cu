// decode_fused.cu -- the bf16 decode form of the routed-experts forward
// ("deepseek-ocr2-moe-experts" model card: fused gather-GEMV for
// n_tokens ~ 1-4) as ONE kernel launch: the expert dedup of the slots, the
// gate/up GEMV with SiLU*up, the down GEMV, the router-weight scale and the
// fixed-order top-K combine (the DeepGEMM Mega MoE news page: the MoE steps in
// a single kernel so that the round trips between kernels disappear).
//
// One CTA per SM, each with a producer warp that streams weight rows into a
// ring of shared-memory stages by bulk copies, and eight compute warps.
//   phase 1  The touched experts (ascending id) laid end to end give n_u * F
//            features; CTA b takes an even, contiguous share (in groups of 8)
//            and computes h[s, f] = bf16(SiLU(G_e[f] . x_t) * (U_e[f] . x_t))
//            for the slots s of each expert e it covers, writes h to the
//            workspace and adds its group count to the expert's counter.
//   phase 2  The n_u * H down-projection rows, likewise split evenly (in
//            units of 8 rows): whole rows, each one contiguous copy of F
//            values.  Before using expert e's rows the compute warps wait
//            (bounded) until e's counter shows all F/8 groups of h; the
//            producer does not wait: it keeps loading rows meanwhile, so the
//            weight stream continues across the dependency.
//            y[s, j] = D_e[j] . h[s] is complete per row (no partial sums).
//   combine  Per (token, 32-row block) a counter collects the rows of the
//            token's K slots; the CTA whose arrival completes it writes
//            out[t, block] = bf16(sum_{k ascending} w[t,k] * y[t*K+k, block])
//            and resets the counter.  Fixed summation order, no
//            floating-point atomics.
// Both GEMVs run on warp-level bf16 tensor-core MMAs (m16n8k16, fp32
// accumulators): a 16-row weight tile (phase 1: the 8 gate rows and the 8 up
// rows of 8 features; phase 2: 16 down rows) times up to 8 slots, the
// reduction dimension split over the eight warps and their partial tiles
// added in warp order.  Weight rows land in shared memory as they lie in
// memory (one bulk copy per chunk); inside each 64-element group the k order
// of the fragments is permuted, identically for weights and activations
// (which leaves every dot product unchanged), and lanes of odd tile rows
// read the group's two halves in the other order, so that every quarter-warp
// load hits eight distinct bank groups.
// The counters live in the workspace header, are zero before the call and
// are zero again after it (the last user of each resets it).  The CTAs wait
// on one another only through those counters, so the grid never exceeds the
// CTAs that are resident at once.  Every wait is bounded; on expiry the
// kernel sets DEV_TIMEOUT in the workspace status word, stops issuing,
// drains its own copies and returns.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kCW = 8;                         // compute warps
constexpr int kFDThreads = 32 * (kCW + 1);     // + one producer warp (the last)
constexpr int kMaxSlots = kDecodeMaxSlots;     // 64
constexpr int kMaxT = kDecodeMaxT;             // 16
constexpr int kSlotGroup = 8;                  // slots per MMA (N = 8)
constexpr int kBlk = 32;                       // rows of a combine block
constexpr int kUnit = 8;                       // rows of a phase-2 work unit
constexpr int kTileRows = 16;                  // weight rows per MMA tile (M = 16)
constexpr int kMaxPieces = 128;                // listed pieces before a flush

struct FDArgs {
    const __nv_bfloat16 *x;        // [T][H]
    const __nv_bfloat16 *gate_up;  // [E][2F][H]
    const __nv_bfloat16 *down;     // [E][H][F]
    const int32_t *idx;            // [T][K]
    const float *w;                // [T][K]
    __nv_bfloat16 *out;            // [T][H]
    __nv_bfloat16 *h;              // [T*K][F] by slot
    float *y;                      // [T*K][H] down-projection rows by slot
    int32_t *hdone;                // [64] h groups published per touched expert
    int32_t *hused;                // [64] down rows (in units of 8) done per touched expert
    int32_t *ctr;                  // [T][H/32] combine arrivals (in units of 8 rows)
    int32_t *status;
    int T, H, F, E, K;
    int stages;
    int sb;                        // ring stage bytes (16 rows at the larger pitch)
    int withhold;                  // test hook: CTA 0 never issues chunk `withhold` (-1: off)
};

// Named barrier of the compute warps (the producer warp never joins it).
__device__ __forceinline__ void compute_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
}

__device__ __forceinline__ int ld_acquire_i32(const int32_t *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Even split of n items over nb parts: the first item of part b (32-bit:
// n * nb stays below 2^31 for every size the kernel takes).
__device__ __forceinline__ int part_start(int b, int n, int nb) { return (b * n) / nb; }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// D (16x8 fp32) += A (16x16 bf16, row-major) * B (16x8 bf16, column-major).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One warp's share of a 16-row tile times 8 activation rows, over K
// elements in groups of 64 (group p for the warps with p % 8 == warp).
// Thread (g, q) takes, of each 128-byte group, the 16-byte chunks q and q+4
// of weight rows g and g+8 and of activation row g (lanes with odd g load
// chunk q+4 first); chunk q feeds k-steps 4p and 4p+1, chunk q+4 k-steps
// 4p+2 and 4p+3, with the same k order on both sides.  act_ok = false gives
// that thread's activation row as zeros (slots past the group).
__device__ __forceinline__ void tile_mma(float (&d)[4], uint32_t wrow_g, uint32_t wrow_g8,
                                         uint32_t arow, bool act_ok, int ngroups, int warp, int g,
                                         int q) {
    const bool odd = g & 1;
    const uint32_t c1 = (uint32_t)(16 * (odd ? q + 4 : q)), c2 = (uint32_t)(16 * (odd ? q : q + 4));
    for (int p = warp; p < ngroups; p += kCW) {
        const uint32_t base = (uint32_t)(128 * p);
        const uint4 w1 = lds128(wrow_g + base + c1), w2 = lds128(wrow_g + base + c2);
        const uint4 v1 = lds128(wrow_g8 + base + c1), v2 = lds128(wrow_g8 + base + c2);
        uint4 x1 = make_uint4(0, 0, 0, 0), x2 = x1;
        if (act_ok) {
            x1 = lds128(arow + base + c1);
            x2 = lds128(arow + base + c2);
        }
        const uint4 wq = odd ? w2 : w1, wq4 = odd ? w1 : w2;     // chunks q and q+4
        const uint4 vq = odd ? v2 : v1, vq4 = odd ? v1 : v2;
        const uint4 xq = odd ? x2 : x1, xq4 = odd ? x1 : x2;
        mma_bf16_16816(d, wq.x, vq.x, wq.y, vq.y, xq.x, xq.y);
        mma_bf16_16816(d, wq.z, vq.z, wq.w, vq.w, xq.z, xq.w);
        mma_bf16_16816(d, wq4.x, vq4.x, wq4.y, vq4.y, xq4.x, xq4.y);
        mma_bf16_16816(d, wq4.z, vq4.z, wq4.w, vq4.w, xq4.z, xq4.w);
    }
}

// Slots, touched experts and the expert-sorted slot order (every CTA builds
// the same in shared memory).
struct FDRouting {
    int nu;
    int e_of[kMaxSlots];     // expert of slot (-1: outside [0, E))
    int u_of[kMaxSlots];     // touched index of slot (-1: invalid)
    int uexp[kMaxSlots];     // expert id of touched index u (ascending)
    int ustart[kMaxSlots + 1];
    int uslot[kMaxSlots];    // slots of u at [ustart[u], ustart[u+1]), ascending
    int nvalid[kMaxT];       // valid slots per token
};

// Builds the routing tables; every thread of the block calls it (E <= 1024,
// T*K <= 64).  A bitmap of the valid experts gives each expert its touched
// index (the set bits below it); the slots of an expert keep their order: a
// slot's rank is the number of earlier slots with the same expert (warp
// match within its warp, plus the count from warp 0 for slots of warp 1).
__device__ void fd_build_routing(const int32_t *__restrict__ idx, int T, int K, int E,
                                 FDRouting &R) {
    __shared__ uint32_t bits[32];
    __shared__ int wpre[33];
    __shared__ int cnt[kMaxSlots], cnt0[kMaxSlots];
    const int N = T * K;
    const int s = threadIdx.x;
    const int lane = s & 31;
    if (s < 32) bits[s] = 0u;
    if (s < kMaxSlots) { cnt[s] = 0; cnt0[s] = 0; }
    int e = -1;
    if (s < N) {
        e = __ldg(idx + s);
        e = (e >= 0 && e < E) ? e : -1;
        R.e_of[s] = e;
    }
    __syncthreads();
    if (e >= 0) atomicOr(&bits[e >> 5], 1u << (e & 31));
    __syncthreads();
    if (s < 32) {   // exclusive prefix of the set bits per word
        const int c = __popc(bits[s]);
        int v = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, v, o);
            if (lane >= o) v += y;
        }
        wpre[s] = v - c;
        if (s == 31) { wpre[32] = v; R.nu = v; }
    }
    __syncthreads();
    int u = -1, rank = 0;
    if (s < 64) {   // warps 0 and 1 hold the slots
        if (e >= 0) u = wpre[e >> 5] + __popc(bits[e >> 5] & ((1u << (e & 31)) - 1u));
        const uint32_t same = __match_any_sync(0xFFFFFFFFu, e);
        rank = __popc(same & ((1u << lane) - 1u));
        if (s < N) R.u_of[s] = u;
        if (e >= 0) {
            R.uexp[u] = e;
            atomicAdd(&cnt[u], 1);
            if (s < 32) atomicAdd(&cnt0[u], 1);
        }
    }
    if (s < T) {
        int nv = 0;
        for (int k = 0; k < K; ++k) nv += (R.e_of[s * K + k] >= 0);
        R.nvalid[s] = nv;
    }
    __syncthreads();
    if (s < 32) {   // ustart: exclusive prefix of cnt over the touched experts
        const int c0 = cnt[2 * s], c1 = cnt[2 * s + 1];
        int v = c0 + c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, v, o);
            if (lane >= o) v += y;
        }
        const int ex = v - c0 - c1;
        R.ustart[2 * s] = ex;
        R.ustart[2 * s + 1] = ex + c0;
        if (s == 31) R.ustart[64] = v;
    }
    __syncthreads();
    if (s < 64 && e >= 0) R.uslot[R.ustart[u] + (s >= 32 ? cnt0[u] : 0) + rank] = s;
    __syncthreads();
}


// ---- chunk sequence shared by the producer and the compute warps ----------
// Phase 1 chunks: the 8 features [f, f+8) of touched expert u (gate rows in
// tile rows 0-7, up rows in tile rows 8-15).  Phase 2 chunks: down rows
// [f, f+n) (n <= 16) of touched expert u inside one 32-row combine block.
struct Chunk {
    int kind;          // 1: gate/up rows, 2: down rows, 0: end
    int u, f, n;
    bool first_u;      // phase 2: this CTA's first chunk of expert u
    bool end_run;      // phase 1: last chunk of a run of one expert; phase 2:
                       // last chunk of a piece (rows of one combine block)
    bool last_u;       // phase 2: this CTA's last chunk of expert u
};

struct Walker {
    int F, H;
    int cur1, end1, cur2, end2, prev_u;

    __device__ void init(int b, int nb, int nu) {
        const int g1 = nu * (F / 8), g2 = nu * (H / kUnit);
        cur1 = 8 * part_start(b, g1, nb);
        end1 = 8 * part_start(b + 1, g1, nb);
        cur2 = kUnit * part_start(b, g2, nb);
        end2 = kUnit * part_start(b + 1, g2, nb);
        prev_u = -1;
    }
    __device__ Chunk next() {
        Chunk k{};
        if (cur1 < end1) {
            const int u = cur1 / F;
            k.kind = 1;
            k.u = u;
            k.f = cur1 - u * F;
            k.n = 8;
            cur1 += 8;
            k.end_run = (cur1 == end1 || cur1 == (u + 1) * F);
            return k;
        }
        if (cur2 < end2) {
            const int u = cur2 / H;
            const int j = cur2 - u * H;
            const int ulast = min(end2, (u + 1) * H);
            const int pend = min(ulast, u * H + (j / kBlk + 1) * kBlk);
            const int e = min(pend, cur2 + kTileRows);
            k.kind = 2;
            k.u = u;
            k.f = j;
            k.n = e - cur2;
            k.first_u = (u != prev_u);
            k.end_run = (e == pend);
            k.last_u = (e == ulast);
            prev_u = u;
            cur2 = e;
            return k;
        }
        k.kind = 0;
        return k;
    }
};

__global__ void __launch_bounds__(kFDThreads, 1) decode_fused_bf16(const FDArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ FDRouting R;
    __shared__ __align__(8) uint64_t full[8], empty[8], xbar;
    __shared__ int abort_flag, n_last;
    __shared__ float red[kCW][kTileRows][kSlotGroup];  // partial tiles of the eight warps
    __shared__ int lcount[kMaxT * (2048 / kBlk)];     // this CTA's arrivals per (token, block)
    __shared__ int last_pair[kMaxT * (2048 / kBlk)];  // (token, block) pairs this CTA completes
    __shared__ int pc_u[kMaxPieces], pc_blk[kMaxPieces], pc_units[kMaxPieces];
    __shared__ int hu_u[kMaxSlots], hu_n[kMaxSlots];

    const int NST = a.stages;
    const int P1 = 2 * a.H, P2 = 2 * a.F;                // row bytes
    uint8_t *ring = smem;
    uint8_t *xs = smem + (size_t)NST * a.sb;              // [T][H] x
    uint8_t *hst = xs + (size_t)a.T * P1;                 // [8][F] staged h
    const uint32_t ring_u = smem_u32(ring), xs_u = smem_u32(xs), hst_u = smem_u32(hst);

    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int tid = threadIdx.x;
    const bool producer = warp == kCW;
    const int nblk = a.H / kBlk;

    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCW);
        }
        mbar_init(&xbar, 1);
        abort_flag = 0;
        n_last = 0;
        fence_mbar_init();
    }
    // every input may come from the previous kernel on the stream
    pdl_wait();
    if (tid == 0) {   // x does not depend on the routing: request it first
        mbar_arrive_expect_tx(&xbar, (uint32_t)(a.T * 2 * a.H));
        bulk_load(xs, a.x, (uint32_t)(a.T * 2 * a.H), &xbar, policy_evict_last());
    }
    fd_build_routing(a.idx, a.T, a.K, a.E, R);   // has __syncthreads
    pdl_launch_dependents();

    // tokens with no valid slot: zeros (CTA 0)
    if (blockIdx.x == 0 && !producer)
        for (int i = tid; i < a.T * a.H; i += kCW * 32)
            if (R.nvalid[i / a.H] == 0) a.out[i] = __float2bfloat16_rn(0.f);

    Walker W;
    W.F = a.F;
    W.H = a.H;
    W.init(blockIdx.x, gridDim.x, R.nu);

    if (producer) {
        // ------------------------------------------------------ producer ----
        // contiguous rows: one bulk copy for x, two (gate, up) per phase-1
        // chunk, one per phase-2 chunk
        const uint64_t pol = policy_evict_first();
        bool ok = true;
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_par = 0;   // stages with copies issued, and their phase parity
        for (int ci = 0;; ++ci) {
            const Chunk k = W.next();
            if (k.kind == 0) break;
            if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1, &abort_flag);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            const bool issue = !(ci == a.withhold && blockIdx.x == 0);   // test hook: never issued
            if (issue) {
                uint8_t *dst = ring + (size_t)stage * a.sb;
                const int e = R.uexp[k.u];
                if (lane == 0) {
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (k.kind == 1) {   // tile rows 0-7: gate f..f+7, rows 8-15: up f..f+7
                        const __nv_bfloat16 *gr = a.gate_up + ((size_t)e * 2 * a.F + k.f) * a.H;
                        mbar_arrive_expect_tx(&full[stage], (uint32_t)(16 * P1));
                        bulk_load(dst, gr, (uint32_t)(8 * P1), &full[stage], pol);
                        bulk_load(dst + 8 * P1, gr + (size_t)a.F * a.H, (uint32_t)(8 * P1), &full[stage],
                                  pol);
                    } else {
                        mbar_arrive_expect_tx(&full[stage], (uint32_t)(k.n * P2));
                        bulk_load(dst, a.down + ((size_t)e * a.H + k.f) * a.F, (uint32_t)(k.n * P2),
                                  &full[stage], pol);
                    }
                }
            }
            if (++stage == NST) { stage = 0; phase ^= 1; }
        }
        if (lane == 0) {
            if (!ok) {
                abort_flag = 1;
                atomicOr(a.status, DEV_TIMEOUT);
            }
            // every copy this warp started has landed before the CTA exits
            volatile int never = 0;
            for (int s = 0; s < NST; ++s)
                if (((armed >> s) & 1u) && !mbar_wait(&full[s], (armed_par >> s) & 1u, &never))
                    atomicOr(a.status, DEV_TIMEOUT);
            if (!mbar_wait(&xbar, 0, &never)) atomicOr(a.status, DEV_TIMEOUT);
        }
        return;
    }

    // --------------------------------------------------------- compute ----
    // every lane waits (acquire for its own reads); the outcome is made
    // warp-uniform, and a timeout raises the CTA's abort flag at once
    auto wait_full = [&](uint64_t *bar, uint32_t par) -> bool {
        bool ok_w = mbar_wait(bar, par, &abort_flag);
        ok_w = __all_sync(0xFFFFFFFFu, ok_w);
        if (!ok_w && lane == 0) {
            abort_flag = 1;
            atomicOr(a.status, DEV_TIMEOUT);
        }
        return ok_w;
    };
    const int g = lane >> 2, q = lane & 3;     // MMA fragment coordinates
    // partial tile of this warp -> red; then the sums in warp order
    auto put_red = [&](const float (&d)[4]) {
        red[warp][g][2 * q] = d[0];
        red[warp][g][2 * q + 1] = d[1];
        red[warp][g + 8][2 * q] = d[2];
        red[warp][g + 8][2 * q + 1] = d[3];
    };
    auto red_sum = [&](int row, int col) -> float {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kCW; ++w) v += red[w][row][col];
        return v;
    };
    bool ok = wait_full(&xbar, 0);
    int stage = 0;
    uint32_t phase = 0;
    Chunk k = W.next();
    // ---- phase 1: h for this CTA's features --------------------------------
    int run_f0 = k.f;
    for (; k.kind == 1; k = W.next()) {
        const int u = k.u;
        const int ns = R.ustart[u + 1] - R.ustart[u];
        if (ok) ok = wait_full(&full[stage], phase);
        const uint32_t wbase = ring_u + (uint32_t)(stage * a.sb);
        for (int s0 = 0; s0 < ns; s0 += kSlotGroup) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            if (ok) {
                const bool act = s0 + g < ns;
                const int tok = act ? R.uslot[R.ustart[u] + s0 + g] / a.K : 0;
                tile_mma(d, wbase + g * P1, wbase + (g + 8) * P1, xs_u + tok * P1, act, a.H / 64,
                         warp, g, q);
            }
            if (s0 + kSlotGroup >= ns) {   // the stage's last reads are done: hand it back
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
            }
            put_red(d);
            compute_sync();
            if (tid < 64) {   // feature f of the chunk, slot s of the group
                const int f = tid >> 3, s = tid & 7;
                if (ok && s0 + s < ns) {
                    const float gs = red_sum(f, s), us = red_sum(f + 8, s);
                    const int slot = R.uslot[R.ustart[u] + s0 + s];
                    a.h[(size_t)slot * a.F + k.f + f] = __float2bfloat16_rn(silu_f(gs) * us);
                }
            }
            compute_sync();
        }
        if (++stage == NST) { stage = 0; phase ^= 1; }
        if (k.end_run) {
            // this CTA's h of expert u is out: count its groups
            __threadfence();
            compute_sync();
            if (tid == 0 && !abort_flag) atomicAdd(a.hdone + u, (k.f + k.n - run_f0) / 8);
            run_f0 = 0;   // a following run starts at feature 0 of the next expert
        }
    }

    // ---- phase 2: down rows of this CTA's units -----------------------------
    // Finished pieces (rows of one expert inside one 32-row block) are listed
    // and counted at the end (or when the list is full), so that the stream
    // of chunks never waits on the bookkeeping.
    int piece_j0 = k.f, rows_u = 0, npc = 0, nhu = 0;
    for (int i = tid; i < a.T * nblk; i += kCW * 32) lcount[i] = 0;
    auto flush = [&]() {
        // this CTA's y rows are out: add its pieces per (token, block), then
        // one global add per pair; the add that completes a pair sums it
        __threadfence();
        compute_sync();
        for (int it = tid; it < npc * kMaxSlots; it += kCW * 32) {
            const int pc = it / kMaxSlots, sl = it - pc * kMaxSlots;
            const int uu = pc_u[pc];
            if (sl < R.ustart[uu + 1] - R.ustart[uu]) {
                const int t = R.uslot[R.ustart[uu] + sl] / a.K;
                atomicAdd(&lcount[t * nblk + pc_blk[pc]], pc_units[pc]);
            }
        }
        compute_sync();
        for (int i = tid; i < a.T * nblk; i += kCW * 32) {
            const int add = lcount[i];
            if (add == 0) continue;
            lcount[i] = 0;
            if (abort_flag) continue;
            const int t = i / nblk;
            const int old = atomicAdd(a.ctr + i, add);
            if (old + add == R.nvalid[t] * (kBlk / kUnit)) {
                __threadfence();
                last_pair[atomicAdd(&n_last, 1)] = i;
            }
        }
        compute_sync();
        const int nl = n_last;
        for (int it = tid; it < nl * kBlk; it += kCW * 32) {
            const int pr = last_pair[it / kBlk];
            const int t = pr / nblk, j = (pr - t * nblk) * kBlk + (it % kBlk);
            float acc = 0.f;
            for (int kk = 0; kk < a.K; ++kk) {
                const int slot = t * a.K + kk;
                if (R.e_of[slot] < 0) continue;
                acc = fmaf(__ldg(a.w + slot), __ldcg(a.y + (size_t)slot * a.H + j), acc);
            }
            a.out[(size_t)t * a.H + j] = __float2bfloat16_rn(acc);
        }
        compute_sync();
        for (int i = tid; i < nl; i += kCW * 32) a.ctr[last_pair[i]] = 0;   // zero for the next call
        if (tid == 0) n_last = 0;
        npc = 0;
    };
    for (; k.kind == 2; k = W.next()) {
        const int u = k.u;
        const int ns = R.ustart[u + 1] - R.ustart[u];
        if (k.first_u) {
            // h of expert u must be complete: all of its F/8 groups published
            if (tid == 0 && !abort_flag) {
                const long long t0 = clock64();
                while (ld_acquire_i32(a.hdone + u) < a.F / 8) {
                    if (abort_flag || clock64() - t0 > kWaitLimitCycles) {
                        abort_flag = 1;
                        atomicOr(a.status, DEV_TIMEOUT);
                        break;
                    }
                    __nanosleep(32);
                }
            }
            compute_sync();
            if (abort_flag) ok = false;
            piece_j0 = k.f;
            rows_u = 0;
        }
        if (ok) ok = wait_full(&full[stage], phase);
        const uint32_t wbase = ring_u + (uint32_t)(stage * a.sb);
        for (int s0 = 0; s0 < ns; s0 += kSlotGroup) {
            const int ng = min(kSlotGroup, ns - s0);
            if (ns > kSlotGroup || k.first_u) {
                // stage h of slots [s0, s0+ng) of expert u
                compute_sync();                      // the previous group's readers are done
                const int nvf = a.F / 8;
                for (int i = tid; i < ng * nvf; i += kCW * 32) {
                    const int si = i / nvf, v = i - si * nvf;
                    const int slot = R.uslot[R.ustart[u] + s0 + si];
                    *reinterpret_cast<uint4 *>(hst + (size_t)si * P2 + v * 16) =
                        __ldcg(reinterpret_cast<const uint4 *>(a.h + (size_t)slot * a.F) + v);
                }
                compute_sync();
            }
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            if (ok)
                tile_mma(d, wbase + g * P2, wbase + (g + 8) * P2, hst_u + g * P2, g < ng, a.F / 64,
                         warp, g, q);
            if (s0 + kSlotGroup >= ns) {   // the stage's last reads are done: hand it back
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
            }
            put_red(d);
            compute_sync();
            if (tid < kTileRows * kSlotGroup) {   // row r of the chunk, slot s of the group
                const int r = tid >> 3, s = tid & 7;
                if (ok && r < k.n && s < ng) {
                    const int slot = R.uslot[R.ustart[u] + s0 + s];
                    a.y[(size_t)slot * a.H + k.f + r] = red_sum(r, s);
                }
            }
            compute_sync();
        }
        if (++stage == NST) { stage = 0; phase ^= 1; }
        rows_u += k.n;
        if (k.end_run) {   // a piece is done: list it
            if (tid == 0) {
                pc_u[npc] = u;
                pc_blk[npc] = piece_j0 / kBlk;
                pc_units[npc] = (k.f + k.n - piece_j0) / kUnit;
            }
            ++npc;
            piece_j0 = k.f + k.n;
            if (npc == kMaxPieces) flush();
        }
        if (k.last_u) {
            if (tid == 0) { hu_u[nhu] = u; hu_n[nhu] = rows_u / kUnit; }
            ++nhu;
        }
    }
    flush();
    // the last CTA done with an expert's h zeroes that expert's counters
    if (tid < nhu && !abort_flag) {
        const int uu = hu_u[tid];
        const int old = atomicAdd(a.hused + uu, hu_n[tid]);
        if (old + hu_n[tid] == a.H / kUnit) {
            a.hdone[uu] = 0;
            a.hused[uu] = 0;
        }
    }
}

// ---- host side ---------------------------------------------------------------

struct FDConfig {
    int ctas = 0;    // CTAs resident at once (grid size); 0: not usable
    int smem = 0;    // dynamic shared memory per CTA (the device's opt-in limit)
};

// Per device (ordinal modulo 64), looked up once.
const FDConfig &fd_config(cudaError_t &err) {
    static FDConfig cache[64];
    static std::atomic<int> state[64];   // 0 unknown, 1 being filled, 2 ready
    static const FDConfig none;
    int dev = 0;
    err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return none;
    std::atomic<int> &st = state[dev & 63];
    if (st.load(std::memory_order_acquire) == 2) return cache[dev & 63];
    int expect = 0;
    if (st.compare_exchange_strong(expect, 1)) {
        FDConfig c;
        int optin = 0, sms = 0, per_sm = 0;
        cudaFuncAttributes fa;
        err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (err == cudaSuccess) err = cudaFuncGetAttributes(&fa, decode_fused_bf16);
        if (err == cudaSuccess) {
            c.smem = optin - (int)fa.sharedSizeBytes;
            err = cudaFuncSetAttribute(decode_fused_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       c.smem);
        }
        if (err == cudaSuccess)
            err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_bf16,
                                                                kFDThreads, c.smem);
        if (err != cudaSuccess) {
            st.store(0, std::memory_order_release);
            return none;
        }
        c.ctas = per_sm * sms;
        cache[dev & 63] = c;
        st.store(2, std::memory_order_release);
        return cache[dev & 63];
    }
    while (st.load(std::memory_order_acquire) == 1) {
    }
    if (st.load(std::memory_order_acquire) == 2) return cache[dev & 63];
    err = cudaErrorNotReady;
    return none;
}

struct FDPlan {
    FDConfig cfg;
    int stages = 0, sb = 0;
};

bool fd_plan(int T, int H, int F, int K, FDPlan &p, cudaError_t &err) {
    err = cudaSuccess;
    if (T < 1 || T > kDecodeMaxT || T * K > kDecodeMaxSlots || H > 2048 || F > 2048) return false;
    const FDConfig &c = fd_config(err);
    if (err != cudaSuccess || c.ctas < 1) return false;
    p.cfg = c;
    const int P1 = 2 * H, P2 = 2 * F;
    p.sb = (int)align_up((size_t)kTileRows * std::max(P1, P2), 128);
    const int fixed = T * P1 + kSlotGroup * P2;          // x rows, staged h rows
    p.stages = std::min(8, (c.smem - fixed) / p.sb);
    return p.stages >= 2;
}

}  // namespace

FusedDecodeWorkspace fused_decode_workspace(int T, int H, int F, int K) {
    FusedDecodeWorkspace L;
    L.status = 0;
    L.hdone = kWorkspaceCounterOffset;
    L.hused = L.hdone + sizeof(int32_t) * kDecodeMaxSlots;
    L.ctr = L.hused + sizeof(int32_t) * kDecodeMaxSlots;
    L.h = kWorkspaceHeaderBytes;
    L.y = align_up(L.h + (size_t)2 * T * K * F, 256);
    L.total = align_up(L.y + sizeof(float) * (size_t)T * K * H, 256);
    return L;
}

bool decode_fused_bf16_fits(int T, int H, int F, int K) {
    FDPlan p;
    cudaError_t e;
    const bool ok = fd_plan(T, H, F, K, p, e);
    if (e != cudaSuccess) cudaGetLastError();
    return ok;
}

cudaError_t launch_decode_fused_bf16(const void *x, const void *gate_up, const void *down,
                                     const int32_t *idx, const float *w, int T, int H, int F,
                                     int E, int K, uint8_t *ws, const FusedDecodeWorkspace &L,
                                     void *out, cudaStream_t st, int withhold) {
    FDPlan p;
    cudaError_t err;
    if (!fd_plan(T, H, F, K, p, err)) return err != cudaSuccess ? err : cudaErrorInvalidValue;
    FDArgs a = {};
    a.x = (const __nv_bfloat16 *)x;
    a.gate_up = (const __nv_bfloat16 *)gate_up;
    a.down = (const __nv_bfloat16 *)down;
    a.idx = idx;
    a.w = w;
    a.out = (__nv_bfloat16 *)out;
    a.h = (__nv_bfloat16 *)(ws + L.h);
    a.y = (float *)(ws + L.y);
    a.hdone = (int32_t *)(ws + L.hdone);
    a.hused = (int32_t *)(ws + L.hused);
    a.ctr = (int32_t *)(ws + L.ctr);
    a.status = (int32_t *)(ws + L.status);
    a.T = T; a.H = H; a.F = F; a.E = E; a.K = K;
    a.stages = p.stages;
    a.sb = p.sb;
    a.withhold = withhold;
    return launch_k(decode_fused_bf16, dim3(p.cfg.ctas), dim3(kFDThreads), (size_t)p.cfg.smem, st,
                    true, a);
}

}  // namespace moe
