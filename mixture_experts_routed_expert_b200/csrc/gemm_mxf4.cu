// gemm_mxf4.cu -- S4 and S5 of the prefill path for MXFP4 routed weights
// (packed E2M1, one E8M0 scale per row and 32 columns) with E4M3 activations
// (power-of-two scale per 128 columns): the FP8 x FP4 precision of the GC MoE
// issue ("FP8 activations, packed FP4 routed weights") and of DeepGEMM's Mega
// MoE (news page: "FP8 x FP4"; sgl-deep-gemm commit list: "MXF4 kind").
//
// Grouped GEMM on tcgen05 with kind::mxf8f6f4.block_scale: the tensor cores
// apply both scales (per 32 k-elements) themselves, so every tile accumulates
// its whole K range in TMEM with no per-k-block promotion.
//   - weights: TMA with the 16U4_ALIGN16B type expands every 16 packed E2M1
//     codes (8 bytes) into a 16-byte slot, giving the same 128-byte rows per
//     128 k-elements as E4M3 and the same 128-byte-swizzled operand tiles;
//   - weight scales are stored in the tensor cores' block layout (a 512-byte
//     block per 128 rows x 128 columns) and arrive with one bulk copy per
//     k-block and operand;
//   - activation scales: the producer warp expands each routed row's E8M0
//     byte (the power-of-two block-128 scale) into the same block layout in
//     shared memory (the byte repeated for the four 32-element slices);
//   - the MMA warp copies the scale blocks into TMEM (tcgen05.cp 32x128b,
//     all four lane quarters) and issues four MMAs of K = 32 per k-block,
//     each selecting its scale byte.
// Tiles as in the E4M3 kernel, of 16, 64 or 112 routed rows (the MMA's N);
// the epilogue walks a tile in chunks of 32 accumulator columns.  Warp roles:
// warps 0 and 11 TMA producers (gate_up: gate weights and the activation
// tile with its scales / up weights; down: weights / activations and scales),
// warps 1 and 10 MMA issue (warp 1 also allocates TMEM), warps 2-9 epilogue
// from double-buffered TMEM accumulators.  With a few routed rows per tile an
// MMA instruction does little tensor work, and two issuing warps keep the
// tensor cores fed where one could not: gate_up issues gate and up from
// separate warps, down the two k-blocks of each stage into two partial
// accumulators that the epilogue adds.
//   S4 (gate_up): h = bf16(SiLU(g) * u), quantised per 128 features (the
//     tile's rows) to E4M3 with a power-of-two scale -> hq [N][F] and the
//     scale's E8M0 byte -> hsf [N][FBp].
//   S5 (down): y[slot, j] = w[slot] * acc (fp32, by original slot).
#include "common.cuh"
#include "gemm_common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kEpiF = 8;
constexpr int kMaxKBF = 128;          // k-blocks (of 128) per row supported

// k-blocks per pipeline stage of the 64-row and the 16-row tiles (measured:
// 1 per stage is 20-25 % slower at 64 rows, 3 per stage 4-5 % slower at 16)
constexpr int KPB64 = 2;
constexpr int KPB16 = 2;

template <bool GATE_UP, int BN>
struct CfgF {
    static_assert(BN == 16 || BN == 64 || BN == 112, "tile heights of the launcher");
    static constexpr int NUM_A = GATE_UP ? 2 : 1;
    // two MMA-issuing warps: the issue of block-scaled MMAs with few routed
    // rows, not the tensor cores, paces a k-block.  gate_up: one per A operand
    // (gate, up); down: one per k-block of a stage, each into its own partial
    // accumulator (summed by the epilogue)
    // and two TMA-issuing warps (A operands on one side, activations and their
    // scales on the other), for the same reason
    static constexpr int MMA1 = 2 + kEpiF, PROD1 = 3 + kEpiF;   // warps 10 and 11
    static constexpr int THREADS = 32 * (PROD1 + 1);
    static constexpr int MAX_STAGES = 12;
    // k-blocks per pipeline stage: one 3-D TMA load per operand and stage, so
    // that the producer's issue cost per byte halves
    static constexpr int KPB = BN == 16 ? KPB16 : KPB64;
    static constexpr int A_KB = kBM * 128;              // 128 rows x 128 E2M1 in 16-byte slots
    static constexpr int A_BYTES = KPB * A_KB;          // one operand, one stage: [kb][row][128]
    static constexpr int B_KB = BN * 128;
    static constexpr int B_BYTES = KPB * B_KB;          // [kb][routed row][128]
    static constexpr int SF_OFF = NUM_A * A_BYTES + B_BYTES;   // scale blocks: [A0][A1][B] x KPB
    static constexpr int STAGE_BYTES = (SF_OFF + (NUM_A + 1) * KPB * 512 + 1023) / 1024 * 1024;
    static constexpr int ACC = 2 * BN;                  // TMEM columns of one accumulator set
    static constexpr int SF_COL = 2 * ACC;              // scale columns after the two sets
    static constexpr int COLS_USED = SF_COL + 16;       // per MMA warp: A and B scale columns
    static constexpr int TMEM_COLS =
        COLS_USED <= 64 ? 64 : (COLS_USED <= 128 ? 128 : (COLS_USED <= 256 ? 256 : 512));
    static_assert(COLS_USED <= 512, "TMEM holds 512 columns");
    static constexpr int NC = BN / 2;                   // columns per epilogue thread
    static size_t smem_bytes(int E, int KBp, int stages) {
        return 1024 + (size_t)stages * STAGE_BYTES + 1024 + 2 * (size_t)BN * KBp +
               sizeof(float) * 5 * BN + 2 * sizeof(int) * (E + 1) + 64;
    }
};

struct GemmFArgs {
    const int32_t *offsets, *tiles;
    int E, MT, KB;
    int a_rows_per_expert, up_offset;
    const uint8_t *wsf;          // E8M0 weight scales in the block layout
    int64_t wsf_per_expert;      // bytes of one expert's weight scales
    const uint8_t *xsf;          // [N][KBp] E8M0 activation scales of the routed rows
    int KBp;                     // row stride of xsf (k-blocks rounded up to 16)
    uint8_t *hq;                 // gate_up: [N][F] e4m3
    uint8_t *hsf;                // gate_up: [N][FBp] E8M0
    int F, FBp;
    float *y;                    // down: [T*K][H]
    int H;
    const int32_t *perm;
    const float *topw;
    int32_t *status;
    int stages;                  // depth of the TMA ring (2..MAX_STAGES)
};

__device__ __forceinline__ void epi_sync_f() {
    asm volatile("bar.sync 2, %0;" ::"n"(32 * kEpiF) : "memory");
}

// CS (8, 16, 24 or 32, warp-uniform) consecutive TMEM columns of this warp's
// lanes into r[0..CS).
__device__ __forceinline__ void load_cols(uint32_t taddr, uint32_t (&r)[32], int CS) {
    if (CS == 32) {
        tmem_ld32(taddr, r);
    } else {
        if (CS & 16) tmem_ld16(taddr, r);
        if (CS & 8) tmem_ld8(taddr + (CS & 16), *reinterpret_cast<uint32_t(*)[8]>(r + (CS & 16)));
    }
    tmem_ld_wait();
}


template <bool GATE_UP, int BN>
__global__ void __launch_bounds__(CfgF<GATE_UP, BN>::THREADS, 1)
    grouped_gemm_mxf4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const GemmFArgs args) {
    using C = CfgF<GATE_UP, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    const int NST = args.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)NST * C::STAGE_BYTES);
    uint64_t *empty = full + C::MAX_STAGES;
    uint64_t *afull = empty + C::MAX_STAGES;
    uint64_t *aempty = afull + 2;
    uint64_t *tbar = aempty + 2;                                         // the two tables' barriers
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tbar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint8_t *sxs = smem + (size_t)NST * C::STAGE_BYTES + 1024;           // [2][BN][KBp]
    float *amax_s = reinterpret_cast<float *>(sxs + 2 * (size_t)BN * args.KBp);   // [4][BN]
    float *scale_s = amax_s + 4 * BN;                                    // [BN]
    int32_t *s_off = reinterpret_cast<int32_t *>(scale_s + BN);
    int32_t *s_tiles = s_off + (args.E + 1);
    const int KB = args.KB;

    const int warp = threadIdx.x >> 5, lane = lane_id();
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 2);
            mbar_init(&empty[s], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&afull[b], 2);
            mbar_init(&aempty[b], 32 * kEpiF);
            mbar_init(&tbar[b], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if ((warp == 0 || warp == C::PROD1) && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    // gate_up reads the permutation's outputs, so it waits for the kernels
    // before it.  down is launched only once gate_up, which waited for the
    // permutation, runs: the offsets and tiles are final, and only the h rows
    // and their scales (gate_up's outputs) need the wait, taken by the
    // producer that loads them -- the weights start streaming at once.
    if (GATE_UP) pdl_wait();
    for (int i = threadIdx.x; i <= args.E; i += blockDim.x) {
        s_off[i] = args.offsets[i];
        s_tiles[i] = args.tiles[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = s_tiles[args.E] * args.MT;
    pdl_launch_dependents();

    if (warp == 0 || warp == C::PROD1) {
        // ------------------------------------------------ TMA producers ----
        // producer p loads A operand p (if it exists); the activations and
        // their scales come from producer 0 in gate_up and producer 1 in down
        const int p = warp == 0 ? 0 : 1;
        const bool do_a = p < C::NUM_A;
        const bool do_b = GATE_UP ? p == 0 : p == 1;
        if (!GATE_UP && do_b) pdl_wait();
        const uint64_t pol_once = policy_evict_first();
        const uint64_t pol_x = policy_evict_last();
        const int KBp = args.KBp;
        int stage = 0, armed[C::MAX_STAGES];
        uint32_t phase = 0;
        for (int s = 0; s < C::MAX_STAGES; ++s) armed[s] = -1;
        bool ok = true;
        // the tile's activation-scale bytes (rows n -> sxs[buf][n][0..KBp)) with
        // one bulk copy into one of two tables, the next tile's requested as
        // soon as the current one is ready
        uint32_t tarmed = 0;                  // table loads issued and not yet waited for
        uint32_t tphase[2] = {0u, 0u};        // the next phase of each table's barrier
        auto load_table = [&](int wt_, int buf) {
            const Tile tn = decode_tile(wt_, s_off, s_tiles, args.E, args.MT, BN);
            mbar_arrive_expect_tx(&tbar[buf], (uint32_t)(tn.nrows * KBp));
            bulk_load(sxs + (size_t)buf * BN * KBp, args.xsf + (size_t)tn.row0 * KBp, (uint32_t)(tn.nrows * KBp),
                      &tbar[buf], pol_x);
            tarmed |= 1u << buf;
        };
        if (do_b && lane == 0 && (int)blockIdx.x < total) load_table(blockIdx.x, 0);
        int it = 0;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
            const Tile t = decode_tile(w, s_off, s_tiles, args.E, args.MT, BN);
            const int cur = it & 1;
            if (do_b) {
                ok = mbar_wait(&tbar[cur], tphase[cur], abort_flag);   // every lane reads the table
                ok = __all_sync(0xFFFFFFFFu, ok);
                if (!ok) break;
                tphase[cur] ^= 1u;
                if (lane == 0) {
                    tarmed &= ~(1u << cur);
                    if (w + (int)gridDim.x < total) load_table(w + gridDim.x, cur ^ 1);
                }
            }
            const uint64_t pol_w = s_tiles[t.e + 1] - s_tiles[t.e] > 1 ? pol_x : pol_once;
            const int arow = t.e * args.a_rows_per_expert + t.m * kBM + p * args.up_offset;
            const uint8_t *sfa = args.wsf + t.e * args.wsf_per_expert +
                                 ((size_t)t.m + (size_t)p * (args.up_offset / kBM)) * KB * 512;
            for (int kb0 = 0; kb0 < KB; kb0 += C::KPB) {
                const int nkb = min(C::KPB, KB - kb0);
                if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1, abort_flag);
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
                uint8_t *sA = ring + stage * C::STAGE_BYTES;
                uint8_t *sB = sA + C::NUM_A * C::A_BYTES;
                uint8_t *sF = sA + C::SF_OFF;
                if (do_b) {
                    // activation scales in the block layout: column n at word
                    // (n % 32) * 4 + n / 32 of its k-block's block, the byte
                    // repeated for the 4 slices
                    // lane l writes the words of rows l, l+32, l+64, l+96
                    const uint8_t *tb = sxs + (size_t)cur * BN * KBp;
#pragma unroll
                    for (int j = 0; j < C::KPB; ++j) {
                        uint32_t v[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int n = lane + 32 * i;
                            v[i] = ((n < t.nrows && j < nkb) ? (uint32_t)tb[(size_t)n * KBp + kb0 + j] : 127u) *
                                   0x01010101u;
                        }
                        *reinterpret_cast<uint4 *>(sF + (C::NUM_A * C::KPB + j) * 512 + 16 * lane) =
                            make_uint4(v[0], v[1], v[2], v[3]);
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    // boxes past the last k-block are zero-filled and still
                    // counted; the E2M1 loads count their packed bytes
                    const uint32_t bytes = (do_a ? C::A_BYTES / 2 + nkb * 512 : 0) + (do_b ? C::B_BYTES : 0);
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    armed[stage] = (int)phase;
                    if (do_a) {
                        tma_load_3d(sA + p * C::A_BYTES, &tmA, &full[stage], 0, arow, kb0, pol_w);
                        bulk_load(sF + p * C::KPB * 512, sfa + (size_t)kb0 * 512, nkb * 512, &full[stage],
                                  pol_w);
                    }
                    if (do_b) tma_load_3d(sB, &tmB, &full[stage], 0, t.row0, kb0, pol_x);
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
            // a table requested for a tile that the loop did not reach
            for (int b = 0; b < 2; ++b)
                if (((tarmed >> b) & 1u) && !mbar_wait(&tbar[b], tphase[b], &never))
                    atomicOr(args.status, DEV_TIMEOUT);
        }
    } else if (warp == 1 || warp == C::MMA1) {
        // ------------------------------------------------ MMA issue (role r) ----
        // gate_up: A operand r, every k-block; down: A operand 0, the k-blocks
        // j == r of each stage, into partial accumulator r
        static_assert(GATE_UP || C::KPB == 2, "down splits each stage's two k-blocks");
        const int r = warp == 1 ? 0 : 1;
        const int op = GATE_UP ? r : 0;
        if (lane == 0) {
            int stage = 0, ab = 0;
            uint32_t phase = 0, aphase = 0;
            bool ok = true;
            const uint32_t tsfa = tmem_base + C::SF_COL + 8 * r;      // A scales
            const uint32_t tsfb = tsfa + 4;                            // B scales
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
                const Tile t = decode_tile(w, s_off, s_tiles, args.E, args.MT, BN);
                const uint32_t idesc = idesc_mxf4_e4m3(kBM, (t.nrows + 15) & ~15);
                if (!mbar_wait(&aempty[ab], aphase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + ab * C::ACC + r * BN;
                for (int kb0 = 0; kb0 < KB; kb0 += C::KPB) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + stage * C::STAGE_BYTES);
                    const uint32_t sf = sa + C::SF_OFF;
                    for (int j = 0; j < C::KPB && kb0 + j < KB; ++j) {
                        if (!GATE_UP && j != r) continue;
                        tmem_cp_32x128b_x4(tsfa, sdesc_rows16(sf + (op * C::KPB + j) * 512));
                        tmem_cp_32x128b_x4(tsfb, sdesc_rows16(sf + (C::NUM_A * C::KPB + j) * 512));
                        const uint64_t da = sdesc_sw128(sa + op * C::A_BYTES + j * C::A_KB);
                        const uint64_t db = sdesc_sw128(sa + C::NUM_A * C::A_BYTES + j * C::B_KB);
                        const int first = GATE_UP ? 0 : r;   // this role's first k-block
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
        constexpr int NC = C::NC;
        const int ew = warp - 2, et = threadIdx.x - 64;
        const int eg = warp & 3;                 // TMEM lanes [32*eg, 32*eg+32)
        const int half = ew >> 2;                // columns [NC*half, NC*half+NC)
        const int row = eg * 32 + lane;
        int ab = 0;
        uint32_t aphase = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const Tile t = decode_tile(w, s_off, s_tiles, args.E, args.MT, BN);
            if (ok && !mbar_wait(&afull[ab], aphase, abort_flag)) {
                ok = false;
                *abort_flag = 1;
                atomicOr(args.status, DEV_TIMEOUT);
            }
            tc_fence_after();
            const uint32_t ta = tmem_base + ((uint32_t)(eg * 32) << 16) + ab * C::ACC + half * NC;
            // this thread's NC columns in chunks of up to 32: TMEM -> registers,
            // then h (gate_up) or y (down); the accumulator set goes back to
            // the MMA warps once the last chunk is loaded
#pragma unroll
            for (int c0 = 0; c0 < NC; c0 += 32) {
                const int CS = NC - c0 < 32 ? NC - c0 : 32;
                float ag[32], au[32];
                {
                    uint32_t r[32];
                    load_cols(ta + c0, r, CS);
#pragma unroll
                    for (int j = 0; j < 32; ++j) ag[j] = j < CS ? __uint_as_float(r[j]) : 0.f;
                    if (GATE_UP || KB > 1) {         // up, or down's second partial accumulator
                        load_cols(ta + BN + c0, r, CS);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float v = j < CS ? __uint_as_float(r[j]) : 0.f;
                            if (GATE_UP) au[j] = v; else ag[j] += v;
                        }
                    }
                }
                if (c0 + 32 >= NC) {
                    tc_fence_before();
                    mbar_arrive(&aempty[ab]);
                }
                const int cbase = half * NC + c0;        // first tile column of this chunk
                if (GATE_UP) {
                    // h = bf16(SiLU(g) * u) for this row (feature) and CS routed rows
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        ag[j] = __bfloat162float(__float2bfloat16_rn(silu_f(ag[j]) * au[j]));
                    // column max of |h| over this warp's 32 rows: lane l ends with column l
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = j < CS ? fabsf(ag[j]) : 0.f;
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
                    if (lane < CS) amax_s[eg * BN + cbase + lane] = v[0];
                    epi_sync_f();
                    if (et < 2 * CS) {                  // one thread per column of the chunk
                        const int col = (et / CS) * NC + c0 + et % CS;
                        const float m = fmaxf(fmaxf(amax_s[col], amax_s[BN + col]),
                                              fmaxf(amax_s[2 * BN + col], amax_s[3 * BN + col]));
                        const int k = fp8_block_exp(m);
                        scale_s[col] = pow2f(-k);
                        if (col < t.nrows)
                            args.hsf[(size_t)(t.row0 + col) * args.FBp + t.m] = (uint8_t)(k + 127);
                    }
                    epi_sync_f();
                    uint8_t *hp = args.hq + (size_t)(t.row0 + cbase) * args.F + t.m * kBM + row;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < CS && cbase + j < t.nrows)
                            hp[(size_t)j * args.F] = (uint8_t)(e4m3x2(ag[j] * scale_s[cbase + j], 0.f) & 0xFF);
                } else {
                    float *yp = args.y + t.m * kBM + row;
                    const int c = cbase + lane;
                    const int my_slot = (lane < CS && c < t.nrows) ? __ldg(args.perm + t.row0 + c) : 0;
                    const float my_w = (lane < CS && c < t.nrows) ? __ldg(args.topw + my_slot) : 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int slot = __shfl_sync(0xFFFFFFFFu, my_slot, j);
                        const float wj = __shfl_sync(0xFFFFFFFFu, my_w, j);
                        if (j < CS && cbase + j < t.nrows) yp[(size_t)slot * args.H] = wj * ag[j];
                    }
                }
            }
            if (++ab == 2) { ab = 0; aphase ^= 1; }
            if (GATE_UP) epi_sync_f();               // amax_s / scale_s are rewritten by the next tile
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <bool GATE_UP, int BN>
cudaError_t launch_oneF(const CUtensorMap &a, const CUtensorMap &b, const GemmFArgs &args,
                        cudaStream_t st) {
    using C = CfgF<GATE_UP, BN>;
    static std::atomic<int> attr_done[64];
    constexpr size_t kSmemMax = 227 * 1024;
    GemmFArgs af = args;
    af.stages = C::MAX_STAGES;
    while (af.stages > 2 && C::smem_bytes(args.E, args.KBp, af.stages) > kSmemMax) --af.stages;
    const size_t need = C::smem_bytes(args.E, args.KBp, af.stages);
    if (need > kSmemMax) return cudaErrorInvalidValue;
    const cudaError_t e = enable_max_dyn_smem((const void *)grouped_gemm_mxf4<GATE_UP, BN>, attr_done);
    if (e != cudaSuccess) return e;
    return launch_k(grouped_gemm_mxf4<GATE_UP, BN>, dim3(num_sms()), dim3(C::THREADS), need, st, true,
                    a, b, af);
}

}  // namespace

cudaError_t launch_gemms_mxf4(const void *w13, const uint8_t *w13sf, const void *w2,
                              const uint8_t *w2sf, const float *topw, int64_t T, int H, int F,
                              int E, int K, int bn, uint8_t *ws, const Workspace &L,
                              cudaStream_t st) {
    if (H / 128 > kMaxKBF || F / 128 > kMaxKBF) return cudaErrorInvalidValue;
    if (bn != kBNFp8 && bn != kBNFp8Decode && bn != kBNMxf4Wide) return cudaErrorInvalidValue;
    const uint64_t N = (uint64_t)T * K;
    const uint32_t kpb = bn == kBNFp8Decode ? CfgF<true, kBNFp8Decode>::KPB : CfgF<true, kBNFp8>::KPB;
    static_assert(CfgF<true, kBNFp8>::KPB == CfgF<true, kBNMxf4Wide>::KPB, "one map per height group");
    CUtensorMap ta, tb, tc, td;
    if (!make_tmap_e2m1(&ta, w13, (uint64_t)E * 2 * F, H, kpb) ||
        !make_tmap_e4m3_kb(&tb, ws + L.xperm, N, H, bn, kpb) ||
        !make_tmap_e2m1(&tc, w2, (uint64_t)E * H, F, kpb) ||
        !make_tmap_e4m3_kb(&td, ws + L.h, N, F, bn, kpb))
        return cudaErrorInvalidValue;
    GemmFArgs g = {};
    g.offsets = (const int32_t *)(ws + L.offsets);
    g.E = E;
    g.perm = (const int32_t *)(ws + L.perm);
    g.topw = topw;
    g.status = (int32_t *)(ws + L.status);
    g.hq = ws + L.h;
    g.hsf = ws + L.hscale;
    g.F = F;
    g.FBp = (int)align_up(F / 128, 16);
    g.y = (float *)(ws + L.y);
    g.H = H;

    GemmFArgs a1 = g;
    a1.tiles = (const int32_t *)(ws + L.tiles_g);
    a1.MT = F / kBM;
    a1.KB = H / 128;
    a1.a_rows_per_expert = 2 * F;
    a1.up_offset = F;
    a1.wsf = w13sf;
    a1.wsf_per_expert = (int64_t)2 * F * H / 32;
    a1.xsf = ws + L.xscale;
    a1.KBp = (int)align_up(H / 128, 16);

    GemmFArgs a2 = g;
    a2.tiles = (const int32_t *)(ws + L.tiles_d);
    a2.MT = H / kBM;
    a2.KB = F / 128;
    a2.a_rows_per_expert = H;
    a2.up_offset = 0;
    a2.wsf = w2sf;
    a2.wsf_per_expert = (int64_t)H * F / 32;
    a2.xsf = ws + L.hscale;
    a2.KBp = g.FBp;
    if (bn == kBNFp8Decode) {
        const cudaError_t err = launch_oneF<true, kBNFp8Decode>(ta, tb, a1, st);
        if (err != cudaSuccess) return err;
        return launch_oneF<false, kBNFp8Decode>(tc, td, a2, st);
    }
    if (bn == kBNMxf4Wide) {
        const cudaError_t err = launch_oneF<true, kBNMxf4Wide>(ta, tb, a1, st);
        if (err != cudaSuccess) return err;
        return launch_oneF<false, kBNMxf4Wide>(tc, td, a2, st);
    }
    const cudaError_t err = launch_oneF<true, kBNFp8>(ta, tb, a1, st);
    if (err != cudaSuccess) return err;
    return launch_oneF<false, kBNFp8>(tc, td, a2, st);
}

}  // namespace moe
