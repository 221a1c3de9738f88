// gemm_fp8.cu -- S4 and S5 of the prefill path for E4M3 expert weights with
// fp32 scales per (row, 128-column block) and E4M3 activations with
// power-of-two scales per 128 columns ("Supporting MegaKernel for DeepSeek
// Models", layer table: moe_w13_fp8_layer, moe_silu_mul_layer,
// bf16_to_fp8_quantize, moe_w2_fp8_layer).
//
// Grouped GEMM on tcgen05, E4M3 x E4M3 -> fp32, K = 32 per instruction.
// Because each 128-wide k-block has its own weight scale, every k-block's
// product goes to a TMEM "partial" buffer (three in rotation for 64-row
// gate_up tiles, three or seven for down, eight for 16-row tiles); epilogue
// warps read it and promote it into fp32 accumulators held in registers
// (column pairs on fp32x2 arithmetic) while later k-blocks' MMAs fill the
// other buffers.  64/128-row tiles run kind::mxf8f6f4.block_scale with the
// power-of-two activation scales as E8M0 block scales (the weights at 2^0),
// so the partial already carries x_scale exactly and
//     acc[row, col] += w_scale[row, kb] * partial[row, col]
// (the rounding of acc += (w_scale * x_scale) * P, which 16-row tiles on
// kind::f8f6f4 compute, from a table of the column scales).
//   S4 (gate_up):  tile = 128 features of expert e (gate rows and up rows,
//     two partials) x up to BN routed rows (64; 16 for a few tokens, where a
//     tile per (expert, 128 features) is all there is to spread over the
//     SMs).  h = bf16(SiLU(g) * u), then quantised per 128 features (the
//     tile's 128 rows): scale = smallest power of two with max|h|/scale <=
//     448, codes E4M3 -> hq [N][F], scales hs [N][F/128] (and their E8M0
//     bytes for the down GEMM's block scales).
//   S5 (down):  tile = 128 hidden rows x up to BN routed rows (64 or 128;
//     16 for a few tokens); y[slot, j] = w[slot] * acc  (fp32, by original
//     slot; combined later).
// Warp roles: warp 0 TMA producer (with block scales, the whole warp also
// writes each stage's scale block), warp 1 TMEM allocation + MMA issue, for
// gate_up with warp 10 (warp 1 the gate MMAs, warp 10 the up MMAs of every
// stage: one thread issuing all eight MMAs of a k-block paced the pipeline,
// ~85 SM cycles per small tcgen05.mma against ~32 of tensor work), warps 2-9
// promotion and epilogue (two warps per TMEM lane quarter, each owning BN/2
// of the BN columns; promotion skips 4-column chunks past the tile's routed
// rows).
#include "common.cuh"
#include "gemm_common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kEpi8 = 8;
constexpr int kMmaWarp2 = 2 + kEpi8;            // gate_up: the warp issuing the up MMAs
constexpr int kMaxKB8 = 128;          // k-blocks (of 128) per row supported

template <bool GATE_UP, int BN>
struct Cfg8 {
    static_assert(BN == 64 || BN == 16 || (!GATE_UP && BN == 128),
                  "one epilogue thread owns 32 or 8 columns (64 of the down GEMM's wide tiles)");
    static constexpr int NUM_A = GATE_UP ? 2 : 1;
    static constexpr int THREADS = 64 + 32 * kEpi8 + (GATE_UP ? 32 : 0);
    static constexpr int MAX_STAGES = 12;               // ring depth: chosen at launch to fill smem
    static constexpr int BOX = BN < 32 ? BN : (BN == 128 ? 64 : 32);   // routed rows per TMA box
    static constexpr int A_BYTES = kBM * 128;           // 128 rows x 128 e4m3
    static constexpr int B_BYTES = BN * 128;
    // BS: the power-of-two activation scales ride on the MMA as E8M0 block
    // scales (kind::mxf8f6f4.block_scale, E4M3 x E4M3, the weights at scale
    // 1): the tensor cores return x_scale * partial exactly, and the
    // promotion multiplies by the weight scale alone.  The 16-row tiles keep
    // kind::f8f6f4 and the promotion by both scales.
    static constexpr bool BS = BN != 16;
    static constexpr int SFB_OFF = NUM_A * A_BYTES + B_BYTES;   // a stage's activation-scale block (BS)
    static constexpr int STAGE_BYTES = BS ? (SFB_OFF + 512 + 1023) / 1024 * 1024 : NUM_A * A_BYTES + B_BYTES;
    static constexpr int PCOLS = NUM_A * BN;            // TMEM columns of one partial buffer
    // per MMA warp (BS): 4 TMEM columns of weight scales, 4 of activation scales
    static constexpr int SF_COLS = BS ? 8 * NUM_A : 0;
    // partial buffers in flight: the rest of TMEM's 512 columns (up to 8);
    // the fp32 accumulators live in registers
    static constexpr int NPB = (512 - SF_COLS) / PCOLS < 8 ? (512 - SF_COLS) / PCOLS : 8;
    static constexpr int SF_COL = NPB * PCOLS;
    static constexpr int COLS_USED = NPB * PCOLS + SF_COLS;
    static constexpr int TMEM_COLS = COLS_USED <= 128 ? 128 : (COLS_USED <= 256 ? 256 : 512);
    static_assert(COLS_USED <= 512, "TMEM holds 512 columns");
    static constexpr int NC = BN / 2;                   // columns per epilogue thread
    // 16-row tiles (one or two per CTA) stage the weight scales in shared
    // memory SG k-blocks ahead; wider tiles read them one k-block ahead.
    static constexpr bool STAGE_SCALES = BN == 16;
    static constexpr int SG = 8;                        // k-blocks per weight-scale group
    static constexpr int WSC_FLOATS = STAGE_SCALES ? 2 * NUM_A * kBM * (SG + 1) : 0;
    // after the ring: barriers (1 KB); BS: the unit weight-scale block (1 KB)
    // and the producer's table of the tile's activation scales [BN][KB];
    // otherwise the staged weight scales and the epilogue's [KB][BN] table;
    // then the h amax / scale arrays and the tile prefixes
    static size_t smem_bytes(int E, int KB, int stages) {
        const size_t table = BS ? 2 * (size_t)BN * ((KB + 15) & ~15) : sizeof(float) * BN * KB;
        return 1024 + (size_t)stages * STAGE_BYTES + 1024 + (BS ? 1024 : 0) + sizeof(float) * WSC_FLOATS +
               table + sizeof(float) * 5 * BN + 2 * sizeof(int) * (E + 1) + 64;
    }
};

struct Gemm8Args {
    const int32_t *offsets, *tiles;
    int E, MT, KB;
    int E_split;             // experts >= E_split read the second weight map and scales
    int a_rows_per_expert, up_offset;
    const float *wscale;     // [E_split * rows][KB] weight scales
    const float *wscale2;    // [(E - E_split) * rows][KB] weight scales of the second set
    const float *xscale;     // [N][KB] activation scales of the routed rows
    const uint8_t *xsb;      // BS: the same as E8M0 bytes, rows of KBp bytes
    int KBp;                 // round16(KB)
    uint8_t *hq;             // gate_up: [N][F] e4m3
    float *hs;               // gate_up: [N][F/128]
    uint8_t *hsb;            // gate_up (BS): the h scales' E8M0 bytes, rows of round16(F/128)
    int F;
    float *y;                // down: [T*K][H]
    int H;
    const int32_t *perm;
    const float *topw;
    int32_t *status;
    int stages;              // depth of the TMA ring (2..MAX_STAGES)
};

__device__ __forceinline__ void epi_sync() {
    asm volatile("bar.sync 2, %0;" ::"n"(32 * kEpi8) : "memory");
}

template <bool GATE_UP, int BN>
__global__ void __launch_bounds__(Cfg8<GATE_UP, BN>::THREADS, 1)
    grouped_gemm_fp8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                     const __grid_constant__ CUtensorMap tmB, const Gemm8Args args) {
    using C = Cfg8<GATE_UP, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    const int NST = args.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)NST * C::STAGE_BYTES);
    uint64_t *empty = full + C::MAX_STAGES;
    uint64_t *pfull = empty + C::MAX_STAGES;
    uint64_t *pempty = pfull + C::NPB;
    uint64_t *tbar = pempty + C::NPB;                                     // BS: the two tables' barriers
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tbar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint32_t *asf = reinterpret_cast<uint32_t *>(smem + (size_t)NST * C::STAGE_BYTES + 1024);   // BS: 512 B
    float *wsc = reinterpret_cast<float *>(smem + (size_t)NST * C::STAGE_BYTES + 1024 + (C::BS ? 1024 : 0));  // [2][NUM_A][128][SG+1]
    float *sx = wsc + C::WSC_FLOATS;              // [KB][BN] (epilogue; not BS)
    uint8_t *tbl = reinterpret_cast<uint8_t *>(sx);   // BS: two [BN][KBp] byte tables (producer)
    float *amax_s = C::BS ? reinterpret_cast<float *>(tbl + 2 * (size_t)BN * args.KBp)
                          : sx + BN * args.KB;                            // [4][BN]
    float *scale_s = amax_s + 4 * BN;                                     // [BN] 1 / h scale
    int32_t *s_off = reinterpret_cast<int32_t *>(scale_s + BN);
    int32_t *s_tiles = s_off + (args.E + 1);
    const int KB = args.KB;

    const int warp = threadIdx.x >> 5, lane = lane_id();
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::NUM_A);   // a commit per MMA-issuing warp
        }
        for (int b = 0; b < C::NPB; ++b) {
            mbar_init(&pfull[b], C::NUM_A);
            mbar_init(&pempty[b], 32 * kEpi8);
        }
        mbar_init(&tbar[0], 1);
        mbar_init(&tbar[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (C::BS && threadIdx.x < 128) {
        // the weights' block scales: 2^0 for every row and 32-element slice
        asf[threadIdx.x] = 0x7F7F7F7Fu;
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmA2);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();
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

    if (warp == 0) {
        // weight tiles: evict-first when only this tile reads them, kept
        // (evict-last) when the expert's other routed-row tiles, running on
        // neighbouring SMs at the same time, read them too.  Lane 0 waits and
        // issues the copies; with BS the whole warp stages the tile's
        // activation scales (asynchronous copies into sx[row][kb]) and writes
        // each stage's block of E8M0 scale bytes -- the exponent field of the
        // power-of-two scale -- in the layout tcgen05.cp 32x128b.warpx4 reads
        // (row n at word (n % 32) * 4 + n / 32, the byte repeated for the
        // four 32-element slices; rows past the tile at 2^0).
        const uint64_t pol_once = policy_evict_first();
        const uint64_t pol_x = policy_evict_last();
        int stage = 0, armed[C::MAX_STAGES];
        uint32_t phase = 0;
        for (int s = 0; s < C::MAX_STAGES; ++s) armed[s] = -1;
        bool ok = true;
        // BS: the tile's E8M0 scale bytes arrive with one bulk copy into one of
        // two tables, the next tile's requested as the current one is ready
        const int KBp = args.KBp;
        uint32_t tarmed = 0;                  // table loads issued and not yet waited for
        uint32_t tphase[2] = {0u, 0u};        // the next phase of each table's barrier
        auto load_table = [&](int wt_, int buf) {
            const Tile tn = decode_tile(wt_, s_off, s_tiles, args.E, args.MT, BN);
            mbar_arrive_expect_tx(&tbar[buf], (uint32_t)(tn.nrows * KBp));
            bulk_load(tbl + (size_t)buf * BN * KBp, args.xsb + (size_t)tn.row0 * KBp, (uint32_t)(tn.nrows * KBp),
                      &tbar[buf], pol_x);
            tarmed |= 1u << buf;
        };
        if (C::BS && lane == 0 && (int)blockIdx.x < total) load_table(blockIdx.x, 0);
        int it = 0;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
            const Tile t = decode_tile(w, s_off, s_tiles, args.E, args.MT, BN);
            const int cur = it & 1;
            if constexpr (C::BS) {
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
            const int nbox = (t.nrows + C::BOX - 1) / C::BOX;
            const uint32_t bytes = C::NUM_A * C::A_BYTES + nbox * C::BOX * 128;
            const bool second = t.e >= args.E_split;
            const CUtensorMap *mA = second ? &tmA2 : &tmA;
            const int arow = (second ? t.e - args.E_split : t.e) * args.a_rows_per_expert + t.m * kBM;
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1, abort_flag);
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
                uint8_t *sA = ring + stage * C::STAGE_BYTES;
                uint8_t *sB = sA + C::NUM_A * C::A_BYTES;
                if constexpr (C::BS) {
                    // lane l holds rows l, l+32, l+64, l+96: words 4l .. 4l+3
                    const uint8_t *tb = tbl + (size_t)cur * BN * KBp + kb;
                    uint32_t v[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = lane + 32 * i;
                        v[i] = (n < t.nrows ? (uint32_t)tb[(size_t)n * KBp] : 127u) * 0x01010101u;
                    }
                    *reinterpret_cast<uint4 *>(sA + C::SFB_OFF + 16 * lane) = make_uint4(v[0], v[1], v[2], v[3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    armed[stage] = (int)phase;
                    tma_load_2d(sA, mA, &full[stage], kb * 128, arow, pol_w);
                    if (GATE_UP)
                        tma_load_2d(sA + C::A_BYTES, mA, &full[stage], kb * 128,
                                    arow + args.up_offset, pol_w);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(sB + b * C::BOX * 128, &tmB, &full[stage], kb * 128,
                                    t.row0 + b * C::BOX, pol_x);
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
    } else if (warp == 1 || (GATE_UP && warp == kMmaWarp2)) {
        if (lane == 0) {
            // operand r: the gate (r = 0) or up (r = 1) weight tile and its
            // half of the partial buffer
            const int r = warp == 1 ? 0 : 1;
            int stage = 0, pb = 0;
            uint32_t phase = 0, pphase = 0;
            bool ok = true;
            // BS: this warp's scale columns in TMEM, weights (2^0, copied once)
            // and the k-block's activation scales
            const uint32_t tsfa = tmem_base + C::SF_COL + 8 * r, tsfb = tsfa + 4;
            if constexpr (C::BS) tmem_cp_32x128b_x4(tsfa, sdesc_rows16(smem_u32(asf)));
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
                const Tile t = decode_tile(w, s_off, s_tiles, args.E, args.MT, BN);
                const uint32_t idesc = C::BS ? idesc_e4m3_bs(kBM, (t.nrows + 15) & ~15)
                                             : idesc_e4m3(kBM, (t.nrows + 15) & ~15);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag) ||
                        !mbar_wait(&pempty[pb], pphase ^ 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + stage * C::STAGE_BYTES);
                    const uint64_t da = sdesc_sw128(sa + r * C::A_BYTES);
                    const uint64_t db = sdesc_sw128(sa + C::NUM_A * C::A_BYTES);
                    const uint32_t d = tmem_base + pb * C::PCOLS + r * BN;
                    if constexpr (C::BS) {
                        // the scale byte of k-step k (32 elements) selected by the
                        // descriptor and the scale addresses' top bits
                        tmem_cp_32x128b_x4(tsfb, sdesc_rows16(sa + C::SFB_OFF));
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t sel = (uint32_t)k << 30;
                            mma_mxf4_ss(d, da + 2 * k, db + 2 * k, idesc | idesc_sf_ids(k, k), tsfa | sel,
                                        tsfb | sel, k > 0 ? 1u : 0u);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 4; ++k) mma_e4m3_ss(d, da + 2 * k, db + 2 * k, idesc, k > 0);
                    }
                    mma_commit(&empty[stage]);
                    mma_commit(&pfull[pb]);
                    if (++stage == NST) { stage = 0; phase ^= 1; }
                    if (++pb == C::NPB) { pb = 0; pphase ^= 1; }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(args.status, DEV_TIMEOUT);
            }
        }
    } else {
        constexpr int NC = C::NC;
        const int ew = warp - 2, et = threadIdx.x - 64;
        const int eg = warp & 3;                 // TMEM lanes [32*eg, 32*eg+32)
        const int half = ew >> 2;                // columns [NC*half, NC*half+NC)
        const int row = eg * 32 + lane;
        int pb = 0;
        uint32_t pphase = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const Tile t = decode_tile(w, s_off, s_tiles, args.E, args.MT, BN);
            if constexpr (C::STAGE_SCALES) {
                epi_sync();
                for (int kb = ew; kb < KB; kb += kEpi8)
                    for (int c = lane; c < t.nrows; c += 32)
                        sx[kb * BN + c] = __ldg(args.xscale + (size_t)(t.row0 + c) * KB + kb);
                epi_sync();
            }
            const int live = t.nrows - half * NC;   // columns of this thread that hold routed rows
            // down: the slots and router weights of columns half*NC + 32*g + lane,
            // for the y stores at the end of the tile
            constexpr int NG = (NC + 31) / 32;
            int my_slot[NG];
            float my_w[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                my_slot[g] = 0;
                my_w[g] = 0.f;
                const int c = half * NC + 32 * g + lane;
                if (!GATE_UP && 32 * g + lane < NC && c < t.nrows) my_slot[g] = __ldg(args.perm + t.row0 + c);
            }
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const int c = half * NC + 32 * g + lane;
                if (!GATE_UP && 32 * g + lane < NC && c < t.nrows) my_w[g] = __ldg(args.topw + my_slot[g]);
            }
            // Weight scales of the tile's 128 rows: with STAGE_SCALES they
            // arrive in shared memory SG k-blocks at a time, one group ahead
            // (asynchronous copies); otherwise each is read one k-block ahead.
            const bool second = t.e >= args.E_split;
            const float *wsrc = (second ? args.wscale2 : args.wscale) +
                                ((size_t)(second ? t.e - args.E_split : t.e) * args.a_rows_per_expert + t.m * kBM) * KB;
            const float *wsg = wsrc + (size_t)row * KB;
            const float *wsu = wsrc + (size_t)(row + args.up_offset) * KB;
            auto issue_scales = [&](int kb0, int buf) {
                for (int i = et; i < C::NUM_A * kBM * C::SG; i += 32 * kEpi8) {
                    const int a = i / (kBM * C::SG), r = (i / C::SG) % kBM, q = i % C::SG;
                    if (kb0 + q < KB)
                        cp_async4(wsc + ((buf * C::NUM_A + a) * kBM + r) * (C::SG + 1) + q,
                                  wsrc + (size_t)(a * args.up_offset + r) * KB + kb0 + q);
                }
                cp_async_commit();
            };
            float ag[NC], au[NC];
#pragma unroll
            for (int j = 0; j < NC; ++j) ag[j] = 0.f;
#pragma unroll
            for (int j = 0; j < NC; ++j) au[j] = 0.f;
            float sg_next = 0.f, su_next = 0.f;
            if constexpr (C::STAGE_SCALES) {
                issue_scales(0, 0);
            } else {
                sg_next = __ldg(wsg);
                if (GATE_UP) su_next = __ldg(wsu);
            }
            for (int kb = 0; kb < KB; ++kb) {
                const int grp = kb / C::SG, q = kb - grp * C::SG, buf = grp & 1;
                float sg, su;
                if constexpr (!C::STAGE_SCALES) {
                    sg = sg_next;
                    su = su_next;
                    if (kb + 1 < KB) {
                        sg_next = __ldg(wsg + kb + 1);
                        if (GATE_UP) su_next = __ldg(wsu + kb + 1);
                    }
                } else {
                    if (q == 0) {
                        epi_sync();                  // everyone is done with the other buffer
                        if (kb + C::SG < KB) {
                            issue_scales(kb + C::SG, buf ^ 1);
                            cp_async_wait<1>();
                        } else {
                            cp_async_wait<0>();
                        }
                        epi_sync();                  // this group's scales are visible
                    }
                    sg = wsc[((buf * C::NUM_A) * kBM + row) * (C::SG + 1) + q];
                    su = GATE_UP ? wsc[((buf * C::NUM_A + 1) * kBM + row) * (C::SG + 1) + q] : 0.f;
                }
                if (ok && !mbar_wait(&pfull[pb], pphase, abort_flag)) {
                    ok = false;
                    *abort_flag = 1;
                    atomicOr(args.status, DEV_TIMEOUT);
                }
                tc_fence_after();
                const uint32_t tb = tmem_base + ((uint32_t)(eg * 32) << 16) + pb * C::PCOLS + half * NC;
                const float *sxk = sx + kb * BN + half * NC;   // this thread's column scales (not BS)
                // Load this thread's columns, hand the partial buffer back to
                // the MMA warp, then promote the live column pairs on fp32x2:
                // acc = (w_scale * x_scale) * partial + acc, or with BS, where
                // the partial already carries x_scale exactly (a power of two),
                // acc = w_scale * partial + acc -- the same single rounding
                uint32_t pr[NC];
                const float2 sg2 = make_float2(sg, sg), su2 = make_float2(su, su);
                auto promote_pairs = [&](float (&acc)[NC], const float2 s2) {
#pragma unroll
                    for (int c = 0; c < NC / 4; ++c) {
                        if (4 * c < live) {          // warp-uniform
                            float4 s4 = make_float4(1.f, 1.f, 1.f, 1.f);
                            if constexpr (!C::BS) s4 = *reinterpret_cast<const float4 *>(sxk + 4 * c);
#pragma unroll
                            for (int h2 = 0; h2 < 2; ++h2) {
                                const int q = 4 * c + 2 * h2;
                                const float2 p2 = make_float2(__uint_as_float(pr[q]), __uint_as_float(pr[q + 1]));
                                const float2 a2 = make_float2(acc[q], acc[q + 1]);
                                float2 r2;
                                if constexpr (C::BS) {
                                    r2 = __ffma2_rn(s2, p2, a2);
                                } else {
                                    const float2 sc = h2 == 0 ? make_float2(s4.x, s4.y) : make_float2(s4.z, s4.w);
                                    r2 = __ffma2_rn(__fmul2_rn(s2, sc), p2, a2);
                                }
                                acc[q] = r2.x;
                                acc[q + 1] = r2.y;
                            }
                        }
                    }
                };
                auto load_partial = [&](uint32_t taddr) {
                    if constexpr (NC == 64) {        // both halves behind one wait
                        tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(pr));
                        tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(pr + 32));
                    } else if constexpr (NC == 32) {
                        tmem_ld32(taddr, pr);
                    } else {
                        tmem_ld8(taddr, pr);
                    }
                    tmem_ld_wait();
                };
                // gate (and down) partial, then the up partial: one 32-column
                // load at a time keeps the live registers under the cap of ten
                // warps; the buffer goes back to the MMA warp after the last load
                load_partial(tb);
                if (!GATE_UP) {
                    tc_fence_before();
                    mbar_arrive(&pempty[pb]);
                }
                promote_pairs(ag, sg2);
                if (GATE_UP) {
                    load_partial(tb + BN);
                    tc_fence_before();
                    mbar_arrive(&pempty[pb]);
                    promote_pairs(au, su2);
                }
                if (++pb == C::NPB) { pb = 0; pphase ^= 1; }
            }
            if (GATE_UP) {
                // h = bf16(SiLU(g) * u) for this row (feature) and NC routed
                // rows (SiLU with the fast division, as the bf16 epilogue)
#pragma unroll
                for (int j = 0; j < NC; ++j) {
                    const float g = ag[j];
                    ag[j] = __bfloat162float(__float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * au[j]));
                }
                // column max of |h| over this warp's 32 rows: |h| >= 0, so the
                // fp32 bit patterns order like the values and one redux.sync
                // per column gives its max; lane j keeps column j
                float cmax = 0.f;
#pragma unroll
                for (int j = 0; j < NC; ++j) {
                    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(fabsf(ag[j])));
                    if (lane == j) cmax = __uint_as_float(m);
                }
                if (lane < NC) amax_s[eg * BN + half * NC + lane] = cmax;
                epi_sync();
                if (et < BN) {
                    const float m = fmaxf(fmaxf(amax_s[et], amax_s[BN + et]),
                                          fmaxf(amax_s[2 * BN + et], amax_s[3 * BN + et]));
                    const int k = fp8_block_exp(m);
                    scale_s[et] = 1.0f / pow2f(k);   // codes are h * (1 / scale), once per column
                    if (et < t.nrows) {
                        args.hs[(size_t)(t.row0 + et) * (args.F / 128) + t.m] = pow2f(k);
                        if constexpr (C::BS)
                            args.hsb[(size_t)(t.row0 + et) * ((args.F / 128 + 15) & ~15) + t.m] = (uint8_t)(k + 127);
                    }
                }
                epi_sync();
                uint8_t *hp = args.hq + (size_t)(t.row0 + half * NC) * args.F + t.m * kBM + row;
#pragma unroll
                for (int j = 0; j < NC; ++j)
                    if (j < live)
                        hp[(size_t)j * args.F] = (uint8_t)(e4m3x2(ag[j] * scale_s[half * NC + j], 0.f) & 0xFF);
            } else {
                // y[slot, row] = w[slot] * acc; lane l's slot and weight were
                // read at the start of the tile
                float *yp = args.y + t.m * kBM + row;
#pragma unroll
                for (int j = 0; j < NC; ++j) {
                    const int slot = __shfl_sync(0xFFFFFFFFu, my_slot[j / 32], j % 32);
                    const float wj = __shfl_sync(0xFFFFFFFFu, my_w[j / 32], j % 32);
                    if (j < live) yp[(size_t)slot * args.H] = wj * ag[j];
                }
            }
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
cudaError_t launch_one8(const CUtensorMap &a, const CUtensorMap &a2, const CUtensorMap &b,
                        const Gemm8Args &args, cudaStream_t st) {
    using C = Cfg8<GATE_UP, BN>;
    static std::atomic<int> attr_done[64];
    constexpr size_t kSmemMax = 227 * 1024;
    Gemm8Args a8 = args;
    a8.stages = C::MAX_STAGES;
    while (a8.stages > 2 && C::smem_bytes(args.E, args.KB, a8.stages) > kSmemMax) --a8.stages;
    const size_t need = C::smem_bytes(args.E, args.KB, a8.stages);
    if (need > kSmemMax) return cudaErrorInvalidValue;
    const cudaError_t e = enable_max_dyn_smem((const void *)grouped_gemm_fp8<GATE_UP, BN>, attr_done);
    if (e != cudaSuccess) return e;
    return launch_k(grouped_gemm_fp8<GATE_UP, BN>, dim3(num_sms()), dim3(C::THREADS), need, st, true,
                    a, a2, b, a8);
}

}  // namespace


cudaError_t launch_gemms_fp8(const void *w13, const float *w13s, const void *w2, const float *w2s,
                             const float *topw, int64_t T, int H, int F, int E, int K, int bn,
                             int bn_d, uint8_t *ws, const Workspace &L, cudaStream_t st,
                             const SharedSet &sh) {
    if (H / 128 > kMaxKB8 || F / 128 > kMaxKB8) return cudaErrorInvalidValue;
    if (bn != kBNFp8 && bn != kBNFp8Decode) return cudaErrorInvalidValue;
    if (bn_d != bn && !(bn == kBNFp8 && bn_d == kBNFp8DownWide)) return cudaErrorInvalidValue;
    const int box = bn < 32 ? bn : 32;
    // down: 128-row tiles (64-row boxes), or the gate_up tile rows
    const int box_d = bn_d == kBNFp8DownWide ? Cfg8<false, kBNFp8DownWide>::BOX : box;
    const uint64_t N = (uint64_t)T * K;
    CUtensorMap ta, tb, tc, td, ta2, tc2;
    const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const int E_split = E - sh.S;  // routed experts; ids E_split.. are the shared set
    if (!make_tmap(&ta, U8, 1, w13, (uint64_t)E_split * 2 * F, H, kBM) ||
        !make_tmap(&tb, U8, 1, ws + L.xperm, N, H, box) ||
        !make_tmap(&tc, U8, 1, w2, (uint64_t)E_split * H, F, kBM) ||
        !make_tmap(&td, U8, 1, ws + L.h, N, F, box_d))
        return cudaErrorInvalidValue;
    if (sh.S > 0) {
        if (!make_tmap(&ta2, U8, 1, sh.gate_up, (uint64_t)sh.S * 2 * F, H, kBM) ||
            !make_tmap(&tc2, U8, 1, sh.down, (uint64_t)sh.S * H, F, kBM))
            return cudaErrorInvalidValue;
    } else {
        ta2 = ta;
        tc2 = tc;
    }
    Gemm8Args g = {};
    g.offsets = (const int32_t *)(ws + L.offsets);
    g.E = E;
    g.E_split = E_split;
    g.perm = (const int32_t *)(ws + L.perm);
    g.topw = topw;
    g.status = (int32_t *)(ws + L.status);
    g.hq = ws + L.h;
    g.hs = (float *)(ws + L.hscale);
    g.hsb = ws + L.hsb;
    g.y = (float *)(ws + L.y);
    g.F = F;
    g.H = H;

    Gemm8Args a1 = g;
    a1.tiles = (const int32_t *)(ws + L.tiles_g);
    a1.MT = F / kBM;
    a1.KB = H / 128;
    a1.a_rows_per_expert = 2 * F;
    a1.up_offset = F;
    a1.wscale = w13s;
    a1.wscale2 = sh.S > 0 ? sh.gate_up_scale : w13s;
    a1.xscale = (const float *)(ws + L.xscale);
    a1.xsb = ws + L.xsb;
    a1.KBp = (a1.KB + 15) & ~15;

    Gemm8Args a2 = g;
    a2.tiles = (const int32_t *)(ws + L.tiles_d);
    a2.MT = H / kBM;
    a2.KB = F / 128;
    a2.a_rows_per_expert = H;
    a2.up_offset = 0;
    a2.wscale = w2s;
    a2.wscale2 = sh.S > 0 ? sh.down_scale : w2s;
    a2.xscale = (const float *)(ws + L.hscale);
    a2.xsb = ws + L.hsb;
    a2.KBp = (a2.KB + 15) & ~15;
    if (bn == kBNFp8Decode) {
        const cudaError_t err = launch_one8<true, kBNFp8Decode>(ta, ta2, tb, a1, st);
        if (err != cudaSuccess) return err;
        return launch_one8<false, kBNFp8Decode>(tc, tc2, td, a2, st);
    }
    const cudaError_t err = launch_one8<true, kBNFp8>(ta, ta2, tb, a1, st);
    if (err != cudaSuccess) return err;
    return bn_d == kBNFp8DownWide ? launch_one8<false, kBNFp8DownWide>(tc, tc2, td, a2, st)
                                  : launch_one8<false, kBNFp8>(tc, tc2, td, a2, st);
}

}  // namespace moe
