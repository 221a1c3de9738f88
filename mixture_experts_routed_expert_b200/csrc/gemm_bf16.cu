// gemm_bf16.cu -- S4 and S5 of the prefill path: grouped GEMMs over experts on
// the 5th-generation tensor cores (tcgen05, accumulators in TMEM, operands
// staged by TMA).
//
// S4 (gate_up, fused SiLU * up):  for the rows r of expert e (routed slots in
//   expert order),  h[r, f] = bf16( SiLU(G_e[f] . x_r) * (U_e[f] . x_r) ).
// S5 (down, fused router-weight scale):  y[s, j] = w[s] * (D_e[j] . h[r]),
//   s = perm[r] the original slot t*K+k; rows are written by slot so that the
//   combine can sum a token's K rows in k order.
// ("deepseek-ocr2-moe-experts" model card, description: grouped GEMM for
// prefill shapes, plain SiLU SwiGLU, router-weight scale + scatter-add.)
//
// Tile = (expert e, 128 weight rows, up to BN routed rows), "swap-AB": the
// weights sit on the MMA M=128 side and the routed rows on N, so small
// experts waste no MMA rows; N is rounded up to 16 per tile.
// Persistent: one CTA per SM walks the tile list (the tile count is read on
// the device; the host never synchronises).  Warp roles:
//   warp 0     TMA producer (4-stage shared-memory ring)
//   warp 1     TMEM allocation + MMA issue (one thread)
//   warps 2-9  epilogue: TMEM -> registers -> global (double-buffered TMEM);
//              two warps per TMEM lane quarter, alternating 32-column chunks
#include <cudaTypedefs.h>

#include "common.cuh"
#include "gemm_common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kStages = 4;
constexpr int kBK = 64;           // bf16 elements per k-block = one 128-byte swizzle row
// Routed rows per TMA box of the B operand, chosen at launch: 128 when the
// experts average >= 64 routed rows (one TMA per k-block; 32-row boxes paced
// the producer: T=2048 / 8192 layers 5 / 13 % slower), 32 for a few rows per
// expert (128-row boxes fetch unused rows: T=4 / 8 decode 12 / 19 % slower).
constexpr int kBoxRowsFew = 32, kBoxRowsMany = 128;
constexpr int kEpiWarps = 8;

template <bool GATE_UP>
struct Cfg {
    static constexpr int BN = GATE_UP ? kBNGateUp : kBNDown;
    static constexpr int NUM_A = GATE_UP ? 2 : 1;      // gate and up weight tiles
    // gate_up: one MMA-issuing warp per weight tile (warps 1 and 10): with
    // 128-row tiles and up to 128 routed rows the issue of the MMAs, not the
    // tensor pipe, paced a k-block when one warp issued both
    static constexpr int THREADS = 64 + 32 * kEpiWarps + 32 * (NUM_A - 1);
    static constexpr int A_BYTES = kBM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = NUM_A * A_BYTES + B_BYTES;
    static constexpr int ACC_COLS = NUM_A * BN;        // TMEM columns per accumulator set
    static constexpr int NUM_ACC = 512 / ACC_COLS;     // accumulator sets (2)
    static constexpr int RING_BYTES = kStages * STAGE_BYTES;
    static constexpr int STAGE_OUT = kEpiWarps * 32 * 32 * 2;   // h staging, 2 KB per warp
    static size_t smem_bytes(int E) {
        return RING_BYTES + 1024 + 1024 + STAGE_OUT + align_up(2 * sizeof(int) * (E + 1), 16);
    }
};

struct GemmArgs {
    const int32_t *offsets;      // [E+1] first routed row of each expert
    const int32_t *tiles;        // [E+1] prefix sum of row tiles per expert
    int E, MT, KB;               // experts, weight-row tiles per expert, k-blocks
    int E_split;                 // experts >= E_split read the second weight map (shared set)
    int a_rows_per_expert;       // 2F (gate_up) or H (down)
    int up_offset;               // F: row offset of the up half (gate_up)
    __nv_bfloat16 *h;            // gate_up output [N][F]
    int F;
    float *y;                    // down output [T*K][H]
    int H;
    const int32_t *perm;         // [N] routed row -> slot
    const float *topw;           // [T*K] router weights
    int32_t *status;
    int box_rows;                // routed rows per B box (kBoxRowsFew or kBoxRowsMany)
};

template <bool GATE_UP>
__global__ void __launch_bounds__(Cfg<GATE_UP>::THREADS, 1)
    grouped_gemm_bf16(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                      const __grid_constant__ CUtensorMap tmB, const GemmArgs args) {
    using C = Cfg<GATE_UP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::RING_BYTES);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + C::NUM_ACC;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + C::NUM_ACC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    __nv_bfloat16 *s_out = reinterpret_cast<__nv_bfloat16 *>(smem + C::RING_BYTES + 1024);
    int32_t *s_off = reinterpret_cast<int32_t *>(smem + C::RING_BYTES + 1024 + C::STAGE_OUT);
    int32_t *s_tiles = s_off + (args.E + 1);

    const int warp = threadIdx.x >> 5, lane = lane_id();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::NUM_A);
        }
        for (int a = 0; a < C::NUM_ACC; ++a) {
            mbar_init(&tfull[a], C::NUM_A);
            mbar_init(&tempty[a], 32 * kEpiWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmA2);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    pdl_wait();  // routed rows, offsets and tiles come from the previous kernels
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
        // ------------------------------------------------ TMA producer ----
        if (lane == 0) {
            // weight tiles: evict-first when only this tile reads them, kept
            // (evict-last) when the expert's other routed-row tiles, running
            // on neighbouring SMs at the same time, read them too
            const uint64_t pol_once = policy_evict_first();
            const uint64_t pol_x = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            int armed[kStages];
#pragma unroll
            for (int s = 0; s < kStages; ++s) armed[s] = -1;
            bool ok = true;
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
                const Tile t = decode_tile(w, s_off, s_tiles, args.E, args.MT, C::BN);
                const uint64_t pol_w = s_tiles[t.e + 1] - s_tiles[t.e] > 1 ? pol_x : pol_once;
                const int box_rows = args.box_rows;
                const int nbox = (t.nrows + box_rows - 1) / box_rows;
                const uint32_t bytes = C::NUM_A * C::A_BYTES + nbox * box_rows * 128;
                const bool second = t.e >= args.E_split;
                const CUtensorMap *mA = second ? &tmA2 : &tmA;
                const int arow = (second ? t.e - args.E_split : t.e) * args.a_rows_per_expert + t.m * kBM;
                for (int kb = 0; kb < args.KB; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t *sA = ring + stage * C::STAGE_BYTES;
                    uint8_t *sB = sA + C::NUM_A * C::A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    armed[stage] = (int)phase;
                    tma_load_2d(sA, mA, &full[stage], kb * kBK, arow, pol_w);
                    if (GATE_UP)
                        tma_load_2d(sA + C::A_BYTES, mA, &full[stage], kb * kBK,
                                    arow + args.up_offset, pol_w);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(sB + b * box_rows * 128, &tmB, &full[stage], kb * kBK,
                                    t.row0 + b * box_rows, pol_x);
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(args.status, DEV_TIMEOUT);
            }
            // drain: every armed stage must have landed before the CTA exits
            volatile int never = 0;
            for (int s = 0; s < kStages; ++s)
                if (armed[s] >= 0 && !mbar_wait(&full[s], (uint32_t)armed[s], &never))
                    atomicOr(args.status, DEV_TIMEOUT);
        }
    } else if (warp == 1 || warp == 2 + kEpiWarps) {
        // ------------------------------------------------ MMA issuer ------
        const int r = warp == 1 ? 0 : 1;          // weight tile (gate, up) of this warp
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
                const Tile t = decode_tile(w, s_off, s_tiles, args.E, args.MT, C::BN);
                const int N = (t.nrows + 15) & ~15;
                const uint32_t idesc = idesc_bf16(kBM, N);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + acc * C::ACC_COLS + r * C::BN;
                for (int kb = 0; kb < args.KB; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + stage * C::STAGE_BYTES);
                    const uint64_t da = sdesc_sw128(sa + r * C::A_BYTES);
                    const uint64_t db = sdesc_sw128(sa + C::NUM_A * C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        mma_bf16_ss(d, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
                    mma_commit(&empty[stage]);
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                if (++acc == C::NUM_ACC) { acc = 0; acc_phase ^= 1; }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(args.status, DEV_TIMEOUT);
            }
        }
    } else {
        // ------------------------------------------------ epilogue --------
        const int ew = warp - 2;                // 0 .. kEpiWarps-1
        const int eg = warp & 3;                // TMEM lanes [32*eg, 32*eg+32)
        const int half = ew >> 2;               // which 32-column chunks
        const int row = eg * 32 + lane;         // weight row inside the tile
        __nv_bfloat16 *stg = s_out + ew * 32 * 32;   // [32 rows][32 features]
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const Tile t = decode_tile(w, s_off, s_tiles, args.E, args.MT, C::BN);
            if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
                *abort_flag = 1;
                atomicOr(args.status, DEV_TIMEOUT);
                break;
            }
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(eg * 32) << 16) + acc * C::ACC_COLS;
            for (int c0 = half * 32; c0 < t.nrows; c0 += 64) {
                uint32_t g[32];
                tmem_ld32(tb + c0, g);
                if (GATE_UP) {
                    uint32_t u[32];
                    tmem_ld32(tb + C::BN + c0, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float gv = __uint_as_float(g[j]);
                        const float hv = __fdividef(gv, 1.0f + __expf(-gv)) * __uint_as_float(u[j]);
                        stg[j * 32 + lane] = __float2bfloat16_rn(hv);
                    }
                    __syncwarp();
                    // 32 routed rows x 64 bytes: four lanes per row, 16 bytes each
                    const int q = lane & 3;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = (lane >> 2) + 8 * i;
                        if (c0 + r < t.nrows) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(stg + r * 32 + q * 8);
                            *reinterpret_cast<uint4 *>(args.h + (size_t)(t.row0 + c0 + r) * args.F +
                                                       t.m * kBM + eg * 32 + q * 8) = v;
                        }
                    }
                    __syncwarp();
                } else {
                    tmem_ld_wait();
                    const int c = c0 + lane;
                    const int my_slot = (c < t.nrows) ? __ldg(args.perm + t.row0 + c) : 0;
                    const float my_w = (c < t.nrows) ? __ldg(args.topw + my_slot) : 0.f;
                    float *yp = args.y + t.m * kBM + row;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int slot = __shfl_sync(0xFFFFFFFFu, my_slot, j);
                        const float wj = __shfl_sync(0xFFFFFFFFu, my_w, j);
                        if (c0 + j < t.nrows) yp[(size_t)slot * args.H] = wj * __uint_as_float(g[j]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (++acc == C::NUM_ACC) { acc = 0; acc_phase ^= 1; }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

template <bool GATE_UP>
cudaError_t launch_one(const CUtensorMap &a, const CUtensorMap &a2, const CUtensorMap &b,
                       const GemmArgs &args,
                       cudaStream_t st) {
    using C = Cfg<GATE_UP>;
    const size_t smem = C::smem_bytes(args.E);
    static std::atomic<int> attr_done[64];
    const cudaError_t e = enable_max_dyn_smem((const void *)grouped_gemm_bf16<GATE_UP>, attr_done);
    if (e != cudaSuccess) return e;
    return launch_k(grouped_gemm_bf16<GATE_UP>, dim3(num_sms()), dim3(C::THREADS), smem, st, true, a,
                    a2, b, args);
}

}  // namespace

cudaError_t launch_gemms_bf16(const void *gate_up, const void *down, const float *topw, int64_t T,
                              int H, int F, int E, int K, uint8_t *ws, const Workspace &L,
                              cudaStream_t st, const SharedSet &sh) {
    const uint64_t N = (uint64_t)T * K;
    const int box_rows = N >= (uint64_t)64 * E ? kBoxRowsMany : kBoxRowsFew;
    CUtensorMap ta, tb, tc, td, ta2, tc2;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int E_split = E - sh.S;  // routed experts; ids E_split.. are the shared set
    if (!make_tmap(&ta, BF, 2, gate_up, (uint64_t)E_split * 2 * F, H, kBM) ||
        !make_tmap(&tb, BF, 2, ws + L.xperm, N, H, box_rows) ||
        !make_tmap(&tc, BF, 2, down, (uint64_t)E_split * H, F, kBM) ||
        !make_tmap(&td, BF, 2, ws + L.h, N, F, box_rows))
        return cudaErrorInvalidValue;
    if (sh.S > 0) {
        if (!make_tmap(&ta2, BF, 2, sh.gate_up, (uint64_t)sh.S * 2 * F, H, kBM) ||
            !make_tmap(&tc2, BF, 2, sh.down, (uint64_t)sh.S * H, F, kBM))
            return cudaErrorInvalidValue;
    } else {
        ta2 = ta;
        tc2 = tc;
    }
    GemmArgs g = {};
    g.offsets = (const int32_t *)(ws + L.offsets);
    g.E = E;
    g.E_split = E_split;
    g.box_rows = box_rows;
    g.perm = (const int32_t *)(ws + L.perm);
    g.topw = topw;
    g.status = (int32_t *)(ws + L.status);
    g.h = (__nv_bfloat16 *)(ws + L.h);
    g.y = (float *)(ws + L.y);
    g.F = F;
    g.H = H;

    GemmArgs a1 = g;
    a1.tiles = (const int32_t *)(ws + L.tiles_g);
    a1.MT = F / kBM;
    a1.KB = H / kBK;
    a1.a_rows_per_expert = 2 * F;
    a1.up_offset = F;
    cudaError_t err = launch_one<true>(ta, ta2, tb, a1, st);
    if (err != cudaSuccess) return err;

    GemmArgs a2 = g;
    a2.tiles = (const int32_t *)(ws + L.tiles_d);
    a2.MT = H / kBM;
    a2.KB = F / kBK;
    a2.a_rows_per_expert = H;
    a2.up_offset = 0;
    return launch_one<false>(tc, tc2, td, a2, st);
}

}  // namespace moe
