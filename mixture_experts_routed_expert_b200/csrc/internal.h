// internal.h -- host-side declarations shared by the translation units of
// libmoe_b200 (launchers, workspace layout, tile configuration).
#pragma once

#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

// ---- grouped-GEMM tiling (shared by the scheduler in the permute kernels) --
constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBNGateUp = 128;    // routed rows (tokens) per gate_up tile
constexpr int kBNDown = 256;      // routed rows per down tile
constexpr int kBNFp8 = 64;        // routed rows per tile of both E4M3 GEMMs
constexpr int kBNFp8Decode = 16;  // the same GEMMs for a few tokens (decode entry)
constexpr int kBNFp8DownWide = 128;  // E4M3 down GEMM tiles with 64-row gate_up tiles
constexpr int kBNMxf4Wide = 112;  // MXFP4 GEMMs with many routed rows per expert

// ---- workspace layout ------------------------------------------------------
// Every workspace starts with a header of kWorkspaceHeaderBytes: the int32
// device status word at offset 0 and, from kWorkspaceCounterOffset, the
// counters of the fused bf16 decode kernel.  The header is zero before a
// workspace's first use and every call that completes leaves it so
// (counters are reset by the kernel that used them).
constexpr size_t kWorkspaceHeaderBytes = 8192;
constexpr size_t kWorkspaceCounterOffset = 256;

struct Workspace {
    size_t status;        // int32 device status word
    size_t ctr;           // fused MXFP4 decode: int32 work counters (cleared with the status word)
    size_t ctr_bytes;
    size_t counts;        // [E] int32
    size_t offsets;       // [E+1] int32
    size_t tiles_g;       // [E+1] int32 prefix of gate_up row tiles per expert
    size_t tiles_d;       // [E+1] int32 prefix of down row tiles per expert
    size_t perm;          // [N] int32
    size_t inv;           // [N] int32
    size_t xperm;         // [N][H] bf16 | e4m3
    size_t xscale;        // [N][H/128] f32 (e4m3 only)
    size_t h;             // [N][F] bf16 | e4m3
    size_t hscale;        // [N][F/128] f32 (e4m3 only)
    size_t xsb, hsb;      // e4m3: the same scales as E8M0 bytes, rows of round16(H/128) / round16(F/128)
    size_t y;             // [N][H] f32 (weighted down-projection rows, by slot)
    size_t total;
};
Workspace prefill_workspace(int64_t T, int H, int F, int E, int K, moe_wtype_t wt);

// Fused bf16 decode (one kernel): header (status; per touched expert the
// published h groups and the finished down rows; per (token, 32-row block)
// the combine arrivals), then h [T*K][F] bf16 and y [T*K][H] fp32 by slot.
struct FusedDecodeWorkspace {
    size_t status, hdone, hused, ctr, h, y, total;
};
FusedDecodeWorkspace fused_decode_workspace(int T, int H, int F, int K);
// True when the fused bf16 decode kernel serves these sizes on the current
// device (T <= 16, T*K <= 64, H, F <= 2048 and the shared-memory plan fits).
bool decode_fused_bf16_fits(int T, int H, int F, int K);
cudaError_t launch_decode_fused_bf16(const void *x, const void *gate_up, const void *down,
                                     const int32_t *idx, const float *w, int T, int H, int F,
                                     int E, int K, uint8_t *ws, const FusedDecodeWorkspace &L,
                                     void *out, cudaStream_t st, int withhold = -1);

struct DecodeWorkspace {
    size_t sync;          // int32 status words (4)
    size_t h;             // [T*K][F] bf16, by slot
    size_t total;
};
// True when the decode kernel's shared-memory staging fits these sizes.
bool decode_shape_ok(int H, int F);
DecodeWorkspace decode_workspace(int T, int H, int F, int E, int K, moe_wtype_t wt);

constexpr int kDecodeMaxSlots = 64;  // T*K served by the decode kernels
constexpr int kDecodeMaxT = 16;
constexpr int kFusedMaxSlots = 64;   // T*K served by the fused MXFP4 decode kernel
constexpr int kFusedMaxT = 16;

// Host-side argument checks of the forward entry points (MOE_OK when valid).
moe_status_t validate_forward(const void *x, const void *gu, const void *dn, const int32_t *idx,
                              const float *w, int K, int T, int H, int F, int E, moe_wtype_t wt,
                              const void *gus, const void *dns, const void *out);
// True when T tokens x K slots are served by the decode kernels.
bool decode_path_fits(int T, int K, int H, int F);

// Always-active (shared) experts served as extra expert ids E_routed..E_routed+S-1
// of the grouped GEMMs; their weights live in their own tensors.
struct SharedSet {
    int S = 0;                          // number of shared experts (0: none)
    const void *gate_up = nullptr;      // [S][2F][H]
    const void *down = nullptr;         // [S][H][F]
    const float *gate_up_scale = nullptr;  // E4M3: [S][2F][H/128]
    const float *down_scale = nullptr;     // E4M3: [S][H][F/128]
};

// ---- launchers (return cudaSuccess or the launch error) --------------------
int num_sms();
// Lets `kernel` take the device's opt-in limit of dynamic shared memory (less
// its static shared memory), once per device; `done` is the caller's
// per-device flag array (device ordinals modulo 64).  Setting the attribute
// is idempotent, so concurrent host threads race only on the atomic flag.
cudaError_t enable_max_dyn_smem(const void *kernel, std::atomic<int> (&done)[64]);

cudaError_t launch_permute(const int32_t *idx, int64_t n_slots, int E, int bn_g, int bn_d,
                           uint8_t *ws, const Workspace &L, cudaStream_t st);
// zero / nzero (MXFP4 only): int32 counters that the kernel also clears.
cudaError_t launch_permute_gather(const void *x, const int32_t *idx, int64_t n_slots, int K, int H,
                                  int E, int bn_g, int bn_d, moe_wtype_t wt, uint8_t *ws,
                                  const Workspace &L, cudaStream_t st, int32_t *zero = nullptr,
                                  int nzero = 0);
cudaError_t launch_debug_outputs(const int32_t *idx, int64_t n_slots, int E, const uint8_t *ws,
                                 const Workspace &L, int32_t *counts, int32_t *offsets,
                                 int32_t *perm, int32_t *inv, cudaStream_t st);
cudaError_t launch_gemms_bf16(const void *gate_up, const void *down, const float *topw, int64_t T,
                              int H, int F, int E, int K, uint8_t *ws, const Workspace &L,
                              cudaStream_t st, const SharedSet &sh = SharedSet());
// E counts the routed and the shared experts (sh.S of them, the last ids).
// bn: gate_up tile rows, kBNFp8 or kBNFp8Decode; bn_d: down tile rows, bn or
// (with kBNFp8) kBNFp8DownWide; both must match the permutation's tile prefixes.
cudaError_t launch_gemms_fp8(const void *w13, const float *w13s, const void *w2, const float *w2s,
                             const float *topw, int64_t T, int H, int F, int E, int K, int bn,
                             int bn_d, uint8_t *ws, const Workspace &L, cudaStream_t st,
                             const SharedSet &sh = SharedSet());
// residual: optional [T][H] bf16 added after the slot sum (nullptr: none).
// The fused MXFP4 decode kernel (one launch for T <= kFusedMaxT,
// T*K <= kFusedMaxSlots): counters, h and y in the workspace L.
bool fused_mxf4_fits(int T, int K);
cudaError_t launch_fused_mxf4(const void *x, const void *w13, const uint8_t *w13sf, const void *w2,
                              const uint8_t *w2sf, const int32_t *idx, const float *w, int T, int H,
                              int F, int E, int K, uint8_t *ws, const Workspace &L, void *out,
                              cudaStream_t st);
// MXFP4 weights (packed E2M1 + E8M0 scales in the block layout), E4M3
// activations with E8M0 scale bytes in the workspace's scale regions.
cudaError_t launch_gemms_mxf4(const void *w13, const uint8_t *w13sf, const void *w2,
                              const uint8_t *w2sf, const float *topw, int64_t T, int H, int F,
                              int E, int K, int bn, uint8_t *ws, const Workspace &L,
                              cudaStream_t st);
cudaError_t launch_combine(const int32_t *idx, int64_t T, int H, int E, int K, const uint8_t *ws,
                           const Workspace &L, void *out, cudaStream_t st,
                           const void *residual = nullptr);
// out[t] = bf16(sum over valid k, ascending, of y[t*K+k]) for caller rows y.
cudaError_t launch_combine_rows(const float *y, const int32_t *idx, int64_t T, int H, int E, int K,
                                void *out, cudaStream_t st);
// idx2/w2 [T][K+S]: the K routed slots (ids outside [0,E) -> -1), then the S
// shared ids E..E+S-1 with weight 1.
cudaError_t launch_widen_routing(const int32_t *idx, const float *w, int64_t T, int E, int K,
                                 int S, int32_t *idx2, float *w2, cudaStream_t st);
cudaError_t launch_decode_bf16(const void *x, const void *gate_up, const void *down,
                               const int32_t *idx, const float *w, int T, int H, int F, int E,
                               int K, uint8_t *ws, const DecodeWorkspace &L, void *out,
                               cudaStream_t st, const SharedSet &sh = SharedSet(),
                               const void *residual = nullptr);
cudaError_t launch_quantize(const void *x, int64_t rows, int cols, void *xq, float *scale,
                            cudaStream_t st);
// One kernel copying bytes (a multiple of 16) from src to dst, src read with
// cache-volatile loads (it may be mapped pinned host memory).
cudaError_t launch_stage_copy(const void *src, void *dst, size_t bytes, cudaStream_t st);
cudaError_t launch_route(const float *logits, const float *bias, int64_t T, int E, int num_groups,
                         int topk_group, int top_k, float scale, int32_t *idx, float *w,
                         int32_t *offsets, cudaStream_t st);

// cudaLaunchKernelEx with optional programmatic dependent launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace moe
