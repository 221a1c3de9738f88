// api.cu -- the C ABI of libmoe_b200 (declared in include/moe_b200.h):
// host-side validation, workspace layout and dispatch to the kernels.
// Nothing here allocates device memory; only moe_workspace_status waits for
// the device (it reads the status word back).
#include <string.h>

#include <algorithm>

#include "internal.h"

namespace moe {

int num_sms() {
    static std::atomic<int> cache[64];   // per device ordinal (modulo 64); 0 = not read yet
    int dev = 0;
    cudaGetDevice(&dev);
    int c = cache[dev & 63].load(std::memory_order_relaxed);
    if (c == 0) {
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0)
            c = 148;
        cache[dev & 63].store(c, std::memory_order_relaxed);
    }
    return c;
}

cudaError_t enable_max_dyn_smem(const void *kernel, std::atomic<int> (&done)[64]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::atomic<int> &d = done[dev & 63];
    if (d.load(std::memory_order_acquire)) return cudaSuccess;
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - (int)fa.sharedSizeBytes);
    if (e != cudaSuccess) return e;
    d.store(1, std::memory_order_release);
    return cudaSuccess;
}

namespace {

struct Bump {
    size_t off = 0;
    size_t take(size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    }
};

constexpr int32_t DEV_TIMEOUT_BIT = 1;   // the kernels' DEV_TIMEOUT status bit

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

moe_status_t from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    cudaGetLastError();  // clear a sticky launch error so later calls can proceed
    return e == cudaErrorInvalidValue ? MOE_ERR_INVALID_ARG : MOE_ERR_CUDA;
}

bool dims_ok(int64_t T, int H, int F, int E, int K) {
    return T >= 0 && T <= (1 << 24) && H >= 128 && H % 128 == 0 && H <= 16384 && F >= 128 &&
           F % 128 == 0 && F <= 16384 && E >= 1 && E <= 1024 && K >= 1 && K <= 16 &&
           (int64_t)T * K < (1LL << 31) / 16;
}

}  // namespace

Workspace prefill_workspace(int64_t T, int H, int F, int E, int K, moe_wtype_t wt) {
    const int64_t N = T * K;
    const size_t eb = (wt == MOE_W_BF16) ? 2 : 1;
    // activation scales: fp32 [N][H/128] (E4M3 weights) or E8M0 bytes in rows
    // of round16(H/128) (MXFP4 weights); the same for h with F
    auto scale_bytes = [&](int cols) -> size_t {
        if (wt == MOE_W_BF16) return 0;
        if (wt == MOE_W_MXFP4) return (size_t)N * align_up(cols / 128, 16);
        return sizeof(float) * (size_t)N * (cols / 128);
    };
    Workspace L;
    Bump b;
    L.status = 0;                       // in the header (see internal.h)
    b.off = kWorkspaceHeaderBytes;
    // work counters of the fused MXFP4 decode kernel (the permutation kernel
    // clears them at the start of every call)
    L.ctr = b.off;
    L.ctr_bytes = (wt == MOE_W_MXFP4 && fused_mxf4_fits((int)T, K))
                      ? sizeof(int32_t) * ((size_t)kFusedMaxSlots + (size_t)T * (H / 128))
                      : 0;
    b.off = align_up(L.ctr + L.ctr_bytes, 256);
    L.counts = b.take(sizeof(int32_t) * E);
    L.offsets = b.take(sizeof(int32_t) * (E + 1));
    L.tiles_g = b.take(sizeof(int32_t) * (E + 1));
    L.tiles_d = b.take(sizeof(int32_t) * (E + 1));
    L.perm = b.take(sizeof(int32_t) * (size_t)std::max<int64_t>(N, 1));
    L.inv = b.take(sizeof(int32_t) * (size_t)std::max<int64_t>(N, 1));
    L.xperm = b.take(eb * (size_t)N * H);
    L.xscale = b.take(scale_bytes(H));
    L.h = b.take(eb * (size_t)N * F);
    L.hscale = b.take(scale_bytes(F));
    L.xsb = b.take(wt == MOE_W_FP8_E4M3 ? (size_t)N * align_up(H / 128, 16) : 0);
    L.hsb = b.take(wt == MOE_W_FP8_E4M3 ? (size_t)N * align_up(F / 128, 16) : 0);
    L.y = b.take(sizeof(float) * (size_t)N * H);
    L.total = b.off;
    return L;
}

DecodeWorkspace decode_workspace(int T, int H, int F, int E, int K, moe_wtype_t wt) {
    (void)H;
    (void)E;
    (void)wt;                        // only bf16 weights take the gather-GEMV kernels
    const size_t N = (size_t)T * K;
    DecodeWorkspace L;
    Bump b;
    L.sync = 0;                         // in the header (see internal.h)
    b.off = kWorkspaceHeaderBytes;
    L.h = b.take(2 * N * F);
    L.total = b.off;
    return L;
}

}  // namespace moe

using namespace moe;

namespace {

bool decode_fits(int T, int K, int H, int F) {
    return T <= kDecodeMaxT && T * K <= kDecodeMaxSlots && decode_shape_ok(H, F);
}

// True when the gather-GEMV decode kernels serve T tokens: bf16 weights and
// at most kGemvMaxSlots slots (beyond that the grouped GEMMs, which stream
// each touched expert once through TMA, are faster: OCR-2 shape T=4 / 8 ->
// 47 / 64 us against 51 / 90 us).  E4M3 weights take the grouped GEMMs with
// 16-row activation tiles instead.
constexpr int kGemvMaxSlots = 16;
bool decode_serves(int T, int K, int H, int F, moe_wtype_t wt) {
    return wt == MOE_W_BF16 && T * K <= kGemvMaxSlots && decode_fits(T, K, H, F);
}
// Sizes of the one-kernel bf16 decode (decode_fused.cu), served by
// moe_experts_decode_fused.  moe_experts_decode keeps the two-kernel GEMV
// pair / grouped GEMMs, faster on every measured OCR-2 size (graph replay,
// isolated / back to back, us): T=1 24.6 / 17.8 vs 26.6 / 21.6; T=2
// 32.8 / 27.6 vs 36.9 / 30.5; T=4 (grouped) 47.1 / 42.6 vs 49.2 / 45.9;
// T=8 (grouped) 65.5 / 57.4 vs 73.7 / 71.1.
bool fused_decode_sizes(int T, int K, int H, int F, moe_wtype_t wt) {
    return wt == MOE_W_BF16 && T <= kDecodeMaxT && T * K <= kDecodeMaxSlots && H <= 2048 &&
           F <= 2048;
}
// Tile height of the E4M3 and MXFP4 grouped GEMMs: 16 routed rows for
// decode-sized calls and whenever the experts average <= 6 routed rows (a
// 64-row tile then loads and multiplies mostly unused rows).  DeepSeek-V3-like
// layer, E4M3 / MXFP4, 16-row vs 64-row tiles: 4 rows per expert (T=128)
// 1177 / 731 vs 1267 / 857 us; 8 rows (T=256) 1562 / 968 vs 1453 / 961 us;
// 12 rows (T=384) 2004 / 1239 vs 1621 / 1082 us.
int tile_rows_8(int64_t T, int K, int E) {
    const int64_t n = T * K;
    return (n <= kDecodeMaxSlots || n <= (int64_t)6 * E) ? kBNFp8Decode : kBNFp8;
}

// MXFP4 weights halve the weight bytes, so with many routed rows per expert
// the weight tiles are re-read once per 64 rows and the block-scaled MMAs
// issue in short bursts; 112-row tiles halve both.  DeepSeek-V3-like layer,
// 112- vs 64-row tiles: 32 rows per expert (T=1024) 1551 vs 1519 us, 64 rows
// (T=2048) 2118 vs 2238 us, 256 rows (T=8192) 5718 vs 6718 us.
int tile_rows_w(int64_t T, int K, int E, moe_wtype_t wt) {
    if (wt == MOE_W_MXFP4 && T * K >= (int64_t)48 * E) return kBNMxf4Wide;
    return tile_rows_8(T, K, E);
}

moe_status_t check_common(const void *x, const void *gu, const void *dn, const int32_t *idx,
                          const float *w, int K, int T, int H, int F, int E, moe_wtype_t wt,
                          const void *gus, const void *dns, const void *out) {
    if (!dims_ok(T, H, F, E, K)) return MOE_ERR_INVALID_ARG;
    if (wt != MOE_W_BF16 && wt != MOE_W_FP8_E4M3 && wt != MOE_W_MXFP4) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !gu || !dn || !idx || !w || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gu) || !aligned16(dn) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(idx) & 3) || (reinterpret_cast<uintptr_t>(w) & 3))
        return MOE_ERR_INVALID_ARG;
    if (wt == MOE_W_FP8_E4M3) {
        if (!gus || !dns || !aligned16(gus) || !aligned16(dns)) return MOE_ERR_INVALID_ARG;
    }
    if (wt == MOE_W_MXFP4) {   // packed weights are read by TMA in 32-byte units
        if (!gus || !dns || !aligned16(gus) || !aligned16(dns) || !aligned32(gu) || !aligned32(dn))
            return MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}

// The grouped path; out == nullptr stops after the down GEMM, leaving the
// weighted rows y [T*K][H] fp32 (by slot) in the workspace at L.y.
moe_status_t run_prefill(const void *x, const void *gu, const void *dn, const int32_t *idx,
                         const float *w, int K, int T, int H, int F, int E, moe_wtype_t wt,
                         const void *gus, const void *dns, void *out, void *ws, size_t ws_bytes,
                         cudaStream_t st, int bn8 = kBNFp8, const SharedSet &sh = SharedSet(),
                         const void *residual = nullptr) {
    const Workspace L = prefill_workspace(T, H, F, E, K, wt);
    if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOE_ERR_WORKSPACE;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    const int64_t N = (int64_t)T * K;
    const bool fp8 = (wt != MOE_W_BF16);   // E4M3 activations (E4M3 or MXFP4 weights)
    // E4M3 weights: 128-row down tiles with 64-row gate_up tiles once the
    // experts average 32 routed rows or more (below that the narrower tiles
    // keep more stages of weights in flight)
    const int bn8_d = (wt == MOE_W_FP8_E4M3 && bn8 == kBNFp8 && N >= (int64_t)32 * E) ? kBNFp8DownWide : bn8;
    cudaError_t e = fp8 ? launch_permute_gather(x, idx, N, K, H, E, bn8, bn8_d, wt, wsb, L, st)
                        : launch_permute_gather(x, idx, N, K, H, E, kBNGateUp, kBNDown, wt, wsb, L, st);
    if (e == cudaSuccess) {
        if (wt == MOE_W_MXFP4)
            e = launch_gemms_mxf4(gu, static_cast<const uint8_t *>(gus), dn,
                                  static_cast<const uint8_t *>(dns), w, T, H, F, E, K, bn8, wsb, L, st);
        else if (fp8)
            e = launch_gemms_fp8(gu, static_cast<const float *>(gus), dn,
                                 static_cast<const float *>(dns), w, T, H, F, E, K, bn8, bn8_d, wsb, L, st,
                                 sh);
        else
            e = launch_gemms_bf16(gu, dn, w, T, H, F, E, K, wsb, L, st, sh);
    }
    if (e == cudaSuccess && out) e = launch_combine(idx, T, H, E, K, wsb, L, out, st, residual);
    return from_cuda(e);
}

// Workspace of moe_experts_with_shared: the prefill workspace of E+S experts
// and K+S slots per token, then the widened routing [T][K+S] (ids, weights).
// Calls served by the gather-GEMV decode kernels (which widen the routing
// themselves) use the decode workspace of K+S slots, which is smaller.
struct SharedLayout {
    Workspace L;
    size_t idx2, w2, total;
};
SharedLayout shared_workspace(int64_t T, int H, int F, int E, int K, int S, moe_wtype_t wt) {
    SharedLayout s;
    s.L = prefill_workspace(T, H, F, E + S, K + S, wt);
    Bump b;
    b.off = align_up(s.L.total, 256);
    const size_t n = (size_t)std::max<int64_t>(T * (K + S), 1);
    s.idx2 = b.take(sizeof(int32_t) * n);
    s.w2 = b.take(sizeof(float) * n);
    s.total = b.off;
    return s;
}
// True when the gather-GEMV decode kernels serve a call with S shared experts.
bool shared_decode_serves(int64_t T, int H, int F, int K, int S, moe_wtype_t wt) {
    return T <= kDecodeMaxT && decode_serves((int)T, K + S, H, F, wt);
}
bool shared_dims_ok(int64_t T, int H, int F, int E, int K, int S) {
    return S >= 0 && K + S <= 16 && E + S <= 1024 && dims_ok(T, H, F, E + S, K + S) &&
           dims_ok(T, H, F, E, K);
}

}  // namespace

namespace moe {
// Validation and decode-size rule shared with the other entry points.
moe_status_t validate_forward(const void *x, const void *gu, const void *dn, const int32_t *idx,
                              const float *w, int K, int T, int H, int F, int E, moe_wtype_t wt,
                              const void *gus, const void *dns, const void *out) {
    return check_common(x, gu, dn, idx, w, K, T, H, F, E, wt, gus, dns, out);
}
bool decode_path_fits(int T, int K, int H, int F) { return decode_fits(T, K, H, F); }
}  // namespace moe

extern "C" {

int moe_abi_version(void) { return 1; }

const char *moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    }
    return "MOE_ERR_UNKNOWN";
}

size_t moe_experts_workspace_size(int T, int H, int F, int E, int K, moe_wtype_t wt, int decode) {
    if (!dims_ok(T, H, F, E, K)) return 0;
    size_t need = (decode && decode_serves(T, K, H, F, wt)) ? decode_workspace(T, H, F, E, K, wt).total
                                                           : prefill_workspace(T, H, F, E, K, wt).total;
    // the fused decode kernel, or the path above where the device cannot run it
    if (decode && fused_decode_sizes(T, K, H, F, wt))
        need = std::max(need, fused_decode_workspace(T, H, F, K).total);
    return need;
}

moe_status_t moe_experts_prefill(const void *hidden_states, const void *gate_up_proj,
                                 const void *down_proj, const int32_t *top_k_index,
                                 const float *top_k_weights, int top_k, int T, int H, int F,
                                 int E, moe_wtype_t wt, const void *gate_up_scale,
                                 const void *down_scale, void *out, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    moe_status_t s = check_common(hidden_states, gate_up_proj, down_proj, top_k_index,
                                  top_k_weights, top_k, T, H, F, E, wt, gate_up_scale, down_scale,
                                  out);
    if (s != MOE_OK || T == 0) return s;
    return run_prefill(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, top_k,
                       T, H, F, E, wt, gate_up_scale, down_scale, out, workspace, workspace_bytes,
                       (cudaStream_t)stream, tile_rows_w(T, top_k, E, wt));
}

moe_status_t moe_experts_decode(const void *hidden_states, const void *gate_up_proj,
                                const void *down_proj, const int32_t *top_k_index,
                                const float *top_k_weights, int top_k, int T, int H, int F, int E,
                                moe_wtype_t wt, const void *gate_up_scale,
                                const void *down_scale, void *out, void *workspace,
                                size_t workspace_bytes, void *stream) {
    moe_status_t s = check_common(hidden_states, gate_up_proj, down_proj, top_k_index,
                                  top_k_weights, top_k, T, H, F, E, wt, gate_up_scale, down_scale,
                                  out);
    if (s != MOE_OK || T == 0) return s;
    cudaStream_t st = (cudaStream_t)stream;
    if (!decode_serves(T, top_k, H, F, wt))
        return run_prefill(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights,
                           top_k, T, H, F, E, wt, gate_up_scale, down_scale, out, workspace,
                           workspace_bytes, st,
                           tile_rows_w(T, top_k, E, wt));
    const DecodeWorkspace L = decode_workspace(T, H, F, E, top_k, wt);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return MOE_ERR_WORKSPACE;
    return from_cuda(launch_decode_bf16(hidden_states, gate_up_proj, down_proj, top_k_index,
                                        top_k_weights, T, H, F, E, top_k,
                                        static_cast<uint8_t *>(workspace), L, out, st));
}

size_t moe_experts_shared_workspace_size(int T, int H, int F, int E, int K, int S,
                                         moe_wtype_t wt) {
    if (!shared_dims_ok(T, H, F, E, K, S)) return 0;
    return shared_workspace(T, H, F, E, K, S, wt).total;
}

moe_status_t moe_experts_with_shared(
    const void *hidden_states, const void *gate_up_proj, const void *down_proj,
    const int32_t *top_k_index, const float *top_k_weights, int top_k, int T, int H, int F, int E,
    moe_wtype_t wt, const void *gate_up_scale, const void *down_scale,
    const void *shared_gate_up_proj, const void *shared_down_proj,
    const float *shared_gate_up_scale, const float *shared_down_scale, int S,
    const void *residual, void *out, void *workspace, size_t workspace_bytes, void *stream) {
    if (!shared_dims_ok(T, H, F, E, top_k, S)) return MOE_ERR_INVALID_ARG;
    if (wt == MOE_W_MXFP4) return MOE_ERR_UNSUPPORTED;
    moe_status_t s = check_common(hidden_states, gate_up_proj, down_proj, top_k_index,
                                  top_k_weights, top_k, T, H, F, E, wt, gate_up_scale, down_scale,
                                  out);
    if (s != MOE_OK || T == 0) return s;
    if (S > 0) {
        if (!shared_gate_up_proj || !shared_down_proj || !aligned16(shared_gate_up_proj) ||
            !aligned16(shared_down_proj))
            return MOE_ERR_INVALID_ARG;
        if (wt == MOE_W_FP8_E4M3 && (!shared_gate_up_scale || !shared_down_scale ||
                                     !aligned16(shared_gate_up_scale) || !aligned16(shared_down_scale)))
            return MOE_ERR_INVALID_ARG;
    }
    if (residual && !aligned16(residual)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    SharedSet sh;
    sh.S = S;
    sh.gate_up = shared_gate_up_proj;
    sh.down = shared_down_proj;
    sh.gate_up_scale = shared_gate_up_scale;
    sh.down_scale = shared_down_scale;
    if (shared_decode_serves(T, H, F, top_k, S, wt)) {
        const DecodeWorkspace D = decode_workspace(T, H, F, E + S, top_k + S, wt);
        if (!workspace || workspace_bytes < D.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
            return MOE_ERR_WORKSPACE;
        return from_cuda(launch_decode_bf16(hidden_states, gate_up_proj, down_proj, top_k_index,
                                            top_k_weights, T, H, F, E, top_k, wsb, D, out, st, sh,
                                            residual));
    }
    const SharedLayout SL = shared_workspace(T, H, F, E, top_k, S, wt);
    if (!workspace || workspace_bytes < SL.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return MOE_ERR_WORKSPACE;
    int32_t *idx2 = reinterpret_cast<int32_t *>(wsb + SL.idx2);
    float *w2 = reinterpret_cast<float *>(wsb + SL.w2);
    const cudaError_t e = launch_widen_routing(top_k_index, top_k_weights, T, E, top_k, S, idx2, w2, st);
    if (e != cudaSuccess) return from_cuda(e);
    // tile height of E4M3 weights: the routed-only call's rule (the shared
    // experts add S experts of T rows each)
    return run_prefill(hidden_states, gate_up_proj, down_proj, idx2, w2, top_k + S, T, H, F, E + S,
                       wt, gate_up_scale, down_scale, out, workspace, SL.L.total, st,
                       tile_rows_w(T, top_k, E, wt),
                       sh, residual);
}

moe_status_t moe_experts_decode_fused(const void *hidden_states, const void *gate_up_proj,
                                      const void *down_proj, const int32_t *top_k_index,
                                      const float *top_k_weights, int top_k, int T, int H, int F,
                                      int E, moe_wtype_t wt, const void *gate_up_scale,
                                      const void *down_scale, void *out, void *workspace,
                                      size_t workspace_bytes, void *stream) {
    moe_status_t s = check_common(hidden_states, gate_up_proj, down_proj, top_k_index,
                                  top_k_weights, top_k, T, H, F, E, wt, gate_up_scale, down_scale,
                                  out);
    if (s != MOE_OK || T == 0) return s;
    if (wt == MOE_W_BF16) {
        if (!fused_decode_sizes(T, top_k, H, F, wt) || !decode_fused_bf16_fits(T, H, F, top_k))
            return MOE_ERR_UNSUPPORTED;
        const FusedDecodeWorkspace FL = fused_decode_workspace(T, H, F, top_k);
        if (!workspace || workspace_bytes < FL.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
            return MOE_ERR_WORKSPACE;
        return from_cuda(launch_decode_fused_bf16(hidden_states, gate_up_proj, down_proj, top_k_index,
                                                  top_k_weights, T, H, F, E, top_k,
                                                  static_cast<uint8_t *>(workspace), FL, out,
                                                  (cudaStream_t)stream));
    }
    if (wt != MOE_W_MXFP4 || !fused_mxf4_fits(T, top_k)) return MOE_ERR_UNSUPPORTED;
    const Workspace L = prefill_workspace(T, H, F, E, top_k, wt);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return MOE_ERR_WORKSPACE;
    return from_cuda(launch_fused_mxf4(hidden_states, gate_up_proj,
                                       static_cast<const uint8_t *>(gate_up_scale), down_proj,
                                       static_cast<const uint8_t *>(down_scale), top_k_index,
                                       top_k_weights, T, H, F, E, top_k,
                                       static_cast<uint8_t *>(workspace), L, out,
                                       (cudaStream_t)stream));
}

moe_status_t moe_route_sigmoid_grouped(const float *logits, const float *bias, int T, int E,
                                       int num_groups, int topk_group, int top_k,
                                       float routed_scaling_factor, int32_t *top_k_index,
                                       float *top_k_weights, int32_t *expert_offsets,
                                       void *stream) {
    if (T < 0 || E < 1 || E > 1024 || num_groups < 1 || num_groups > 32 || E % num_groups ||
        topk_group < 1 || topk_group > num_groups || top_k < 1 || top_k > 16 ||
        top_k > topk_group * (E / num_groups))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) {
        if (expert_offsets) return from_cuda(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), (cudaStream_t)stream));
        return MOE_OK;
    }
    if (!logits || !bias || !top_k_index || !top_k_weights) return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_route(logits, bias, T, E, num_groups, topk_group, top_k,
                                  routed_scaling_factor, top_k_index, top_k_weights, expert_offsets,
                                  (cudaStream_t)stream));
}

moe_status_t quantize_fp8_block128(const void *x, int rows, int cols, void *xq, float *scale,
                                   void *stream) {
    if (rows < 0 || cols <= 0 || cols % 128) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!x || !xq || !scale || !aligned16(x) || !aligned16(xq) ||
        (reinterpret_cast<uintptr_t>(scale) & 3))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_quantize(x, rows, cols, xq, scale, (cudaStream_t)stream));
}

moe_status_t moe_debug_permute(const int32_t *top_k_index, int T, int K, int E, int32_t *counts,
                               int32_t *offsets, int32_t *perm, int32_t *inv, void *workspace,
                               size_t workspace_bytes, void *stream) {
    if (!dims_ok(T, 128, 128, E, K)) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || (T > 0 && (!top_k_index || !perm || !inv)))
        return MOE_ERR_INVALID_ARG;
    const Workspace L = prefill_workspace(T, 128, 128, E, K, MOE_W_BF16);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return MOE_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int64_t N = (int64_t)T * K;
    if (N == 0) {
        cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st);
        return from_cuda(e);
    }
    cudaError_t e = launch_permute(top_k_index, N, E, kBNGateUp, kBNDown, ws, L, st);
    if (e == cudaSuccess) e = launch_debug_outputs(top_k_index, N, E, ws, L, counts, offsets, perm, inv, st);
    return from_cuda(e);
}

moe_status_t moe_debug_decode_withhold(const void *hidden_states, const void *gate_up_proj,
                                       const void *down_proj, const int32_t *top_k_index,
                                       const float *top_k_weights, int top_k, int T, int H, int F,
                                       int E, void *out, void *workspace, size_t workspace_bytes,
                                       int withhold_chunk, void *stream) {
    moe_status_t s = check_common(hidden_states, gate_up_proj, down_proj, top_k_index,
                                  top_k_weights, top_k, T, H, F, E, MOE_W_BF16, nullptr, nullptr,
                                  out);
    if (s != MOE_OK || T == 0) return s;
    if (withhold_chunk < 0) return MOE_ERR_INVALID_ARG;
    if (!fused_decode_sizes(T, top_k, H, F, MOE_W_BF16) || !decode_fused_bf16_fits(T, H, F, top_k))
        return MOE_ERR_UNSUPPORTED;
    const FusedDecodeWorkspace FL = fused_decode_workspace(T, H, F, top_k);
    if (!workspace || workspace_bytes < FL.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return MOE_ERR_WORKSPACE;
    return from_cuda(launch_decode_fused_bf16(hidden_states, gate_up_proj, down_proj, top_k_index,
                                              top_k_weights, T, H, F, E, top_k,
                                              static_cast<uint8_t *>(workspace), FL, out,
                                              (cudaStream_t)stream, withhold_chunk));
}

moe_status_t moe_experts_rows(const void *hidden_states, const void *gate_up_proj,
                              const void *down_proj, const int32_t *top_k_index,
                              const float *top_k_weights, int top_k, int T, int H, int F, int E,
                              moe_wtype_t wt, const void *gate_up_scale, const void *down_scale,
                              void *workspace, size_t workspace_bytes, size_t *y_offset,
                              void *stream) {
    if (!y_offset) return MOE_ERR_INVALID_ARG;
    const void *dummy_out = reinterpret_cast<const void *>(uintptr_t(256));   // checked, never used
    moe_status_t s = check_common(hidden_states, gate_up_proj, down_proj, top_k_index,
                                  top_k_weights, top_k, T, H, F, E, wt, gate_up_scale, down_scale,
                                  dummy_out);
    if (s != MOE_OK) return s;
    *y_offset = prefill_workspace(T, H, F, E, top_k, wt).y;
    if (T == 0) return MOE_OK;
    return run_prefill(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, top_k,
                       T, H, F, E, wt, gate_up_scale, down_scale, nullptr, workspace,
                       workspace_bytes, (cudaStream_t)stream, tile_rows_w(T, top_k, E, wt));
}

moe_status_t moe_combine_rows(const float *y, const int32_t *top_k_index, int top_k, int T, int H,
                              int E, void *out, void *stream) {
    if (!dims_ok(T, H, 128, E, top_k)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y || !top_k_index || !out || !aligned16(y) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(top_k_index) & 3))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_combine_rows(y, top_k_index, T, H, E, top_k, out, (cudaStream_t)stream));
}

moe_status_t moe_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
    if (!workspace || workspace_bytes < kWorkspaceHeaderBytes ||
        (reinterpret_cast<uintptr_t>(workspace) & 255))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(cudaMemsetAsync(workspace, 0, kWorkspaceHeaderBytes, (cudaStream_t)stream));
}

moe_status_t moe_workspace_status(void *workspace, int clear, void *stream) {
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    int32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear) {
        e = cudaMemsetAsync(workspace, 0, kWorkspaceHeaderBytes, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) return from_cuda(e);
    return (word & DEV_TIMEOUT_BIT) ? MOE_ERR_TIMEOUT : MOE_OK;
}

moe_status_t moe_stage_inputs(const void *src, void *dst, size_t bytes, void *stream) {
    if (bytes == 0) return MOE_OK;
    if (!src || !dst || (bytes & 15) || !aligned16(src) || !aligned16(dst) || bytes > ((size_t)1 << 30))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_stage_copy(src, dst, bytes, (cudaStream_t)stream));
}

}  // extern "C"
