// static_scratch.cu -- moe_experts_decode_static: the decode form of the
// routed-experts forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run the layer: code recorded into a CUDA graph while capture forbids
// allocation, serving loops and real-time hosts that fix their device memory
// budget at start-up, and plugin or embedded hosts that expose no allocator to
// the code they load.  They still own their inputs and outputs; this entry
// point takes its scratch memory from a fixed array that is part of the
// library image instead of a caller-provided workspace.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds kStaticScratchBytes of it until the process exits.  Host code
// must not use the array's name as a device address: on the host the name
// only denotes a stand-in object.  Every call looks up the device address
// with cudaGetSymbolAddress in the caller's current context (a host-side
// query: no stream work, no allocation), so the address stays right after a
// cudaDeviceReset or when another context is current.  The first call in a
// context also loads the library's module there, so it should come before
// any stream capture.  All calls share the one array and it keeps whatever
// the last call left there: calls that may overlap on the GPU (different
// streams, or different host threads without ordering) race on it.
#include "internal.h"

namespace moe {

namespace {

constexpr size_t kStaticScratchBytes = 1u << 20;   // 1 MiB

__device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

// The largest decode scratch (T*K <= kDecodeMaxSlots slots of h, F <= 2048
// features, plus the status words) fits the array, so every size the decode
// kernels accept is served.
static_assert(kWorkspaceHeaderBytes + (size_t)kDecodeMaxSlots * 2048 * 2 <= kStaticScratchBytes,
              "static decode scratch smaller than the largest decode workspace");

// Device address of g_decode_scratch in the current context.
cudaError_t scratch_address(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" MOE_API moe_status_t moe_experts_decode_static(
    const void *hidden_states, const void *gate_up_proj, const void *down_proj,
    const int32_t *top_k_index, const float *top_k_weights, int top_k, int T, int H, int F, int E,
    moe_wtype_t wt, const void *gate_up_scale, const void *down_scale, void *out,
    void *stream) {
    moe_status_t s = validate_forward(hidden_states, gate_up_proj, down_proj, top_k_index,
                                      top_k_weights, top_k, T, H, F, E, wt, gate_up_scale,
                                      down_scale, out);
    if (s != MOE_OK || T == 0) return s;
    if (wt != MOE_W_BF16) return MOE_ERR_UNSUPPORTED;
    if (!decode_path_fits(T, top_k, H, F)) return MOE_ERR_WORKSPACE;
    const DecodeWorkspace L = decode_workspace(T, H, F, E, top_k, wt);
    if (L.total > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
    void *scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    e = launch_decode_bf16(hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, T,
                           H, F, E, top_k, static_cast<uint8_t *>(scratch), L, out,
                           (cudaStream_t)stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}
