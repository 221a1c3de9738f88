// stage.cu -- moves a step's small inputs (hidden states, top-k ids and
// weights of a decode call, a few KB) from memory the device reads over the
// bus (mapped pinned host memory) into device memory with one kernel.  For a
// few KB a kernel's loads finish sooner than a copy-engine transfer, and the
// decode kernels that follow then read device memory.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kStageThreads = 256;

// dst[i] = src[i] for n 16-byte vectors; the loads are cache-volatile
// (ld.global.cv), so host writes made between steps are always seen.
__global__ void __launch_bounds__(kStageThreads) stage_copy_kernel(const uint4 *__restrict__ src,
                                                                   uint4 *__restrict__ dst,
                                                                   size_t n) {
    const size_t step = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += step)
        dst[i] = __ldcv(src + i);
}

}  // namespace

cudaError_t launch_stage_copy(const void *src, void *dst, size_t bytes, cudaStream_t st) {
    const size_t n = bytes / 16;
    const size_t want = (n + kStageThreads - 1) / kStageThreads;
    const unsigned grid = (unsigned)std::min<size_t>(want, (size_t)4 * num_sms());
    return launch_k(stage_copy_kernel, dim3(grid), dim3(kStageThreads), 0, st, false,
                    static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), n);
}

}  // namespace moe
