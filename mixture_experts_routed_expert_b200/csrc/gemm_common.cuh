// gemm_common.cuh -- pieces shared by the grouped GEMM kernels (bf16 and
// E4M3): the tile list over experts and the TMA descriptor encoder.
#pragma once

#include <cudaTypedefs.h>

#include "common.cuh"

namespace moe {

struct Tile {
    int e, m, row0, nrows;
};

// Work item w -> (expert, weight-row tile, routed rows).  Items of one expert
// are contiguous, routed-row tiles fastest; an expert's n_e rows are split in
// ceil(n_e/BN) near-equal tiles of a multiple of 16 rows.
__device__ __forceinline__ Tile decode_tile(int w, const int32_t *s_off, const int32_t *s_tiles,
                                            int E, int MT, int BN) {
    int lo = 0, hi = E;  // s_tiles[lo]*MT <= w < s_tiles[hi]*MT
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_tiles[mid] * MT <= w) lo = mid; else hi = mid;
    }
    Tile t;
    t.e = lo;
    const int nt = s_tiles[lo + 1] - s_tiles[lo];
    const int local = w - s_tiles[lo] * MT;
    t.m = local / nt;
    const int n = local - t.m * nt;
    const int n_e = s_off[lo + 1] - s_off[lo];
    const int rpt = min(BN, ((n_e + nt - 1) / nt + 15) & ~15);
    t.row0 = s_off[lo] + n * rpt;
    t.nrows = min(rpt, n_e - n * rpt);
    return t;
}


// The driver's tensor-map encoder, looked up once (a function-local static
// is initialised exactly once even with concurrent callers).
inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    }();
    return fn;
}

// Row-major [rows, cols] matrix, box = box_rows x 128 bytes, 128-byte swizzle.
inline bool make_tmap(CUtensorMap *m, CUtensorMapDataType dt, int elem_bytes, const void *ptr,
               uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto enc = tmap_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
    cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// A row-major [rows][cols] matrix seen as 3-D (k-element within a 128-block,
// row, 128-block) so that one box brings `kpb` k-blocks of `box_rows` rows as
// [k-block][row][128 bytes] tiles with the 128-byte swizzle.
// Packed E2M1 (cols/2 bytes a row): each 16 codes land in a 16-byte slot.
inline bool make_tmap_e2m1(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t kpb) {
    auto enc = tmap_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, rows, cols / 128};
    cuuint64_t strides[2] = {cols / 2, 64};
    cuuint32_t box[3] = {128, 128, kpb};   // 128 weight rows (one MMA tile)
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void *>(ptr), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// E4M3 activations [rows][cols] bytes, the same 3-D view.
inline bool make_tmap_e4m3_kb(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols,
                       uint32_t box_rows, uint32_t kpb) {
    auto enc = tmap_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, rows, cols / 128};
    cuuint64_t strides[2] = {cols, 128};
    cuuint32_t box[3] = {128, box_rows, kpb};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


}  // namespace moe
