// Host side of the TMA copies: tensor maps for bf16 matrices, encoded with the
// driver's cuTensorMapEncodeTiled (fetched through the runtime, so the
// library does not link the driver library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "tpl.h"

namespace tpl {

// ---- tensor maps (driver entry point fetched through the runtime) ---------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline std::atomic<EncodeTiledFn> g_encode{nullptr};

inline EncodeTiledFn encode_fn() {
    EncodeTiledFn f = g_encode.load();
    if (f) return f;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
        return nullptr;
    f = reinterpret_cast<EncodeTiledFn>(p);
    g_encode.store(f);
    return f;
}

// bf16 matrix [rows][cols] with `row_bytes` between rows (and, for 3-D,
// `planes` of them `plane_bytes` apart); boxes of box_cols x box_rows with the
// 128-byte swizzle the MMA descriptors expect; out-of-range elements read 0.
inline int make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t row_bytes, uint32_t box_cols,
             uint32_t box_rows, uint64_t planes = 0, uint64_t plane_bytes = 0, uint32_t box_planes = 1) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return TPL_ECUDA;
    if (((uintptr_t)base & 15u) || (row_bytes & 15u) || (plane_bytes & 15u)) return TPL_EINVAL;
    const cuuint64_t gdim[3] = {cols, rows, planes};
    const cuuint64_t gstr[2] = {row_bytes, plane_bytes};
    const cuuint32_t box[3] = {box_cols, box_rows, box_planes};
    const cuuint32_t es[3] = {1, 1, 1};
    const cuuint32_t rank = planes ? 3 : 2;
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), gdim, gstr, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? TPL_OK : TPL_EINVAL;
}

// The bf16 KV cache of one layer, [t][batch_cap][n_kv/t][seq_cap][128], as a
// 4-D map (128 dims, `keys` rows, n_kv/t, t * batch_cap): the rows at or past
// `keys` read as 0, so a block that runs past the cache length needs no
// masking of its values.  Boxes of 64 dims x box_keys rows, 128-byte swizzle.
inline int make_kv_map(CUtensorMap *m, const void *base, uint64_t keys, uint64_t nkv_s, uint64_t sb, uint64_t seq_cap,
                       uint32_t box_keys) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return TPL_ECUDA;
    if (((uintptr_t)base & 15u) || keys == 0) return TPL_EINVAL;
    const cuuint64_t gdim[4] = {128, keys, nkv_s, sb};
    const cuuint64_t gstr[3] = {256, seq_cap * 256, nkv_s * seq_cap * 256};
    const cuuint32_t box[4] = {64, box_keys, 1, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), gdim, gstr, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? TPL_OK : TPL_EINVAL;
}

}  // namespace tpl
