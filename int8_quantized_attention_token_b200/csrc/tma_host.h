// tma_host.h -- host-side creation of TMA tensor maps (cuTensorMapEncodeTiled
// through the runtime's driver entry point), shared by the attention kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace intfa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            (void)cudaGetLastError();
    }
    return fn;
}

// 3-D tensor map (uint8 unless dtype says otherwise): dims (x = inner, y, z) in
// elements, byte strides of y and z, box (bx, by, 1) in elements.
inline int make_map(CUtensorMap *map, const void *base, uint64_t x, uint64_t y, uint64_t z,
                    uint64_t stride_y, uint64_t stride_z, uint32_t bx, uint32_t by,
                    CUtensorMapSwizzle swz, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_UINT8) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return INTFA_ERR_CUDA;
    const cuuint64_t dims[3] = {x, y, z};
    const cuuint64_t strides[2] = {stride_y, stride_z};
    const cuuint32_t box[3] = {bx, by, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(map, dtype, 3, const_cast<void *>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? INTFA_OK : INTFA_ERR_CUDA;
}

}  // namespace intfa
