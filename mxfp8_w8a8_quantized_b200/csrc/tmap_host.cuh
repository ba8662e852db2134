/*
 * tmap_host.cuh -- host-side construction of TMA tensor maps (CUtensorMap)
 * through the driver's cuTensorMapEncodeTiled, reached via the runtime's
 * entry-point query so that the library links against cudart only.
 */
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace mx {

typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static inline PFN_encodeTiled get_encode_fn()
{
    static PFN_encodeTiled fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(p);
    }
    return fn;
}

/*
 * Row-major 2-D tensor [rows, inner] of `type` with a row pitch of
 * `pitch_bytes`; box = box_inner x box_rows elements.  Out-of-range boxes
 * read as zero and stores are clipped at the tensor's extent.
 */
static inline bool encode_2d(CUtensorMap *m, CUtensorMapDataType type, const void *base, int64_t inner, int64_t rows,
                             int64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle)
{
    PFN_encodeTiled enc = get_encode_fn();
    if (!enc)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, type, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

} // namespace mx
