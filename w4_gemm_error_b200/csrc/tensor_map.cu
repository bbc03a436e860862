// Host-side encoding of TMA tensor maps (cuTensorMapEncodeTiled, reached
// through the runtime's driver entry point so no driver library is linked).
#include <cudaTypedefs.h>

#include <mutex>

#include "tensor_map.h"

namespace spear {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D row-major tensor [rows][cols] of `elem` bytes, boxes of box_cols x box_rows.
}  // namespace

cudaError_t make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int elem, uint64_t cols,
                     uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw)
{
    const uint64_t dims[2] = {cols, rows};
    const uint64_t strides[1] = {cols * (uint64_t)elem};
    const uint32_t box[2] = {box_cols, box_rows};
    return make_map_nd(m, ptr, dt, 2, dims, strides, box, sw);
}

cudaError_t make_map_nd(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int rank, const uint64_t *dims,
                        const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle sw)
{
    auto fn = encode_fn();
    if (!fn || rank < 1 || rank > 5)
        return cudaErrorNotSupported;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i + 1 < rank)
            s[i] = strides[i];
    }
    CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void *>(ptr), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

bool tensor_maps_available() { return encode_fn() != nullptr; }

}  // namespace spear
