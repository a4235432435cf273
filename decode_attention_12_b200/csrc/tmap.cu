// tmap.cu -- access to the driver's tensor-map encoder (cuTensorMapEncodeTiled) through
// the runtime's driver entry-point query, so the library does not link libcuda directly.
#include <mutex>

#include "mma_common.cuh"

namespace lla {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}


namespace mma {

// 2-D map over one layer's latent plane [rows][r bf16]: boxes of `cols` columns x 32 rows
// with the swizzle that matches the box's row bytes.
static bool plane_map(CUtensorMap *map, const void *base, int r, int64_t rows, int cols)
{
    auto fn = tensor_map_encoder();
    if (fn == nullptr)
        return false;
    const int rb = cols * 2;
    const CUtensorMapSwizzle sw = rb == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                           : (rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
    const cuuint64_t dims[2] = {(cuuint64_t)r, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)r * 2};
    const cuuint32_t box[2] = {(cuuint32_t)cols, (cuuint32_t)kBox};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Maps for the 64-column blocks and the tail of one plane (an unused map is a copy).
bool plane_maps(CUtensorMap *main, CUtensorMap *tail, const void *base, int r, int64_t rows)
{
    const int nblk = r / 64, t = r % 64;
    bool ok = true;
    if (nblk > 0)
        ok = ok && plane_map(main, base, r, rows, 64);
    if (t > 0)
        ok = ok && plane_map(tail, base, r, rows, t);
    if (nblk == 0)
        *main = *tail;
    if (t == 0)
        *tail = *main;
    return ok;
}


} // namespace mma

} // namespace lla
