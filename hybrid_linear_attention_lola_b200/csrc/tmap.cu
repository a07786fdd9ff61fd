// Host-side encoding of the TMA tensor maps the kernels gather rows with.
//
// A "row map" views a row-major bfloat16 array [rows][cols] as a 2-D tensor
// whose box is box_rows rows of 64 elements (128 bytes each) with 128-byte
// swizzle. With box_rows = 1 the kernels load it with tile::gather4 (four
// arbitrary rows of one 64-column block per instruction); with box_rows = 128
// one instruction loads 128 consecutive rows of one 64-column block, exactly
// one column of atoms of a K-major operand tile. Rows at or past `rows` and
// columns at or past `cols` read as zero.
//
// A "3-D map" views a bfloat16 array [d2][d1][d0] (d0 contiguous, a multiple of
// 64) with boxes of 64 x box1 x box2 elements and 128-byte swizzle: one box lands
// as box1 * box2 rows of 128 bytes, i.e. one 64-column atom block of a K-major
// operand whose rows run over (d2, d1) with d1 fastest. Used for the query and
// key/value tensors [batch * tokens][heads][head_dim] of a prefill call.
#include <cudaTypedefs.h>

#include "lola_internal.cuh"

namespace lola {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tiled_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (encode == nullptr) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return nullptr;
        encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    }
    return encode;
}

}  // namespace

bool make_row_map(CUtensorMap *m, const void *base, unsigned long long rows, int cols, int box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 encode = tiled_encoder();
    if (encode == nullptr || base == nullptr || rows == 0 || cols <= 0 || (cols * 2) % 16 != 0 || box_rows < 1 ||
        box_rows > 256)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_3d(CUtensorMap *m, const void *base, int d0, int d1, unsigned long long d2, int box1, int box2)
{
    PFN_cuTensorMapEncodeTiled_v12000 encode = tiled_encoder();
    if (encode == nullptr || base == nullptr || d0 < 64 || d0 % 64 != 0 || d1 < 1 || d2 == 0 || box1 < 1 ||
        box1 > 256 || box2 < 1 || box2 > 256)
        return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d0, (cuuint64_t)d1, (cuuint64_t)d2};
    const cuuint64_t strides[2] = {(cuuint64_t)d0 * 2, (cuuint64_t)d0 * d1 * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box1, (cuuint32_t)box2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lola
