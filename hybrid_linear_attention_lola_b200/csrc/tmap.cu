// Host-side encoding of the TMA tensor maps the kernels gather rows with.
//
// A "row map" views a row-major bfloat16 array [rows][cols] as a 2-D tensor
// whose box is box_rows rows of 64 elements (128 bytes each) with 128-byte
// swizzle. With box_rows = 1 the kernels load it with tile::gather4 (four
// arbitrary rows of one 64-column block per instruction); with box_rows = 128
// one instruction loads 128 consecutive rows of one 64-column block, exactly
// one column of atoms of a K-major operand tile. Rows at or past `rows` and
// columns at or past `cols` read as zero.
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

}  // namespace lola
