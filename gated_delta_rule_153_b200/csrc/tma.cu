// tma.cu -- host-side tensor-map encoding through the driver entry point.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "tma.cuh"

namespace gdn {

static PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool encode_token_map(CUtensorMap* map, const void* base, int B, int T, int H, int box_cols, int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encoder();
    if (!fn) return false;
    const cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)B * (cuuint64_t)T};
    const cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
    const cuuint32_t box[3] = {(cuuint32_t)box_cols, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace gdn
