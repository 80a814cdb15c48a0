// Tensor maps (TMA descriptors) over the library's device tensors.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"
#include "tma_host.h"

namespace pa {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

CUtensorMapDataType tma_type(pa_dtype dt) {
    switch (dt) {
    case PA_F32: return CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    case PA_F16: return CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    case PA_BF16: return CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    default: return CU_TENSOR_MAP_DATA_TYPE_UINT8;
    }
}

}  // namespace

// The cache [NB, bs, Hkv, D] as a 4-D tensor {D, Hkv, bs, NB} (innermost
// first).  A box {128 bytes of D, 1, bs, 1} is one 128-byte segment of the
// K (or V) tile of one block for one kv head, swizzled per 128-byte row; a
// tile takes D * elt / 128 boxes, at x = 0, 128 / elt, ...
pa_status make_cache_map(CUtensorMap* m, const void* base, pa_dtype dt, int64_t NB, int bs,
                         int Hkv, int D) {
    auto fn = encode_fn();
    if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const int e = elem_size(dt);
    const cuuint64_t row = (cuuint64_t)D * e;            // bytes of one (token, head) row
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)bs, (cuuint64_t)NB};
    cuuint64_t strides[3] = {row, row * Hkv, row * Hkv * bs};
    cuuint32_t box[4] = {(cuuint32_t)(128 / e), 1, (cuuint32_t)bs, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, tma_type(dt), 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PA_OK;
}

pa_status make_cache_map_heads(CUtensorMap* m, const void* base, pa_dtype dt, int64_t NB, int bs,
                               int Hkv, int D, int hg) {
    auto fn = encode_fn();
    if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const int e = elem_size(dt);
    const cuuint64_t row = (cuuint64_t)D * e;            // bytes of one (token, head) row
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)bs, (cuuint64_t)Hkv, (cuuint64_t)NB};
    cuuint64_t strides[3] = {row * Hkv, row, row * Hkv * bs};   // token, head, block
    cuuint32_t box[4] = {(cuuint32_t)(128 / e), (cuuint32_t)bs, (cuuint32_t)hg, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, tma_type(dt), 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (head groups) failed (%d)", (int)r);
    return PA_OK;
}

pa_status make_rows_map(CUtensorMap* m, const void* base, pa_dtype dt, int64_t T, int H, int D,
                        int box_h, int box_t) {
    auto fn = encode_fn();
    if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const int e = elem_size(dt);
    const cuuint64_t row = (cuuint64_t)D * e;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {row, row * H};
    cuuint32_t box[3] = {(cuuint32_t)(128 / e), (cuuint32_t)box_h, (cuuint32_t)box_t};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, tma_type(dt), 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PA_OK;
}

}  // namespace pa
