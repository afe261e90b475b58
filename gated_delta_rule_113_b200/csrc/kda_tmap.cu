// kda_tmap.cu -- host-side TMA descriptor encoding for the prefill kernels.
// The driver entry point is looked up through the runtime, so the library
// does not link against libcuda.
#include "kda_internal.cuh"

namespace kda {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxSetCurrentFn)(CUcontext);

}  // namespace

void *driver_fn(const char *name) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return ptr;
}

bool DeviceGuard::use(int dev) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (cur == dev) return true;
    if (!switched_) {
        static CtxGetCurrentFn get_cur =
            reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
        if (!get_cur || get_cur(&saved_) != CUDA_SUCCESS) return false;
        switched_ = true;
    }
    if (cudaSetDevice(dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return true;
}

DeviceGuard::~DeviceGuard() {
    if (!switched_) return;
    static CtxSetCurrentFn set_cur =
        reinterpret_cast<CtxSetCurrentFn>(driver_fn("cuCtxSetCurrent"));
    if (set_cur) set_cur(saved_);
}

bool make_tmap_bf16_3d(CUtensorMap *m, const void *base, int T, int H, int D, int box_x,
                       int swizzle_bytes) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE;
    if (swizzle_bytes == 32) swz = CU_TENSOR_MAP_SWIZZLE_32B;
    if (swizzle_bytes == 64) swz = CU_TENSOR_MAP_SWIZZLE_64B;
    if (swizzle_bytes == 128) swz = CU_TENSOR_MAP_SWIZZLE_128B;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    const cuuint32_t box[3] = {(cuuint32_t)box_x, 1, (cuuint32_t)kChunk};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace kda
