// nf4_tmap.cu -- cached 2-D TMA tensor-map encoding (see nf4_tmap.h).
#include <cudaTypedefs.h>

#include <mutex>

#include "nf4_tmap.h"

namespace nf4 {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

constexpr int kCache = 512;
struct Entry {
    bool used = false;
    TmapKey key{};
    CUtensorMap map{};
};

}  // namespace

cudaError_t tmap_2d(CUtensorMap* out, CUtensorMapDataType dtype, const void* base, uint64_t dim0,
                    uint64_t dim1, uint64_t stride1, uint32_t box0, uint32_t box1,
                    CUtensorMapSwizzle swizzle) {
    static std::mutex mu;
    static Entry cache[kCache];
    static int next = 0;
    const TmapKey key{base, dim0, dim1, stride1, box0, box1, static_cast<int>(dtype),
                      static_cast<int>(swizzle)};
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < kCache; ++i)
            if (cache[i].used && cache[i].key == key) {
                *out = cache[i].map;
                return cudaSuccess;
            }
    }
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {dim0, dim1};
    const cuuint64_t strides[1] = {stride1};
    const cuuint32_t box[2] = {box0, box1};
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMap map;
    const CUresult r = fn(&map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    std::lock_guard<std::mutex> lock(mu);
    cache[next].used = true;
    cache[next].key = key;
    cache[next].map = map;
    next = (next + 1) % kCache;
    *out = map;
    return cudaSuccess;
}

}  // namespace nf4
