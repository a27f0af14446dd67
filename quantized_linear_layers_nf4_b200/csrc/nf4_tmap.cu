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

static cudaError_t tmap_nd(CUtensorMap* out, const TmapKey& key) {
    static std::mutex mu;
    static Entry cache[kCache];
    static int next = 0;
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
    const cuuint64_t dims[3] = {key.dim0, key.dim1, key.dim2};
    const cuuint64_t strides[2] = {key.stride1, key.stride2};
    const cuuint32_t box[3] = {key.box0, key.box1, key.box2};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUtensorMap map;
    const CUresult r = fn(&map, static_cast<CUtensorMapDataType>(key.dtype), static_cast<cuuint32_t>(key.rank),
                          const_cast<void*>(key.base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          static_cast<CUtensorMapSwizzle>(key.swizzle), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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

cudaError_t tmap_2d(CUtensorMap* out, CUtensorMapDataType dtype, const void* base, uint64_t dim0,
                    uint64_t dim1, uint64_t stride1, uint32_t box0, uint32_t box1,
                    CUtensorMapSwizzle swizzle) {
    const TmapKey key{base, dim0, dim1, 1, stride1, 0, box0, box1, 1, 2, static_cast<int>(dtype),
                      static_cast<int>(swizzle)};
    return tmap_nd(out, key);
}

}  // namespace nf4
