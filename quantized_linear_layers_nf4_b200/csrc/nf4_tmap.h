// nf4_tmap.h -- host-side TMA tensor-map encoding (2-D, tiled), cached.
//
// cuTensorMapEncodeTiled is fetched through cudaGetDriverEntryPoint, so the
// library needs no link-time dependency on the driver library and still loads
// on hosts without a GPU.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nf4 {

struct TmapKey {
    const void* base;
    uint64_t dim0, dim1, dim2, stride1, stride2;
    uint32_t box0, box1, box2;
    int rank, dtype, swizzle;
    bool operator==(const TmapKey& o) const {
        return base == o.base && dim0 == o.dim0 && dim1 == o.dim1 && dim2 == o.dim2 && stride1 == o.stride1 &&
               stride2 == o.stride2 && box0 == o.box0 && box1 == o.box1 && box2 == o.box2 && rank == o.rank &&
               dtype == o.dtype && swizzle == o.swizzle;
    }
};

// Encodes (or returns a cached copy of) a 2-D tiled tensor map:
//   dim0 = innermost extent (elements), dim1 = rows, stride1 = row pitch in bytes,
//   box = {box0, box1} elements, zero fill out of bounds, no interleave.
cudaError_t tmap_2d(CUtensorMap* out, CUtensorMapDataType dtype, const void* base, uint64_t dim0,
                    uint64_t dim1, uint64_t stride1, uint32_t box0, uint32_t box1,
                    CUtensorMapSwizzle swizzle);

}  // namespace nf4
