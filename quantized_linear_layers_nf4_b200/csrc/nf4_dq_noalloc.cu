// nf4_dq_noalloc.cu -- double quantization for callers that cannot allocate.
//
// Some callers cannot hand this library a workspace: a plugin or custom op
// running inside a host framework that owns all device memory and exposes no
// allocator to it, or a deployment whose memory plan is fixed at start-up and
// forbids any allocation afterwards.  nf4_double_quant needs scratch space for
// its fp64 partial sums, so this file offers the same computation with that
// scratch held in a fixed array in device memory instead of a caller buffer.
//
// The array lives for the life of the process on every GPU that loads the
// library (NF4_DQ_NOALLOC_MAX_NB / 256 doubles = 512 KiB).  Its address is taken
// once per device, on the first call made with that device current.  All calls
// on a device share the one array: calls whose work overlaps on the GPU (on
// different streams, or from different host threads) race on it, so callers
// must order them.  Nothing in it needs to start at zero: every call writes
// each partial sum before it reads it, so stale contents from an earlier call
// are never used.
#include <mutex>

#include "nf4.h"
#include "nf4_internal.h"

namespace {

constexpr int64_t kMaxPartials = NF4_DQ_NOALLOC_MAX_NB / 256;

// File-scope scratch for the fp64 per-256 partial sums.  In host code this name
// is only a stand-in for the device symbol: its device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) double g_dq_partials[kMaxPartials];

// Device address of g_dq_partials for the current device, looked up on the
// first call with that device current.
cudaError_t scratch_address(int device, double** out) {
    static std::mutex mu;
    static double* addr[64] = {};
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[device] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_dq_partials);
        if (e != cudaSuccess) return e;
        addr[device] = static_cast<double*>(p);
    }
    *out = addr[device];
    return cudaSuccess;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" nf4_status_t nf4_double_quant_noalloc(const float* absmax, int64_t nb, int8_t* absmax_q,
                                                 float* absmax_scale, float* absmax_offset,
                                                 nf4_stream_t stream) {
    if (!absmax || !absmax_q || !absmax_scale || !absmax_offset) return NF4_ERR_NULL;
    if (nb <= 0) return NF4_ERR_SHAPE;
    if (nb > NF4_DQ_NOALLOC_MAX_NB) return NF4_ERR_WORKSPACE;  // beyond the fixed scratch
    if (!aligned4(absmax) || !aligned4(absmax_scale) || !aligned4(absmax_offset)) return NF4_ERR_ALIGN;
    nf4::DeviceInfo dev;
    if (nf4::current_device(&dev) != cudaSuccess) {
        cudaGetLastError();
        return NF4_ERR_CUDA;
    }
    if (dev.major != 10) return NF4_ERR_UNSUPPORTED;
    double* scratch = nullptr;
    if (scratch_address(dev.device, &scratch) != cudaSuccess) {
        cudaGetLastError();
        return NF4_ERR_CUDA;
    }
    const cudaError_t e = nf4::launch_double_quant(absmax, nb, scratch, absmax_q, absmax_scale,
                                                   absmax_offset, dev,
                                                   reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}
