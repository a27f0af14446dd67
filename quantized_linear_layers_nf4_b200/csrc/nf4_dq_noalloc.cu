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

#include <cuda.h>

#include "nf4.h"
#include "nf4_internal.h"

namespace {

constexpr int64_t kMaxPartials = NF4_DQ_NOALLOC_MAX_NB / 256;

// File-scope scratch for the fp64 per-256 partial sums.  In host code this name
// is only a stand-in for the device symbol: its device address comes from
// cudaGetSymbolAddress, once per context.
static __device__ __align__(256) double g_dq_partials[kMaxPartials];

// Device address of g_dq_partials in the current context.  Each context (a
// device's primary context, or one the caller created) has its own copy of the
// module, so the address is cached per context, looked up the first time a
// context makes the call.  The context comes from cuCtxGetCurrent, fetched
// through the runtime's driver entry point (no link-time driver dependency);
// without it the address is looked up on every call.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

cudaError_t scratch_address(double** out) {
    constexpr int kSlots = 64;
    static std::mutex mu;
    static CUcontext ctx_of[kSlots] = {};
    static double* addr_of[kSlots] = {};
    static int used = 0;
    CUcontext ctx = nullptr;
    const CtxGetCurrentFn get = ctx_get_current();
    const bool keyed = get != nullptr && get(&ctx) == CUDA_SUCCESS && ctx != nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (keyed)
        for (int i = 0; i < used; ++i)
            if (ctx_of[i] == ctx) {
                *out = addr_of[i];
                return cudaSuccess;
            }
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_dq_partials);
    if (e != cudaSuccess) return e;
    *out = static_cast<double*>(p);
    if (keyed && used < kSlots) {
        ctx_of[used] = ctx;
        addr_of[used] = *out;
        ++used;
    }
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
    if (scratch_address(&scratch) != cudaSuccess) {
        cudaGetLastError();
        return NF4_ERR_CUDA;
    }
    const cudaError_t e = nf4::launch_double_quant(absmax, nb, scratch, absmax_q, absmax_scale,
                                                   absmax_offset, dev,
                                                   reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}
