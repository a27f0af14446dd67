// nf4_api.cu -- the extern "C" entry points of libnf4.so (declared in include/nf4.h).
//
// Each entry point validates its arguments on the host, then enqueues kernels
// on the caller's stream.  Nothing is launched when validation fails, nothing
// is allocated, and the host is never synchronized.
#include <cstdint>
#include <cstring>
#include <mutex>

#include "nf4.h"
#include "nf4_internal.h"
#include "nf4_levels.h"

namespace nf4 {

cudaError_t current_device(DeviceInfo* out) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev].device != dev) {
        DeviceInfo d;
        d.device = dev;
        if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return e;
        int optin = 0;
        if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
        d.smem_optin = static_cast<size_t>(optin);
        cache[dev] = d;
    }
    *out = cache[dev];
    return cudaSuccess;
}

}  // namespace nf4

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Device check shared by every launching entry point.
nf4_status_t device_ok(nf4::DeviceInfo* dev) {
    if (nf4::current_device(dev) != cudaSuccess) {
        cudaGetLastError();
        return NF4_ERR_CUDA;
    }
    if (dev->major != 10) return NF4_ERR_UNSUPPORTED;
    return NF4_OK;
}

nf4_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA; }

nf4_status_t check_weight(const nf4_weight_t* w) {
    if (!w) return NF4_ERR_NULL;
    if ((w->magic != NF4_WEIGHT_MAGIC && w->magic != NF4_FP4_WEIGHT_MAGIC) || w->version != NF4_WEIGHT_VERSION ||
        w->blocksize != NF4_BLOCKSIZE || w->blocksize2 != NF4_BLOCKSIZE2)
        return NF4_ERR_STATE;
    if (!w->wq || !w->absmax_q || !w->absmax_scale || !w->absmax_offset) return NF4_ERR_NULL;
    if (w->n <= 0 || w->k <= 0) return NF4_ERR_SHAPE;
    if (w->n > INT64_MAX / w->k) return NF4_ERR_SHAPE;
    if ((w->n * w->k) % NF4_BLOCKSIZE != 0) return NF4_ERR_SHAPE;
    if (!aligned(w->wq, 16) || !aligned(w->absmax_scale, 4) || !aligned(w->absmax_offset, 4))
        return NF4_ERR_ALIGN;
    return NF4_OK;
}

// The codebook a (checked) weight's codes index: its magic says NF4 or FP4.
int codebook_of(const nf4_weight_t* w) { return w->magic == NF4_FP4_WEIGHT_MAGIC ? 1 : 0; }

}  // namespace

extern "C" {

int nf4_abi_version(void) { return NF4_ABI_VERSION; }

const char* nf4_status_str(int status) {
    switch (status) {
        case NF4_OK: return "NF4_OK";
        case NF4_ERR_NULL: return "NF4_ERR_NULL: a required pointer is NULL";
        case NF4_ERR_SHAPE: return "NF4_ERR_SHAPE: size out of range or not a multiple of the block size";
        case NF4_ERR_ALIGN: return "NF4_ERR_ALIGN: pointer not 16-byte aligned";
        case NF4_ERR_DTYPE: return "NF4_ERR_DTYPE: unsupported dtype";
        case NF4_ERR_STATE: return "NF4_ERR_STATE: bad nf4_weight_t magic, version or block size";
        case NF4_ERR_WORKSPACE: return "NF4_ERR_WORKSPACE: workspace missing or too small";
        case NF4_ERR_CUDA: return "NF4_ERR_CUDA: CUDA runtime error";
        case NF4_ERR_DEVICE_TIMEOUT: return "NF4_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
        case NF4_ERR_UNSUPPORTED: return "NF4_ERR_UNSUPPORTED: device is not compute capability 10.x";
        default: return "unknown nf4 status";
    }
}

nf4_status_t nf4_codebook(float* levels_out) { return nf4_codebook_typed(NF4_QUANT_NF4, levels_out); }

nf4_status_t nf4_codebook_typed(nf4_quant_type_t quant_type, float* levels_out) {
    if (!levels_out) return NF4_ERR_NULL;
    static const float nf4_levels[16] = NF4_LEVELS_INIT;
    static const float fp4_levels[16] = FP4_LEVELS_INIT;
    if (quant_type == NF4_QUANT_NF4)
        std::memcpy(levels_out, nf4_levels, sizeof nf4_levels);
    else if (quant_type == NF4_QUANT_FP4)
        std::memcpy(levels_out, fp4_levels, sizeof fp4_levels);
    else
        return NF4_ERR_DTYPE;
    return NF4_OK;
}

nf4_status_t nf4_quantize(const void* W, nf4_dtype_t w_dtype, int64_t n, int64_t k, uint8_t* wq,
                          float* absmax, nf4_stream_t stream) {
    return nf4_quantize_typed(W, w_dtype, n, k, NF4_QUANT_NF4, wq, absmax, stream);
}

nf4_status_t nf4_quantize_typed(const void* W, nf4_dtype_t w_dtype, int64_t n, int64_t k,
                                nf4_quant_type_t quant_type, uint8_t* wq, float* absmax, nf4_stream_t stream) {
    if (!W || !wq || !absmax) return NF4_ERR_NULL;
    if (quant_type != NF4_QUANT_NF4 && quant_type != NF4_QUANT_FP4) return NF4_ERR_DTYPE;
    if (w_dtype != NF4_F32 && w_dtype != NF4_BF16) return NF4_ERR_DTYPE;
    if (n <= 0 || k <= 0 || n > INT64_MAX / k || (n * k) % NF4_BLOCKSIZE != 0) return NF4_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(wq, 16) || !aligned(absmax, 4)) return NF4_ERR_ALIGN;
    nf4::DeviceInfo dev;
    nf4_status_t st = device_ok(&dev);
    if (st != NF4_OK) return st;
    return from_cuda(nf4::launch_quantize(W, w_dtype == NF4_BF16, n * k, wq, absmax,
                                          quant_type == NF4_QUANT_FP4 ? 1 : 0, dev,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

size_t nf4_double_quant_workspace_bytes(int64_t nb) { return nf4::dq_workspace_bytes(nb); }

nf4_status_t nf4_double_quant(const float* absmax, int64_t nb, void* workspace,
                              size_t workspace_bytes, int8_t* absmax_q, float* absmax_scale,
                              float* absmax_offset, nf4_stream_t stream) {
    if (!absmax || !absmax_q || !absmax_scale || !absmax_offset) return NF4_ERR_NULL;
    if (nb <= 0 || nb > nf4::dq_max_nb()) return NF4_ERR_SHAPE;
    if (!workspace || workspace_bytes < nf4::dq_workspace_bytes(nb)) return NF4_ERR_WORKSPACE;
    if (!aligned(absmax, 4) || !aligned(absmax_scale, 4) || !aligned(absmax_offset, 4) ||
        !aligned(workspace, 8))
        return NF4_ERR_ALIGN;
    nf4::DeviceInfo dev;
    nf4_status_t st = device_ok(&dev);
    if (st != NF4_OK) return st;
    return from_cuda(nf4::launch_double_quant(absmax, nb, static_cast<double*>(workspace), absmax_q,
                                              absmax_scale, absmax_offset, dev,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

nf4_status_t nf4_dequantize(const nf4_weight_t* w, void* out, nf4_dtype_t out_dtype,
                            nf4_stream_t stream) {
    nf4_status_t st = check_weight(w);
    if (st != NF4_OK) return st;
    if (!out) return NF4_ERR_NULL;
    if (out_dtype != NF4_F32 && out_dtype != NF4_BF16) return NF4_ERR_DTYPE;
    if (!aligned(out, 16)) return NF4_ERR_ALIGN;
    nf4::DeviceInfo dev;
    if ((st = device_ok(&dev)) != NF4_OK) return st;
    return from_cuda(nf4::launch_dequantize(w->wq, w->absmax_q, w->absmax_scale, w->absmax_offset,
                                            w->n * w->k, out, out_dtype == NF4_BF16, codebook_of(w), dev,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

static_assert(NF4_DEQUANT_BATCH_MAX == nf4::kMaxDequantBatch, "batch bound of the header and the kernel agree");

nf4_status_t nf4_dequantize_batch(const nf4_weight_t* const* w, int32_t count, void* const* out,
                                  nf4_dtype_t out_dtype, nf4_stream_t stream) {
    if (!w || !out) return NF4_ERR_NULL;
    if (count < 1 || count > NF4_DEQUANT_BATCH_MAX) return NF4_ERR_SHAPE;
    if (out_dtype != NF4_F32 && out_dtype != NF4_BF16) return NF4_ERR_DTYPE;
    nf4::DequantItem items[NF4_DEQUANT_BATCH_MAX];
    for (int32_t i = 0; i < count; ++i) {
        if (!w[i] || !out[i]) return NF4_ERR_NULL;
        const nf4_status_t st = check_weight(w[i]);
        if (st != NF4_OK) return st;
        if (!aligned(out[i], 16)) return NF4_ERR_ALIGN;
        items[i] = {w[i]->wq, w[i]->absmax_q, w[i]->absmax_scale, w[i]->absmax_offset, w[i]->n * w[i]->k, out[i],
                    codebook_of(w[i])};
    }
    nf4::DeviceInfo dev;
    nf4_status_t st;
    if ((st = device_ok(&dev)) != NF4_OK) return st;
    return from_cuda(nf4::launch_dequantize_batch(items, count, out_dtype == NF4_BF16, dev,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

// LoRA workspace: t fp32 [m, r], then its bf16 halves t_hi, t_lo [m, r] (each
// region padded to 256 bytes), then for m > 16 the scratch of the tensor-core
// down-projection, then the split-k area of the decode path.
static size_t lora_t_region(int64_t m, int32_t r, size_t elem) {
    return (static_cast<size_t>(m) * static_cast<size_t>(r) * elem + 255) / 256 * 256;
}
static size_t lora_tc_region(int64_t m, int64_t k, int32_t r) {
    return m > nf4::kGemvMaxTokens ? (nf4::lora_tc_scratch_bytes(m, k, r) + 255) / 256 * 256 : 0;
}
static size_t lora_t_bytes(int64_t m, int64_t k, int32_t r) {
    return lora_t_region(m, r, sizeof(float)) + 2 * lora_t_region(m, r, 2) + lora_tc_region(m, k, r);
}

nf4_status_t nf4_linear_lora(const void* X, int64_t m, const nf4_weight_t* w, const void* lora_down,
                             const void* lora_up, int32_t r, float scale, void* Y, nf4_dtype_t y_dtype,
                             int32_t* dev_status, uint32_t flags, void* workspace, size_t ws_bytes,
                             nf4_stream_t stream) {
    nf4_status_t st = check_weight(w);
    if (st != NF4_OK) return st;
    if (!X || !Y || !lora_down || !lora_up || !workspace) return NF4_ERR_NULL;
    if (y_dtype != NF4_F32 && y_dtype != NF4_BF16) return NF4_ERR_DTYPE;
    if ((flags & ~static_cast<uint32_t>(NF4_LINEAR_WEIGHTS_EARLY)) != 0) return NF4_ERR_DTYPE;
    if (m < 1 || w->k % NF4_BLOCKSIZE != 0 || r < 1 || r > 256) return NF4_ERR_SHAPE;
    if (m > INT64_MAX / w->k || m > INT64_MAX / w->n || m > INT64_MAX / 1024) return NF4_ERR_SHAPE;
    if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(lora_down, 16) || !aligned(lora_up, 16) ||
        !aligned(workspace, 16) || (dev_status && !aligned(dev_status, 4)))
        return NF4_ERR_ALIGN;
    nf4::DeviceInfo dev;
    if ((st = device_ok(&dev)) != NF4_OK) return st;
    const size_t tb = lora_t_bytes(m, w->k, r);
    if (ws_bytes < tb + nf4::linear_workspace_bytes(m, w->n, w->k, dev)) return NF4_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    nf4::LoraArgs lora;
    lora.up = static_cast<const __nv_bfloat16*>(lora_up);
    lora.r = r;
    if (nf4::gemv_fuses_lora(m, w->n, w->k, r, true, dev)) {
        // decode with r = 8 or 16: the dequant-GEMV forms t itself
        lora.down = static_cast<const __nv_bfloat16*>(lora_down);
        lora.scale = scale;
    } else {
        float* t = static_cast<float*>(workspace);
        __nv_bfloat16* t_hi = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(workspace) + lora_t_region(m, r, 4));
        __nv_bfloat16* t_lo = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<char*>(t_hi) + lora_t_region(m, r, 2));
        const bool early = (flags & NF4_LINEAR_WEIGHTS_EARLY) != 0;
        if (m > nf4::kGemvMaxTokens) {
            void* scratch = lora_tc_region(m, w->k, r) ? reinterpret_cast<char*>(t_lo) + lora_t_region(m, r, 2) : nullptr;
            st = from_cuda(nf4::launch_lora_down_tc(X, m, w->k, lora_down, r, scale, t, t_hi, t_lo, scratch, early,
                                                    dev, s));
        } else {
            st = from_cuda(nf4::launch_lora_down(X, m, w->k, lora_down, r, scale, t, t_hi, t_lo, early, s));
        }
        if (st != NF4_OK) return st;
        lora.t = t;
        lora.t_hi = t_hi;
        lora.t_lo = t_lo;
    }
    return from_cuda(nf4::launch_linear(X, m, w->wq, w->absmax_q, w->absmax_scale, w->absmax_offset, w->n, w->k,
                                        Y, y_dtype == NF4_BF16, dev_status, (flags & NF4_LINEAR_WEIGHTS_EARLY) != 0,
                                        static_cast<char*>(workspace) + tb, lora, codebook_of(w), dev, s));
}

nf4_status_t nf4_merge_lora(const nf4_weight_t* w, const void* lora_down, const void* lora_up, int32_t r,
                            float scale, void* w_new, uint8_t* wq_out, float* absmax_out,
                            nf4_stream_t stream) {
    nf4_status_t st = check_weight(w);
    if (st != NF4_OK) return st;
    if (!lora_down || !lora_up || !wq_out || !absmax_out) return NF4_ERR_NULL;
    if (w->k % NF4_BLOCKSIZE != 0 || r < 1 || r > 256) return NF4_ERR_SHAPE;
    if (!aligned(lora_down, 16) || !aligned(lora_up, 16) || !aligned(wq_out, 16) || !aligned(absmax_out, 4) ||
        (w_new && !aligned(w_new, 16)))
        return NF4_ERR_ALIGN;
    nf4::DeviceInfo dev;
    if ((st = device_ok(&dev)) != NF4_OK) return st;
    return from_cuda(nf4::launch_merge_lora(w->wq, w->absmax_q, w->absmax_scale, w->absmax_offset, w->n, w->k,
                                            lora_down, lora_up, r, scale, w_new, wq_out, absmax_out,
                                            codebook_of(w), dev,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

size_t nf4_linear_lora_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t r) {
    if (m < 1 || n < 1 || k < 1 || k % NF4_BLOCKSIZE != 0 || r < 1 || r > 256) return 0;
    nf4::DeviceInfo dev;
    if (device_ok(&dev) != NF4_OK) return 0;
    return lora_t_bytes(m, k, r) + nf4::linear_workspace_bytes(m, n, k, dev);
}

nf4_status_t nf4_linear_group(const void* X, int64_t m, const nf4_weight_t* const* w, int32_t count,
                              void* const* Y, nf4_dtype_t y_dtype, int32_t* dev_status, uint32_t flags,
                              void* workspace, size_t ws_bytes, nf4_stream_t stream) {
    if (!X || !w || !Y) return NF4_ERR_NULL;
    if (count < 1 || count > nf4::kMaxGroup) return NF4_ERR_SHAPE;
    nf4_status_t st;
    for (int32_t i = 0; i < count; ++i) {
        if ((st = check_weight(w[i])) != NF4_OK) return st;
        if (!Y[i]) return NF4_ERR_NULL;
        if (w[i]->k != w[0]->k) return NF4_ERR_SHAPE;
        if (w[i]->magic != w[0]->magic) return NF4_ERR_STATE;
        if (m >= 1 && m > INT64_MAX / w[i]->n) return NF4_ERR_SHAPE;
        if (!aligned(Y[i], 16)) return NF4_ERR_ALIGN;
    }
    const int64_t k = w[0]->k;
    if (y_dtype != NF4_F32 && y_dtype != NF4_BF16) return NF4_ERR_DTYPE;
    if ((flags & ~static_cast<uint32_t>(NF4_LINEAR_WEIGHTS_EARLY | NF4_LINEAR_TEST_TIMEOUT)) != 0)
        return NF4_ERR_DTYPE;
    if (m < 1 || k % NF4_BLOCKSIZE != 0 || m > INT64_MAX / k) return NF4_ERR_SHAPE;
    if (!aligned(X, 16) || (dev_status && !aligned(dev_status, 4))) return NF4_ERR_ALIGN;
    if (workspace && !aligned(workspace, 16)) return NF4_ERR_ALIGN;
    nf4::DeviceInfo dev;
    if ((st = device_ok(&dev)) != NF4_OK) return st;
    nf4::LinearWeight lw[nf4::kMaxGroup];
    for (int32_t i = 0; i < count; ++i) {
        if (workspace && ws_bytes < nf4::linear_workspace_bytes(m, w[i]->n, k, dev)) return NF4_ERR_WORKSPACE;
        lw[i].wq = w[i]->wq;
        lw[i].absmax_q = w[i]->absmax_q;
        lw[i].absmax_scale = w[i]->absmax_scale;
        lw[i].absmax_offset = w[i]->absmax_offset;
        lw[i].n = w[i]->n;
        lw[i].y = Y[i];
    }
    const uint32_t test = (flags & NF4_LINEAR_TEST_TIMEOUT) ? nf4::kTestStall : 0u;
    return from_cuda(nf4::launch_linear_group(X, m, k, lw, count, y_dtype == NF4_BF16, dev_status,
                                              (flags & NF4_LINEAR_WEIGHTS_EARLY) != 0, workspace, nf4::LoraArgs(),
                                              codebook_of(w[0]), test, dev, reinterpret_cast<cudaStream_t>(stream)));
}

int32_t nf4_linear_group_launches(int64_t m, const int64_t* n, int32_t count, int64_t k) {
    if (!n || count < 1 || count > nf4::kMaxGroup || m < 1 || k < 1 || k % NF4_BLOCKSIZE != 0) return -1;
    for (int32_t i = 0; i < count; ++i)
        if (n[i] < 1) return -1;
    nf4::DeviceInfo dev;
    if (device_ok(&dev) != NF4_OK) return -1;
    return nf4::group_in_one_launch(m, n, count, k, false, dev) ? 1 : count;
}

nf4_status_t nf4_linear_ws(const void* X, int64_t m, const nf4_weight_t* w, void* Y,
                           nf4_dtype_t y_dtype, int32_t* dev_status, uint32_t flags, void* workspace,
                           size_t ws_bytes, nf4_stream_t stream) {
    if (!w) return NF4_ERR_NULL;
    return nf4_linear_group(X, m, &w, 1, &Y, y_dtype, dev_status, flags, workspace, ws_bytes, stream);
}

nf4_status_t nf4_linear_ex(const void* X, int64_t m, const nf4_weight_t* w, void* Y,
                           nf4_dtype_t y_dtype, int32_t* dev_status, uint32_t flags, nf4_stream_t stream) {
    return nf4_linear_ws(X, m, w, Y, y_dtype, dev_status, flags, nullptr, 0, stream);
}

nf4_status_t nf4_linear_dx(const void* dY, int64_t m, const nf4_weight_t* w, void* dX,
                           nf4_dtype_t dx_dtype, int32_t* dev_status, nf4_stream_t stream) {
    nf4_status_t st = check_weight(w);
    if (st != NF4_OK) return st;
    if (!dY || !dX) return NF4_ERR_NULL;
    if (dx_dtype != NF4_F32 && dx_dtype != NF4_BF16) return NF4_ERR_DTYPE;
    if (m < 1 || w->k % NF4_BLOCKSIZE != 0 || w->n % 8 != 0) return NF4_ERR_SHAPE;
    if (m > INT64_MAX / w->k || m > INT64_MAX / w->n) return NF4_ERR_SHAPE;
    if (!aligned(dY, 16) || !aligned(dX, 16) || (dev_status && !aligned(dev_status, 4))) return NF4_ERR_ALIGN;
    nf4::DeviceInfo dev;
    if ((st = device_ok(&dev)) != NF4_OK) return st;
    return from_cuda(nf4::launch_gemm_dx(dY, m, w->wq, w->absmax_q, w->absmax_scale, w->absmax_offset, w->n,
                                         w->k, dX, dx_dtype == NF4_BF16, dev_status, codebook_of(w), dev,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

size_t nf4_linear_workspace_bytes(int64_t m, int64_t n, int64_t k) {
    if (m < 1 || n < 1 || k < 1 || k % NF4_BLOCKSIZE != 0) return 0;
    nf4::DeviceInfo dev;
    if (device_ok(&dev) != NF4_OK) return 0;
    return nf4::linear_workspace_bytes(m, n, k, dev);
}

nf4_status_t nf4_linear(const void* X, int64_t m, const nf4_weight_t* w, void* Y,
                        nf4_dtype_t y_dtype, int32_t* dev_status, nf4_stream_t stream) {
    return nf4_linear_ex(X, m, w, Y, y_dtype, dev_status, 0u, stream);
}

}  // extern "C"
