// nf4_internal.h -- launchers behind the C ABI (nf4_api.cu validates, these launch).
// Every launcher enqueues on `stream` and returns the cudaGetLastError() of its
// launches.  Arguments arrive already validated.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

namespace nf4 {

struct DeviceInfo {
    int device = -1;
    int sm_count = 0;
    int major = 0;
    int minor = 0;
    size_t smem_optin = 0;
};

// Low-rank (LoRA) term added in a linear's epilogue: Y[t, o] += sum_j t[t * r + j] * up[o * r + j]
// (t = scale * X down^T, fp32 [m, r]; up bf16 [n, r]).  t == nullptr: none.
// t_hi / t_lo: t split into two bf16 halves (t_hi = bf16(t), t_lo = bf16(t - t_hi)),
// [m, r] each, for the tensor-core form of the term in the large-m GEMM.
struct LoraArgs {
    const float* t = nullptr;
    const __nv_bfloat16* up = nullptr;
    int r = 0;
    const __nv_bfloat16* t_hi = nullptr;
    const __nv_bfloat16* t_lo = nullptr;
    // Set (with t null) when the dequant-GEMV computes t = scale * X down^T
    // itself, in its k loop (see gemv_fuses_lora).
    const __nv_bfloat16* down = nullptr;
    float scale = 0.f;
};

// A launch as a programmatic dependent of the preceding kernel on the stream:
// it may start while that kernel drains, and waits for it (griddepcontrol.wait)
// before it touches memory.  Used for kernels that begin with that wait.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Properties of the current device (cached per device).
cudaError_t current_device(DeviceInfo* out);

// `codebook` in the launchers below: 0 = NF4 levels, 1 = FP4 values.
cudaError_t launch_quantize(const void* W, bool w_bf16, int64_t n_elem, uint8_t* wq, float* absmax, int codebook,
                            const DeviceInfo& dev, cudaStream_t stream);

// Maximum number of absmax values double quantization accepts in one call.
int64_t dq_max_nb();
size_t dq_workspace_bytes(int64_t nb);
cudaError_t launch_double_quant(const float* absmax, int64_t nb, double* workspace, int8_t* absmax_q,
                                float* absmax_scale, float* absmax_offset, const DeviceInfo& dev,
                                cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t* wq, const int8_t* absmax_q, const float* absmax_scale,
                              const float* absmax_offset, int64_t n_elem, void* out, bool out_bf16, int codebook,
                              const DeviceInfo& dev, cudaStream_t stream);

// Several weights dequantized by one launch (same output dtype).
constexpr int kMaxDequantBatch = 16;
struct DequantItem {
    const uint8_t* wq;
    const int8_t* absmax_q;
    const float* absmax_scale;
    const float* absmax_offset;
    int64_t n_elem;
    void* out;
    int codebook;
};
cudaError_t launch_dequantize_batch(const DequantItem* items, int count, bool out_bf16, const DeviceInfo& dev,
                                    cudaStream_t stream);

// Bytes of the split-k workspace the decode path needs for (m, n, k); 0 if none.
size_t linear_workspace_bytes(int64_t m, int64_t n, int64_t k, const DeviceInfo& dev);

// Weights one decode launch may serve together (they share X and k).
constexpr int kMaxGroup = 4;

// Test hook for the bounded waits: the kernel's copy producers issue nothing
// and every wait gives up after a few polls, so the call ends with
// NF4_ERR_DEVICE_TIMEOUT in dev_status and nothing left in flight.
constexpr uint32_t kTestStall = 1u;

// One weight of a (grouped) linear and the output it writes, Y [m, n].
struct LinearWeight {
    const uint8_t* wq = nullptr;
    const int8_t* absmax_q = nullptr;
    const float* absmax_scale = nullptr;
    const float* absmax_offset = nullptr;
    int64_t n = 0;
    void* y = nullptr;
};

// Y_i = X * What_i^T for `count` (1 .. kMaxGroup) weights of the same k in one
// launch (m <= kGemvMaxTokens); larger m runs the GEMM once per weight.
cudaError_t launch_linear_group(const void* X, int64_t m, int64_t k, const LinearWeight* w, int count,
                                bool y_bf16, int32_t* dev_status, bool weights_early, void* ws, const LoraArgs& lora,
                                int codebook, uint32_t test_flags, const DeviceInfo& dev, cudaStream_t stream);

// True when the dequant-GEMV of an [n, k] weight at m tokens computes a LoRA
// down-projection of rank r in its own k loop (r = 8 or 16, and the split of k
// is 1 or runs through a workspace): no separate down-projection launch.
bool gemv_fuses_lora(int64_t m, int64_t n, int64_t k, int r, bool has_ws, const DeviceInfo& dev);

// True when launch_linear_group runs these weights (rows n[0 .. count-1], one
// k) as a single dequant-GEMV launch rather than one launch per weight.
bool group_in_one_launch(int64_t m, const int64_t* n, int count, int64_t k, bool lora, const DeviceInfo& dev);

// `ws` (nullable) must hold linear_workspace_bytes(m, n, k, dev) bytes, 16-byte aligned.
cudaError_t launch_linear(const void* X, int64_t m, const uint8_t* wq, const int8_t* absmax_q,
                          const float* absmax_scale, const float* absmax_offset, int64_t n,
                          int64_t k, void* Y, bool y_bf16, int32_t* dev_status, bool weights_early,
                          void* ws, const LoraArgs& lora, int codebook, const DeviceInfo& dev,
                          cudaStream_t stream);

// t[m, r] = scale * X[m, k] down[r, k]^T in fp32 (fixed order); also its two bf16
// halves when t_hi / t_lo are given.
// With `early`, launched as a programmatic dependent of the preceding kernel
// (it waits for it before reading X) and letting the next kernel start at once.
cudaError_t launch_lora_down(const void* X, int64_t m, int64_t k, const void* down, int r, float scale, float* t,
                             __nv_bfloat16* t_hi, __nv_bfloat16* t_lo, bool early, cudaStream_t stream);

// The same t on the tensor cores for the prefill path (m > 16): k split into up
// to kLoraTcMaxSplit ranges whose fp32 partials are added in split order.
// `scratch` (zero-filled before first use; the kernel leaves it zeroed) holds
// lora_tc_scratch_bytes(m, k, r) bytes: counters, then the partials.
constexpr int kLoraTcMaxSplit = 16;
int lora_tc_splits(int64_t m, int64_t k, int r, int sm_count);
size_t lora_tc_scratch_bytes(int64_t m, int64_t k, int r);
cudaError_t launch_lora_down_tc(const void* X, int64_t m, int64_t k, const void* down, int r, float scale, float* t,
                                __nv_bfloat16* t_hi, __nv_bfloat16* t_lo, void* scratch, bool early,
                                const DeviceInfo& dev, cudaStream_t stream);

// Merge a LoRA update into the quantized weight and requantize: w_new (bf16
// [n, k], may be null), wq_out [n*k/2] and absmax_out [n*k/64] fp32.
cudaError_t launch_merge_lora(const uint8_t* wq, const int8_t* absmax_q, const float* absmax_scale,
                              const float* absmax_offset, int64_t n, int64_t k, const void* down, const void* up,
                              int r, float scale, void* w_new, uint8_t* wq_out, float* absmax_out, int codebook,
                              const DeviceInfo& dev, cudaStream_t stream);

cudaError_t launch_gemm_dx(const void* dY, int64_t m, const uint8_t* wq, const int8_t* absmax_q,
                           const float* absmax_scale, const float* absmax_offset, int64_t n, int64_t k, void* dX,
                           bool dx_bf16, int32_t* dev_status, int codebook, const DeviceInfo& dev,
                           cudaStream_t stream);

cudaError_t launch_gemm(const void* X, int64_t m, const uint8_t* wq, const int8_t* absmax_q,
                        const float* absmax_scale, const float* absmax_offset, int64_t n, int64_t k, void* Y,
                        bool y_bf16, int32_t* dev_status, const LoraArgs& lora, int codebook,
                        uint32_t test_flags, const DeviceInfo& dev, cudaStream_t stream);

// Token counts up to this run the decode GEMV; larger ones the tcgen05 GEMM.
constexpr int64_t kGemvMaxTokens = 16;

}  // namespace nf4
