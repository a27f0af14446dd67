/*
 * nf4.h -- C ABI of libnf4.so: NF4 weight quantization, double quantization,
 * dequantization and the fused dequantize + bf16 linear, for NVIDIA B200
 * (sm_100a).
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "Tim Dettmers 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？" (yololab.net)
 *   [P3] "bitsandbytes：让大语言模型在消费级硬件上运行的量化神器" (zingnex.cn)
 *   [P4] "LLM 相關知識" (technicalnotes, tag qlora)
 *   [P5] "篇2-bitsandbytes-具体观-算法与实现剖析" (xyzblog)
 *
 * General rules for every entry point:
 *   - All tensor arguments are DEVICE pointers on the current CUDA device, except
 *     the nf4_weight_t struct itself, which lives in host memory and borrows
 *     device pointers.  The caller allocates and frees every buffer; the library
 *     never allocates, never frees and never synchronizes the host.
 *   - Work is enqueued on `stream` (NULL = the legacy default stream) and runs
 *     asynchronously; outputs are valid once the stream reaches that point.
 *   - Arguments are validated on the host BEFORE anything is launched; on an
 *     error nothing is enqueued and the status says why.  A launch failure
 *     reported by the runtime maps to NF4_ERR_CUDA.
 *   - Inputs must be finite (documented precondition, not checked on device).
 *   - Layouts are row-major and dense.  "Element e" of a weight W[n, k] is
 *     W[e / k][e % k]; blocks of 64 are consecutive runs of elements.
 *   - The library requires a compute-capability 10.x device; other devices get
 *     NF4_ERR_UNSUPPORTED.
 */
#ifndef NF4_H
#define NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (a pointer to the runtime's opaque stream object). */
struct CUstream_st;
typedef struct CUstream_st* nf4_stream_t;

typedef enum nf4_status {
    NF4_OK = 0,
    NF4_ERR_NULL = -1,            /* a required pointer is NULL */
    NF4_ERR_SHAPE = -2,           /* a size is out of range or not a multiple of the block size */
    NF4_ERR_ALIGN = -3,           /* a pointer is not 16-byte aligned */
    NF4_ERR_DTYPE = -4,           /* unsupported dtype code */
    NF4_ERR_STATE = -5,           /* nf4_weight_t has a bad magic, version or block size */
    NF4_ERR_WORKSPACE = -6,       /* workspace missing or smaller than required */
    NF4_ERR_CUDA = -7,            /* the CUDA runtime reported an error */
    NF4_ERR_DEVICE_TIMEOUT = -8,  /* a bounded device-side wait ran out (written to dev_status) */
    NF4_ERR_UNSUPPORTED = -9      /* current device is not compute capability 10.x */
} nf4_status_t;

/* Element types of weights, activations and outputs. */
typedef enum nf4_dtype {
    NF4_F32 = 0,   /* IEEE binary32 */
    NF4_BF16 = 1   /* bfloat16 (top half of a binary32) */
} nf4_dtype_t;

#define NF4_ABI_VERSION 1
#define NF4_BLOCKSIZE 64          /* weights per absmax ([P5] §2.2 example: "split by 64") */
#define NF4_BLOCKSIZE2 256        /* absmax values per double-quantization block */
#define NF4_WEIGHT_MAGIC 0x4E463442u /* "NF4B": codes index the NF4 levels */
#define NF4_FP4_WEIGHT_MAGIC 0x46503442u /* "FP4B": codes index the FP4 values (same layout) */
#define NF4_WEIGHT_VERSION 1u

/* The 4-bit codebook of a quantization ([P5] §2.2 code walk: quant_type "nf4"
 * or "fp4"; FP4 is the generic float format with a sign bit, 2 exponent bits
 * and 1 mantissa bit, [P3] "4-bit 量化"). */
typedef enum nf4_quant_type {
    NF4_QUANT_NF4 = 0,  /* the 16 NF4 levels, ascending, exact zero at code 7 */
    NF4_QUANT_FP4 = 1   /* the 16 FP4 values in code order: code = s|e1 e0|m, exponent
                           bias 1, subnormal at e = 0, magnitudes 0, 0.5, 1, 1.5, 2, 3,
                           4, 6 divided by 6; code 8 is -0 */
} nf4_quant_type_t;

/*
 * A quantized weight W[n, k] (out_features n, in_features k) as produced by
 * nf4_quantize + nf4_double_quant: the nested quantization state of [P5] §2.2
 * code walk (packed 4-bit weight, absmax quantized again as "state2", plus the
 * offset that double quantization subtracts).  Host struct; the pointers are
 * device pointers owned by the caller.
 *   wq            uint8  [n*k/2]      two 4-bit level indices per byte, element 2i
 *                                     in the high nibble of byte i
 *   absmax_q      int8   [n*k/64]     double-quantized absmax codes
 *   absmax_scale  fp32   [ceil(n*k/64/256)]  one scale per 256 absmax values
 *   absmax_offset fp32   [1]          the mean subtracted before double quantization
 */
typedef struct nf4_weight {
    uint32_t magic;       /* NF4_WEIGHT_MAGIC, or NF4_FP4_WEIGHT_MAGIC for FP4 codes */
    uint32_t version;     /* NF4_WEIGHT_VERSION */
    int64_t n;            /* rows (out_features) */
    int64_t k;            /* columns (in_features) */
    int32_t blocksize;    /* must be NF4_BLOCKSIZE */
    int32_t blocksize2;   /* must be NF4_BLOCKSIZE2 */
    const uint8_t* wq;
    const int8_t* absmax_q;
    const float* absmax_scale;
    const float* absmax_offset;
} nf4_weight_t;

/* ABI version of the loaded library (NF4_ABI_VERSION it was built with). */
int nf4_abi_version(void);

/* Static, human-readable name of a status code. */
const char* nf4_status_str(int status);

/* The 16 NF4 levels the library uses, ascending, copied to host memory
 * `levels_out[16]` ([P5] §2.2 principle ①: N(0,1) quantiles normalised to
 * [-1, 1]; [P1] section on NF4 not being a generic FP4).  Returns NF4_OK or
 * NF4_ERR_NULL.  Host-only; launches nothing. */
nf4_status_t nf4_codebook(float* levels_out);

/* The 16 values of either codebook (NF4 ascending, FP4 in code order) copied to
 * host memory `levels_out[16]`.  Returns NF4_OK, NF4_ERR_NULL or NF4_ERR_DTYPE
 * (unknown quant_type).  Host-only. */
nf4_status_t nf4_codebook_typed(nf4_quant_type_t quant_type, float* levels_out);

/*
 * nf4_quantize -- blockwise NF4 quantization ([P5] §2.2 worked example and
 * Figure 2-2 steps 1-4; [P1] "NF4 不是一般四位元浮點格式").
 * For every block b of 64 consecutive elements of W:
 *     absmax[b] = max_j |w_j|;  x_j = w_j / absmax[b]  (IEEE fp32, round to nearest even);
 *     idx_j = index of the level nearest to x_j, ties to the lower index
 *     (a block whose absmax is 0 maps every element to the zero level, index 7);
 *     wq[32b + i] = (idx_{2i} << 4) | idx_{2i+1}.
 *   W        device, [n, k] of w_dtype (NF4_F32 or NF4_BF16; bf16 is widened exactly)
 *   wq       device, uint8 [n*k/2]       (output)
 *   absmax   device, fp32  [n*k/64]      (output)
 * Errors: NF4_ERR_NULL, NF4_ERR_SHAPE (n <= 0, k <= 0 or n*k % 64 != 0),
 * NF4_ERR_ALIGN (W or wq not 16-byte aligned, absmax not 4-byte aligned),
 * NF4_ERR_DTYPE, NF4_ERR_UNSUPPORTED, NF4_ERR_CUDA.
 */
nf4_status_t nf4_quantize(const void* W, nf4_dtype_t w_dtype, int64_t n, int64_t k,
                          uint8_t* wq, float* absmax, nf4_stream_t stream);

/*
 * nf4_quantize_typed -- nf4_quantize with either codebook.  NF4_QUANT_NF4 is
 * nf4_quantize.  NF4_QUANT_FP4 runs the same pipeline with the FP4 values:
 * code = the nearest FP4 value to x_j, ties to the lower code (toward zero),
 * so that every x_j nearest to zero, of either sign, is code 0 (+0) and code 8
 * is never written; a zero block is code 0.  Describe the result with
 * magic = NF4_FP4_WEIGHT_MAGIC; every other entry point then decodes it with
 * the FP4 values.  Errors: as nf4_quantize; NF4_ERR_DTYPE also for an unknown
 * quant_type.
 */
nf4_status_t nf4_quantize_typed(const void* W, nf4_dtype_t w_dtype, int64_t n, int64_t k,
                                nf4_quant_type_t quant_type, uint8_t* wq, float* absmax, nf4_stream_t stream);

/* Bytes of workspace nf4_double_quant needs for nb absmax values (0 if nb <= 0). */
size_t nf4_double_quant_workspace_bytes(int64_t nb);

/*
 * nf4_double_quant -- double quantization of the absmax constants ([P5] §2.2
 * principle ② and Figure 2-2 step 5; [P1] "Double quantization 連 scale 本身也壓縮";
 * [P3] "分页优化器与双量化").
 *     mu = fp32(S / nb), S the fp64 sum of all absmax in a fixed tree order:
 *          the list is cut into chunks of 256 (last chunk zero-padded), each chunk
 *          reduced by a[i] += a[i + h] for h = 128, 64, ..., 1, the chunk results
 *          form the next list, until one value is left;
 *     r_b = fp32(absmax[b] - mu);
 *     per block j of 256 absmax: s_j = max |r_b|,
 *          q_b = round_half_even(fp32(fp32(r_b / s_j) * 127)), q_b = 0 when s_j = 0.
 *   absmax        device, fp32 [nb]                 (input)
 *   workspace     device, >= nf4_double_quant_workspace_bytes(nb), 8-byte aligned;
 *                 scratch, contents undefined afterwards
 *   absmax_q      device, int8 [nb]                 (output)
 *   absmax_scale  device, fp32 [ceil(nb/256)]       (output)
 *   absmax_offset device, fp32 [1]                  (output: mu)
 * Errors: NF4_ERR_NULL, NF4_ERR_SHAPE (nb <= 0), NF4_ERR_ALIGN, NF4_ERR_WORKSPACE,
 * NF4_ERR_UNSUPPORTED, NF4_ERR_CUDA.
 */
nf4_status_t nf4_double_quant(const float* absmax, int64_t nb, void* workspace,
                              size_t workspace_bytes, int8_t* absmax_q, float* absmax_scale,
                              float* absmax_offset, nf4_stream_t stream);

/* Largest nb that nf4_double_quant_noalloc accepts: 65536 blocks of 256 absmax
 * values, i.e. weights of up to 2^30 elements per call. */
#define NF4_DQ_NOALLOC_MAX_NB 16777216

/*
 * nf4_double_quant_noalloc -- the same double quantization as nf4_double_quant,
 * with identical outputs, but without a workspace argument and without
 * allocating anything.  The pages have no counterpart to this entry point; it
 * exists for callers that cannot allocate device memory: a plugin or custom op
 * inside a host framework that owns all device memory and gives it no
 * allocator, or a deployment whose memory plan is fixed at start-up.
 *   Scratch: a fixed array of NF4_DQ_NOALLOC_MAX_NB / 256 doubles (512 KiB) in
 *   device memory, held by every GPU that loads the library until the process
 *   exits.  The first call on a device (with that device current) looks up the
 *   array's device address; make that first call before any stream capture.
 *   Every call on a device shares the array, so calls that overlap on the GPU
 *   (different streams or host threads) race and must be ordered by the
 *   caller.  No part of the array needs to start at zero.
 *   absmax, absmax_q, absmax_scale, absmax_offset: as for nf4_double_quant.
 * Errors: NF4_ERR_NULL, NF4_ERR_SHAPE (nb <= 0), NF4_ERR_WORKSPACE (nb >
 * NF4_DQ_NOALLOC_MAX_NB: the request does not fit the fixed scratch),
 * NF4_ERR_ALIGN, NF4_ERR_UNSUPPORTED, NF4_ERR_CUDA.
 */
nf4_status_t nf4_double_quant_noalloc(const float* absmax, int64_t nb, int8_t* absmax_q,
                                      float* absmax_scale, float* absmax_offset,
                                      nf4_stream_t stream);

/*
 * nf4_dequantize -- NF4 + double-quantization state back to real values ([P4]
 * §5 "動態反量化": restore the 4-bit weights to the compute dtype; [P1] the frozen
 * 4-bit base is dequantized in forward and backward).  For element e in block b:
 *     a_b = fp32(fp32(fp32(q_b / 127) * s_{b/256}) + mu);
 *     out[e] = fp32(c[idx_e] * a_b)          for out_dtype NF4_F32,
 *     out[e] = bf16_round_nearest_even(...)  for out_dtype NF4_BF16.
 *   w    host struct (validated: magic, version, block sizes, n*k % 64 == 0)
 *   out  device, [n, k] of out_dtype, 16-byte aligned  (output)
 * Errors: NF4_ERR_NULL, NF4_ERR_STATE, NF4_ERR_SHAPE, NF4_ERR_ALIGN, NF4_ERR_DTYPE,
 * NF4_ERR_UNSUPPORTED, NF4_ERR_CUDA.
 */
nf4_status_t nf4_dequantize(const nf4_weight_t* w, void* out, nf4_dtype_t out_dtype,
                            nf4_stream_t stream);

/*
 * nf4_dequantize_batch -- nf4_dequantize of up to NF4_DEQUANT_BATCH_MAX weights
 * in one launch (the weights of a layer restored together, [P4] §5), with the
 * same bits as one call per weight.  The weights may differ in shape and
 * codebook; every output has out_dtype.
 *   w      host array of count weight structs (each validated as for nf4_dequantize)
 *   count  1 .. NF4_DEQUANT_BATCH_MAX
 *   out    host array of count device pointers, out[i] [n_i, k_i] of out_dtype,
 *          16-byte aligned (outputs; they must not overlap each other or any input)
 * Errors: NF4_ERR_NULL (w, out or an entry NULL), NF4_ERR_SHAPE (count out of
 * range, or a weight's), NF4_ERR_STATE, NF4_ERR_ALIGN, NF4_ERR_DTYPE,
 * NF4_ERR_UNSUPPORTED, NF4_ERR_CUDA.  Nothing is launched on an error.
 */
#define NF4_DEQUANT_BATCH_MAX 16
nf4_status_t nf4_dequantize_batch(const nf4_weight_t* const* w, int32_t count, void* const* out,
                                  nf4_dtype_t out_dtype, nf4_stream_t stream);

/*
 * nf4_linear -- Y = X * What^T with What the bf16 dequantized weight, fused:
 * the weight is dequantized tile by tile on chip and never written out ([P5]
 * §2.2 code walk: matmul_4bit(x, weight, bias, quant_state) dequantizes and
 * multiplies; [P4] §5: per layer, 4-bit weights are restored to BF16 for the
 * matrix multiply and discarded; [P1] "量化速度取決於硬體與 kernel": without fusion
 * 4-bit can be slower than fp16, and the batch size moves the work between
 * memory- and compute-bound).  What[r][c] = bf16_round(fp32(c[idx] * a_b)); the
 * products are accumulated in fp32 in an unspecified order.  Small m (decode)
 * runs a bandwidth-bound dequant-GEMV on the tensor cores; large m (prefill)
 * runs a tcgen05 dequant-GEMM.
 *   X          device, bf16 [m, k], 16-byte aligned rows (k % 64 == 0 required)
 *   m          rows of X (tokens), >= 1
 *   w          host struct describing the [n, k] quantized weight
 *   Y          device, [m, n] of y_dtype (NF4_F32 or NF4_BF16), 16-byte aligned (output)
 *   dev_status device int32 [1] or NULL; kernels with bounded waits write
 *              NF4_ERR_DEVICE_TIMEOUT there if a wait runs out (never cleared by
 *              the library; the caller zeroes it)
 * Errors: NF4_ERR_NULL, NF4_ERR_STATE, NF4_ERR_SHAPE (m < 1, k % 64 != 0),
 * NF4_ERR_ALIGN, NF4_ERR_DTYPE, NF4_ERR_UNSUPPORTED, NF4_ERR_CUDA.
 */
nf4_status_t nf4_linear(const void* X, int64_t m, const nf4_weight_t* w, void* Y,
                        nf4_dtype_t y_dtype, int32_t* dev_status, nf4_stream_t stream);

/* Flag for nf4_linear_ex: the weight and its quantization state were NOT written
 * by the work enqueued immediately before this call on the stream (the usual
 * case at inference time, when weights are quantized once at load time).  The
 * kernel is then launched as a programmatic dependent launch: it may start
 * loading the weight while the preceding kernel is still running, and reads X
 * and writes Y only after that kernel has completed. */
#define NF4_LINEAR_WEIGHTS_EARLY 1u

/*
 * nf4_linear_ex -- nf4_linear with launch flags (0, NF4_LINEAR_WEIGHTS_EARLY,
 * NF4_LINEAR_TEST_TIMEOUT);
 * same arithmetic and results.  Arguments and errors as for nf4_linear, plus
 * NF4_ERR_DTYPE for an unknown flag bit.  Same source passages as nf4_linear;
 * the overlap of consecutive layers follows the per-layer dequantize-then-
 * multiply loop of [P4] §5, where layer N+1's weights do not depend on layer N.
 */
nf4_status_t nf4_linear_ex(const void* X, int64_t m, const nf4_weight_t* w, void* Y,
                           nf4_dtype_t y_dtype, int32_t* dev_status, uint32_t flags,
                           nf4_stream_t stream);

/* Flag for nf4_linear_ex / nf4_linear_ws / nf4_linear_group, for tests of the
 * bounded device waits only: the kernel's copy producers issue nothing and every
 * device wait gives up after a few polls, so the call writes
 * NF4_ERR_DEVICE_TIMEOUT to dev_status (when given) with no copy or tensor-core
 * operation left in flight (the GEMM frees its tensor memory).  Y is not
 * written.  The split-k workspace is left as it was. */
#define NF4_LINEAR_TEST_TIMEOUT 0x80000000u

/*
 * nf4_linear_dx -- backward through the frozen quantized base:
 * dX = dY * What, with What the bf16 dequantized weight, fused like nf4_linear:
 * the weight is dequantized tile by tile on chip and never written out ([P1]
 * "QLoRA 把 frozen 4-bit base 與可訓練 adapter 分開": the 4-bit base is dequantized
 * to the compute dtype in the backward pass as in the forward one and is not
 * updated; the gradient reaches the adapters through it).  The products
 * dY[i][r] * What[r][c] are accumulated in fp32 in an unspecified order.  Runs
 * a tcgen05 dequant-GEMM that contracts over the rows of W.
 *   dY         device, bf16 [m, n], 16-byte aligned rows (n % 8 == 0 required)
 *   m          rows of dY (tokens), >= 1
 *   w          host struct describing the [n, k] quantized weight
 *   dX         device, [m, k] of dx_dtype (NF4_F32 or NF4_BF16), 16-byte aligned (output)
 *   dev_status as for nf4_linear
 * Errors: NF4_ERR_NULL, NF4_ERR_STATE, NF4_ERR_SHAPE (m < 1, k % 64 != 0,
 * n % 8 != 0), NF4_ERR_ALIGN, NF4_ERR_DTYPE, NF4_ERR_UNSUPPORTED, NF4_ERR_CUDA.
 */
nf4_status_t nf4_linear_dx(const void* dY, int64_t m, const nf4_weight_t* w, void* dX,
                           nf4_dtype_t dx_dtype, int32_t* dev_status, nf4_stream_t stream);

/*
 * nf4_linear_lora_workspace_bytes -- bytes of the workspace nf4_linear_lora
 * needs for m tokens, an [n, k] weight and rank r: the low-rank projection
 * t [m, r] in fp32 and as two bf16 halves, for m > 16 the counters and
 * partial sums of its k-split tensor-core computation, then the split-k area
 * of nf4_linear_ws.  0 for invalid sizes.
 */
size_t nf4_linear_lora_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t r);

/*
 * nf4_linear_lora -- the QLoRA layer: the frozen quantized base plus a trained
 * low-rank update, Y = X * What^T + scale * (X * down^T) * up^T ([P4] "2-2. LoRA
 * （低秩適應）": W acts as W + dW with dW = A x B of rank r; section 4: base frozen
 * INT4, LoRA matrices bf16).  With W stored [n, k], dW = up * down.
 * t = scale * X down^T is formed in fp32.  For m <= 16 with r = 8 or 16 the
 * dequant-GEMV forms it itself: tensor-core products over the same X tiles as
 * the base, each CTA's share of k added into the split-k exchange in a fixed
 * order (no separate launch).  Other m <= 16 cases compute it first in a small
 * kernel (fixed summation order); m > 16 computes it first on the tensor cores
 * (fp32 accumulation, k split into ranges whose partial sums are added in
 * range order).  For m <= 16 the linear then adds
 * sum_j t[i][j] * up[o][j] (j in order, fp32) to each fp32 output before
 * rounding it to y_dtype.  For larger m with r % 8 == 0
 * the term runs on the tensor cores as extra K steps, t_hi up^T + t_lo up^T
 * with t = t_hi + t_lo split into bf16 halves (t kept to about 16 bits) and
 * accumulated in fp32; other ranks use the fp32 epilogue.  Same path and flags
 * as nf4_linear_ws.
 *   X          device, bf16 [m, k], 16-byte aligned
 *   w          the [n, k] quantized weight
 *   lora_down  device, bf16 [r, k] row-major (PEFT's lora_A.weight), 16-byte aligned
 *   lora_up    device, bf16 [n, r] row-major (PEFT's lora_B.weight), 16-byte aligned
 *   r          rank, 1 .. 256
 *   scale      e.g. lora_alpha / r
 *   Y          device, [m, n] of y_dtype, 16-byte aligned (output)
 *   dev_status, flags  as for nf4_linear_ex
 *   workspace  device, 16-byte aligned, >= nf4_linear_lora_workspace_bytes(m, n,
 *              k, r) bytes, zero-filled before first use (as for nf4_linear_ws)
 * Errors: as nf4_linear_ws; NF4_ERR_NULL also for a missing LoRA matrix or
 * workspace; NF4_ERR_SHAPE for r out of range.
 */
nf4_status_t nf4_linear_lora(const void* X, int64_t m, const nf4_weight_t* w, const void* lora_down,
                             const void* lora_up, int32_t r, float scale, void* Y, nf4_dtype_t y_dtype,
                             int32_t* dev_status, uint32_t flags, void* workspace, size_t ws_bytes,
                             nf4_stream_t stream);

/*
 * nf4_merge_lora -- fold a trained LoRA update into the quantized weight for
 * deployment ([P4] "8. LoRA 的合併（Merge）": the 4-bit weight is dequantized to
 * bf16, the product of the LoRA matrices is added in bf16, and the result is
 * quantized to 4 bits again).  Per element (o, c):
 *   What  = bf16_rn(level * ahat)                       (as nf4_dequantize to bf16)
 *   delta = fp32 fused-multiply-add chain over j = 0 .. r-1 of up[o][j] * down[j][c]
 *   Wnew  = bf16_rn(What + fp32(scale * delta))
 * Wnew is then quantized blockwise exactly as nf4_quantize quantizes a bf16
 * weight.  The result is bit-identical to dequantize -> add -> quantize done
 * in that arithmetic; run nf4_double_quant on absmax_out to finish the
 * storage format.  The input weight is not modified (wq_out may not alias w->wq).
 *   w          the [n, k] quantized weight (k % 64 == 0)
 *   lora_down  device, bf16 [r, k] row-major, 16-byte aligned
 *   lora_up    device, bf16 [n, r] row-major, 16-byte aligned
 *   r          rank, 1 .. 256
 *   scale      e.g. lora_alpha / r
 *   w_new      device, bf16 [n, k], 16-byte aligned, or NULL to skip writing the
 *              merged bf16 weight (output)
 *   wq_out     device, uint8 [n * k / 2] packed codes, 16-byte aligned (output)
 *   absmax_out device, fp32 [n * k / 64], 4-byte aligned (output)
 * Errors: NF4_ERR_NULL, NF4_ERR_STATE, NF4_ERR_SHAPE (k % 64 != 0, r out of
 * range), NF4_ERR_ALIGN, NF4_ERR_UNSUPPORTED, NF4_ERR_CUDA.
 */
nf4_status_t nf4_merge_lora(const nf4_weight_t* w, const void* lora_down, const void* lora_up, int32_t r,
                            float scale, void* w_new, uint8_t* wq_out, float* absmax_out,
                            nf4_stream_t stream);

/*
 * nf4_linear_workspace_bytes -- bytes of the optional split-k workspace that
 * nf4_linear_ws / nf4_linear_group can use for Y[m, n] = X[m, k] * What^T on the
 * current device; 0 when that product splits no k range (then no workspace is
 * needed), and always for m > 16 (the dequant-GEMM path).  The workspace holds
 * 1024 counters (one per 128-row tile of a launch) and room for the fp32 partial
 * sums of two CTAs per SM (each with the CTA's share of a fused LoRA
 * down-projection); the non-zero size is the same for every shape, so one
 * buffer serves every call and group of a model.  Returns 0 for invalid sizes.
 * Same source passages as nf4_linear.
 */
size_t nf4_linear_workspace_bytes(int64_t m, int64_t n, int64_t k);

/*
 * nf4_linear_ws -- nf4_linear_ex with an optional caller-owned workspace; the
 * results are bit-identical.  In the decode path (m <= 16) the k range of each
 * 128-row tile is split across several CTAs.  Without a workspace those CTAs
 * form a thread-block cluster and add their partial sums through distributed
 * shared memory, each waiting for the others.  With a workspace they meet in
 * global memory instead: every CTA stores its partial sums and counts itself in;
 * the last one adds the partials in k order and writes Y, and the others exit at
 * once.  (Same source passages as nf4_linear.)
 *   workspace  device, 16-byte aligned, at least nf4_linear_workspace_bytes(m,
 *              n, k) bytes, or NULL (the cluster path).  Its counters must be
 *              zero before first use:
 *              zero-fill the buffer once; every call leaves them zero again (a
 *              call that ends in NF4_ERR_DEVICE_TIMEOUT may not: zero it again).
 *              A workspace must not serve two calls that can run at the same
 *              time (for example on two streams).
 *   ws_bytes   size of workspace in bytes
 * Errors: as nf4_linear_ex, plus NF4_ERR_WORKSPACE (workspace smaller than
 * required) and NF4_ERR_ALIGN (workspace not 16-byte aligned).
 */
nf4_status_t nf4_linear_ws(const void* X, int64_t m, const nf4_weight_t* w, void* Y,
                           nf4_dtype_t y_dtype, int32_t* dev_status, uint32_t flags,
                           void* workspace, size_t ws_bytes, nf4_stream_t stream);

/* Most weights one nf4_linear_group call takes. */
#define NF4_LINEAR_GROUP_MAX 4

/*
 * nf4_linear_group -- Y_i = X * What_i^T for up to NF4_LINEAR_GROUP_MAX quantized
 * weights that share the input X (the query, key and value projections of an
 * attention block, the gate and up projections of an MLP), in one call.  Same
 * source passages as nf4_linear: per layer, each 4-bit weight is dequantized on
 * chip and multiplied in bf16 ([P4] §5; [P5] §2.2 code walk).  For m <= 16 the
 * weights run as one dequant-GEMV launch over all their row tiles when that is
 * predicted to be faster than one launch per weight (the query, key and value
 * projections of a layer), otherwise one launch each; larger m runs the
 * dequant-GEMM once per weight.  A grouped launch may split k differently from a
 * single-weight one, so an output can differ from nf4_linear_ws on that weight
 * alone in the fp32 summation order (not beyond it); with and without a
 * workspace the bits are the same.
 *   X          device, bf16 [m, k], 16-byte aligned
 *   w          host array of `count` pointers to weight structs, all with the same
 *              k and the same codebook (magic)
 *   count      1 .. NF4_LINEAR_GROUP_MAX
 *   Y          host array of `count` device pointers, Y[i] [m, w[i]->n] of y_dtype,
 *              16-byte aligned (outputs)
 *   dev_status, flags, workspace, ws_bytes  as for nf4_linear_ws (the workspace
 *              must meet nf4_linear_workspace_bytes for every weight)
 * Errors: as nf4_linear_ws; NF4_ERR_SHAPE also for a count out of range or
 * weights of different k, NF4_ERR_STATE for mixed codebooks.
 */
nf4_status_t nf4_linear_group(const void* X, int64_t m, const nf4_weight_t* const* w, int32_t count,
                              void* const* Y, nf4_dtype_t y_dtype, int32_t* dev_status, uint32_t flags,
                              void* workspace, size_t ws_bytes, nf4_stream_t stream);

/*
 * nf4_linear_group_launches -- how many kernel launches nf4_linear_group makes
 * for weights of rows n[0 .. count-1] and width k at m tokens on the current
 * device: 1 when they run as one grouped launch, count otherwise.  Returns -1
 * for invalid sizes or when no usable device is current.  Host only; n is a
 * host array.
 */
int32_t nf4_linear_group_launches(int64_t m, const int64_t* n, int32_t count, int64_t k);

#ifdef __cplusplus
}
#endif
#endif /* NF4_H */
