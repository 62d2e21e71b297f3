/*
 * coat.h -- C ABI of the B200 (sm_100a) COAT library, libcoat.so.
 *
 * COAT compresses AdamW's optimizer states and the saved activations of a
 * transformer to FP8.  This library implements the data-parallel hot path:
 * one fused AdamW step over FP8 first and second moments with COAT's
 * dynamic-range expansion, plus COAT's two activation quantizers.
 *
 * Sources, by page title and section:
 *   [COAT]  "COAT: 压缩优化器状态和激活以实现内存高效的 FP8 训练"
 *           (blog.daoxuan.cc/posts/57954).  Sections used:
 *           "为什么二阶动量对量化比一阶动量更敏感" -- the AdamW rule and its
 *             hyper-parameters beta1, beta2, eta, eps, lambda;
 *           "二阶动量的动态范围反而更小" -- E4M3 range 448 / 2^-9;
 *           "扩展函数：把窄分布拉宽" -- f(x) = sign(x)|x|^k applied before
 *             quantization, k = log(R_E4M3) / log(R_X) recomputed for every
 *             group at every step, dequantization by the 1/k power, and the
 *             E4M3+E4M3 / E4M3+E5M2 format pairs;
 *           "混合粒度：线性层和非线性层分开处理" -- 1xG group quantization
 *             along channels for nonlinear-layer inputs, and Group Scaling
 *             (max per 1xG run, then max of that small intermediate) for the
 *             per-tensor scale of linear-layer inputs;
 *           "结果和边界" -- k follows the target format's range; training
 *             on several GPUs (data-parallel ranks, every rank computing a
 *             full gradient).
 *   [ATLAS] "LLM Atlas / systems / numerics" (llm-atlas.k1412.top),
 *           section 03 "FP8" (E4M3 max 448, min subnormal 2^-9; E5M2 max
 *           57344, min subnormal 2^-16) and section 08 "Adam -> AdamW"
 *           (m_t, v_t, the bias-corrected update with eps outside the root,
 *           theta <- (1 - eta*lambda) theta + delta).
 *   [QA]    "AI 低精度格式（bfloat16/FP8/TF32）" (codechuan.com): BF16 keeps
 *           FP32's 8 exponent bits with 7 mantissa bits (conversion is a
 *           rounding of the low 16 bits); FP32 master weights with
 *           low-precision gradients.
 *
 * Common conventions
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless
 *     stated otherwise.  The library allocates no memory on any call.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call is asynchronous on that stream; the return value reports only
 *     the host-side argument checks and the launch itself.
 *   - Buffers that the kernels access with 16-byte vector instructions
 *     (parameters, gradients, codes, activations) must start on a 16-byte
 *     boundary, otherwise COAT_ERR_MISALIGNED is returned and nothing runs.
 *     Float32 metadata arrays (per-group k and s, scales, maxima) need only
 *     natural (4-byte) alignment, and every element pointer its element
 *     size's; a pointer short of that is also COAT_ERR_MISALIGNED.
 *   - Group size G: a power of two, 16 <= G <= 4096
 *     (COAT_ERR_UNSUPPORTED otherwise).
 *   - Sizes are element counts.  n == 0 is valid and launches nothing.
 *   - Errors never leave partial work behind: argument errors are found
 *     before any launch.  COAT_ERR_CUDA means a launch failed; call
 *     coat_last_cuda_error() for the CUDA error code.
 *   - FP8 encoding is round-to-nearest-even with saturation to +-max
 *     (hardware cvt ... satfinite); NaN encodes as 0x7F.
 */
#ifndef COAT_H
#define COAT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum coat_status {
    COAT_OK = 0,
    COAT_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad hyper-parameter */
    COAT_ERR_MISALIGNED = 2,  /* a buffer short of its required alignment (16-byte for vector-accessed ones) */
    COAT_ERR_UNSUPPORTED = 3, /* format / group size / flag combination not built */
    COAT_ERR_CUDA = 4,        /* a CUDA launch or query failed */
    COAT_ERR_NONFINITE = 5,   /* reserved */
    COAT_ERR_TIMEOUT = 6      /* reserved: no kernel of this library waits on the device */
} coat_status_t;

typedef enum coat_fp8 {
    COAT_E4M3 = 0, /* 1 sign, 4 exponent (bias 7), 3 mantissa; max 448, no inf */
    COAT_E5M2 = 1  /* 1 sign, 5 exponent (bias 15), 2 mantissa; max 57344 */
} coat_fp8_t;

/* cfg.flags */
#define COAT_FORCE_K1 0x1 /* ablation: k = 1 for every group (no expansion) */
/* The step takes no `stats` argument and has no finite-check or statistics
 * flags: the finite check is coat_count_nonfinite_bf16 followed by
 * coat_adamw_fp8_step_guarded (a step that becomes a no-op when the count
 * is nonzero, with no host round trip), and the per-state statistics are
 * coat_state_stats -- separate calls, so the step kernel carries none of
 * that counting. */

/* Hyper-parameters and layout of one COAT AdamW step ([COAT] AdamW
 * section; [ATLAS] section 08). */
typedef struct coat_adamw_cfg {
    float beta1;        /* first-moment decay, 0 <= beta1 < 1 */
    float beta2;        /* second-moment decay, 0 <= beta2 < 1 */
    float lr;           /* eta */
    float eps;          /* added to sqrt(v_hat) */
    float weight_decay; /* lambda; the decay applied is (1 - eta*lambda) */
    int64_t step;       /* t >= 1, already incremented for this step */
    int32_t group_size; /* G, power of two in [16, 4096] */
    int32_t m_fmt;      /* COAT_E4M3 (the only first-moment format COAT uses) */
    int32_t v_fmt;      /* COAT_E4M3 or COAT_E5M2 */
    int32_t k_range;    /* 0: k targets the E4M3 range for both states;
                           1: k targets the storage format's own range */
    float k_max;        /* upper clamp for k (0 = none); 64 recommended */
    int32_t flags;      /* COAT_FORCE_K1 or 0 */
} coat_adamw_cfg_t;

/*
 * coat_adamw_fp8_step -- one fused COAT AdamW step, in place.
 * [COAT] sections on AdamW and on the expansion function; [ATLAS] 08.
 *
 * Layout: n parameters in one flat buffer; groups are the runs
 * [i*G, (i+1)*G) of that buffer (the last may be shorter);
 * ngroups = ceil(n / G).
 *   param    float32[n]   FP32 master weights theta (read, written)
 *   grad     uint16[n]    BF16 gradient bit patterns (read)
 *   m_code   uint8[n]     first moment, FP8 codes in m_fmt (read, written)
 *   m_k      float32[ngroups]  per-group expansion exponent k of m
 *   m_scale  float32[ngroups]  per-group scale s of m
 *   v_code, v_k, v_scale  the same for the second moment in v_fmt
 * Stored state per group: x = sign(d) * |d|^(1/k) * s for decoded FP8 d
 * (an all-zero group stores k = 1, s = 0).
 *
 * Per element: g = float(grad); m, v = dequantized states;
 *   m_t = beta1*m + (1-beta1)*g;  v_t = beta2*v + (1-beta2)*g*g;
 *   theta = (1 - lr*wd)*theta - lr * (m_t/(1-beta1^t)) / (sqrt(v_t/(1-beta2^t)) + eps).
 * Per group, for each of m_t and v_t: M = max|x|, mn = min nonzero |x|,
 *   k = log(R)/log(M/mn) with R = 448/2^-9 (k_range 0) or the storage
 *   format's max/min-subnormal (k_range 1), clamped to k_max, k = 1 when
 *   M == mn; s = M * fmt_max^(-1/k); code = sign(x) . RNE(fmt_max * (|x|/M)^k).
 * Alignment: param, grad, m_code, v_code 16-byte aligned.
 * Errors: INVALID_ARG (null pointer, n < 0, step < 1, betas outside [0,1),
 * k_max < 0), UNSUPPORTED (G, formats, flags), MISALIGNED, CUDA.
 * Buffers must not overlap.  Results are bit-reproducible run to run.
 */
coat_status_t coat_adamw_fp8_step(float *param, const uint16_t *grad, uint8_t *m_code,
                                  float *m_k, float *m_scale, uint8_t *v_code, float *v_k,
                                  float *v_scale, int64_t n, const coat_adamw_cfg_t *cfg,
                                  void *stream);

/*
 * coat_count_nonfinite_bf16 -- *count += the number of BF16 values in x that
 * are +-inf or NaN (all-ones exponent).  The caller zeroes *count first.
 * With coat_adamw_fp8_step_guarded this skips a step on overflowed
 * gradients without a host round trip (the pages define no behaviour for
 * non-finite gradients; skipping the step is the usual mixed-precision
 * convention).
 *   x      BF16 bits [n] (16-byte aligned)
 *   count  uint32[1] (4-byte aligned), accumulated atomically
 * Errors: INVALID_ARG, UNSUPPORTED (n too large), MISALIGNED, CUDA.
 */
coat_status_t coat_count_nonfinite_bf16(const uint16_t *x, int64_t n, uint32_t *count,
                                        void *stream);

/*
 * coat_adamw_fp8_step_fp32grad -- coat_adamw_fp8_step with float32 gradients
 * (e.g. a flat float32 gradient buffer that a framework accumulates into):
 * each gradient is rounded to BF16 (nearest even) as it is loaded and the
 * step then proceeds exactly as with that BF16 gradient ([QA]: BF16
 * gradients, FP32 master weights), so the results are those of
 * coat_adamw_fp8_step on the rounded gradients.  It saves the separate
 * float32 -> BF16 pass (6 B per parameter of HBM traffic) at the cost of
 * reading 4 instead of 2 gradient bytes in the step.
 *   grad   float32[n] (16-byte aligned)
 * Other arguments and errors as coat_adamw_fp8_step.
 */
coat_status_t coat_adamw_fp8_step_fp32grad(float *param, const float *grad, uint8_t *m_code,
                                           float *m_k, float *m_scale, uint8_t *v_code,
                                           float *v_k, float *v_scale, int64_t n,
                                           const coat_adamw_cfg_t *cfg, void *stream);

/*
 * coat_adamw_fp8_step_guarded -- coat_adamw_fp8_step, except that the
 * kernel first reads the device word *skip_if_nonzero and, if it is not
 * zero, returns without reading or writing anything else: parameters,
 * codes, k and s keep their values (for example, skip_if_nonzero = the
 * count of coat_count_nonfinite_bf16 on grad).  The decision is made on the
 * device, so the call stays asynchronous; cfg->step is still the caller's
 * step count (a skipped step leaves it to the caller whether to advance it).
 * Arguments and errors as coat_adamw_fp8_step; skip_if_nonzero must be a
 * 4-byte-aligned device pointer (INVALID_ARG if NULL, MISALIGNED).
 */
coat_status_t coat_adamw_fp8_step_guarded(float *param, const uint16_t *grad, uint8_t *m_code,
                                          float *m_k, float *m_scale, uint8_t *v_code,
                                          float *v_k, float *v_scale, int64_t n,
                                          const coat_adamw_cfg_t *cfg,
                                          const uint32_t *skip_if_nonzero, void *stream);

/*
 * coat_adamw_fp8_step_peers -- one ZeRO-1 data-parallel step of this rank's
 * shard in one kernel ([COAT] "结果和边界": multi-GPU data-parallel
 * training; the optimizer state is partitioned over the ranks at 1xG group
 * boundaries): the reduce-scatter of the ranks' gradients, the step of
 * coat_adamw_fp8_step on the shard, and the all-gather of the updated
 * parameters, over peer memory (plain loads and stores; NVLink between
 * GPUs).
 *   grads      host array of `world` device pointers: rank r's full BF16
 *              gradient buffer, mapped into this process; the shard's
 *              gradient element i is the mean of grads[r][grad_offset + i]
 *              over r, RN_bf16(RN32(sum) / world) with the sum in binary32
 *              in rank order (world = 1: the gradient itself)
 *   world      1 .. COAT_MAX_PEERS
 *   param      float32[n]: this rank's FP32 master weights (its shard),
 *              updated in place
 *   params_out host array of `world` device pointers or NULL: rank r's full
 *              parameter buffer (float32, or BF16 when params_out_bf16 = 1);
 *              every updated parameter i is also stored at
 *              params_out[r][params_out_offset + i] (an entry may be NULL:
 *              that rank gets no copy)
 *   m_code .. v_scale, n, cfg   this rank's shard, as coat_adamw_fp8_step
 * Every grads[r] + grad_offset and params_out[r] + params_out_offset must be
 * 16-byte aligned, and the current device must be able to access each of
 * them (coat_enable_peer_access for another GPU's memory).  The caller orders the call between two barriers of all
 * ranks: after every rank's gradient is complete, and before any rank
 * reads its parameters (the kernel reads other ranks' gradients and writes
 * their parameter buffers; it waits for nothing on the device).  The
 * kernel makes its stores to other ranks' memory visible system-wide
 * before it finishes.
 * Errors: INVALID_ARG (world, a NULL gradient pointer, offsets < 0,
 * params_out_bf16 not 0/1, and as coat_adamw_fp8_step), MISALIGNED,
 * UNSUPPORTED, CUDA.
 */
#define COAT_MAX_PEERS 8

/*
 * coat_enable_peer_access -- let kernels launched on the current device read
 * and write the memory of GPU `peer_device` (a rank's buffers mapped into
 * this process live there): cudaDeviceEnablePeerAccess from the current
 * device, where the two can reach each other.  A call for the current
 * device, or for a peer already enabled, does nothing.
 * Errors: INVALID_ARG (no such device), UNSUPPORTED (the two devices cannot
 * reach each other), CUDA.
 */
coat_status_t coat_enable_peer_access(int32_t peer_device);
coat_status_t coat_adamw_fp8_step_peers(const uint16_t *const *grads, int32_t world,
                                        int64_t grad_offset, float *param,
                                        void *const *params_out, int32_t params_out_bf16,
                                        int64_t params_out_offset, uint8_t *m_code, float *m_k,
                                        float *m_scale, uint8_t *v_code, float *v_k,
                                        float *v_scale, int64_t n, const coat_adamw_cfg_t *cfg,
                                        void *stream);

/*
 * coat_quantize_state -- compress an FP32 optimizer state into COAT's FP8
 * form (the re-quantization half of the step, on its own): used to
 * initialize or convert states.  [COAT] "扩展函数".
 *   x      float32[n]        input (16-byte aligned)
 *   code   uint8[n]          output codes in `fmt` (16-byte aligned)
 *   k, scale float32[ceil(n/G)]  outputs
 * k_range, k_max, flags as in coat_adamw_cfg_t.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, CUDA.
 */
coat_status_t coat_quantize_state(const float *x, int64_t n, int32_t group_size, int32_t fmt,
                                  int32_t k_range, float k_max, int32_t flags, uint8_t *code,
                                  float *k, float *scale, void *stream);

/*
 * coat_dequant -- decode FP8 codes to FP32 or BF16.
 * [COAT] "扩展函数" (inverse by the 1/k power) and "混合粒度" (activation
 * scales).
 *   q      uint8[n] codes in `fmt` (16-byte aligned)
 *   k      float32[ceil(n/G)] per-group exponents, or NULL for k = 1
 *          (activations: x = decode(q) * s exactly)
 *   scale  float32[ceil(n/G)] per-group scales; G = n (or any G >= n)
 *          with a single scale gives per-tensor dequantization
 *   out    float32[n] (out_bf16 == 0) or BF16 bits uint16[n] (out_bf16 != 0,
 *          nearest-even rounding of the FP32 value), 16-byte aligned
 * Here G may be any positive count (it only maps element -> scale index).
 * Errors: INVALID_ARG, UNSUPPORTED (fmt), MISALIGNED, CUDA.
 */
coat_status_t coat_dequant(const uint8_t *q, const float *k, const float *scale, int64_t n,
                           int64_t group_size, int32_t fmt, int32_t out_bf16, void *out,
                           void *stream);

/*
 * coat_group_quant_1xG -- COAT's 1xG group quantization of a nonlinear-layer
 * input.  [COAT] "混合粒度": groups of G consecutive channels of one token.
 *   x      BF16 bits, row-major [rows, cols] with row stride ld >= cols
 *          (16-byte aligned; ld a multiple of 8)
 *   q      uint8 [rows, cols], row stride cols (16-byte aligned)
 *   scale  float32 [rows, cols/G], s = amax/fmt_max per group
 * Codes: RNE_satfinite(x * (fmt_max/amax)), the product rounded to FP32
 * first; a group with amax <= 2^-100 (e.g. all zero) uses s = 1.
 * Requires cols % G == 0.  Bit-exact by construction.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, CUDA.
 */
coat_status_t coat_group_quant_1xG(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                   int32_t group_size, int32_t fmt, uint8_t *q, float *scale,
                                   void *stream);

/* Bytes of workspace coat_group_scaling_quant_pertensor needs for n values
 * in groups of G: (ceil(n/G) + 1) float32 slots.  Host function, no GPU. */
int64_t coat_group_scaling_workspace_bytes(int64_t n, int32_t group_size);

/*
 * coat_group_scaling_quant_pertensor -- COAT's "Group Scaling" per-tensor
 * FP8 quantization of a linear-layer input.  [COAT] "混合粒度": (i) the max
 * of each 1xG run goes to a small intermediate; (ii) the max of that
 * intermediate is the tensor's amax; (iii) one cast with s = amax/fmt_max.
 *   x          BF16 bits [n] (16-byte aligned)
 *   workspace  float32[ceil(n/G) + 1] (4-byte aligned).  Slots
 *              [0, ceil(n/G)) hold the per-group maxima: written by step (i)
 *              when amax_precomputed == 0, or filled beforehand by the
 *              producing kernel when amax_precomputed == 1 (step (i) is then
 *              skipped).  The last slot holds the tensor maximum of step
 *              (ii); amax_precomputed == 2: the producer also wrote that
 *              slot (its tensor_amax output), and only the cast runs.
 *              Other amax_precomputed values: INVALID_ARG.
 *   q          uint8[n] codes (16-byte aligned)
 *   scale      float32[1], the per-tensor scale s (amax <= 2^-100 gives 1)
 * Bit-exact: amax is an exact max and s, the reciprocal and the product
 * are single IEEE operations.  Calls on the same workspace must not
 * overlap on the GPU.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, CUDA.
 */
coat_status_t coat_group_scaling_quant_pertensor(const uint16_t *x, int64_t n,
                                                 int32_t group_size, int32_t fmt,
                                                 float *workspace, int32_t amax_precomputed,
                                                 uint8_t *q, float *scale, void *stream);

/* Capacity, in 1xG groups, of the library-owned scratch that
 * coat_group_scaling_quant_pertensor_noalloc uses (4 MiB of device memory
 * per GPU, plus one slot). */
#define COAT_NOALLOC_MAX_GROUPS (1 << 20)

/*
 * coat_group_scaling_quant_pertensor_noalloc -- the same Group Scaling
 * quantization as coat_group_scaling_quant_pertensor (amax_precomputed = 0),
 * for callers that cannot allocate device memory: for example a serving
 * process that reserves its whole memory budget at start-up and forbids
 * allocation afterwards, or a plug-in hosted by a framework that owns every
 * device allocation and hands the plug-in no allocator.  It takes no
 * workspace and allocates nothing (no cudaMalloc, no allocating library
 * call).  (The COAT pages have no counterpart: this is an interface
 * convenience only.)
 *
 * Scratch: a fixed array of COAT_NOALLOC_MAX_GROUPS + 1 float32 slots
 * compiled into the library as a device variable; every GPU that loads the
 * library holds it until the process exits.  The first call on a device
 * resolves that array's address for the current device (a one-time,
 * non-allocating runtime query), so make the first call on each device
 * before any stream capture.  The address is kept for the life of the
 * process: after cudaDeviceReset (which gives the device a new context and
 * the array a new address) this entry point must not be called again in
 * that process.  Every call shares the array: calls that
 * overlap on the GPU (on different streams, or from different threads
 * without ordering) race on it and must be serialised by the caller.
 *   x      BF16 bits [n] (16-byte aligned)
 *   q      uint8[n] codes (16-byte aligned)
 *   scale  float32[1], the per-tensor scale s
 * Errors: INVALID_ARG, MISALIGNED, CUDA, and UNSUPPORTED for an unsupported
 * format or group size or when ceil(n/G) > COAT_NOALLOC_MAX_GROUPS.
 */
coat_status_t coat_group_scaling_quant_pertensor_noalloc(const uint16_t *x, int64_t n,
                                                         int32_t group_size, int32_t fmt,
                                                         uint8_t *q, float *scale,
                                                         void *stream);

/*
 * coat_fp8_encode -- the FP8 cast alone: code = RNE_satfinite(y), the last
 * operation of every quantizer here.  [ATLAS] 03 "FP8": E4M3 (bias 7, max
 * 448, no infinity) and E5M2 (bias 15, max 57344); round to nearest even;
 * finite values beyond the largest magnitude and infinities saturate to
 * +-max; NaN gives a NaN code (either sign).
 *   y  float32[n] (16-byte aligned)
 *   q  uint8[n] codes (16-byte aligned)
 * Errors: INVALID_ARG, UNSUPPORTED (format), MISALIGNED, CUDA.
 */
coat_status_t coat_fp8_encode(const float *y, int64_t n, int32_t fmt, uint8_t *q, void *stream);

/*
 * coat_swiglu_group_amax -- a producing kernel with Group Scaling's step (i)
 * fused in.  [COAT] "混合粒度": the per-1xG maxima of a linear layer's
 * input are emitted by the kernel that produces it, so the per-tensor
 * quantizer only reads the G-times-smaller intermediate before its cast.
 * This producer is the SwiGLU of a GLU MLP ([COAT] "激活为什么难压"), whose
 * output feeds the down projection:
 *   out[i] = RN_bf16(silu(gate[i]) * up[i]),  silu(g) = g / (1 + e^-g),
 * evaluated in binary32 with the hardware exp2 and reciprocal estimates
 * (relative error ~2^-20), then rounded to nearest even BF16: the correctly
 * rounded BF16 value except next to a rounding midpoint.
 *   gate, up    BF16 bits [n] (16-byte aligned)
 *   out         BF16 bits [n] (16-byte aligned)
 *   group_amax  float32[ceil(n/G)] (4-byte aligned): max |out| over each
 *               1xG run of the flat output (the last run may be shorter) --
 *               exactly the slots coat_group_scaling_quant_pertensor reads
 *               when called on `out` with amax_precomputed != 0
 *   tensor_amax float32[1] or NULL (4-byte aligned): when given, zeroed and
 *               then set to max |out| over the whole output (step (ii),
 *               folded into the producer with one atomic max per block):
 *               pass workspace + ceil(n/G) and call Group Scaling with
 *               amax_precomputed == 2 to run the cast alone.
 * Errors: INVALID_ARG, UNSUPPORTED (group size), MISALIGNED, CUDA.
 */
coat_status_t coat_swiglu_group_amax(const uint16_t *gate, const uint16_t *up, int64_t n,
                                     int32_t group_size, uint16_t *out, float *group_amax,
                                     float *tensor_amax, void *stream);

/*
 * coat_pack_bf16 -- gather `count` tensors into one flat BF16 buffer with
 * one launch per 128 tensors: element j of tensor i goes to
 * dst[offset[i] + j], converted from float32 (round to nearest even, as a
 * BF16 cast does; NaN stays a NaN) when src_f32 != 0, else copied as BF16
 * bits; a NULL src[i] fills its slice with zeros.  This lays the
 * per-parameter BF16 gradients of a parameter group out for one
 * coat_adamw_fp8_step ([QA]: FP32 -> BF16 by rounding away the low 16 bits;
 * the flat 1xG layout is this library's, see coat_adamw_fp8_step).
 *   src     HOST array [count] of device pointers (float32 or BF16 bits)
 *   numel   HOST array [count]: elements of each tensor (>= 0)
 *   offset  HOST array [count]: destination offset of each tensor, a
 *           multiple of 8 (MISALIGNED otherwise), offset + numel <= n
 *   dst     BF16 bits [n] device buffer (16-byte aligned)
 * The tables are copied into the kernels' parameter blocks, so nothing is
 * allocated.  Slices must not overlap (not checked); elements of dst
 * outside every slice are left as they are.
 * Errors: INVALID_ARG (NULL tables with count > 0, negative sizes, a slice
 * outside [0, n), dst NULL), MISALIGNED, UNSUPPORTED (over 2^31 2048-element
 * chunks in one launch), CUDA.
 */
coat_status_t coat_pack_bf16(const void *const *src, const int64_t *numel, const int64_t *offset,
                             int32_t count, int32_t src_f32, uint16_t *dst, int64_t n,
                             void *stream);

/*
 * coat_unpack_bf16 -- the reverse for BF16 parameters: dst[i][j] =
 * BF16(src[offset[i] + j]) (nearest even) for the `count` tensors, e.g. the
 * updated float32 master weights of a parameter group written back into its
 * BF16 parameters.
 *   src     float32 [n] device buffer (16-byte aligned)
 *   numel, offset  HOST arrays as in coat_pack_bf16
 *   dst     HOST array [count] of device pointers to BF16 tensors (not NULL
 *           where numel > 0)
 * Errors as coat_pack_bf16.
 */
coat_status_t coat_unpack_bf16(const float *src, const int64_t *numel, const int64_t *offset,
                               int32_t count, void *const *dst, int64_t n, void *stream);

/*
 * coat_state_stats -- monitoring of one compressed optimizer state (codes in
 * `fmt` with per-group k and s, as coat_adamw_fp8_step leaves them).  The
 * pages define no such report; it counts what COAT's expansion is meant to
 * produce ([COAT] "扩展函数": every group's maximum on the format's largest
 * value, k per group and step, typically 1-3 for m and 5-15 for v).  Two
 * launches: one initialising *stats, one accumulating into it; read it after
 * the stream reaches them.
 *   code   uint8[n] (16-byte aligned);  k, scale  float32[ceil(n/G)]
 *   stats  DEVICE pointer to a coat_state_stats_t (8-byte aligned):
 *     groups          ceil(n/G)
 *     zero_groups     groups with scale 0 (all-zero groups)
 *     k1_groups       other groups stored with k == 1 (no expansion)
 *     max_codes       codes whose magnitude is the format's largest finite
 *                     value (0x7E E4M3, 0x7B E5M2): at least one per
 *                     nonzero group
 *     zero_codes      codes +-0
 *     nonfinite_codes inf / NaN codes (0 for states the library wrote)
 *     k_sum, k_min, k_max  over the nonzero groups (+inf / -inf / 0 when
 *                     there are none); mean k = k_sum / (groups - zero_groups);
 *                     k_sum is summed with floating-point atomics, so its
 *                     last bits can differ between runs (the counts and
 *                     k_min / k_max are exact)
 * Errors: INVALID_ARG, UNSUPPORTED (G, fmt), MISALIGNED, CUDA.
 */
typedef struct {
  uint64_t groups, zero_groups, k1_groups;
  uint64_t max_codes, zero_codes, nonfinite_codes;
  double k_sum;
  float k_min, k_max;
} coat_state_stats_t;

coat_status_t coat_state_stats(const uint8_t *code, const float *k, const float *scale,
                               int64_t n, int32_t group_size, int32_t fmt,
                               coat_state_stats_t *stats, void *stream);

/*
 * coat_norm_group_amax -- a second producer with Group Scaling's step (i)
 * fused in ([COAT] "混合粒度"; the norm is one of the nonlinear layers of
 * "激活为什么难压" and produces the input of the QKV and MLP up/gate
 * projections): row-wise LayerNorm (rms = 0: y = (x - mean) / sqrt(var +
 * eps), var the mean squared deviation) or RMSNorm (rms = 1: y = x /
 * sqrt(mean(x^2) + eps)), times weight[c] and plus bias[c] (LayerNorm only)
 * when given (with both, y weight + bias is one fused multiply-add),
 * rounded to BF16; plus the maxima of |out| over every 1xG run of each row.
 * Evaluated in binary32 (row sums in a fixed order, divided by cols with
 * the correctly rounded quotient, so a row whose sum is exact -- a constant
 * row, say -- gets its exact mean), with an error of about 1e-6 x (|out| +
 * (|x - mean| + |mean|) / std x |weight|) (x - mean carries the rounding
 * of the mean; with a bias the error is relative to the product, not to
 * the sum): the output is the correctly rounded norm except within that
 * distance of a BF16 rounding midpoint.  weight and bias are read 16 bytes
 * at a time when both (those given) are 16-byte aligned.
 *   x           BF16 bits [rows, cols] row-major (16-byte aligned),
 *               cols a multiple of 16 and of G, cols <= 16384
 *   weight,bias float32 [cols] or NULL (bias must be NULL when rms = 1)
 *   out         BF16 bits [rows, cols] (16-byte aligned)
 *   group_amax  float32 [rows * cols / G]: the slots
 *               coat_group_scaling_quant_pertensor reads on `out` (flat,
 *               the same G) with amax_precomputed != 0
 *   tensor_amax float32[1] or NULL: as for coat_swiglu_group_amax
 * Errors: INVALID_ARG (sizes, eps < 0 or not finite, rms not 0/1, bias with
 * rms), UNSUPPORTED (G, cols > 16384, rows > 2^31 - 1), MISALIGNED, CUDA.
 */
coat_status_t coat_norm_group_amax(const uint16_t *x, int64_t rows, int64_t cols, int32_t rms,
                                   float eps, const float *weight, const float *bias,
                                   int32_t group_size, uint16_t *out, float *group_amax,
                                   float *tensor_amax, void *stream);

/* The last CUDA error code seen by a call that returned COAT_ERR_CUDA in
 * this thread (0 if none). */
int32_t coat_last_cuda_error(void);

/* A static, human-readable name for a status code. */
const char *coat_status_string(coat_status_t status);

/* Library version as (major << 16) | (minor << 8) | patch. */
int32_t coat_version(void);

#ifdef __cplusplus
}
#endif

#endif /* COAT_H */
