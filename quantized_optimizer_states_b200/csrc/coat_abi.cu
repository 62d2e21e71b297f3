// C ABI of libcoat.so: argument checks, the per-call scalar set-up, and the
// kernel launches.  Declarations and the contract of every entry point are
// in include/coat.h.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "coat.h"

#include "act_kernels.cuh"
#include "fp8_device.cuh"
#include "pack_kernels.cuh"
#include "resident_grid.cuh"
#include "stats_kernels.cuh"
#include "step_kernels.cuh"

namespace {

thread_local int32_t g_last_cuda_error = 0;

// Every compute entry point is one NVTX range named after it, so a profiler's
// timeline shows which library call issued which launches (header-only
// NVTX: without a tool attached a range costs a couple of branches).
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

coat_status_t launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int32_t>(e);
    return COAT_ERR_CUDA;
  }
  return COAT_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 4-byte alignment of a float array the kernels read or write (null passes)
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool valid_fmt(int32_t f) { return f == COAT_E4M3 || f == COAT_E5M2; }

// log2(G) for a supported group size, else -1.
int group_log2(int64_t G) {
  if (G < 16 || G > 4096 || (G & (G - 1)) != 0) return -1;
  int l = 0;
  while ((int64_t{1} << l) < G) ++l;
  return l;
}

double fmt_max_host(int32_t f) { return f == COAT_E4M3 ? 448.0 : 57344.0; }

double fmt_min_subnormal_host(int32_t f) {
  return f == COAT_E4M3 ? std::ldexp(1.0, -9) : std::ldexp(1.0, -16);
}

// The range that k fills: E4M3's for both states (k_range 0), or the
// storage format's own (k_range 1).
coat::StateFmtParams state_fmt_params(int32_t store_fmt, int32_t k_range) {
  const int32_t rf = k_range == 1 ? store_fmt : COAT_E4M3;
  coat::StateFmtParams f;
  f.ln_range = std::log(fmt_max_host(rf) / fmt_min_subnormal_host(rf));
  f.fmax = static_cast<float>(fmt_max_host(store_fmt));
  f.log2_fmax = static_cast<float>(std::log2(fmt_max_host(store_fmt)));
  volatile float one = 1.0f;
  f.rfmax = one / f.fmax;  // correctly rounded reciprocal
  return f;
}

void fill_log2_table(double *tab) {
  for (int i = 0; i < 8; ++i) tab[i] = std::log2(1.0 + i / 8.0);
}

unsigned int blocks_for(int64_t elems) {
  return static_cast<unsigned int>((elems + coat::kElemsPerBlock - 1) / coat::kElemsPerBlock);
}

// Launch of an activation-side kernel with programmatic stream serialization:
// the kernel may be scheduled while the kernel before it on `s` drains, and
// it waits for that kernel (pdl_enter) before its first global access.
template <class... KArgs, class... Args>
void launch_act_threads(void (*kernel)(KArgs...), unsigned int grid, unsigned int threads,
                        size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, args...);  // a failure is reported by launch_status()
}

template <class... KArgs, class... Args>
void launch_act(void (*kernel)(KArgs...), unsigned int grid, size_t smem, cudaStream_t s,
                Args... args) {
  launch_act_threads(kernel, grid, coat::kThreads, smem, s, args...);
}

// Group Scaling step (iii): the per-tensor cast.
void launch_pertensor_cast(const coat::GroupScalingParams &p, int32_t fmt, cudaStream_t s) {
  const unsigned int grid = coat::act_blocks(p.n);
  if (fmt == COAT_E4M3)
    launch_act(coat::pertensor_cast_kernel<coat::kE4M3>, grid, 0, s, p);
  else
    launch_act(coat::pertensor_cast_kernel<coat::kE5M2>, grid, 0, s, p);
}

constexpr int64_t kMaxElems = int64_t{1} << 42;  // within the grid-size bound (2^31 - 1 blocks x 2048)

// Launch one instantiation of the step kernel, raising its dynamic shared
// memory limit first when the decode tables need more than the default.
coat_status_t launch_step(void (*kernel)(coat::StepParams), unsigned int grid, int block,
                          size_t smem, cudaStream_t s, const coat::StepParams &p) {
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(
        kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) {
      g_last_cuda_error = static_cast<int32_t>(e);
      return COAT_ERR_CUDA;
    }
  }
  kernel<<<grid, block, smem, s>>>(p);
  return launch_status();
}

// The step kernel is instantiated for each supported group size, for full
// blocks / the ragged tail block, and per gradient source (BF16, float32,
// or the ranks' BF16 gradients in peer memory).
template <int VF, bool FULL, int GS>
coat_status_t launch_step_for(int lg, unsigned int grid, int block, size_t smem, cudaStream_t s,
                              const coat::StepParams &p) {
  switch (lg) {
#define COAT_LAUNCH(LGV) \
  case LGV:              \
    return launch_step(coat::adamw_fp8_step_kernel<VF, LGV, FULL, GS>, grid, block, smem, s, p);
    COAT_LAUNCH(4) COAT_LAUNCH(5) COAT_LAUNCH(6) COAT_LAUNCH(7) COAT_LAUNCH(8)
    COAT_LAUNCH(9) COAT_LAUNCH(10) COAT_LAUNCH(11) COAT_LAUNCH(12)
#undef COAT_LAUNCH
  }
  return COAT_ERR_UNSUPPORTED;
}

// One launch over the full blocks (no bounds checks), then, if n is not a
// multiple of the block's parameter count, one block for the ragged tail.
template <int VF, int GS>
coat_status_t launch_step_all(int lg, int64_t n, cudaStream_t s, coat::StepParams p) {
  size_t smem = 0;
  int block = 0;
  coat::step_launch_shape(lg, smem, block);
  if (block == 0) return COAT_ERR_UNSUPPORTED;
  const int64_t per = static_cast<int64_t>(block) * coat::kVec;
  const int64_t full = n / per;
  if (full > 0) {
    p.block0 = 0;
    const coat_status_t st =
        launch_step_for<VF, true, GS>(lg, static_cast<unsigned int>(full), block, smem, s, p);
    if (st != COAT_OK) return st;
  }
  if (n % per != 0) {
    p.block0 = full;
    return launch_step_for<VF, false, GS>(lg, 1u, block, smem, s, p);
  }
  return COAT_OK;
}

static_assert(COAT_MAX_PEERS == coat::kMaxPeers, "peer count of the header and the kernel");

// The ranks' buffers of the peer form (coat_adamw_fp8_step_peers), already
// offset to this shard.
struct PeerArgs {
  const uint16_t *grad[coat::kMaxPeers];
  void *param[coat::kMaxPeers];
  int world;
  int param_bf16;
};

coat_status_t step_impl(float *param, const void *grad, bool grad_f32, uint8_t *m_code,
                        float *m_k, float *m_scale, uint8_t *v_code, float *v_k,
                        float *v_scale, int64_t n, const coat_adamw_cfg_t *cfg,
                        const uint32_t *skip, void *stream, const PeerArgs *peers = nullptr) {
  if (!cfg || n < 0) return COAT_ERR_INVALID_ARG;
  if (n > 0 && (!param || (!grad && !peers) || !m_code || !m_k || !m_scale || !v_code ||
                !v_k || !v_scale))
    return COAT_ERR_INVALID_ARG;
  if (cfg->step < 1 || !(cfg->beta1 >= 0.0f && cfg->beta1 < 1.0f) ||
      !(cfg->beta2 >= 0.0f && cfg->beta2 < 1.0f) || !(cfg->k_max >= 0.0f) ||
      !std::isfinite(cfg->lr) || !std::isfinite(cfg->eps) || !std::isfinite(cfg->weight_decay))
    return COAT_ERR_INVALID_ARG;
  const int lg = group_log2(cfg->group_size);
  if (lg < 0 || cfg->m_fmt != COAT_E4M3 || !valid_fmt(cfg->v_fmt) ||
      (cfg->k_range != 0 && cfg->k_range != 1) || (cfg->flags & ~COAT_FORCE_K1) != 0)
    return COAT_ERR_UNSUPPORTED;
  if (n > kMaxElems) return COAT_ERR_UNSUPPORTED;
  if (n == 0) return COAT_OK;
  if (!aligned16(param) || !aligned16(grad) || !aligned16(m_code) || !aligned16(v_code) ||
      !aligned4(m_k) || !aligned4(m_scale) || !aligned4(v_k) || !aligned4(v_scale))
    return COAT_ERR_MISALIGNED;

  coat::StepParams p;
  p.world = 1;
  p.param_peer_bf16 = 0;
  for (int r = 0; r < coat::kMaxPeers; ++r) {
    p.grad_peer[r] = nullptr;
    p.param_peer[r] = nullptr;
  }
  if (peers) {
    p.world = peers->world;
    p.param_peer_bf16 = peers->param_bf16;
    for (int r = 0; r < peers->world; ++r) {
      p.grad_peer[r] = peers->grad[r];
      p.param_peer[r] = peers->param[r];
    }
  }
  p.theta = param;
  p.grad = grad_f32 ? nullptr : static_cast<const uint16_t *>(grad);
  p.grad_f32 = grad_f32 ? static_cast<const float *>(grad) : nullptr;
  p.m_code = m_code;
  p.m_k = m_k;
  p.m_s = m_scale;
  p.v_code = v_code;
  p.v_k = v_k;
  p.v_s = v_scale;
  p.n = n;
  p.ngroups = (n + cfg->group_size - 1) / cfg->group_size;
  p.beta1 = cfg->beta1;
  p.beta2 = cfg->beta2;
  // scalar factors of the rule, each rounded to binary32 once
  p.c1 = 1.0f - cfg->beta1;
  p.c2 = 1.0f - cfg->beta2;
  p.bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(cfg->beta1),
                                            static_cast<double>(cfg->step)));
  p.bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(cfg->beta2),
                                            static_cast<double>(cfg->step)));
  {
    volatile float lr_wd = cfg->lr * cfg->weight_decay;  // keep the product rounded alone
    p.decay = 1.0f - lr_wd;
    volatile float one = 1.0f;
    p.rbc1 = one / p.bc1;  // correctly rounded reciprocals for the corrected quotients
    p.rbc2 = one / p.bc2;
  }
  p.lr = cfg->lr;
  p.eps = cfg->eps;
  p.k_max = cfg->k_max;
  p.force_k1 = (cfg->flags & COAT_FORCE_K1) ? 1 : 0;
  p.m = state_fmt_params(COAT_E4M3, cfg->k_range);
  p.v = state_fmt_params(cfg->v_fmt, cfg->k_range);
  fill_log2_table(p.log2_tab);
  if (!(p.bc1 > 0.0f) || !(p.bc2 > 0.0f)) return COAT_ERR_INVALID_ARG;

  // Bounds of the estimate-based quotient (see step_kernels.cuh): v^ = v_t / bc2
  // within [2^-120, 2^100] keeps the rsqrt / rcp estimates on normal
  // numbers, and |m_t| <= 2^100 bc1 eps keeps m^ / (sqrt(v^) + eps) below
  // 2^100.  A non-normal eps disables the fast form.
  p.block0 = 0;
  p.skip = skip;
  if (p.eps >= 0x1p-100f && p.eps <= 0x1p+20f) {
    p.fast_vmin = 0x1p-120f;
    p.fast_vmax = static_cast<float>(std::ldexp(static_cast<double>(p.bc2), 100));
    p.fast_mmax = static_cast<float>(std::ldexp(static_cast<double>(p.bc1) * p.eps, 100));
  } else {
    p.fast_vmin = 0.0f;
    p.fast_vmax = 0.0f;
    p.fast_mmax = -1.0f;
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool e4 = cfg->v_fmt == COAT_E4M3;
  if (peers)
    return e4 ? launch_step_all<coat::kE4M3, coat::kGradPeers>(lg, n, s, p)
              : launch_step_all<coat::kE5M2, coat::kGradPeers>(lg, n, s, p);
  if (grad_f32)
    return e4 ? launch_step_all<coat::kE4M3, coat::kGradF32>(lg, n, s, p)
              : launch_step_all<coat::kE5M2, coat::kGradF32>(lg, n, s, p);
  return e4 ? launch_step_all<coat::kE4M3, coat::kGradBf16>(lg, n, s, p)
            : launch_step_all<coat::kE5M2, coat::kGradBf16>(lg, n, s, p);
}

// Register-resident norm rows of 256 NC columns: persistent grid of the
// blocks that fit the GPU at once (or fewer, for few rows), the occupancy
// looked up once per device.
template <int NC, bool kAffine>
coat_status_t launch_norm_reg_form(cudaStream_t s, const coat::NormParams &p) {
  constexpr auto kernel = coat::norm_reg_group_amax_kernel<NC, kAffine>;
  constexpr size_t smem = coat::norm_reg_smem<NC>();
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int32_t>(e);
    return COAT_ERR_CUDA;
  }
  const int64_t blocks_needed = (p.rows + coat::kNormRegWarps - 1) / coat::kNormRegWarps;
  const unsigned int grid = coat::resident_grid<kernel>(32 * coat::kNormRegWarps, smem, blocks_needed);
  launch_act_threads(kernel, grid, 32u * coat::kNormRegWarps, smem, s, p);
  return launch_status();
}

// weight or bias given: the instantiation with the affine terms
template <int NC>
coat_status_t launch_norm_reg(cudaStream_t s, const coat::NormParams &p) {
  return (p.weight || p.bias) ? launch_norm_reg_form<NC, true>(s, p)
                              : launch_norm_reg_form<NC, false>(s, p);
}

// Rows of 512 NCH columns, two warps a row, persistent blocks of four warp
// pairs (as many as fit the GPU at once, or fewer, for few rows).
template <int NCH, bool kAffine>
coat_status_t launch_norm_split_form(cudaStream_t s, const coat::NormParams &p) {
  constexpr auto kernel = coat::norm_split_group_amax_kernel<NCH, kAffine>;
  const int64_t need = (p.rows + coat::kSplitPairs - 1) / coat::kSplitPairs;
  const unsigned int grid = coat::resident_grid<kernel>(256, 0, need);
  launch_act_threads(kernel, grid, 256u, 0, s, p);
  return launch_status();
}

template <int NCH>
coat_status_t launch_norm_split(cudaStream_t s, const coat::NormParams &p) {
  return (p.weight || p.bias) ? launch_norm_split_form<NCH, true>(s, p)
                              : launch_norm_split_form<NCH, false>(s, p);
}

}  // namespace

extern "C" {

coat_status_t coat_adamw_fp8_step(float *param, const uint16_t *grad, uint8_t *m_code,
                                  float *m_k, float *m_scale, uint8_t *v_code, float *v_k,
                                  float *v_scale, int64_t n, const coat_adamw_cfg_t *cfg,
                                  void *stream) {
  NvtxRange nvtx_range("coat_adamw_fp8_step");
  return step_impl(param, grad, false, m_code, m_k, m_scale, v_code, v_k, v_scale, n, cfg,
                   nullptr, stream);
}

coat_status_t coat_adamw_fp8_step_fp32grad(float *param, const float *grad, uint8_t *m_code,
                                           float *m_k, float *m_scale, uint8_t *v_code,
                                           float *v_k, float *v_scale, int64_t n,
                                           const coat_adamw_cfg_t *cfg, void *stream) {
  NvtxRange nvtx_range("coat_adamw_fp8_step_fp32grad");
  return step_impl(param, grad, true, m_code, m_k, m_scale, v_code, v_k, v_scale, n, cfg,
                   nullptr, stream);
}

coat_status_t coat_adamw_fp8_step_guarded(float *param, const uint16_t *grad, uint8_t *m_code,
                                          float *m_k, float *m_scale, uint8_t *v_code,
                                          float *v_k, float *v_scale, int64_t n,
                                          const coat_adamw_cfg_t *cfg,
                                          const uint32_t *skip_if_nonzero, void *stream) {
  NvtxRange nvtx_range("coat_adamw_fp8_step_guarded");
  if (!skip_if_nonzero || (reinterpret_cast<uintptr_t>(skip_if_nonzero) & 3u) != 0)
    return skip_if_nonzero ? COAT_ERR_MISALIGNED : COAT_ERR_INVALID_ARG;
  return step_impl(param, grad, false, m_code, m_k, m_scale, v_code, v_k, v_scale, n, cfg,
                   skip_if_nonzero, stream);
}

coat_status_t coat_adamw_fp8_step_peers(const uint16_t *const *grads, int32_t world,
                                        int64_t grad_offset, float *param,
                                        void *const *params_out, int32_t params_out_bf16,
                                        int64_t params_out_offset, uint8_t *m_code, float *m_k,
                                        float *m_scale, uint8_t *v_code, float *v_k,
                                        float *v_scale, int64_t n, const coat_adamw_cfg_t *cfg,
                                        void *stream) {
  NvtxRange nvtx_range("coat_adamw_fp8_step_peers");
  if (world < 1 || world > COAT_MAX_PEERS || !grads || grad_offset < 0 ||
      params_out_offset < 0 || (params_out_bf16 != 0 && params_out_bf16 != 1))
    return COAT_ERR_INVALID_ARG;
  PeerArgs pa;
  pa.world = world;
  pa.param_bf16 = params_out_bf16;
  const size_t pesz = params_out_bf16 ? 2 : 4;
  for (int r = 0; r < COAT_MAX_PEERS; ++r) {
    pa.grad[r] = nullptr;
    pa.param[r] = nullptr;
  }
  for (int r = 0; r < world; ++r) {
    if (!grads[r]) return COAT_ERR_INVALID_ARG;
    pa.grad[r] = grads[r] + grad_offset;
    if (!aligned16(pa.grad[r])) return COAT_ERR_MISALIGNED;
    if (params_out && params_out[r]) {
      pa.param[r] = static_cast<unsigned char *>(params_out[r]) +
                    static_cast<size_t>(params_out_offset) * pesz;
      if (!aligned16(pa.param[r])) return COAT_ERR_MISALIGNED;
    }
  }
  return step_impl(param, nullptr, false, m_code, m_k, m_scale, v_code, v_k, v_scale, n, cfg,
                   nullptr, stream, &pa);
}

coat_status_t coat_enable_peer_access(int32_t peer_device) {
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return launch_status();
  if (peer_device == cur) return COAT_OK;
  int count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess) return launch_status();
  if (peer_device < 0 || peer_device >= count) return COAT_ERR_INVALID_ARG;
  int can = 0;
  if (cudaDeviceCanAccessPeer(&can, cur, peer_device) != cudaSuccess) return launch_status();
  if (!can) return COAT_ERR_UNSUPPORTED;
  const cudaError_t e = cudaDeviceEnablePeerAccess(peer_device, 0);
  if (e == cudaErrorPeerAccessAlreadyEnabled) {
    cudaGetLastError();   // not an error here: clear it
    return COAT_OK;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_last_cuda_error = static_cast<int32_t>(e);
    return COAT_ERR_CUDA;
  }
  return COAT_OK;
}

coat_status_t coat_count_nonfinite_bf16(const uint16_t *x, int64_t n, uint32_t *count,
                                        void *stream) {
  NvtxRange nvtx_range("coat_count_nonfinite_bf16");
  if (n < 0 || !count) return COAT_ERR_INVALID_ARG;
  if (n > 0 && !x) return COAT_ERR_INVALID_ARG;
  if (n > kMaxElems) return COAT_ERR_UNSUPPORTED;
  if (n == 0) return COAT_OK;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(count) & 3u) != 0) return COAT_ERR_MISALIGNED;
  coat::CountParams p;
  p.x = x;
  p.n = n;
  p.count = count;
  coat::count_nonfinite_bf16_kernel<<<coat::act_blocks(n), coat::kThreads, 0,
                                      static_cast<cudaStream_t>(stream)>>>(p);
  return launch_status();
}

coat_status_t coat_quantize_state(const float *x, int64_t n, int32_t group_size, int32_t fmt,
                                  int32_t k_range, float k_max, int32_t flags, uint8_t *code,
                                  float *k, float *scale, void *stream) {
  NvtxRange nvtx_range("coat_quantize_state");
  if (n < 0 || !(k_max >= 0.0f)) return COAT_ERR_INVALID_ARG;
  if (n > 0 && (!x || !code || !k || !scale)) return COAT_ERR_INVALID_ARG;
  const int lg = group_log2(group_size);
  if (lg < 0 || !valid_fmt(fmt) || (k_range != 0 && k_range != 1) ||
      (flags & ~COAT_FORCE_K1) != 0 || n > kMaxElems)
    return COAT_ERR_UNSUPPORTED;
  if (n == 0) return COAT_OK;
  if (!aligned16(x) || !aligned16(code) || !aligned4(k) || !aligned4(scale))
    return COAT_ERR_MISALIGNED;
  coat::QuantParams p;
  p.x = x;
  p.code = code;
  p.k = k;
  p.s = scale;
  p.n = n;
  p.log2G = lg;
  p.k_max = k_max;
  p.force_k1 = (flags & COAT_FORCE_K1) ? 1 : 0;
  p.f = state_fmt_params(fmt, k_range);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned int grid = blocks_for(n);
  if (fmt == COAT_E4M3)
    coat::quantize_state_kernel<coat::kE4M3><<<grid, coat::kThreads, 0, s>>>(p);
  else
    coat::quantize_state_kernel<coat::kE5M2><<<grid, coat::kThreads, 0, s>>>(p);
  return launch_status();
}

coat_status_t coat_dequant(const uint8_t *q, const float *k, const float *scale, int64_t n,
                           int64_t group_size, int32_t fmt, int32_t out_bf16, void *out,
                           void *stream) {
  NvtxRange nvtx_range("coat_dequant");
  if (n < 0 || group_size < 1) return COAT_ERR_INVALID_ARG;
  if (n > 0 && (!q || !scale || !out)) return COAT_ERR_INVALID_ARG;
  if (!valid_fmt(fmt) || n > kMaxElems) return COAT_ERR_UNSUPPORTED;
  int lg = -1;
  if (group_size < n) {
    lg = group_log2(group_size);
    if (lg < 0) return COAT_ERR_UNSUPPORTED;
  }
  if (n == 0) return COAT_OK;
  if (!aligned16(q) || !aligned16(out) || !aligned4(k) || !aligned4(scale))
    return COAT_ERR_MISALIGNED;
  coat::DequantParams p;
  p.q = q;
  p.k = k;
  p.scale = scale;
  p.n = n;
  p.log2G = lg;
  p.out_bf16 = out_bf16 ? 1 : 0;
  p.out = out;
  fill_log2_table(p.log2_tab);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k) {
    const unsigned int grid = blocks_for(n);
    if (fmt == COAT_E4M3)
      coat::dequant_kernel<coat::kE4M3><<<grid, coat::kThreads, 0, s>>>(p);
    else
      coat::dequant_kernel<coat::kE5M2><<<grid, coat::kThreads, 0, s>>>(p);
  } else {
    // plain loads: a streamed form (bulk copies of the codes) measured
    // slower here, the kernel being bound by its 4-byte-per-element writes
    const unsigned int grid = coat::deq_blocks(n);
    if (fmt == COAT_E4M3)
      launch_act(coat::dequant_linear_kernel<coat::kE4M3>, grid, 0, s, p);
    else
      launch_act(coat::dequant_linear_kernel<coat::kE5M2>, grid, 0, s, p);
  }
  return launch_status();
}

coat_status_t coat_group_quant_1xG(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                   int32_t group_size, int32_t fmt, uint8_t *q, float *scale,
                                   void *stream) {
  NvtxRange nvtx_range("coat_group_quant_1xG");
  if (rows < 0 || cols < 0 || ld < cols) return COAT_ERR_INVALID_ARG;
  if (rows > 0 && cols > 0 && (!x || !q || !scale)) return COAT_ERR_INVALID_ARG;
  const int lg = group_log2(group_size);
  if (lg < 0 || !valid_fmt(fmt)) return COAT_ERR_UNSUPPORTED;
  if (cols % group_size != 0) return COAT_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return COAT_OK;
  if (rows * cols > kMaxElems) return COAT_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(q) || (ld % 8) != 0 || !aligned4(scale))
    return COAT_ERR_MISALIGNED;
  coat::GroupQuantParams p;
  p.x = x;
  p.rows = rows;
  p.cols = cols;
  p.ld = ld;
  p.vec_per_row = cols / coat::kVec;
  p.log2G = lg;
  p.q = q;
  p.scale = scale;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (ld == cols) {
    // contiguous rows: one flat run, every group G consecutive elements
    const int64_t n = rows * cols;
    if (fmt == COAT_E4M3)
      launch_act(coat::group_quant_1xG_flat_kernel<coat::kE4M3>, coat::act_blocks(n), 0, s, p, n);
    else
      launch_act(coat::group_quant_1xG_flat_kernel<coat::kE5M2>, coat::act_blocks(n), 0, s, p, n);
    return launch_status();
  }
  const unsigned int grid = coat::act_blocks(p.rows * p.cols);
  if (fmt == COAT_E4M3)
    launch_act(coat::group_quant_1xG_kernel<coat::kE4M3>, grid, 0, s, p);
  else
    launch_act(coat::group_quant_1xG_kernel<coat::kE5M2>, grid, 0, s, p);
  return launch_status();
}

int64_t coat_group_scaling_workspace_bytes(int64_t n, int32_t group_size) {
  if (n < 0 || group_size < 1) return -1;
  return ((n + group_size - 1) / group_size + 1) * static_cast<int64_t>(sizeof(float));
}

coat_status_t coat_group_scaling_quant_pertensor(const uint16_t *x, int64_t n,
                                                 int32_t group_size, int32_t fmt,
                                                 float *workspace, int32_t amax_precomputed,
                                                 uint8_t *q, float *scale, void *stream) {
  NvtxRange nvtx_range("coat_group_scaling_quant_pertensor");
  if (n < 0 || amax_precomputed < 0 || amax_precomputed > 2) return COAT_ERR_INVALID_ARG;
  if (n > 0 && (!x || !workspace || !q || !scale)) return COAT_ERR_INVALID_ARG;
  const int lg = group_log2(group_size);
  if (lg < 0 || !valid_fmt(fmt) || n > kMaxElems) return COAT_ERR_UNSUPPORTED;
  if (n == 0) return COAT_OK;
  if (!aligned16(x) || !aligned16(q) || !aligned4(workspace) || !aligned4(scale))
    return COAT_ERR_MISALIGNED;
  const int64_t ng = (n + group_size - 1) / group_size;
  coat::GroupScalingParams p;
  p.x = x;
  p.n = n;
  p.ngroups = ng;
  p.log2G = lg;
  p.group_amax = workspace;
  p.tensor_amax = reinterpret_cast<uint32_t *>(workspace + ng);
  p.q = q;
  p.scale = scale;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (amax_precomputed == 2) {
    // the producer also folded its maxima into workspace[ng]: the cast alone
    launch_pertensor_cast(p, fmt, s);
    return launch_status();
  }
  // the tensor maximum accumulates with atomicMax from zero (a kernel, not a
  // memset, so the launches stay one programmatic-dependent-launch chain)
  launch_act_threads(coat::zero_word_kernel, 1u, 32u, 0, s, p.tensor_amax);
  if (amax_precomputed) {
    // one pass over the small intermediate: a few blocks per SM suffice (a
    // single 8- or 16-block cluster that reduces it through distributed
    // shared memory and stores the maximum without atomics, one launch
    // fewer, measured 0.8-1.4 us slower)
    const int64_t want = (ng + coat::kThreads - 1) / coat::kThreads;
    const unsigned int grid = static_cast<unsigned int>(want < 1184 ? want : 1184);
    launch_act(coat::amax_of_groups_kernel, grid, 0, s, p);
  } else {
    launch_act(coat::group_amax_kernel, coat::act_blocks(n), 0, s, p);
  }
  launch_pertensor_cast(p, fmt, s);
  return launch_status();
}

coat_status_t coat_swiglu_group_amax(const uint16_t *gate, const uint16_t *up, int64_t n,
                                     int32_t group_size, uint16_t *out, float *group_amax,
                                     float *tensor_amax, void *stream) {
  NvtxRange nvtx_range("coat_swiglu_group_amax");
  if (n < 0) return COAT_ERR_INVALID_ARG;
  if (n > 0 && (!gate || !up || !out || !group_amax)) return COAT_ERR_INVALID_ARG;
  const int lg = group_log2(group_size);
  if (lg < 0 || n > kMaxElems) return COAT_ERR_UNSUPPORTED;
  if (n == 0) return COAT_OK;
  if (!aligned16(gate) || !aligned16(up) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(group_amax) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(tensor_amax) & 3u) != 0)
    return COAT_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the producer's block maxima accumulate with atomicMax from zero
  if (tensor_amax)
    launch_act_threads(coat::zero_word_kernel, 1u, 32u, 0, s,
                       reinterpret_cast<uint32_t *>(tensor_amax));
  coat::SwigluParams p;
  p.gate = gate;
  p.up = up;
  p.n = n;
  p.log2G = lg;
  p.out = out;
  p.group_amax = group_amax;
  p.tensor_amax = reinterpret_cast<uint32_t *>(tensor_amax);
  launch_act(coat::swiglu_group_amax_kernel, coat::act_blocks(n), 0, s, p);
  return launch_status();
}

coat_status_t coat_norm_group_amax(const uint16_t *x, int64_t rows, int64_t cols, int32_t rms,
                                   float eps, const float *weight, const float *bias,
                                   int32_t group_size, uint16_t *out, float *group_amax,
                                   float *tensor_amax, void *stream) {
  NvtxRange nvtx_range("coat_norm_group_amax");
  if (rows < 0 || cols < 1 || (rms != 0 && rms != 1) || !(eps >= 0.0f) || !std::isfinite(eps))
    return COAT_ERR_INVALID_ARG;
  if (rms && bias) return COAT_ERR_INVALID_ARG;
  const int lg = group_log2(group_size);
  if (lg < 0) return COAT_ERR_UNSUPPORTED;
  if (cols % group_size != 0 || cols % 16 != 0) return COAT_ERR_INVALID_ARG;
  if (cols > coat::kNormMaxCols || rows > 0x7fffffff) return COAT_ERR_UNSUPPORTED;
  if (rows == 0) return COAT_OK;
  if (!x || !out || !group_amax) return COAT_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out) || (reinterpret_cast<uintptr_t>(group_amax) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(weight) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(bias) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(tensor_amax) & 3u) != 0)
    return COAT_ERR_MISALIGNED;
  coat::NormParams p;
  p.x = x;
  p.out = out;
  p.group_amax = group_amax;
  p.weight = weight;
  p.bias = bias;
  p.rows = rows;
  p.cols = cols;
  p.log2G = lg;
  p.rms = rms;
  p.eps = eps;
  p.tensor_amax = reinterpret_cast<uint32_t *>(tensor_amax);
  p.affine_vec = aligned16(weight) && aligned16(bias);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tensor_amax)
    launch_act_threads(coat::zero_word_kernel, 1u, 32u, 0, s,
                       reinterpret_cast<uint32_t *>(tensor_amax));
  if (cols % 512 == 0 && cols / 512 <= coat::kNormRegMaxChunks / 2 &&
      (cols / 2) % group_size == 0) {
    // even chunk counts whose 1xG runs lie within a half row: two warps a row
    switch (cols / 512) {
      case 1: return launch_norm_split<1>(s, p);
      case 2: return launch_norm_split<2>(s, p);
      case 3: return launch_norm_split<3>(s, p);
      default: return launch_norm_split<4>(s, p);
    }
  }
  if (cols % 256 == 0 && cols / 256 <= coat::kNormRegMaxChunks) {
    switch (cols / 256) {
      case 1: return launch_norm_reg<1>(s, p);
      case 2: return launch_norm_reg<2>(s, p);
      case 3: return launch_norm_reg<3>(s, p);
      case 4: return launch_norm_reg<4>(s, p);
      case 5: return launch_norm_reg<5>(s, p);
      case 6: return launch_norm_reg<6>(s, p);
      case 7: return launch_norm_reg<7>(s, p);
      default: return launch_norm_reg<8>(s, p);
    }
  }
  // other widths: persistent warps, each staging two rows in shared memory
  const int wpb = coat::norm_warps_per_block(cols);
  const size_t smem = static_cast<size_t>(wpb) * 2 * static_cast<size_t>(cols) * 2;
  {
    // always: the kernel's static shared memory comes on top of smem, so
    // even smem == 48 KB needs the opt-in
    const cudaError_t e = cudaFuncSetAttribute(coat::norm_group_amax_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) {
      g_last_cuda_error = static_cast<int32_t>(e);
      return COAT_ERR_CUDA;
    }
  }
  int dev = 0, sms = 1, per_sm = 1;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, coat::norm_group_amax_kernel,
                                                    32 * wpb, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t blocks_needed = (rows + wpb - 1) / wpb;
  const int64_t resident = static_cast<int64_t>(sms) * per_sm;
  const unsigned int grid =
      static_cast<unsigned int>(blocks_needed < resident ? blocks_needed : resident);
  launch_act_threads(coat::norm_group_amax_kernel, grid, 32u * wpb, smem, s, p);
  return launch_status();
}

coat_status_t coat_fp8_encode(const float *y, int64_t n, int32_t fmt, uint8_t *q,
                              void *stream) {
  NvtxRange nvtx_range("coat_fp8_encode");
  if (n < 0) return COAT_ERR_INVALID_ARG;
  if (n > 0 && (!y || !q)) return COAT_ERR_INVALID_ARG;
  if (!valid_fmt(fmt) || n > kMaxElems) return COAT_ERR_UNSUPPORTED;
  if (n == 0) return COAT_OK;
  if (!aligned16(y) || !aligned16(q)) return COAT_ERR_MISALIGNED;
  coat::EncodeParams p;
  p.y = y;
  p.n = n;
  p.q = q;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (fmt == COAT_E4M3)
    launch_act(coat::fp8_encode_kernel<coat::kE4M3>, coat::act_blocks(n), 0, s, p);
  else
    launch_act(coat::fp8_encode_kernel<coat::kE5M2>, coat::act_blocks(n), 0, s, p);
  return launch_status();
}

int32_t coat_last_cuda_error(void) { return g_last_cuda_error; }

const char *coat_status_string(coat_status_t status) {
  switch (status) {
    case COAT_OK: return "ok";
    case COAT_ERR_INVALID_ARG: return "invalid argument";
    case COAT_ERR_MISALIGNED: return "buffer not 16-byte aligned";
    case COAT_ERR_UNSUPPORTED: return "unsupported format, group size or flag";
    case COAT_ERR_CUDA: return "CUDA error";
    case COAT_ERR_NONFINITE: return "non-finite input";
    case COAT_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int32_t coat_version(void) { return (0 << 16) | (1 << 8) | 0; }

}  // extern "C"

// ---- Group Scaling with library-owned scratch (no allocation) -----------------

namespace {

constexpr int64_t kNoAllocGroups = COAT_NOALLOC_MAX_GROUPS;
constexpr int kMaxDevices = 64;

// The per-group maxima [0, kNoAllocGroups) and the tensor-max slot
// [kNoAllocGroups] of the no-allocation variant, shared by all its calls.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocGroups + 1];

std::mutex g_noalloc_mu;
float *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, resolved once
// per device (host code cannot use the symbol's name as an address).
coat_status_t noalloc_scratch(float **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int32_t>(e);
    return COAT_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return COAT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void *ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      g_last_cuda_error = static_cast<int32_t>(e);
      return COAT_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = static_cast<float *>(ptr);
  }
  *out = g_noalloc_ptr[dev];
  return COAT_OK;
}

// Multi-tensor pack / unpack: argument checks, then one launch per
// kPackTensors tensors.
coat_status_t pack_launch(bool unpack, const void *const *ptrs, const int64_t *numel,
                          const int64_t *offset, int32_t count, int32_t src_f32, void *flat,
                          int64_t n, void *stream) {
  if (count < 0 || n < 0) return COAT_ERR_INVALID_ARG;
  if (count == 0) return COAT_OK;
  if (!ptrs || !numel || !offset) return COAT_ERR_INVALID_ARG;
  bool any = false;
  int64_t chunks_in_launch = 0;
  for (int32_t i = 0; i < count; ++i) {
    if (numel[i] < 0 || offset[i] < 0 || offset[i] > n - numel[i]) return COAT_ERR_INVALID_ARG;
    if (numel[i] > 0 && unpack && !ptrs[i]) return COAT_ERR_INVALID_ARG;
    if (numel[i] > 0 && (offset[i] % 8) != 0) return COAT_ERR_MISALIGNED;
    // element alignment of a source (float32: 4 bytes, BF16: 2) or BF16 target
    const uintptr_t elem_mask = (!unpack && src_f32) ? 3u : 1u;
    if (numel[i] > 0 && (reinterpret_cast<uintptr_t>(ptrs[i]) & elem_mask) != 0)
      return COAT_ERR_MISALIGNED;
    any = any || numel[i] > 0;
    // one launch per kPackTensors tensors, its blocks counted in an int32
    if (i % coat::kPackTensors == 0) chunks_in_launch = 0;
    chunks_in_launch += (numel[i] + coat::kPackChunk - 1) / coat::kPackChunk;
    if (chunks_in_launch > 0x7fffffff) return COAT_ERR_UNSUPPORTED;
  }
  if (!any) return COAT_OK;
  if (!flat) return COAT_ERR_INVALID_ARG;
  if (!aligned16(flat)) return COAT_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int32_t base = 0; base < count; base += coat::kPackTensors) {
    const int32_t c = count - base < coat::kPackTensors ? count - base : coat::kPackTensors;
    coat::PackParams p;
    int64_t chunks = 0;
    for (int32_t i = 0; i < c; ++i) {
      p.ptr[i] = ptrs[base + i];
      p.numel[i] = numel[base + i];
      p.offset[i] = offset[base + i];
      p.chunk0[i] = static_cast<int32_t>(chunks);
      chunks += (numel[base + i] + coat::kPackChunk - 1) / coat::kPackChunk;
    }
    p.chunk0[c] = static_cast<int32_t>(chunks);
    p.count = c;
    p.src_f32 = src_f32 ? 1 : 0;
    p.flat = flat;
    if (chunks == 0) continue;
    const unsigned int grid = static_cast<unsigned int>(chunks);
    if (unpack)
      coat::unpack_bf16_kernel<<<grid, coat::kPackThreads, 0, s>>>(p);
    else
      coat::pack_bf16_kernel<<<grid, coat::kPackThreads, 0, s>>>(p);
  }
  return launch_status();
}

}  // namespace

extern "C" coat_status_t coat_state_stats(const uint8_t *code, const float *k,
                                          const float *scale, int64_t n, int32_t group_size,
                                          int32_t fmt, coat_state_stats_t *stats,
                                          void *stream) {
  NvtxRange nvtx_range("coat_state_stats");
  if (n < 0 || !stats) return COAT_ERR_INVALID_ARG;
  if (n > 0 && (!code || !k || !scale)) return COAT_ERR_INVALID_ARG;
  if (group_log2(group_size) < 0 || !valid_fmt(fmt) || n > kMaxElems)
    return COAT_ERR_UNSUPPORTED;
  if ((n > 0 && (!aligned16(code) || !aligned4(k) || !aligned4(scale))) ||
      (reinterpret_cast<uintptr_t>(stats) & 7u) != 0)
    return COAT_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  coat::state_stats_init_kernel<<<1, 1, 0, s>>>(stats);
  if (n > 0) {
    coat::StatsParams p;
    p.code = code;
    p.k = k;
    p.s = scale;
    p.n = n;
    p.ngroups = (n + group_size - 1) / group_size;
    p.max_mag = fmt == COAT_E4M3 ? 0x7Eu : 0x7Bu;
    p.out = stats;
    const int64_t want = (n / 16 + coat::kStatsThreads - 1) / coat::kStatsThreads;
    const unsigned int grid = static_cast<unsigned int>(want < 1184 ? (want > 0 ? want : 1) : 1184);
    coat::state_stats_kernel<<<grid, coat::kStatsThreads, 0, s>>>(p);
  }
  return launch_status();
}

extern "C" coat_status_t coat_pack_bf16(const void *const *src, const int64_t *numel,
                                        const int64_t *offset, int32_t count, int32_t src_f32,
                                        uint16_t *dst, int64_t n, void *stream) {
  NvtxRange nvtx_range("coat_pack_bf16");
  return pack_launch(false, src, numel, offset, count, src_f32, dst, n, stream);
}

extern "C" coat_status_t coat_unpack_bf16(const float *src, const int64_t *numel,
                                          const int64_t *offset, int32_t count, void *const *dst,
                                          int64_t n, void *stream) {
  NvtxRange nvtx_range("coat_unpack_bf16");
  return pack_launch(true, const_cast<const void *const *>(dst), numel, offset, count, 1,
                     const_cast<float *>(src), n, stream);
}

extern "C" coat_status_t coat_group_scaling_quant_pertensor_noalloc(
    const uint16_t *x, int64_t n, int32_t group_size, int32_t fmt, uint8_t *q, float *scale,
    void *stream) {
  NvtxRange nvtx_range("coat_group_scaling_quant_pertensor_noalloc");
  if (n < 0) return COAT_ERR_INVALID_ARG;
  if (n > 0 && (!x || !q || !scale)) return COAT_ERR_INVALID_ARG;
  const int lg = group_log2(group_size);
  if (lg < 0 || !valid_fmt(fmt) || n > kMaxElems) return COAT_ERR_UNSUPPORTED;
  if (n == 0) return COAT_OK;
  if (!aligned16(x) || !aligned16(q) || !aligned4(scale)) return COAT_ERR_MISALIGNED;
  const int64_t ng = (n + group_size - 1) / group_size;
  if (ng > kNoAllocGroups) return COAT_ERR_UNSUPPORTED;
  float *ws = nullptr;
  const coat_status_t st = noalloc_scratch(&ws);
  if (st != COAT_OK) return st;
  coat::GroupScalingParams p;
  p.x = x;
  p.n = n;
  p.ngroups = ng;
  p.log2G = lg;
  p.group_amax = ws;
  p.tensor_amax = reinterpret_cast<uint32_t *>(ws + kNoAllocGroups);
  p.q = q;
  p.scale = scale;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the tensor maximum accumulates with atomicMax and must start at zero
  launch_act_threads(coat::zero_word_kernel, 1u, 32u, 0, s, p.tensor_amax);
  launch_act(coat::group_amax_kernel, coat::act_blocks(n), 0, s, p);
  launch_pertensor_cast(p, fmt, s);
  return launch_status();
}
