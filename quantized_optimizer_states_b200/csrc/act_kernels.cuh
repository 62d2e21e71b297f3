// COAT activation quantizers and FP8 dequantization.
//
// COAT summary page (blog.daoxuan.cc/posts/57954), section
// "混合粒度：线性层和非线性层分开处理":
//   - nonlinear-layer inputs: 1xG group quantization along the channel axis
//     of each token (not BxB tiles);
//   - linear-layer inputs: one scale per tensor, found by "Group Scaling":
//     (i) the max of every 1xG run, cached in a small intermediate (which
//     the producing kernel can emit), (ii) the max of that G-times-smaller
//     intermediate, (iii) the cast.
// Scale convention: s = amax / fmt_max; codes = RNE_satfinite(x * (fmt_max /
// amax)) with the product rounded to binary32 first, so GPU and CPU agree
// bit for bit.  amax <= 2^-100 (e.g. an all-zero group) uses s = 1.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "fp8_device.cuh"
#include "state_codec.cuh"
#include "step_kernels.cuh"

namespace coat {

// Programmatic dependent launch.  The host launches these kernels with
// programmatic stream serialization, so a kernel may be scheduled while the
// kernel before it on the stream is still draining.  First thing, each block
// allows the next kernel to be scheduled likewise (only once every block of
// this grid has started, so no waiting block ever takes a slot this grid
// still needs), then waits until the previous grid has completed and its
// writes are visible -- stream order is kept for every global access.
// Launched without the attribute, both instructions do nothing.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// 16-byte global -> shared copy on the asynchronous copy path (no registers
// held), and the waits for this thread's own outstanding copy groups.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_one() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

__device__ __forceinline__ void act_scale(float amax, float fmax, float &s, float &inv) {
  if (amax > 0x1p-100f) {
    s = __fdiv_rn(amax, fmax);
    inv = __fdiv_rn(fmax, amax);
  } else {
    s = 1.0f;
    inv = 1.0f;
  }
}

// 16 BF16 values (eight words) -> 16 floats.
__device__ __forceinline__ void unpack16_bf16(const uint32_t *w, float *x) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = bf16lo_to_float(w[i]);
    x[2 * i + 1] = bf16hi_to_float(w[i]);
  }
}

__device__ __forceinline__ float amax16(const float *x) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
  return a;
}

// Max over the threads of one group (lanes = G/16).
__device__ __forceinline__ float group_max(float a, int lanes, float *red) {
  const int lim = lanes < 32 ? lanes : 32;
  for (int off = 1; off < lim; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  if (lanes > 32) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[warp] = a;
    __syncthreads();
    const int wpg = lanes >> 5;
    const int w0 = (warp / wpg) * wpg;
    a = red[w0];
    for (int i = 1; i < wpg; ++i) a = fmaxf(a, red[w0 + i]);
  }
  return a;
}

// Zeroes the tensor-maximum word a producer then accumulates into (a
// kernel rather than a memset, so that it joins the programmatic
// dependent launch chain of the kernels around it).
__global__ void zero_word_kernel(uint32_t *w) {
  pdl_enter();
  if (threadIdx.x == 0) *w = 0u;
}

// Group Scaling's step (ii) folded into a producer: the maximum of the
// block's group maxima (non-negative, so their bits order as unsigned
// integers) joins the tensor maximum with one atomic per block.  Every
// thread of the block calls it.
__device__ __forceinline__ void block_max_to_tensor(float m, uint32_t *tensor_amax) {
  __shared__ float bred[kWarps];
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) bred[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = bred[0];
    for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) t = fmaxf(t, bred[i]);
    atomicMax(tensor_amax, __float_as_uint(t));
  }
}

template <int F>
__device__ __forceinline__ void cast16(const float *x, float inv, uint32_t *out) {
#pragma unroll
  for (int w = 0; w < 4; ++w)
    out[w] = float4_to_fp8x4<F>(__fmul_rn(x[4 * w], inv), __fmul_rn(x[4 * w + 1], inv),
                                __fmul_rn(x[4 * w + 2], inv), __fmul_rn(x[4 * w + 3], inv));
}

// These kernels stream 2-6 bytes per element and nothing else, so each thread
// handles kActV vectors of 16 elements (kActV consecutive 256-thread tiles
// per block) and issues all of their loads before any arithmetic: twice the
// bytes in flight per thread.
constexpr int kActV = 2;

inline unsigned int act_blocks(int64_t elems) {
  const int64_t per = static_cast<int64_t>(kElemsPerBlock) * kActV;
  return static_cast<unsigned int>((elems + per - 1) / per);
}

// ---- 1xG group quantization ---------------------------------------------------

struct GroupQuantParams {
  const uint16_t *x;
  int64_t rows, cols, ld;
  int64_t vec_per_row;  // cols / 16
  int log2G;
  uint8_t *q;
  float *scale;
};

template <int F>
__global__ void __launch_bounds__(kThreads) group_quant_1xG_kernel(const GroupQuantParams p) {
  __shared__ float red[kActV][kWarps];
  pdl_enter();
  const int lanes = 1 << (p.log2G - 4);
  const int64_t nvec = p.rows * p.vec_per_row;
  uint32_t w[kActV][8];
  int64_t row[kActV], c0[kActV];
  bool active[kActV];
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    const int64_t vid = (static_cast<int64_t>(blockIdx.x) * kActV + v) * kThreads + threadIdx.x;
    active[v] = vid < nvec;
    row[v] = active[v] ? vid / p.vec_per_row : 0;
    c0[v] = (vid - row[v] * p.vec_per_row) * kVec;
    if (active[v]) {
      const uint4 *src = reinterpret_cast<const uint4 *>(p.x + row[v] * p.ld + c0[v]);
      const uint4 a = src[0], b = src[1];
      w[v][0] = a.x; w[v][1] = a.y; w[v][2] = a.z; w[v][3] = a.w;
      w[v][4] = b.x; w[v][5] = b.y; w[v][6] = b.z; w[v][7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[v][i] = 0;
    }
  }
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    float x[16];
    unpack16_bf16(w[v], x);
    const float amax = group_max(amax16(x), lanes, red[v]);
    float s, inv;
    act_scale(amax, fmt_max<F>(), s, inv);
    uint32_t o[4];
    cast16<F>(x, inv, o);
    if (active[v]) {
      *reinterpret_cast<uint4 *>(p.q + row[v] * p.cols + c0[v]) = make_uint4(o[0], o[1], o[2], o[3]);
      if ((threadIdx.x & (lanes - 1)) == 0)
        p.scale[row[v] * (p.cols >> p.log2G) + (c0[v] >> p.log2G)] = s;
    }
  }
}

// 1xG quantization of a tensor with contiguous rows (ld == cols) as one
// flat run of n elements: every 1xG group is G consecutive elements, so no
// row / column split is needed.
template <int F>
__global__ void __launch_bounds__(kThreads)
    group_quant_1xG_flat_kernel(const GroupQuantParams p, int64_t n) {
  __shared__ float red[kActV][kWarps];
  pdl_enter();
  const int lanes = 1 << (p.log2G - 4);
  uint32_t w[kActV][8];
  int64_t e0[kActV];
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    e0[v] = ((static_cast<int64_t>(blockIdx.x) * kActV + v) * kThreads + threadIdx.x) * kVec;
    if (e0[v] < n) {
      load16_bf16<false>(p.x, e0[v], n, w[v]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[v][i] = 0;
    }
  }
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    float x[16];
    unpack16_bf16(w[v], x);
    const float amax = group_max(amax16(x), lanes, red[v]);
    float s, inv;
    act_scale(amax, fmt_max<F>(), s, inv);
    uint32_t o[4];
    cast16<F>(x, inv, o);
    if (e0[v] < n) {
      store16_u8<false>(p.q, e0[v], n, o);
      if ((threadIdx.x & (lanes - 1)) == 0) p.scale[e0[v] >> p.log2G] = s;
    }
  }
}

// ---- Group Scaling per-tensor quantization -------------------------------------

struct GroupScalingParams {
  const uint16_t *x;
  int64_t n;
  int64_t ngroups;
  int log2G;
  float *group_amax;     // [ngroups]
  uint32_t *tensor_amax; // bits of the running max (non-negative floats order as integers)
  uint8_t *q;
  float *scale;
};

// Step (i) (+ the block's share of step (ii)): per-group maxima of the BF16
// input into group_amax, and the block maximum folded into tensor_amax.
__global__ void __launch_bounds__(kThreads) group_amax_kernel(const GroupScalingParams p) {
  __shared__ float red[kActV][kWarps];
  __shared__ float blockred[kWarps];
  pdl_enter();
  const int lanes = 1 << (p.log2G - 4);
  uint32_t w[kActV][8];
  int64_t e0[kActV];
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    e0[v] = ((static_cast<int64_t>(blockIdx.x) * kActV + v) * kThreads + threadIdx.x) * kVec;
    if (e0[v] < p.n) {
      load16_bf16<false>(p.x, e0[v], p.n, w[v]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[v][i] = 0;
    }
  }
  float b = 0.0f;
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    float x[16];
    unpack16_bf16(w[v], x);
    const float gmax = group_max(amax16(x), lanes, red[v]);
    if (e0[v] < p.n && (threadIdx.x & (lanes - 1)) == 0) p.group_amax[e0[v] >> p.log2G] = gmax;
    b = fmaxf(b, gmax);
  }
  // block max of the group maxima
  for (int off = 16; off > 0; off >>= 1) b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, off));
  if ((threadIdx.x & 31) == 0) blockred[threadIdx.x >> 5] = b;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = blockred[0];
    for (int i = 1; i < kWarps; ++i) m = fmaxf(m, blockred[i]);
    atomicMax(p.tensor_amax, __float_as_uint(m));
  }
}

// Step (ii) alone, when the producer already wrote group_amax: a grid-wide
// max of the intermediate into tensor_amax.
__global__ void __launch_bounds__(kThreads) amax_of_groups_kernel(const GroupScalingParams p) {
  __shared__ float blockred[kWarps];
  pdl_enter();
  float m = 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < p.ngroups;
       i += static_cast<int64_t>(gridDim.x) * kThreads)
    m = fmaxf(m, p.group_amax[i]);
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) blockred[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = blockred[0];
    for (int i = 1; i < kWarps; ++i) r = fmaxf(r, blockred[i]);
    atomicMax(p.tensor_amax, __float_as_uint(r));
  }
}

// Step (iii): the per-tensor cast.
template <int F>
__global__ void __launch_bounds__(kThreads) pertensor_cast_kernel(const GroupScalingParams p) {
  pdl_enter();
  uint32_t w[kActV][8];
  int64_t e0[kActV];
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    e0[v] = ((static_cast<int64_t>(blockIdx.x) * kActV + v) * kThreads + threadIdx.x) * kVec;
    if (e0[v] < p.n) load16_bf16<false>(p.x, e0[v], p.n, w[v]);
  }
  const float amax = __uint_as_float(*p.tensor_amax);
  float s, inv;
  act_scale(amax, fmt_max<F>(), s, inv);
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.scale = s;
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    if (e0[v] >= p.n) continue;
    float x[16];
    unpack16_bf16(w[v], x);
    uint32_t o[4];
    cast16<F>(x, inv, o);
    store16_u8<false>(p.q, e0[v], p.n, o);
  }
}

// ---- a producer with Group Scaling's step (i) fused in: SwiGLU -------------------
// COAT summary page, section "混合粒度": the per-1xG maxima of a linear
// layer's input are emitted by the kernel that produces that input, so the
// per-tensor quantizer only reads the G-times-smaller intermediate (step
// (ii)) before its cast.  SwiGLU produces the input of an MLP's down
// projection (the GLU layers of section "激活为什么难压"):
//   out = RN_bf16(silu(gate) * up), silu(g) = g / (1 + e^-g),
// evaluated in binary32 with the special-function exp2 and reciprocal
// (relative error ~2^-20 for |g| < 64, far below BF16's 2^-9 spacing: the
// BF16 result is the correctly rounded one except next to a rounding
// midpoint); the maxima are taken over the BF16 outputs, i.e. exactly the
// values the quantizer will read.

struct SwigluParams {
  const uint16_t *gate;
  const uint16_t *up;
  int64_t n;
  int log2G;
  uint16_t *out;
  float *group_amax;     // [ceil(n / G)]
  uint32_t *tensor_amax; // nullable: also the maximum of all outputs (bits, zeroed first)
};

__global__ void __launch_bounds__(kThreads) swiglu_group_amax_kernel(const SwigluParams p) {
  __shared__ float red[kActV][kWarps];
  pdl_enter();
  const int lanes = 1 << (p.log2G - 4);
  float tmax = 0.0f;
  uint32_t gw[kActV][8], uw[kActV][8];
  int64_t e0[kActV];
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    e0[v] = ((static_cast<int64_t>(blockIdx.x) * kActV + v) * kThreads + threadIdx.x) * kVec;
    if (e0[v] < p.n) {
      load16_bf16<false>(p.gate, e0[v], p.n, gw[v]);
      load16_bf16<false>(p.up, e0[v], p.n, uw[v]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) gw[v][i] = uw[v][i] = 0;
    }
  }
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    float g[16], u[16], h[16];
    unpack16_bf16(gw[v], g);
    unpack16_bf16(uw[v], u);
    uint32_t ow[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a = __fmul_rn(__fdividef(g[2 * i], 1.0f + __expf(-g[2 * i])), u[2 * i]);
      const float b =
          __fmul_rn(__fdividef(g[2 * i + 1], 1.0f + __expf(-g[2 * i + 1])), u[2 * i + 1]);
      const uint32_t ba = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(a)));
      const uint32_t bb = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(b)));
      ow[i] = ba | (bb << 16);
      h[2 * i] = bf16lo_to_float(ow[i]);
      h[2 * i + 1] = bf16hi_to_float(ow[i]);
    }
    const float gmax = group_max(amax16(h), lanes, red[v]);
    tmax = fmaxf(tmax, gmax);
    if (e0[v] >= p.n) continue;
    if (e0[v] + 16 <= p.n) {
      uint4 *dst = reinterpret_cast<uint4 *>(p.out + e0[v]);
      dst[0] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      dst[1] = make_uint4(ow[4], ow[5], ow[6], ow[7]);
    } else {
      for (int i = 0; i < 16; ++i)
        if (e0[v] + i < p.n) p.out[e0[v] + i] = static_cast<uint16_t>(ow[i >> 1] >> (16 * (i & 1)));
    }
    if ((threadIdx.x & (lanes - 1)) == 0) p.group_amax[e0[v] >> p.log2G] = gmax;
  }
  if (p.tensor_amax) block_max_to_tensor(tmax, p.tensor_amax);
}

// ---- a second producer with the maxima fused in: LayerNorm / RMSNorm ---------------------
// The norm of a transformer block (COAT summary page, section "激活为什么难压":
// LayerNorm/RMSNorm are among the nonlinear layers) produces the input of
// the linear layers that follow it (QKV, MLP up/gate), so, as for SwiGLU,
// it emits the per-1xG maxima of its BF16 output for Group Scaling (section
// "混合粒度").  Per row (token):
//   LayerNorm  y = (x - mean) / sqrt(var + eps)   (var: mean of squared deviations)
//   RMSNorm    y = x / sqrt(mean(x^2) + eps)
// then y * weight[c] (+ bias[c] for LayerNorm) when given, rounded to BF16.
// One warp per row: the warp stages its row in shared memory (16-byte
// asynchronous copies, the next row's issued before the current one is
// computed), takes the row sums over it in binary32 (per-lane sums, then a
// fixed xor shuffle tree, so every lane holds the same value), divides them
// by the row length with the correctly rounded quotient (a row whose sum is
// exact, such as a constant row, gets its exact mean: x - mean is then 0,
// where a product with a rounded 1/n could leave one ulp of x, multiplied by
// 1/sqrt(eps)), and writes the BF16 output and each 1xG run's maximum.  The binary32
// statistics (sums of a few thousand terms) and y carry an error of about
// 1e-6 x (|y| + |mean| / std), so the BF16 output is the correctly rounded
// norm except within that distance of a rounding midpoint.

struct NormParams {
  const uint16_t *x;
  uint16_t *out;
  float *group_amax;     // [rows * cols / G]
  const float *weight;   // nullable, [cols]
  const float *bias;     // nullable, [cols] (LayerNorm)
  int64_t rows, cols;
  int log2G;
  int rms;
  float eps;
  uint32_t *tensor_amax; // nullable: also the maximum of all outputs (bits, zeroed first)
  bool affine_vec;       // weight and bias (those given) are 16-byte aligned
};

constexpr int kNormMaxCols = 16384;

// Warps (rows in flight) of a block: up to kWarps, fewer for long rows so
// that the two staged rows of every warp fit 96 KB of shared memory.
inline int norm_warps_per_block(int64_t cols) {
  const int64_t fit = (96 * 1024) / (2 * 2 * cols);
  return static_cast<int>(fit < 1 ? 1 : (fit > kWarps ? kWarps : fit));
}

__device__ __forceinline__ float warp_sum_f(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max_f(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Issue the 16-byte asynchronous copies of one row into shared memory (one
// commit group per row).
__device__ __forceinline__ void norm_prefetch_row(const NormParams &p, uint4 *dst, int64_t row,
                                                  int nq, int lane) {
  const uint4 *src = reinterpret_cast<const uint4 *>(p.x + row * p.cols);
  for (int q = lane; q < nq; q += 32) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst + q));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src + q) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// One row from its staged copy rs: statistics, output, 1xG maxima; returns
// the row's maximum |output| (in every lane).
__device__ __forceinline__ float norm_one_row(const NormParams &p, const uint4 *rs, int64_t row,
                                              int lane) {
  const int nq = static_cast<int>(p.cols >> 3);
  const float nf = static_cast<float>(p.cols);   // exact (cols <= 16384)
  float acc = 0.0f;
  for (int q = lane; q < nq; q += 32) {
    const uint4 c = rs[q];
    const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = bf16lo_to_float(wv[i]), b = bf16hi_to_float(wv[i]);
      acc += p.rms ? a * a + b * b : a + b;
    }
  }
  const float s1 = warp_sum_f(acc);
  float mean = 0.0f, var;
  if (p.rms) {
    var = __fdiv_rn(s1, nf);
  } else {
    mean = __fdiv_rn(s1, nf);
    float ss = 0.0f;
    for (int q = lane; q < nq; q += 32) {
      const uint4 c = rs[q];
      const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = bf16lo_to_float(wv[i]) - mean, b = bf16hi_to_float(wv[i]) - mean;
        ss += a * a + b * b;
      }
    }
    var = __fdiv_rn(warp_sum_f(ss), nf);
  }
  const float rstd = 1.0f / sqrtf(var + p.eps);

  // output: lane handles 16-element vectors j = lane + 32 v
  const int nv = static_cast<int>(p.cols >> 4);
  const int lanes = 1 << (p.log2G - 4);
  const int64_t groups_per_row = p.cols >> p.log2G;
  float run = 0.0f;   // running maximum of a group spanning several iterations
  float rowmax = 0.0f;
  for (int v = 0; 32 * v < nv; ++v) {
    const int j = lane + 32 * v;
    const bool on = j < nv;
    uint32_t ow[8];
    float a = 0.0f;
    if (on) {
      const uint4 c0 = rs[2 * j], c1 = rs[2 * j + 1];
      const uint32_t wv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = 16 * j + 2 * i;
        float y0 = (bf16lo_to_float(wv[i]) - mean) * rstd;
        float y1 = (bf16hi_to_float(wv[i]) - mean) * rstd;
        if (p.weight && p.bias) {   // y w + b, one fused multiply-add
          y0 = __fmaf_rn(y0, p.weight[c], p.bias[c]);
          y1 = __fmaf_rn(y1, p.weight[c + 1], p.bias[c + 1]);
        } else if (p.weight) {
          y0 = __fmul_rn(y0, p.weight[c]);
          y1 = __fmul_rn(y1, p.weight[c + 1]);
        } else if (p.bias) {
          y0 = __fadd_rn(y0, p.bias[c]);
          y1 = __fadd_rn(y1, p.bias[c + 1]);
        }
        ow[i] = bf16x2_rn(y0, y1);
        a = fmaxf(a, fmaxf(fabsf(bf16lo_to_float(ow[i])), fabsf(bf16hi_to_float(ow[i]))));
      }
      uint4 *dst = reinterpret_cast<uint4 *>(p.out + row * p.cols + 16 * j);
      dst[0] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      dst[1] = make_uint4(ow[4], ow[5], ow[6], ow[7]);
    }
    rowmax = fmaxf(rowmax, a);
    if (lanes <= 32) {
      for (int off = 1; off < lanes; off <<= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      if (on && (lane & (lanes - 1)) == 0)
        p.group_amax[row * groups_per_row + ((16 * j) >> p.log2G)] = a;
    } else {
      for (int off = 1; off < 32; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      run = fmaxf(run, a);
      if (((32 * (v + 1)) & (lanes - 1)) == 0) {   // the group's last iteration
        if (lane == 0) p.group_amax[row * groups_per_row + ((16 * 32 * v) >> p.log2G)] = run;
        run = 0.0f;
      }
    }
  }
  return warp_max_f(rowmax);
}

// Persistent warps: warp w of the grid takes rows w, w + W, w + 2W, ... (W
// the grid's warps), staging each row in one of its two shared-memory
// buffers while the previous row is computed.
__global__ void __launch_bounds__(kThreads) norm_group_amax_kernel(const NormParams p) {
  extern __shared__ uint4 norm_rows[];
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nq = static_cast<int>(p.cols >> 3);    // 16-byte chunks of a row
  uint4 *buf = norm_rows + static_cast<int64_t>(warp) * 2 * nq;
  const int64_t step = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
  float wmax = 0.0f;
  if (row < p.rows) {   // warp-uniform; a warp without rows only joins the block max
    norm_prefetch_row(p, buf, row, nq, lane);
    for (int it = 0; row < p.rows; ++it, row += step) {
      const bool more = row + step < p.rows;
      if (more) norm_prefetch_row(p, buf + ((it + 1) & 1) * nq, row + step, nq, lane);
      if (more)
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      else
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncwarp();   // every lane's copies of this row have landed
      wmax = fmaxf(wmax, norm_one_row(p, buf + (it & 1) * nq, row, lane));
      __syncwarp();   // every lane is done with the buffer the next prefetch reuses
    }
  }
  if (p.tensor_amax) block_max_to_tensor(wmax, p.tensor_amax);
}

// Rows of 256 NC columns (NC = 1..8: up to 2048 columns) that the two-warp
// form further below does not take (an odd chunk count, or 1xG runs wider
// than half a row) are held in registers by one warp: lane l loads the
// row's 16-byte chunks l, l + 32, ..., l + 32 (NC - 1) (every load
// instruction of the warp reads 512 contiguous bytes) and takes the sums,
// the output and the maxima from them.  Fully unrolled over the row, it
// executes far fewer instructions than the staged form's three loops over
// shared memory, which are what limit that form.  Persistent warps, 8 to a
// block, 2 blocks per SM (the row and its sums take ~110 registers).
constexpr int kNormRegWarps = 8;
constexpr int kNormRegMaxChunks = 8;

// max of two BF16 pairs, lane by lane (NaN ignored)
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(bf16lo_to_float(w), bf16hi_to_float(w));
}

// 8 consecutive floats as 4 pairs: two 16-byte loads when `vec` (the
// vector's base, and so every 8-column chunk of it, is 16-byte aligned),
// else one load a float.
__device__ __forceinline__ void load8_f32(const float *a, bool vec, float2 (&o)[4]) {
  if (vec) {
    const float4 u = __ldg(reinterpret_cast<const float4 *>(a));
    const float4 v = __ldg(reinterpret_cast<const float4 *>(a) + 1);
    o[0] = make_float2(u.x, u.y); o[1] = make_float2(u.z, u.w);
    o[2] = make_float2(v.x, v.y); o[3] = make_float2(v.z, v.w);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = make_float2(__ldg(a + 2 * j), __ldg(a + 2 * j + 1));
  }
}

// One row of 256 NC columns held in registers: src is the row (its 32 NC
// 16-byte chunks, in global or shared memory), lane l takes chunks l + 32 i.
// The arithmetic runs on packed binary32 pairs: the row sums as four partial
// sums a lane (two packed pairs, alternate pairs of columns), the
// normalisation two columns an instruction, and each 1xG maximum of |out|
// on the BF16 outputs themselves (pairs with their sign bits cleared).
// kAffine: a weight and/or a bias is given (an instantiation of its own, so
// the plain norm carries no affine code at all).
template <int NC, bool kAffine>
__device__ __forceinline__ float norm_reg_row(const NormParams &p, const uint4 *src, int64_t row,
                                              int lane) {
  uint4 c[NC];
#pragma unroll
  for (int i = 0; i < NC; ++i) c[i] = src[lane + 32 * i];
  const float nf = static_cast<float>(p.cols);   // exact (cols <= 16384)
  float2 s0 = make_float2(0.0f, 0.0f), s1 = s0;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const uint32_t wv[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 x2 = bf16x2_to_float2(wv[j]);
      float2 &acc = (j & 1) ? s1 : s0;
      acc = p.rms ? fma2_rn(x2, x2, acc) : add2_rn(acc, x2);
    }
  }
  const float sum = warp_sum_f((s0.x + s0.y) + (s1.x + s1.y));
  float mean = 0.0f, var;
  if (p.rms) {
    var = __fdiv_rn(sum, nf);
  } else {
    mean = __fdiv_rn(sum, nf);
    const float2 nm = make_float2(-mean, -mean);
    float2 q0 = make_float2(0.0f, 0.0f), q1 = q0;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const uint32_t wv[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 d = add2_rn(bf16x2_to_float2(wv[j]), nm);
        float2 &acc = (j & 1) ? q1 : q0;
        acc = fma2_rn(d, d, acc);
      }
    }
    var = __fdiv_rn(warp_sum_f((q0.x + q0.y) + (q1.x + q1.y)), nf);
  }
  const float rstd = 1.0f / sqrtf(var + p.eps);
  const float2 NM = make_float2(-mean, -mean), RS = make_float2(rstd, rstd);

  // chunk q = lane + 32 i holds columns 8q .. 8q + 7; a 1xG run is G / 8
  // chunks: consecutive lanes of one i for G <= 256, else all lanes of
  // G / 256 consecutive i
  const int clanes = 1 << (p.log2G - 3);
  const int64_t gbase = (row * p.cols) >> p.log2G;
  uint4 *dst = reinterpret_cast<uint4 *>(p.out + row * p.cols);
  float run = 0.0f, rowmax = 0.0f;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const uint32_t wv[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
    const int col0 = 8 * (lane + 32 * i);
    uint32_t ow[4];
    uint32_t am = 0u;
    if constexpr (kAffine) {
      // the affine terms of the chunk's 8 columns: two 16-byte loads each
      // where the vectors allow it (one load a column otherwise); with both,
      // y w + b is one fused multiply-add
      float2 w2[4], b2[4];
      if (p.weight) load8_f32(p.weight + col0, p.affine_vec, w2);
      if (p.bias) load8_f32(p.bias + col0, p.affine_vec, b2);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 y = mul2_rn(add2_rn(bf16x2_to_float2(wv[j]), NM), RS);
        if (p.weight && p.bias) y = fma2_rn(y, w2[j], b2[j]);
        else if (p.weight) y = mul2_rn(y, w2[j]);
        else y = add2_rn(y, b2[j]);
        ow[j] = bf16x2_rn(y.x, y.y);
        am = bmax2(am, ow[j] & 0x7FFF7FFFu);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 y = mul2_rn(add2_rn(bf16x2_to_float2(wv[j]), NM), RS);
        ow[j] = bf16x2_rn(y.x, y.y);
        am = bmax2(am, ow[j] & 0x7FFF7FFFu);
      }
    }
    dst[lane + 32 * i] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
    float a = fmaxf(bf16lo_to_float(am), bf16hi_to_float(am));
    rowmax = fmaxf(rowmax, a);
    if (clanes <= 32) {
      for (int off = 1; off < clanes; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      if ((lane & (clanes - 1)) == 0) p.group_amax[gbase + (col0 >> p.log2G)] = a;
    } else {
      run = fmaxf(run, warp_max_f(a));
      if (((i + 1) & ((clanes >> 5) - 1)) == 0) {   // the run's last chunk column
        if (lane == 0) p.group_amax[gbase + ((256 * i) >> p.log2G)] = run;
        run = 0.0f;
      }
    }
  }
  return warp_max_f(rowmax);
}

// Shared memory of norm_reg_group_amax_kernel<NC>: two row buffers a warp.
template <int NC>
constexpr size_t norm_reg_smem() {
  return static_cast<size_t>(kNormRegWarps) * 2 * 32 * NC * sizeof(uint4);
}

// Persistent blocks, one contiguous share of the rows each.  A warp takes
// the block's next untaken row whenever it starts one (a shared-memory
// counter), so warps the scheduler favours take more rows and the block's
// warps finish together, and it copies that next row into the second of its
// two shared-memory buffers (cp.async, its own chunks only, so no barrier)
// while it normalises the current one.
template <int NC, bool kAffine>
__global__ void __launch_bounds__(32 * kNormRegWarps, 2) norm_reg_group_amax_kernel(const NormParams p) {
  extern __shared__ __align__(16) uint4 nbuf[];
  __shared__ unsigned int next_row;
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t r0 = p.rows * blockIdx.x / gridDim.x;
  const int64_t r1 = p.rows * (blockIdx.x + 1) / gridDim.x;
  if (threadIdx.x == 0) next_row = kNormRegWarps;
  __syncthreads();
  uint4 *wb = nbuf + warp * 2 * 32 * NC;
  const int64_t cv = p.cols / 8;   // 16-byte chunks a row
  auto fetch = [&](int64_t row, uint4 *dst) {
    const uint4 *src = reinterpret_cast<const uint4 *>(p.x) + row * cv;
#pragma unroll
    for (int i = 0; i < NC; ++i) cp_async16(dst + lane + 32 * i, src + lane + 32 * i);
    cp_async_commit();
  };
  float wmax = 0.0f;
  int64_t row = r0 + warp;
  if (row < r1) fetch(row, wb);
  for (int k = 0; row < r1; ++k) {
    unsigned int g = 0;
    if (lane == 0) g = atomicAdd(&next_row, 1u);
    const int64_t nxt = r0 + __shfl_sync(0xffffffffu, g, 0);
    if (nxt < r1) {
      fetch(nxt, wb + ((k + 1) & 1) * 32 * NC);
      cp_async_wait_one();   // the current row's copies (all but the newest group)
    } else {
      cp_async_wait_all();
    }
    wmax = fmaxf(wmax, norm_reg_row<NC, kAffine>(p, wb + (k & 1) * 32 * NC, row, lane));
    row = nxt;
  }
  if (p.tensor_amax) block_max_to_tensor(wmax, p.tensor_amax);
}

// Rows of 512 NCH columns, two warps a row: warp half h of a pair holds
// chunk columns NCH h .. NCH h + NCH - 1 (lane l: chunks l + 32 i), so a
// row's data takes half the registers of the one-warp form and twice the
// warps fit an SM (latency, not bandwidth, bounds that form: 16 warps per
// SM).  Each half sums its columns (four partial sums a lane, then the
// warp), the two halves' sums meet in shared memory (half 0 + half 1), and
// the mean and the variance follow as in the one-warp form.  The block's
// four pairs advance in lockstep, two block barriers a round; every warp
// takes part in every round (a pair without a row in the last round skips
// only its arithmetic), so every barrier is reached by the whole block.
// Each warp loads the next round's half row into registers while it works
// on the current one.  A 1xG run lies within one half (G divides 256 NCH).
constexpr int kSplitPairs = 4;

template <int NCH, bool kAffine>
__global__ void __launch_bounds__(256, kAffine ? 3 : 4) norm_split_group_amax_kernel(const NormParams p) {
  __shared__ float sum_red[kSplitPairs][2], var_red[kSplitPairs][2];
  pdl_enter();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int pair = warp >> 1, h = warp & 1;
  const int64_t r0 = p.rows * blockIdx.x / gridDim.x;
  const int64_t r1 = p.rows * (blockIdx.x + 1) / gridDim.x;
  const int64_t rounds = (r1 - r0 + kSplitPairs - 1) / kSplitPairs;
  const float nf = static_cast<float>(p.cols);   // exact (cols <= 16384)
  const int clanes = 1 << (p.log2G - 3);
  uint32_t rowmax2 = 0u, prev = 0u;   // BF16 pairs of |out| maxima
  uint4 nxt[NCH];
  auto load = [&](int64_t row, uint4 *c) {
    const uint4 *src = reinterpret_cast<const uint4 *>(p.x + row * p.cols);
#pragma unroll
    for (int j = 0; j < NCH; ++j) c[j] = src[lane + 32 * (NCH * h + j)];
  };
  int64_t row = r0 + pair;
  if (row < r1) load(row, nxt);
  for (int64_t k = 0; k < rounds; ++k, row += kSplitPairs) {
    const bool on = row < r1;
    uint4 c[NCH];
#pragma unroll
    for (int j = 0; j < NCH; ++j) c[j] = nxt[j];
    if (row + kSplitPairs < r1) load(row + kSplitPairs, nxt);
    float2 s0 = make_float2(0.0f, 0.0f), s1 = s0;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const uint32_t wv[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 x2 = bf16x2_to_float2(wv[j]);
        float2 &acc = (j & 1) ? s1 : s0;
        acc = p.rms ? fma2_rn(x2, x2, acc) : add2_rn(acc, x2);
      }
    }
    const float ws = warp_sum_f((s0.x + s0.y) + (s1.x + s1.y));
    if (lane == 0) sum_red[pair][h] = ws;
    __syncthreads();
    const float sum = sum_red[pair][0] + sum_red[pair][1];
    float mean = 0.0f, var;
    if (p.rms) {
      var = __fdiv_rn(sum, nf);
      __syncthreads();   // the same two barriers a round on both forms
    } else {
      mean = __fdiv_rn(sum, nf);
      const float2 nm = make_float2(-mean, -mean);
      float2 q0 = make_float2(0.0f, 0.0f), q1 = q0;
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const uint32_t wv[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 d = add2_rn(bf16x2_to_float2(wv[j]), nm);
          float2 &acc = (j & 1) ? q1 : q0;
          acc = fma2_rn(d, d, acc);
        }
      }
      const float wq = warp_sum_f((q0.x + q0.y) + (q1.x + q1.y));
      if (lane == 0) var_red[pair][h] = wq;
      __syncthreads();
      var = __fdiv_rn(var_red[pair][0] + var_red[pair][1], nf);
    }
    if (!on) continue;   // after both barriers of the round
    const float rstd = 1.0f / sqrtf(var + p.eps);
    const float2 NM = make_float2(-mean, -mean), RS = make_float2(rstd, rstd);
    const int64_t gbase = (row * p.cols) >> p.log2G;
    uint4 *dst = reinterpret_cast<uint4 *>(p.out + row * p.cols);
    float run = 0.0f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const uint32_t wv[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
      const int ci = NCH * h + i;                     // chunk column in the row
      const int col0 = 8 * (lane + 32 * ci);
      uint32_t ow[4], am = 0u;
      if constexpr (kAffine) {
        float2 w2[4], b2[4];
        if (p.weight) load8_f32(p.weight + col0, p.affine_vec, w2);
        if (p.bias) load8_f32(p.bias + col0, p.affine_vec, b2);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 y = mul2_rn(add2_rn(bf16x2_to_float2(wv[j]), NM), RS);
          if (p.weight && p.bias) y = fma2_rn(y, w2[j], b2[j]);
          else if (p.weight) y = mul2_rn(y, w2[j]);
          else y = add2_rn(y, b2[j]);
          ow[j] = bf16x2_rn(y.x, y.y);
          am = bmax2(am, ow[j] & 0x7FFF7FFFu);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 y = mul2_rn(add2_rn(bf16x2_to_float2(wv[j]), NM), RS);
          ow[j] = bf16x2_rn(y.x, y.y);
          am = bmax2(am, ow[j] & 0x7FFF7FFFu);
        }
      }
      dst[lane + 32 * ci] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      rowmax2 = bmax2(rowmax2, am);
      // the chunk's maximum in the low half-word (BF16, exact)
      const uint32_t m = bmax2(am, am >> 16);
      if (clanes <= 32) {
        // two chunk columns reduced together: chunk i - 1 in the low half,
        // chunk i in the high half of one word
        if ((i & 1) == 0 && i + 1 < NCH) {
          prev = m;
          continue;
        }
        uint32_t w = (i & 1) ? __byte_perm(prev, m, 0x5410) : m;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1)
          if (off < clanes) w = bmax2(w, __shfl_xor_sync(0xffffffffu, w, off));
        if ((lane & (clanes - 1)) == 0) {
          if (i & 1) {
            p.group_amax[gbase + ((col0 - 256) >> p.log2G)] = bf16lo_to_float(w);
            p.group_amax[gbase + (col0 >> p.log2G)] = bf16hi_to_float(w);
          } else {
            p.group_amax[gbase + (col0 >> p.log2G)] = bf16lo_to_float(w);
          }
        }
      } else {
        run = fmaxf(run, warp_max_f(bf16lo_to_float(m)));
        if (((ci + 1) & ((clanes >> 5) - 1)) == 0) {   // the run's last chunk column
          if (lane == 0) p.group_amax[gbase + ((256 * ci) >> p.log2G)] = run;
          run = 0.0f;
        }
      }
    }
  }
  if (p.tensor_amax)
    block_max_to_tensor(warp_max_f(fmaxf(bf16lo_to_float(rowmax2), bf16hi_to_float(rowmax2))),
                        p.tensor_amax);
}

// ---- the FP8 cast alone -------------------------------------------------------------
// code = RNE_satfinite(y): round to nearest even, finite values beyond the
// format's largest magnitude (and infinities) saturate to +-max, NaN gives a
// NaN code (LLM Atlas "systems/numerics", section 03 "FP8": E4M3 max 448,
// E5M2 max 57344).  The hardware cvt that every quantizer here ends with.
struct EncodeParams {
  const float *y;
  int64_t n;
  uint8_t *q;
};

template <int F>
__global__ void __launch_bounds__(kThreads) fp8_encode_kernel(const EncodeParams p) {
  pdl_enter();
  float x[kActV][16];
  int64_t e0[kActV];
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    e0[v] = ((static_cast<int64_t>(blockIdx.x) * kActV + v) * kThreads + threadIdx.x) * kVec;
    if (e0[v] < p.n) load16_f32<false>(p.y, e0[v], p.n, x[v]);
  }
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    if (e0[v] >= p.n) continue;
    uint32_t o[4];
#pragma unroll
    for (int w = 0; w < 4; ++w)
      o[w] = float4_to_fp8x4<F>(x[v][4 * w], x[v][4 * w + 1], x[v][4 * w + 2], x[v][4 * w + 3]);
    store16_u8<false>(p.q, e0[v], p.n, o);
  }
}

// ---- non-finite gradient count ----------------------------------------------------
// *count += number of BF16 values with an all-ones exponent (inf or NaN).
struct CountParams {
  const uint16_t *x;
  int64_t n;
  uint32_t *count;
};

__global__ void __launch_bounds__(kThreads) count_nonfinite_bf16_kernel(const CountParams p) {
  __shared__ uint32_t part[kWarps];
  uint32_t c = 0;
#pragma unroll
  for (int v = 0; v < kActV; ++v) {
    const int64_t e0 =
        ((static_cast<int64_t>(blockIdx.x) * kActV + v) * kThreads + threadIdx.x) * kVec;
    if (e0 < p.n) {
      uint32_t w[8];
      load16_bf16<false>(p.x, e0, p.n, w);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c += ((w[i] & 0x7F80u) == 0x7F80u) ? 1u : 0u;
        c += ((w[i] & 0x7F800000u) == 0x7F800000u) ? 1u : 0u;
      }
    }
  }
  for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int i = 0; i < kWarps; ++i) t += part[i];
    if (t) atomicAdd(p.count, t);
  }
}

// ---- dequantization ----------------------------------------------------------------

struct DequantParams {
  const uint8_t *q;
  const float *k;  // nullable
  const float *scale;
  int64_t n;
  int log2G;       // -1: one scale for the whole tensor
  int out_bf16;
  void *out;
  double log2_tab[8];
};

__device__ __forceinline__ uint32_t float_to_bf16_rn(float f) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

__device__ __forceinline__ void store16_out(const DequantParams &p, int64_t e0, const float *x) {
  if (p.out_bf16) {
    uint16_t *o = static_cast<uint16_t *>(p.out);
    if (e0 + 16 <= p.n) {
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        pk[i] = float_to_bf16_rn(x[2 * i]) | (float_to_bf16_rn(x[2 * i + 1]) << 16);
      uint4 *dst = reinterpret_cast<uint4 *>(o + e0);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    } else {
      for (int i = 0; i < 16; ++i)
        if (e0 + i < p.n) o[e0 + i] = static_cast<uint16_t>(float_to_bf16_rn(x[i]));
    }
  } else {
    store16_f32<false>(static_cast<float *>(p.out), e0, p.n, x);
  }
}

// States (k given): x = sign(d) RN32(|d|^(1/k)) s per element, binary64.
template <int F>
__global__ void __launch_bounds__(kThreads) dequant_kernel(const DequantParams p) {
  __shared__ double tab8[8];
  if (threadIdx.x < 8) tab8[threadIdx.x] = p.log2_tab[threadIdx.x];
  __syncthreads();
  const int64_t e0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) * kVec;
  if (e0 >= p.n) return;
  const int64_t grp = p.log2G < 0 ? 0 : (e0 >> p.log2G);
  const float s = p.scale[grp];
  const double rk = 1.0 / static_cast<double>(p.k[grp]);
  uint32_t w[4];
  load16_u8<false>(p.q, e0, p.n, w);
  float x[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float d[4];
    fp8x4_to_float<F>(w[i], d);
#pragma unroll
    for (int j = 0; j < 4; ++j) x[4 * i + j] = dequant_exact(d[j], s, rk, tab8);
  }
  store16_out(p, e0, x);
}

// Activations (no k): x = d * s, one binary32 product.  Written 4 B (or 2 B)
// per element, the kernel is bound by its stores, so the warp's elements
// are interleaved for them: lane l owns the 4-element pieces at 128 j + 4 l
// of the warp's 512 elements, and every store instruction of the warp
// writes one contiguous 512 B run (16 consecutive elements per lane left
// each 32-byte sector to two instructions: 4.4 instead of 6.2 TB/s).
constexpr int kDeqV = 1;

inline unsigned int deq_blocks(int64_t elems) {
  const int64_t per = static_cast<int64_t>(kElemsPerBlock) * kDeqV;
  return static_cast<unsigned int>((elems + per - 1) / per);
}

template <int F>
__global__ void __launch_bounds__(kThreads) dequant_linear_kernel(const DequantParams p) {
  pdl_enter();
  // each warp covers 512 consecutive elements per unit; lane owns the
  // 4-element pieces at 128 j + 4 lane, so every load and store instruction
  // of the warp touches one contiguous run (128 B of codes, 512 B of FP32)
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
#pragma unroll
  for (int v = 0; v < kDeqV; ++v) {
    const int64_t cb = (static_cast<int64_t>(blockIdx.x) * kDeqV + v) * kElemsPerBlock + warp * 512;
    uint32_t w[4];
    float sc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t e = cb + 128 * j + 4 * lane;
      w[j] = 0;
      sc[j] = 0.0f;
      if (e + 4 <= p.n) {
        w[j] = *reinterpret_cast<const uint32_t *>(p.q + e);
      } else {
        for (int i = 0; i < 4; ++i)
          if (e + i < p.n) w[j] |= static_cast<uint32_t>(p.q[e + i]) << (8 * i);
      }
      if (e < p.n) sc[j] = p.scale[p.log2G < 0 ? 0 : (e >> p.log2G)];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t e = cb + 128 * j + 4 * lane;
      if (e >= p.n) continue;
      float d[4];
      fp8x4_to_float<F>(w[j], d);
      float x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = __fmul_rn(d[i], sc[j]);
      if (e + 4 <= p.n) {
        if (p.out_bf16) {
          uint2 o;
          o.x = float_to_bf16_rn(x[0]) | (float_to_bf16_rn(x[1]) << 16);
          o.y = float_to_bf16_rn(x[2]) | (float_to_bf16_rn(x[3]) << 16);
          *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(p.out) + e) = o;
        } else {
          *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + e) =
              make_float4(x[0], x[1], x[2], x[3]);
        }
      } else {
        for (int i = 0; i < 4 && e + i < p.n; ++i) {
          if (p.out_bf16)
            static_cast<uint16_t *>(p.out)[e + i] = static_cast<uint16_t>(float_to_bf16_rn(x[i]));
          else
            static_cast<float *>(p.out)[e + i] = x[i];
        }
      }
    }
  }
}

}  // namespace coat
