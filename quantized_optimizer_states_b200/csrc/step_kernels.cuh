// COAT FP8-state AdamW step (fused) and the stand-alone state quantizer.
//
// COAT summary page (blog.daoxuan.cc/posts/57954):
//   section "为什么二阶动量对量化比一阶动量更敏感" -- AdamW with decoupled
//   weight decay on the FP32 master weights;
//   section "扩展函数：把窄分布拉宽" -- before FP8 encoding each 1xG group of
//   a moment is expanded by f(x) = sign(x)|x|^k with
//   k = log(R_target) / log(R_X), R_X = max|x| / min nonzero |x|, k
//   recomputed per group at every step; decoding takes the 1/k power.
// LLM Atlas "systems/numerics", section 08 "Adam -> AdamW" -- m_t, v_t,
// bias correction, eps outside the root, theta <- (1 - eta*lambda) theta + delta.
//
// Work decomposition: one thread owns 16 consecutive parameters, so every
// stream moves in 16-byte vectors (4 x 16 B of theta, 2 x 16 B of BF16
// gradient, 16 B of each code stream); blocks are small (64 threads, more
// only where one group needs it, see StepLayout).  Dynamic shared memory
// holds only the warps' decode tables.  A 1xG group is G/16 consecutive
// threads: up to 32 of them reduce with warp shuffles, larger groups (G >=
// 1024) finish the reduction through shared memory among their warps.  The
// whole group stays in registers between the range reduction and the
// encode, so every byte crosses HBM exactly once.
//
// Dequantization must reproduce RN32(|d|^(1/k)) exactly (the new group
// range depends on the smallest |m_t|, which cancellation in
// beta1*m + (1-beta1)*g makes sensitive to the last bit).  For G >= 64 every
// warp first builds, in shared memory, the 128-entry decode table of each of
// its (group, moment) pairs (binary64 power chains, state_codec.cuh) --
// holding beta1*m or beta2*v directly -- so an element costs one table
// lookup; for G < 64 each element is decoded directly in binary64.
//
// The update quotient u = m^ / (sqrt(v^) + eps) is evaluated branch-free with
// one correction step per operation (division by the bias corrections with
// their correctly rounded reciprocals, the square root from the rsqrt
// estimate, the quotient from the rcp estimate), each of which yields the
// correctly rounded result except in vanishingly rare near-midpoint cases;
// a warp whose moments fall outside the range where those estimates are
// valid (zero-free tiny, huge or infinite values) takes the fully IEEE path.
//
// The kernel is instantiated per group size, so lane counts, table counts
// and shifts are compile-time, and per launch shape: full blocks (no bounds
// checks) and the one ragged tail block of a launch.
//
// kThreads / kElemsPerBlock below are the 256-thread block shape of the
// other kernels of the library (the stand-alone quantizer and the
// activation kernels).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "fp8_device.cuh"
#include "state_codec.cuh"

namespace coat {


constexpr int kThreads = 256;
constexpr int kVec = 16;                           // parameters per thread
constexpr int kElemsPerBlock = kThreads * kVec;    // 4096
constexpr int kWarps = kThreads / 32;
constexpr int kMinTableLog2G = 6;                  // decode tables for G >= 64

// Where the step's gradient comes from (a template parameter of the kernel):
// BF16 words, float32 values rounded to BF16 as they load, or the mean of
// the BF16 gradients of `world` data-parallel ranks read from their own
// buffers (peer memory), with the updated parameters also written into
// every rank's parameter buffer -- the reduce-scatter, the step and the
// all-gather of a ZeRO-1 step in one kernel.
constexpr int kGradBf16 = 0;
constexpr int kGradF32 = 1;
constexpr int kGradPeers = 2;
constexpr int kMaxPeers = 8;

struct StepParams {
  float *theta;
  const uint16_t *grad;       // BF16 gradients (kGradBf16)
  const float *grad_f32;      // float32 gradients, rounded to BF16 on load (kGradF32)
  // kGradPeers: rank r's gradient slice of this shard (element i at
  // grad_peer[r][i]) and rank r's parameter slice (param_peer[r][i], FP32 or
  // BF16 by param_peer_bf16; null: not replicated), r < world
  const uint16_t *grad_peer[kMaxPeers];
  void *param_peer[kMaxPeers];
  int world;
  int param_peer_bf16;
  uint8_t *m_code;
  float *m_k;
  float *m_s;
  uint8_t *v_code;
  float *v_k;
  float *v_s;
  int64_t n;
  int64_t ngroups;
  int64_t block0;     // index of this launch's first block (of StepLayout::kBlockElems)
  const uint32_t *skip;  // nullable: a nonzero word here makes the step a no-op
  float beta1, beta2, c1, c2, bc1, bc2, rbc1, rbc2, decay, lr, eps;
  // The estimate-based quotient is used for a thread's 16 elements when
  // max|m_t| <= fast_mmax, max v_t <= fast_vmax and every nonzero v_t >=
  // fast_vmin (bounds from the bias corrections and eps); otherwise, or when
  // fast_mmax < 0, the warp takes the fully IEEE path.
  float fast_mmax, fast_vmin, fast_vmax;
  float k_max;        // <= 0: no clamp
  int force_k1;
  StateFmtParams m, v;
  double log2_tab[8]; // log2(1 + i/8)
};

struct QuantParams {
  const float *x;
  uint8_t *code;
  float *k;
  float *s;
  int64_t n;
  int log2G;
  float k_max;
  int force_k1;
  StateFmtParams f;
};

// Compile-time layout of the step kernel for group size 2^LG.
template <int LG>
struct StepLayout {
  // Threads per block: 64 (2 warps), or the threads of one group where that
  // is more (128 for G = 2048, 256 for G = 4096).  Small blocks finish at
  // different times, so the warps of an SM spread over the kernel's phases
  // (table build, update, encode) and use the special-function, FP64 and
  // shared-memory pipes more evenly (measured against 256-thread blocks:
  // +7% at G = 128, +10% at G = 256, +15% at G = 1024).
  static constexpr int kBlock = LG >= 12 ? 256 : (LG == 11 ? 128 : 64);
  static constexpr int kBlockWarps = kBlock / 32;
  static constexpr int kBlockElems = kBlock * kVec;
  static constexpr int kLanes = 1 << (LG - 4);               // threads per group
  static constexpr bool kTable = LG >= kMinTableLog2G;
  static constexpr int kGPW = LG <= 9 ? (512 >> LG) : 1;     // groups a warp touches
  static constexpr int kTW = 2 * kGPW;                       // tables per warp (m and v)
  static constexpr int kL = kTW >= 8 ? 4 : 32 / kTW;         // lanes building one table
  static constexpr int kRounds = kTW >= 8 ? kTW / 8 : 1;     // tables per lane
  static constexpr int kTableBytesPerWarp = kTable ? kTW * kTableBytes : 0;
  static constexpr int kWarpTotal = kTableBytesPerWarp;  // multiple of 512
  static constexpr int kSmemBytes = kBlockWarps * kWarpTotal;
  // resident warps per SM the register budget is sized for: 32 (64
  // registers per thread); 24 for G = 64 (16 tables, 32 KB of shared memory
  // per 4 warps) and for groups spanning several warps (G >= 1024), which run
  // faster with 80 registers (measured: 311 vs 196 G params/s at G = 1024,
  // 260 vs 233 at G = 64); 16 for the direct-decode G < 64 kernels
  static constexpr int kMinWarps = LG <= 5 ? 16 : ((LG == 6 || LG >= 10) ? 24 : 32);
  static constexpr int kMinBlocks = kMinWarps / kBlockWarps;
  // groups per block, and whether warp 0 evaluates every (k, s) of the
  // block (each pair once, read back through shared memory) instead of each
  // lane of a group evaluating its own copy: for G = 64 and 128, where a
  // group has 4 or 8 lanes (measured: +3.5% at G = 64, +1-2% at G = 128;
  // at G = 256 and 512 the two block barriers cost more than they save)
  static constexpr int kBlockGroups = kBlockElems >> LG;
  static constexpr bool kShareParams = kTable && LG <= 7 && kBlockWarps >= 2 &&
                                       2 * kBlockGroups <= 32;
};

// Dynamic shared memory, threads per block and parameters per block of the
// step kernel for group size 2^log2G (host side).
template <int LG>
struct StepLaunch {
  static constexpr size_t kSmem = StepLayout<LG>::kSmemBytes;
  static constexpr int kBlock = StepLayout<LG>::kBlock;
};

inline void step_launch_shape(int log2G, size_t &smem, int &block) {
  switch (log2G) {
#define COAT_STEP_SHAPE(LGV) \
  case LGV: smem = StepLaunch<LGV>::kSmem; block = StepLaunch<LGV>::kBlock; return;
    COAT_STEP_SHAPE(4) COAT_STEP_SHAPE(5) COAT_STEP_SHAPE(6) COAT_STEP_SHAPE(7)
    COAT_STEP_SHAPE(8) COAT_STEP_SHAPE(9) COAT_STEP_SHAPE(10) COAT_STEP_SHAPE(11)
    COAT_STEP_SHAPE(12)
#undef COAT_STEP_SHAPE
    default: smem = 0; block = 0; return;
  }
}

// a / b for a per-launch constant b with r = RN(1/b): q = RN(a r) corrected
// once with the exact residual a - q b (Markstein's FMA division step).
__device__ __forceinline__ float div_by_const(float a, float b, float r) {
  const float q = __fmul_rn(a, r);
  const float res = __fmaf_rn(-q, b, a);
  return __fmaf_rn(res, r, q);
}

__device__ __forceinline__ float rsqrt_approx(float x) {
  float y;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed binary32 pairs through PTX.  The code generator may still fuse a
// packed product that feeds a packed sum into one packed fma, even with the
// explicit rounding mode, so a product whose rounding the rule fixes is
// never summed with add2_rn: those sums are scalar __fadd_rn, which is never
// contracted.  The packed fma below is used only where a fused operation is
// intended (the correction steps).
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

// theta_t for one element with every operation of the rule correctly
// rounded: m^ = m_t / bc1, v^ = v_t / bc2, u = m^ / (sqrt(v^) + eps).
template <class P>
__device__ __forceinline__ float exact_update(float th, float mt, float vt, const P &p) {
  const float mh = div_by_const(mt, p.bc1, p.rbc1);
  const float vh = div_by_const(vt, p.bc2, p.rbc2);
  const float u = __fdiv_rn(mh, __fadd_rn(__fsqrt_rn(vh), p.eps));
  return __fsub_rn(__fmul_rn(th, p.decay), __fmul_rn(p.lr, u));
}

// The same for two elements from the estimates (see the file comment):
// m^, v^ by Markstein division; sqrt(v^) = s + (v^ - s^2) y/2 with s = v^ y,
// y = rsqrt(v^); u = q0 + (m^ - q0 d) r with d = sqrt(v^) + eps, r = rcp(d),
// q0 = m^ r.  v^ = 0 is covered by evaluating y at max(v^, 2^-126).
template <class P>
__device__ __forceinline__ float2 fast_update2(float2 th, float2 mt, float2 vt, const P &p) {
  const float2 RB1 = make_float2(p.rbc1, p.rbc1), NB1 = make_float2(-p.bc1, -p.bc1);
  const float2 RB2 = make_float2(p.rbc2, p.rbc2), NB2 = make_float2(-p.bc2, -p.bc2);
  const float2 EPS = make_float2(p.eps, p.eps), DEC = make_float2(p.decay, p.decay);
  const float2 NLR = make_float2(-p.lr, -p.lr), HALF = make_float2(0.5f, 0.5f);
  float2 q = mul2_rn(mt, RB1);
  const float2 mh = fma2_rn(fma2_rn(q, NB1, mt), RB1, q);
  q = mul2_rn(vt, RB2);
  const float2 vh = fma2_rn(fma2_rn(q, NB2, vt), RB2, q);
  const float2 y = make_float2(rsqrt_approx(fmaxf(vh.x, 0x1p-126f)),
                               rsqrt_approx(fmaxf(vh.y, 0x1p-126f)));
  const float2 sv = mul2_rn(vh, y);
  const float2 e = fma2_rn(neg2(sv), sv, vh);
  const float2 sq = fma2_rn(e, mul2_rn(y, HALF), sv);
  const float2 den = add2_rn(sq, EPS);
  const float2 r = make_float2(rcp_approx(den.x), rcp_approx(den.y));
  const float2 q0 = mul2_rn(mh, r);
  const float2 u = fma2_rn(fma2_rn(neg2(q0), den, mh), r, q0);
  const float2 a = mul2_rn(th, DEC), t2 = mul2_rn(NLR, u);
  return make_float2(__fadd_rn(a.x, t2.x), __fadd_rn(a.y, t2.y));
}

// Max of |x| and min of nonzero |x| over 16 values (NaN ignored by the max).
// The minimum runs on 2*bits(x) - 2 as unsigned integers: the doubling drops
// the sign bit, and the -2 wraps +-0 to the largest value, so zeros never win;
// for non-negative floats the integer order is the numeric order.
__device__ __forceinline__ void range16(const float *x, float &mx, float &mn) {
  mx = 0.0f;
  uint32_t key = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    mx = fmaxf(mx, fabsf(x[i]));
    key = min(key, __float_as_uint(x[i]) * 2u - 2u);
  }
  // all-zero (or all-NaN) input gives an infinite minimum
  mn = key >= 0xFF000000u - 2u ? __int_as_float(0x7f800000) : __uint_as_float((key + 2u) >> 1);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// The same for 16 values that are +0, positive or NaN (the second moment):
// the maximum needs no |.|, and bits(x) - 1 read as a float is, for x > 0,
// the float just below x (order preserved) and NaN for +0, which the
// minimum ignores.
__device__ __forceinline__ void range16_nonneg(const float *x, float &mx, float &mn) {
  float a = fmax3(x[0], x[1], x[2]);
  a = fmax3(a, x[3], x[4]);
  a = fmax3(a, x[5], x[6]);
  a = fmax3(a, x[7], x[8]);
  a = fmax3(a, x[9], x[10]);
  a = fmax3(a, x[11], x[12]);
  a = fmax3(a, x[13], x[14]);
  mx = fmaxf(fmaxf(a, x[15]), 0.0f);
  float k[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) k[i] = __uint_as_float(__float_as_uint(x[i]) - 1u);
  float b = fmin3(k[0], k[1], k[2]);
  b = fmin3(b, k[3], k[4]);
  b = fmin3(b, k[5], k[6]);
  b = fmin3(b, k[7], k[8]);
  b = fmin3(b, k[9], k[10]);
  b = fmin3(b, k[11], k[12]);
  b = fmin3(b, k[13], k[14]);
  b = fminf(b, k[15]);
  // all-zero input leaves NaN: infinite minimum
  mn = b != b ? __int_as_float(0x7f800000) : __uint_as_float(__float_as_uint(b) + 1u);
}

// Reduce (max, min) pairs for two states over the LANES threads of a group.
// For LANES <= 32 the group lives inside one warp; otherwise warp results
// are combined through shared memory.
template <int LANES, int BLOCK_WARPS>
__device__ __forceinline__ void group_reduce2(float &mx0, float &mn0, float &mx1, float &mn1,
                                              float (*red)[BLOCK_WARPS]) {
  constexpr int lim = LANES < 32 ? LANES : 32;
#pragma unroll
  for (int off = 1; off < lim; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mn0 = fminf(mn0, __shfl_xor_sync(0xffffffffu, mn0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    mn1 = fminf(mn1, __shfl_xor_sync(0xffffffffu, mn1, off));
  }
  if constexpr (LANES > 32) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
      red[0][warp] = mx0;
      red[1][warp] = mn0;
      red[2][warp] = mx1;
      red[3][warp] = mn1;
    }
    constexpr int wpg = LANES >> 5;
    if constexpr (wpg == BLOCK_WARPS) {
      __syncthreads();
    } else {
      // only the warps of this group wait for one another (named barrier
      // 1 + group index, wpg * 32 threads), so the other groups of the
      // block keep their own pace
      asm volatile("bar.sync %0, %1;" ::"r"(1 + warp / wpg), "r"(wpg * 32) : "memory");
    }
    const int w0 = (warp / wpg) * wpg;
    mx0 = red[0][w0];
    mn0 = red[1][w0];
    mx1 = red[2][w0];
    mn1 = red[3][w0];
#pragma unroll
    for (int i = 1; i < wpg; ++i) {
      mx0 = fmaxf(mx0, red[0][w0 + i]);
      mn0 = fminf(mn0, red[1][w0 + i]);
      mx1 = fmaxf(mx1, red[2][w0 + i]);
      mn1 = fminf(mn1, red[3][w0 + i]);
    }
  }
}

// Runtime-lane form for the stand-alone quantizer.
__device__ __forceinline__ void group_reduce2_rt(float &mx0, float &mn0, float &mx1, float &mn1,
                                                 int lanes, float (*red)[kWarps]) {
  const int lim = lanes < 32 ? lanes : 32;
  for (int off = 1; off < lim; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mn0 = fminf(mn0, __shfl_xor_sync(0xffffffffu, mn0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    mn1 = fminf(mn1, __shfl_xor_sync(0xffffffffu, mn1, off));
  }
  if (lanes > 32) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
      red[0][warp] = mx0;
      red[1][warp] = mn0;
      red[2][warp] = mx1;
      red[3][warp] = mn1;
    }
    __syncthreads();
    const int wpg = lanes >> 5;
    const int w0 = (warp / wpg) * wpg;
    mx0 = red[0][w0];
    mn0 = red[1][w0];
    mx1 = red[2][w0];
    mn1 = red[3][w0];
    for (int i = 1; i < wpg; ++i) {
      mx0 = fmaxf(mx0, red[0][w0 + i]);
      mn0 = fminf(mn0, red[1][w0 + i]);
      mx1 = fmaxf(mx1, red[2][w0 + i]);
      mn1 = fminf(mn1, red[3][w0 + i]);
    }
  }
}

// ---- vector I/O; FULL = the 16 values are all inside [0, n) --------------------

template <bool FULL>
__device__ __forceinline__ void load16_f32(const float *p, int64_t e0, int64_t n, float *v) {
  if (FULL || e0 + 16 <= n) {
    const float4 *q = reinterpret_cast<const float4 *>(p + e0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 t = q[i];
      v[4 * i + 0] = t.x;
      v[4 * i + 1] = t.y;
      v[4 * i + 2] = t.z;
      v[4 * i + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = (e0 + i < n) ? p[e0 + i] : 0.0f;
  }
}

template <bool FULL>
__device__ __forceinline__ void store16_f32(float *p, int64_t e0, int64_t n, const float *v) {
  if (FULL || e0 + 16 <= n) {
    float4 *q = reinterpret_cast<float4 *>(p + e0);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else {
    for (int i = 0; i < 16; ++i)
      if (e0 + i < n) p[e0 + i] = v[i];
  }
}

// 16 bytes (16 codes) as four words.
template <bool FULL>
__device__ __forceinline__ void load16_u8(const uint8_t *p, int64_t e0, int64_t n, uint32_t *w) {
  if (FULL || e0 + 16 <= n) {
    uint4 t = *reinterpret_cast<const uint4 *>(p + e0);
    w[0] = t.x;
    w[1] = t.y;
    w[2] = t.z;
    w[3] = t.w;
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = 0;
    for (int i = 0; i < 16; ++i)
      if (e0 + i < n) w[i >> 2] |= static_cast<uint32_t>(p[e0 + i]) << (8 * (i & 3));
  }
}

template <bool FULL>
__device__ __forceinline__ void store16_u8(uint8_t *p, int64_t e0, int64_t n, const uint32_t *w) {
  if (FULL || e0 + 16 <= n) {
    *reinterpret_cast<uint4 *>(p + e0) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    for (int i = 0; i < 16; ++i)
      if (e0 + i < n) p[e0 + i] = static_cast<uint8_t>(w[i >> 2] >> (8 * (i & 3)));
  }
}

// 16 BF16 values as eight words (element 2i in the low half of word i).
template <bool FULL>
__device__ __forceinline__ void load16_bf16(const uint16_t *p, int64_t e0, int64_t n,
                                            uint32_t *w) {
  if (FULL || e0 + 16 <= n) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p + e0);
    uint4 a = q[0], b = q[1];
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = 0;
    for (int i = 0; i < 16; ++i)
      if (e0 + i < n) w[i >> 1] |= static_cast<uint32_t>(p[e0 + i]) << (16 * (i & 1));
  }
}

// ---- the fused step ----------------------------------------------------------

// BF16 pair from two binary32 values, each rounded to nearest even
// (element lo in the low half, as BF16 words are stored)
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// kGradPeers: the 16 gradients of this thread as BF16 words, each the mean
// over the ranks of their BF16 gradients, RN_bf16(RN32(sum) / world) with
// the sum taken in binary32 in rank order (one rounding per addition); one
// rank gives its own gradient unchanged.
template <bool FULL>
__device__ __forceinline__ void peer_mean_bf16(const StepParams &p, int64_t e0, uint32_t *gw) {
  if (p.world == 1) {   // one rank: its own gradient, as it is
    load16_bf16<FULL>(p.grad_peer[0], e0, p.n, gw);
    return;
  }
  float acc[16];
  {
    uint32_t w[8];
    load16_bf16<FULL>(p.grad_peer[0], e0, p.n, w);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[2 * i] = bf16lo_to_float(w[i]);
      acc[2 * i + 1] = bf16hi_to_float(w[i]);
    }
  }
#pragma unroll 1
  for (int r = 1; r < p.world; ++r) {
    uint32_t w[8];
    load16_bf16<FULL>(p.grad_peer[r], e0, p.n, w);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[2 * i] = __fadd_rn(acc[2 * i], bf16lo_to_float(w[i]));
      acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], bf16hi_to_float(w[i]));
    }
  }
  const float wf = static_cast<float>(p.world);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    gw[i] = bf16x2_rn(__fdiv_rn(acc[2 * i], wf), __fdiv_rn(acc[2 * i + 1], wf));
}

// kGradPeers: four updated parameters (elements base .. base + 3 of the
// shard) into every rank's parameter slice, as FP32 or rounded to BF16.
template <bool FULL>
__device__ __forceinline__ void store4_to_peers(const StepParams &p, int64_t base,
                                                const float *o) {
  const bool whole = FULL || base + 4 <= p.n;
  if (p.param_peer_bf16) {
    const uint2 b = make_uint2(bf16x2_rn(o[0], o[1]), bf16x2_rn(o[2], o[3]));
#pragma unroll 1
    for (int r = 0; r < p.world; ++r) {
      uint16_t *d = static_cast<uint16_t *>(p.param_peer[r]);
      if (d == nullptr) continue;
      d += base;
      if (whole) {
        *reinterpret_cast<uint2 *>(d) = b;
      } else {
        const uint16_t h[4] = {static_cast<uint16_t>(b.x), static_cast<uint16_t>(b.x >> 16),
                               static_cast<uint16_t>(b.y), static_cast<uint16_t>(b.y >> 16)};
        for (int j = 0; j < 4; ++j)
          if (base + j < p.n) d[j] = h[j];
      }
    }
  } else {
#pragma unroll 1
    for (int r = 0; r < p.world; ++r) {
      float *d = static_cast<float *>(p.param_peer[r]);
      if (d == nullptr) continue;
      d += base;
      if (whole) {
        *reinterpret_cast<float4 *>(d) = make_float4(o[0], o[1], o[2], o[3]);
      } else {
        for (int j = 0; j < 4; ++j)
          if (base + j < p.n) d[j] = o[j];
      }
    }
  }
}

// The peer form holds the rank count's loop state and the replica pointers
// as well: it is sized for 7/8 of the resident blocks (72 instead of 64
// registers at G = 128; with 64 it spilled and ran 20% slower at one rank).
template <int VF, int LG, bool FULL, int GS>
__global__ void __launch_bounds__(StepLayout<LG>::kBlock,
                                  GS == kGradPeers ? StepLayout<LG>::kMinBlocks * 7 / 8
                                                   : StepLayout<LG>::kMinBlocks)
adamw_fp8_step_kernel(const StepParams p) {
  using L = StepLayout<LG>;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ double tab8[8];   // log2(1 + i/8), direct decode (G < 64)
  __shared__ float red[4][L::kBlockWarps];
  if constexpr (!L::kTable) {
    if (threadIdx.x < 8) tab8[threadIdx.x] = p.log2_tab[threadIdx.x];
  }

  // guarded form: the whole grid leaves before touching anything (the word
  // is the same for every thread, so no barrier below is split)
  if (p.skip != nullptr && *p.skip != 0u) return;

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t blk0 = (p.block0 + static_cast<int64_t>(blockIdx.x)) * L::kBlockElems;
  const int64_t e0 = blk0 + threadIdx.x * kVec;
  const bool active = FULL || e0 < p.n;
  const int64_t grp = e0 >> LG;
  const uint32_t warp_off = static_cast<uint32_t>(warp * L::kWarpTotal);

  // Per-group (k, s) of the decode tables this lane builds (or of its own
  // group on the direct path), loaded first so that they arrive while the
  // bulk streams are requested.
  const int64_t warp_g0 = (blk0 + warp * 32 * kVec) >> LG;
  float kk[L::kRounds], ss[L::kRounds];
  float mk = 1.0f, ms = 0.0f, vk = 1.0f, vs = 0.0f;
  if constexpr (L::kTable) {
#pragma unroll
    for (int r = 0; r < L::kRounds; ++r) {
      const int j = r * (32 / L::kL) + lane / L::kL;
      const bool vst = j >= L::kGPW;
      const int64_t g = warp_g0 + (vst ? j - L::kGPW : j);
      kk[r] = 1.0f;
      ss[r] = 0.0f;
      if (FULL || g < p.ngroups) {
        kk[r] = vst ? p.v_k[g] : p.m_k[g];
        ss[r] = vst ? p.v_s[g] : p.m_s[g];
      }
    }
  } else if (active) {
    mk = p.m_k[grp];
    ms = p.m_s[grp];
    vk = p.v_k[grp];
    vs = p.v_s[grp];
  }

  float m[16], v[16];
  uint32_t gw[8], mw[4], vw[4];
  if (active) {
    if constexpr (GS == kGradF32) {
      // float32 gradients become the BF16 gradients of the rule right here
      float g16[16];
      load16_f32<FULL>(p.grad_f32, e0, p.n, g16);
#pragma unroll
      for (int i = 0; i < 8; ++i) gw[i] = bf16x2_rn(g16[2 * i], g16[2 * i + 1]);
    } else if constexpr (GS == kGradPeers) {
      peer_mean_bf16<FULL>(p, e0, gw);
    } else {
      load16_bf16<FULL>(p.grad, e0, p.n, gw);
    }
    load16_u8<FULL>(p.m_code, e0, p.n, mw);
    load16_u8<FULL>(p.v_code, e0, p.n, vw);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) gw[i] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) mw[i] = vw[i] = 0;
  }

  // ---- beta1 * m and beta2 * v from the stored states (exact binary32) ----
  if constexpr (L::kTable) {
    // warp-local decode tables: [0, GPW) first moment, [GPW, 2 GPW) second
#pragma unroll
    for (int r = 0; r < L::kRounds; ++r) {
      const int j = r * (32 / L::kL) + lane / L::kL;
      const bool vst = j >= L::kGPW;
      const uint32_t key = (warp_off + j * kTableBytes) | (32u * (j & 3));
      build_table<L::kL, VF != kE4M3>(smem, key, lane % L::kL, VF == kE4M3 || !vst, kk[r],
                                      ss[r], vst ? p.beta2 : p.beta1);
    }
    __syncwarp();
    const int lg = L::kGPW > 1 ? (lane >> (LG - 4)) : 0;
    const int jm = lg, jv = L::kGPW + lg;
    lookup16(smem, (warp_off + jm * kTableBytes) | (32u * (jm & 3)), mw, m);
    lookup16(smem, (warp_off + jv * kTableBytes) | (32u * (jv & 3)), vw, v);
  } else {
    __syncthreads();  // tab8
    const double mrk = 1.0 / static_cast<double>(mk), vrk = 1.0 / static_cast<double>(vk);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      float dm[4], dv[4];
      fp8x4_to_float<kE4M3>(mw[w], dm);
      fp8x4_to_float<VF>(vw[w], dv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        m[4 * w + j] = __fmul_rn(p.beta1, dequant_exact(dm[j], ms, mrk, tab8));
        v[4 * w + j] = __fmul_rn(p.beta2, dequant_exact(dv[j], vs, vrk, tab8));
      }
    }
  }

  // ---- the new moments, binary32, one rounding per operation (scalar sums) ----
  {
    const float2 C1 = make_float2(p.c1, p.c1), C2 = make_float2(p.c2, p.c2);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 g = make_float2(bf16lo_to_float(gw[i]), bf16hi_to_float(gw[i]));
      const float2 cg = mul2_rn(C1, g), cgg = mul2_rn(C2, mul2_rn(g, g));
      m[2 * i] = __fadd_rn(m[2 * i], cg.x);
      m[2 * i + 1] = __fadd_rn(m[2 * i + 1], cg.y);
      v[2 * i] = __fadd_rn(v[2 * i], cgg.x);
      v[2 * i + 1] = __fadd_rn(v[2 * i + 1], cgg.y);
    }
  }
  // theta is loaded only now, when the codes and gradients are consumed, so
  // that its 16 registers are not held through the table build; the range
  // below runs while it is in flight
  float4 th[4];
  if (FULL || e0 + 16 <= p.n) {
#pragma unroll
    for (int c = 0; c < 4; ++c) th[c] = *reinterpret_cast<const float4 *>(p.theta + e0 + 4 * c);
  } else {
    float t16[16];
    load16_f32<false>(p.theta, e0, p.n, t16);
#pragma unroll
    for (int c = 0; c < 4; ++c)
      th[c] = make_float4(t16[4 * c], t16[4 * c + 1], t16[4 * c + 2], t16[4 * c + 3]);
  }
  // tail elements beyond n must not take part in the group range
  if (!FULL && e0 + 16 > p.n) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (e0 + i >= p.n) m[i] = v[i] = 0.0f;
  }

  // ---- this thread's range of the new moments ----
  float mmx, mmn, vmx, vmn;
  range16(m, mmx, mmn);
  range16_nonneg(v, vmx, vmn);

  const bool slow = __any_sync(0xffffffffu, !(mmx <= p.fast_mmax && vmx <= p.fast_vmax &&
                                                 vmn >= p.fast_vmin));

  // ---- theta_t = (1 - lr wd) theta - lr m^ / (sqrt(v^) + eps) ----
  // The estimate-based form runs unconditionally; a warp with a thread
  // outside its range then recomputes and rewrites its parameters with the
  // fully IEEE operations.
  {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 th4 = th[c];
      const float2 a = fast_update2(make_float2(th4.x, th4.y),
                                    make_float2(m[4 * c], m[4 * c + 1]),
                                    make_float2(v[4 * c], v[4 * c + 1]), p);
      const float2 b = fast_update2(make_float2(th4.z, th4.w),
                                    make_float2(m[4 * c + 2], m[4 * c + 3]),
                                    make_float2(v[4 * c + 2], v[4 * c + 3]), p);
      const int64_t base = e0 + 4 * c;
      if (FULL || base + 4 <= p.n) {
        *reinterpret_cast<float4 *>(p.theta + base) = make_float4(a.x, a.y, b.x, b.y);
      } else {
        const float o[4] = {a.x, a.y, b.x, b.y};
        for (int j = 0; j < 4; ++j)
          if (base + j < p.n) p.theta[base + j] = o[j];
      }
      if constexpr (GS == kGradPeers) {
        const float o[4] = {a.x, a.y, b.x, b.y};
        store4_to_peers<FULL>(p, base, o);
      }
    }
    if (slow) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 th4 = th[c];
        const float o[4] = {exact_update(th4.x, m[4 * c], v[4 * c], p),
                            exact_update(th4.y, m[4 * c + 1], v[4 * c + 1], p),
                            exact_update(th4.z, m[4 * c + 2], v[4 * c + 2], p),
                            exact_update(th4.w, m[4 * c + 3], v[4 * c + 3], p)};
        const int64_t base = e0 + 4 * c;
        for (int j = 0; j < 4; ++j)
          if (FULL || base + j < p.n) p.theta[base + j] = o[j];
        if constexpr (GS == kGradPeers) store4_to_peers<FULL>(p, base, o);
      }
    }
    if constexpr (GS == kGradPeers) {
      // the replicas written into other ranks' memory are visible to them
      // (after the host-side barrier that follows the launch) before the
      // kernel counts as finished
      if (p.world > 1) __threadfence_system();
    }
  }

  // ---- per-group range of the new moments, then k and s ----
  group_reduce2<L::kLanes, L::kBlockWarps>(mmx, mmn, vmx, vmn, red);
  GroupQ gm, gv;
  if constexpr (L::kShareParams) {
    // The block's (group, state) pairs fit one warp: warp 0 evaluates each
    // pair once (lane 2 g for group g's first moment, 2 g + 1 for its second)
    // and the block reads them back, instead of every lane of a group
    // evaluating its own copy.
    __shared__ float rng[L::kBlockGroups][4];
    __shared__ float gq[L::kBlockGroups][2][4];
    const int gib = threadIdx.x >> (LG - 4);
    if ((threadIdx.x & (L::kLanes - 1)) == 0) {
      rng[gib][0] = mmx;
      rng[gib][1] = mmn;
      rng[gib][2] = vmx;
      rng[gib][3] = vmn;
    }
    __syncthreads();
    if (threadIdx.x < 2 * L::kBlockGroups) {
      const int gi = threadIdx.x >> 1;
      const int odd = threadIdx.x & 1;
      const GroupQ q = group_params(rng[gi][2 * odd], rng[gi][2 * odd + 1],
                                    odd ? p.v.ln_range : p.m.ln_range,
                                    odd ? p.v.fmax : p.m.fmax,
                                    odd ? p.v.log2_fmax : p.m.log2_fmax,
                                    odd ? p.v.rfmax : p.m.rfmax, p.k_max, p.force_k1);
      gq[gi][odd][0] = q.k;
      gq[gi][odd][1] = q.s;
      gq[gi][odd][2] = q.rM;
    }
    __syncthreads();
    gm.k = gq[gib][0][0];
    gm.s = gq[gib][0][1];
    gm.rM = gq[gib][0][2];
    gv.k = gq[gib][1][0];
    gv.s = gq[gib][1][1];
    gv.rM = gq[gib][1][2];
    gm.zero = gm.s == 0.0f;
    gv.zero = gv.s == 0.0f;
  } else if constexpr (L::kLanes >= 2) {
    // even lanes evaluate m's parameters, odd lanes v's; then swap
    const bool odd = threadIdx.x & 1;
    const GroupQ mine = group_params(odd ? vmx : mmx, odd ? vmn : mmn,
                                     odd ? p.v.ln_range : p.m.ln_range,
                                     odd ? p.v.fmax : p.m.fmax,
                                     odd ? p.v.log2_fmax : p.m.log2_fmax,
                                     odd ? p.v.rfmax : p.m.rfmax, p.k_max, p.force_k1);
    GroupQ other;
    other.k = __shfl_xor_sync(0xffffffffu, mine.k, 1);
    other.s = __shfl_xor_sync(0xffffffffu, mine.s, 1);
    other.rM = __shfl_xor_sync(0xffffffffu, mine.rM, 1);
    other.zero = __shfl_xor_sync(0xffffffffu, static_cast<int>(mine.zero), 1) != 0;
    gm = odd ? other : mine;
    gv = odd ? mine : other;
  } else {
    gm = group_params(mmx, mmn, p.m.ln_range, p.m.fmax, p.m.log2_fmax, p.m.rfmax, p.k_max,
                      p.force_k1);
    gv = group_params(vmx, vmn, p.v.ln_range, p.v.fmax, p.v.log2_fmax, p.v.rfmax, p.k_max,
                      p.force_k1);
  }

  // ---- re-expand, rescale and encode ----
  uint32_t mo[4], vo[4];
  encode16<kE4M3>(m, gm, p.m.log2_fmax, mo);
  encode16<VF>(v, gv, p.v.log2_fmax, vo);
  if (active) {
    store16_u8<FULL>(p.m_code, e0, p.n, mo);
    store16_u8<FULL>(p.v_code, e0, p.n, vo);
    if ((threadIdx.x & (L::kLanes - 1)) == 0) {
      p.m_k[grp] = gm.k;
      p.m_s[grp] = gm.s;
      p.v_k[grp] = gv.k;
      p.v_s[grp] = gv.s;
    }
  }
}

// ---- stand-alone state quantizer --------------------------------------------

template <int F>
__global__ void __launch_bounds__(kThreads)
quantize_state_kernel(const QuantParams p) {
  __shared__ float red[4][kWarps];
  const int64_t e0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) * kVec;
  const bool active = e0 < p.n;
  const int64_t grp = e0 >> p.log2G;
  const int lanes = 1 << (p.log2G - 4);
  float x[16];
  if (active) {
    load16_f32<false>(p.x, e0, p.n, x);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = 0.0f;
  }
  float mx, mn, dmx = 0.0f, dmn = 0.0f;
  range16(x, mx, mn);
  group_reduce2_rt(mx, mn, dmx, dmn, lanes, red);
  const GroupQ g = group_params(mx, mn, p.f.ln_range, p.f.fmax, p.f.log2_fmax, p.f.rfmax,
                                p.k_max, p.force_k1);
  uint32_t o[4];
  encode16<F>(x, g, p.f.log2_fmax, o);
  if (active) {
    store16_u8<false>(p.code, e0, p.n, o);
    if ((threadIdx.x & (lanes - 1)) == 0) {
      p.k[grp] = g.k;
      p.s[grp] = g.s;
    }
  }
}

}  // namespace coat
