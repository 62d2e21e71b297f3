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
// gradient, 16 B of each code stream).  A 1xG group is G/16 consecutive
// threads: up to 32 of them reduce with warp shuffles, larger groups (G >=
// 1024) finish the reduction through shared memory inside the block.  The
// whole group stays in registers between the range reduction and the
// encode, so every byte crosses HBM exactly once.
//
// Dequantization must reproduce RN32(|d|^(1/k)) exactly (the new group
// range depends on the smallest |m_t|, which cancellation in
// beta1*m + (1-beta1)*g makes sensitive to the last bit).  For G >= 64 every
// warp first builds, in shared memory, the 128-entry decode table of each of
// its (group, moment) pairs from binary64 factors -- holding beta1*m or
// beta2*v directly -- so an element costs one table lookup; for G < 64 each
// element is decoded directly in binary64.  The kernel is instantiated per
// group size, so lane counts, table counts and shifts are compile-time.
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

struct StepParams {
  float *theta;
  const uint16_t *grad;
  uint8_t *m_code;
  float *m_k;
  float *m_s;
  uint8_t *v_code;
  float *v_k;
  float *v_s;
  int64_t n;
  int64_t ngroups;
  float beta1, beta2, c1, c2, bc1, bc2, rbc1, rbc2, decay, lr, eps;
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
  static constexpr int kLanes = 1 << (LG - 4);               // threads per group
  static constexpr bool kTable = LG >= kMinTableLog2G;
  static constexpr int kGroupsPerWarp = LG <= 9 ? (512 >> LG) : 1;
  static constexpr int kTablesPerWarp = 2 * kGroupsPerWarp;  // m and v per group
  static constexpr int kJobs = 8 * kTablesPerWarp;           // per phase, per warp
  static constexpr int kRounds = (kJobs + 31) / 32;
  // 128 magnitude entries per table, the code's sign applied at lookup (the
  // signed 256-entry form measured slower: twice the shared-memory stores)
  static constexpr int kEnt = 128;
  static constexpr int kWarpBytes = kTable ? warp_table_bytes<kEnt>(kTablesPerWarp) : 0;
  // each warp also stages its 512 theta values (2 KB) through shared memory
  static constexpr int kThetaBytes = 32 * kVec * 4;
  static constexpr int kWarpTotal = kThetaBytes + kWarpBytes;
  static constexpr int kSmemBytes = kWarps * kWarpTotal;
  // resident blocks per SM the register budget is sized for (64 registers
  // per thread at 4 blocks); G = 64 is held to 2 by its 16 tables per warp
  static constexpr int kMinBlocks = LG <= 6 ? 2 : (LG == 11 ? 3 : 4);
};

// Dynamic shared memory of the step kernel for group size 2^log2G.
inline size_t step_smem_bytes(int log2G) {
  switch (log2G) {
    case 4: return StepLayout<4>::kSmemBytes;
    case 5: return StepLayout<5>::kSmemBytes;
    case 6: return StepLayout<6>::kSmemBytes;
    case 7: return StepLayout<7>::kSmemBytes;
    case 8: return StepLayout<8>::kSmemBytes;
    case 9: return StepLayout<9>::kSmemBytes;
    case 10: return StepLayout<10>::kSmemBytes;
    case 11: return StepLayout<11>::kSmemBytes;
    case 12: return StepLayout<12>::kSmemBytes;
    default: return 0;
  }
}

// a / b for a per-launch constant b with r = RN(1/b): q = RN(a r) corrected
// once with the exact residual a - q b (Markstein's FMA division step).
__device__ __forceinline__ float div_by_const(float a, float b, float r) {
  const float q = __fmul_rn(a, r);
  const float res = __fmaf_rn(-q, b, a);
  return __fmaf_rn(res, r, q);
}

__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// theta_t for one element with every operation of the rule correctly
// rounded: m^ = m_t / bc1, v^ = v_t / bc2, u = m^ / (sqrt(v^) + eps).
template <class P>
__device__ __forceinline__ float exact_update(float th, float mt, float vt, const P &p) {
  const float mh = div_by_const(mt, p.bc1, p.rbc1);
  const float vh = div_by_const(vt, p.bc2, p.rbc2);
  const float u = __fdiv_rn(mh, __fadd_rn(__fsqrt_rn(vh), p.eps));
  return __fsub_rn(__fmul_rn(th, p.decay), __fmul_rn(p.lr, u));
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

// Reduce (max, min) pairs for two states over the LANES threads of a group.
// For LANES <= 32 the group lives inside one warp; otherwise warp results
// are combined through shared memory.
template <int LANES>
__device__ __forceinline__ void group_reduce2(float &mx0, float &mn0, float &mx1, float &mn1,
                                              float (*red)[kWarps]) {
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
    __syncthreads();
    constexpr int wpg = LANES >> 5;
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

// ---- vector I/O with a ragged tail -----------------------------------------

__device__ __forceinline__ void load16_f32(const float *p, int64_t e0, int64_t n, float *v) {
  if (e0 + 16 <= n) {
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

__device__ __forceinline__ void store16_f32(float *p, int64_t e0, int64_t n, const float *v) {
  if (e0 + 16 <= n) {
    float4 *q = reinterpret_cast<float4 *>(p + e0);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else {
    for (int i = 0; i < 16; ++i)
      if (e0 + i < n) p[e0 + i] = v[i];
  }
}

// 16 bytes (16 codes or 8 BF16) as four words.
__device__ __forceinline__ void load16_u8(const uint8_t *p, int64_t e0, int64_t n, uint32_t *w) {
  if (e0 + 16 <= n) {
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

__device__ __forceinline__ void store16_u8(uint8_t *p, int64_t e0, int64_t n, const uint32_t *w) {
  if (e0 + 16 <= n) {
    *reinterpret_cast<uint4 *>(p + e0) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    for (int i = 0; i < 16; ++i)
      if (e0 + i < n) p[e0 + i] = static_cast<uint8_t>(w[i >> 2] >> (8 * (i & 3)));
  }
}

// 16 BF16 values as eight words (element 2i in the low half of word i).
__device__ __forceinline__ void load16_bf16(const uint16_t *p, int64_t e0, int64_t n,
                                            uint32_t *w) {
  if (e0 + 16 <= n) {
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

// theta of one thread (16 values) copied asynchronously into shared memory
// (cp.async, zero-filled past n), so no registers are held while it loads.
// The warp's 512 values are stored chunk-major -- chunk c (values 4c..4c+3)
// of lane l at float4 index 32c + l -- so that every 16-byte access of the
// warp touches 512 consecutive bytes (no bank conflicts).
__device__ __forceinline__ void stage_theta(float4 *warp_th, const float *theta, int64_t e0,
                                            int64_t n, int lane) {
  const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(warp_th + lane));
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int64_t base = e0 + 4 * c;
    const int bytes = base + 4 <= n ? 16 : (base < n ? static_cast<int>(n - base) * 4 : 0);
    const float *src = bytes > 0 ? theta + base : theta;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(sa + 512 * c), "l"(src),
                 "r"(bytes)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

__device__ __forceinline__ void wait_staged() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

template <int VF, int LG>
__global__ void __launch_bounds__(kThreads, StepLayout<LG>::kMinBlocks)
adamw_fp8_step_kernel(const StepParams p) {
  using L = StepLayout<LG>;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ double tab8[8];   // log2(1 + i/8)
  __shared__ double mult8[8];  // 1, -1, log2(1 + i/8) for i = 2..7
  __shared__ float red[4][kWarps];
  if (threadIdx.x < 8) {
    const double t = p.log2_tab[threadIdx.x];
    tab8[threadIdx.x] = t;
    mult8[threadIdx.x] = threadIdx.x == 0 ? 1.0 : (threadIdx.x == 1 ? -1.0 : t);
  }

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t blk0 = static_cast<int64_t>(blockIdx.x) * kElemsPerBlock;
  const int64_t e0 = blk0 + threadIdx.x * kVec;
  const bool active = e0 < p.n;
  const int64_t grp = e0 >> LG;

  // Per-group (k, s) of the decode tables this thread helps to build (or of
  // its own group on the direct path), loaded first so that they arrive
  // while the bulk streams are requested.
  const int64_t warp_g0 = (blk0 + warp * 32 * kVec) >> LG;
  float kk[L::kRounds], ss[L::kRounds];
  float mk = 1.0f, ms = 0.0f, vk = 1.0f, vs = 0.0f;
  if constexpr (L::kTable) {
#pragma unroll
    for (int r = 0; r < L::kRounds; ++r) {
      const int job = lane + 32 * r;
      const int j = job >> 3;
      const bool vst = j >= L::kGroupsPerWarp;
      const int64_t g = warp_g0 + (vst ? j - L::kGroupsPerWarp : j);
      kk[r] = 1.0f;
      ss[r] = 0.0f;
      if (job < L::kJobs && g < p.ngroups) {
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

  float4 *th_s = reinterpret_cast<float4 *>(smem + static_cast<size_t>(warp) * L::kWarpTotal);
  stage_theta(th_s, p.theta, e0, p.n, lane);
  float m[16], v[16];
  uint32_t gw[8], mw[4], vw[4];
  if (active) {
    load16_bf16(p.grad, e0, p.n, gw);
    load16_u8(p.m_code, e0, p.n, mw);
    load16_u8(p.v_code, e0, p.n, vw);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) gw[i] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) mw[i] = vw[i] = 0;
  }
  __syncthreads();  // tab8, mult8

  // ---- beta1 * m and beta2 * v from the stored states (exact binary32) ----
  if constexpr (L::kTable) {
    // warp-local decode tables: [0, GPW) first moment, [GPW, 2 GPW) second
    const WarpTables<L::kEnt> tw = warp_tables<L::kEnt>(
        smem + static_cast<size_t>(warp) * L::kWarpTotal + L::kThetaBytes, L::kTablesPerWarp);
#pragma unroll
    for (int r = 0; r < L::kRounds; ++r) {
      const int job = lane + 32 * r;
      if (job < L::kJobs) table_slot(tw, job >> 3, job & 7, kk[r], ss[r], mult8);
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < L::kRounds; ++r) {
      const int job = lane + 32 * r;
      if (job < L::kJobs) {
        const int j = job >> 3;
        const bool first = j < L::kGroupsPerWarp;
        table_codes(tw, j, job & 7, VF == kE4M3 || first, first ? p.beta1 : p.beta2);
      }
    }
    __syncwarp();
    const int lg = L::kGroupsPerWarp > 1 ? (lane >> (LG - 4)) : 0;
    lookup16<L::kEnt>(tw.ent + lg * L::kEnt, mw, m);
    lookup16<L::kEnt>(tw.ent + (L::kGroupsPerWarp + lg) * L::kEnt, vw, v);
  } else {
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

  // ---- AdamW, binary32, one rounding per operation in the order of the rule ----
  // m_t and v_t are computed exactly as the rule rounds them (they are the
  // new states): scalar IEEE sums of separately rounded products.  The
  // update quotient u = m^ / (sqrt(v^) + eps) is first formed with
  // the reciprocal-square-root estimate (relative error below 1e-6, so lr*u
  // is off by at most ~1e-6 of itself); wherever |lr*u| is not at least twice
  // below max(|theta|, lr), or eps is not negligible next to sqrt(v^), that
  // error could matter for theta, and the element is recomputed with
  // correctly rounded division and square root.
  {
    const float2 C1 = make_float2(p.c1, p.c1), C2 = make_float2(p.c2, p.c2);
    const float2 RB1 = make_float2(p.rbc1, p.rbc1), RB2 = make_float2(p.rbc2, p.rbc2);
    const float2 EPS = make_float2(p.eps, p.eps), DEC = make_float2(p.decay, p.decay);
    const float2 NLR = make_float2(-p.lr, -p.lr), TWO = make_float2(2.0f, 2.0f);
    const float2 ONE = make_float2(1.0f, 1.0f), MONE = make_float2(-1.0f, -1.0f);
    wait_staged();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 th4 = th_s[32 * c + lane];
      float2 out[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = 2 * c + h;
        const uint32_t gword = gw[i];
        const float2 g = make_float2(bf16lo_to_float(gword), bf16hi_to_float(gword));
        const float2 cg = fmul2(C1, g);
        const float2 cgg = fmul2(C2, fmul2(g, g));
        float2 mt, vt;
        mt.x = __fadd_rn(m[2 * i], cg.x);
        mt.y = __fadd_rn(m[2 * i + 1], cg.y);
        vt.x = __fadd_rn(v[2 * i], cgg.x);
        vt.y = __fadd_rn(v[2 * i + 1], cgg.y);
        // 1 / (sqrt(v^) + eps) = r / (1 + d) with r = 1/sqrt(v^), d = eps r;
        // for d <= 2^-10, 1 - d + d^2 is within 2^-30 of 1/(1 + d)
        const float2 vh = fmul2(vt, RB2);
        const float2 r = make_float2(rsqrt_approx(vh.x), rsqrt_approx(vh.y));
        const float2 d = fmul2(EPS, r);
        const float2 cc = ffma2(d, fadd2(d, MONE), ONE);
        const float2 u = fmul2(fmul2(fmul2(mt, RB1), r), cc);
        const float2 th0 = h ? make_float2(th4.z, th4.w) : make_float2(th4.x, th4.y);
        const float2 t2 = fmul2(NLR, u);
        float2 tn = fadd2(fmul2(th0, DEC), t2);
        const float2 w2 = fmul2(TWO, t2);
        const bool slow = fabsf(w2.x) > fmaxf(fabsf(tn.x), p.lr) ||
                          fabsf(w2.y) > fmaxf(fabsf(tn.y), p.lr) || !(d.x <= 0x1p-10f) ||
                          !(d.y <= 0x1p-10f);
        if (__any_sync(0xffffffffu, slow)) {
          if (slow) {
            tn.x = exact_update(th0.x, mt.x, vt.x, p);
            tn.y = exact_update(th0.y, mt.y, vt.y, p);
          }
        }
        out[h] = tn;
        m[2 * i] = mt.x;
        m[2 * i + 1] = mt.y;
        v[2 * i] = vt.x;
        v[2 * i + 1] = vt.y;
      }
      if (active) {
        const int64_t base = e0 + 4 * c;
        if (base + 4 <= p.n) {
          *reinterpret_cast<float4 *>(p.theta + base) =
              make_float4(out[0].x, out[0].y, out[1].x, out[1].y);
        } else {
          const float o[4] = {out[0].x, out[0].y, out[1].x, out[1].y};
          for (int j = 0; j < 4; ++j)
            if (base + j < p.n) p.theta[base + j] = o[j];
        }
      }
    }
  }

  // tail elements beyond n must not take part in the group range
  if (e0 + 16 > p.n) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (e0 + i >= p.n) m[i] = v[i] = 0.0f;
  }

  // ---- per-group range of the new moments, then k and s ----
  float mmx, mmn, vmx, vmn;
  range16(m, mmx, mmn);
  range16(v, vmx, vmn);
  group_reduce2<L::kLanes>(mmx, mmn, vmx, vmn, red);
  GroupQ gm, gv;
  if constexpr (L::kLanes >= 2) {
    // even lanes evaluate m's parameters, odd lanes v's; then swap
    const bool odd = threadIdx.x & 1;
    const GroupQ mine = group_params(odd ? vmx : mmx, odd ? vmn : mmn,
                                     odd ? p.v.ln_range : p.m.ln_range,
                                     odd ? p.v.fmax : p.m.fmax,
                                     odd ? p.v.log2_fmax : p.m.log2_fmax, p.k_max, p.force_k1);
    GroupQ other;
    other.k = __shfl_xor_sync(0xffffffffu, mine.k, 1);
    other.s = __shfl_xor_sync(0xffffffffu, mine.s, 1);
    other.rM = __shfl_xor_sync(0xffffffffu, mine.rM, 1);
    other.zero = __shfl_xor_sync(0xffffffffu, static_cast<int>(mine.zero), 1) != 0;
    gm = odd ? other : mine;
    gv = odd ? mine : other;
  } else {
    gm = group_params(mmx, mmn, p.m.ln_range, p.m.fmax, p.m.log2_fmax, p.k_max, p.force_k1);
    gv = group_params(vmx, vmn, p.v.ln_range, p.v.fmax, p.v.log2_fmax, p.k_max, p.force_k1);
  }

  // ---- re-expand, rescale and encode ----
  uint32_t mo[4], vo[4];
  encode16<kE4M3>(m, gm, p.m.log2_fmax, mo);
  encode16<VF>(v, gv, p.v.log2_fmax, vo);
  if (active) {
    store16_u8(p.m_code, e0, p.n, mo);
    store16_u8(p.v_code, e0, p.n, vo);
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
    load16_f32(p.x, e0, p.n, x);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = 0.0f;
  }
  float mx, mn, dmx = 0.0f, dmn = 0.0f;
  range16(x, mx, mn);
  group_reduce2_rt(mx, mn, dmx, dmn, lanes, red);
  const GroupQ g = group_params(mx, mn, p.f.ln_range, p.f.fmax, p.f.log2_fmax, p.k_max,
                                p.force_k1);
  uint32_t o[4];
  encode16<F>(x, g, p.f.log2_fmax, o);
  if (active) {
    store16_u8(p.code, e0, p.n, o);
    if ((threadIdx.x & (lanes - 1)) == 0) {
      p.k[grp] = g.k;
      p.s[grp] = g.s;
    }
  }
}

}  // namespace coat
