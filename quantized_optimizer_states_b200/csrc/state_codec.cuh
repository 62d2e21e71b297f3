// Per-group state codec pieces of the COAT step: the range -> (k, s)
// computation, the expansion + FP8 encode, and correctly rounded inverse
// expansion (dequantization).
//
// COAT summary page (blog.daoxuan.cc/posts/57954), section
// "扩展函数：把窄分布拉宽": each 1xG group of a moment is expanded by
// f(x) = sign(x)|x|^k before FP8 encoding, with k = log(R_target)/log(R_X),
// R_X = max|x| / min nonzero |x|, recomputed for every group at every step;
// dequantization takes the 1/k power.  Stored per group: k and the scale s
// with x = sign(d) |d|^(1/k) s, so that the group maximum maps to the
// format's maximum: s = M * fmt_max^(-1/k).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "fp8_device.cuh"

namespace coat {

struct StateFmtParams {
  double ln_range;   // ln of the range k aims to fill
  float fmax;        // storage format's largest finite value
  float log2_fmax;   // log2(fmax), binary32
  float rfmax;       // RN(1 / fmax)
};

// ---- binary64 exp2 -----------------------------------------------------------
// 2^y for |y| < 1000.  Method: y = n + r with n the nearest integer (|r| <=
// 1/2, found by the 1.5 * 2^52 rounding trick), 2^r = e^(r ln 2) from its
// Taylor series to degree 13 (remainder < 5e-18 for |r ln 2| <= 0.347),
// evaluated by Horner's rule, then scaled by 2^n through the exponent field.
// Relative error a few units of 2^-53.
struct TaylorExp {
  double c[14];
  constexpr TaylorExp() : c() {
    double f = 1.0;
    for (int i = 0; i < 14; ++i) {
      if (i > 0) f *= static_cast<double>(i);
      c[i] = 1.0 / f;
    }
  }
};

__device__ __forceinline__ double exp2_d(double y) {
  constexpr TaylorExp T;
  constexpr double kRound = 6755399441055744.0;  // 1.5 * 2^52
  constexpr double kLn2 = 0.6931471805599453094;  // ln 2 rounded to binary64
  const double t = y + kRound;
  const int n = __double2loint(t);
  const double r = y - (t - kRound);
  const double z = r * kLn2;
  double q = T.c[13];
#pragma unroll
  for (int i = 12; i >= 0; --i) q = fma(q, z, T.c[i]);
  return q * __hiloint2double((n + 1023) << 20, 0);
}

// 1/x in binary64 from the hardware estimate and two Newton steps.
__device__ __forceinline__ double recip_d(double x) {
  double y;
  asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(y) : "d"(x));
  double e = fma(-x, y, 1.0);
  y = fma(e, y, y);
  e = fma(-x, y, 1.0);
  return fma(e, y, y);
}

// ---- per-group parameters from the group range --------------------------------

struct GroupQ {
  float k;     // expansion exponent (binary32, as stored)
  float s;     // scale, x = |d|^(1/k) * s
  float rM;    // 1 / max|x| (binary32)
  bool zero;   // all-zero group
};

// ln(x) for a positive normal binary64 x (+inf and NaN are returned as they
// are), without branches: x = 2^e m with
// m in [~sqrt(1/2), ~sqrt(2)), ln m = 2 atanh(s) = 2 (s + s^3/3 + s^5/5 + ...)
// with s = (m - 1)/(m + 1), |s| <= 0.1716, summed to s^21 (remainder below
// 2^-56 of the result); e ln 2 with ln 2 split in two parts.  Error a few
// units of 2^-53.
__device__ __forceinline__ double log_d(double x) {
  const int hi = __double2hiint(x), lo = __double2loint(x);
  const int frac = hi & 0x000FFFFF;
  const int big = frac > 0x6A09E ? 1 : 0;  // m >= ~sqrt(2): use m/2, e + 1
  const int e = (hi >> 20) - 1023 + big;
  const double m = __hiloint2double((frac | 0x3FF00000) - (big << 20), lo);
  const double s = (m - 1.0) * recip_d(m + 1.0);
  const double s2 = s * s;
  double p = 1.0 / 21.0;
  p = fma(p, s2, 1.0 / 19.0);
  p = fma(p, s2, 1.0 / 17.0);
  p = fma(p, s2, 1.0 / 15.0);
  p = fma(p, s2, 1.0 / 13.0);
  p = fma(p, s2, 1.0 / 11.0);
  p = fma(p, s2, 1.0 / 9.0);
  p = fma(p, s2, 1.0 / 7.0);
  p = fma(p, s2, 1.0 / 5.0);
  p = fma(p, s2, 1.0 / 3.0);
  const double lnm = fma(2.0 * s * s2, p, 2.0 * s);
  constexpr double kLn2Hi = 0x1.62e42fefa3800p-1;  // ln 2, leading 43 bits
  constexpr double kLn2Lo = 0x1.ef35793c76730p-45; // ln 2 - kLn2Hi
  const double ed = static_cast<double>(e);
  const double r = fma(ed, kLn2Hi, fma(ed, kLn2Lo, lnm));
  return x < __longlong_as_double(0x7FF0000000000000LL) ? r : x;  // inf, NaN pass through
}

// k = ln(R_target) / ln(M / mn) in binary64, rounded once, clamped to k_max;
// k = 1 when M == mn (or for an all-zero group, or when forced).
// s = M * fmax^(-1/k) (binary32 through the exp2 unit), or the correctly
// rounded quotient M / fmax when k == 1 (Markstein division by the constant
// fmax with its rounded reciprocal).  Every branch is a select, so the
// binary64 chain can be scheduled together with independent work.
__device__ __forceinline__ GroupQ group_params(float M, float mn, double ln_range, float fmax,
                                               float log2_fmax, float rfmax, float k_max,
                                               int force_k1) {
  GroupQ g;
  g.zero = !(M > 0.0f);
  const bool expand = !g.zero && !force_k1 && M != mn;
  const double Md = static_cast<double>(expand ? M : 2.0f);
  const double mnd = static_cast<double>(expand ? mn : 1.0f);
  double kd = ln_range * recip_d(log_d(Md * recip_d(mnd)));
  kd = (k_max > 0.0f && kd > static_cast<double>(k_max)) ? static_cast<double>(k_max) : kd;
  const float k = expand ? static_cast<float>(kd) : 1.0f;
  g.k = k;
  float rk, rM;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rk) : "f"(k));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rM) : "f"(M));
  const float q = __fmul_rn(M, rfmax);
  const float s1 = __fmaf_rn(__fmaf_rn(-q, fmax, M), rfmax, q);  // M / fmax
  const float sk = __fmul_rn(M, ex2_approx(-log2_fmax * rk));
  g.s = g.zero ? 0.0f : (k == 1.0f ? s1 : sk);
  g.rM = g.zero ? 0.0f : rM;
  return g;
}

// ---- expansion + encode ---------------------------------------------------------
// y = fmax * (|x| / M)^k = 2^(k log2(|x| / M) + log2 fmax), carrying x's sign
// bit (+0 encodes as 0x00; -0, which the update can produce only from a
// negative-zero gradient on a zero moment, as the equal-valued 0x80).
template <int F>
__device__ __forceinline__ void encode16(const float *x, const GroupQ &g, float log2_fmax,
                                         uint32_t *out) {
  // an all-zero group has rM = 0, so every y is 0 and every code 0x00
  const float2 RM = make_float2(g.rM, g.rM), K = make_float2(g.k, g.k);
  const float2 LF = make_float2(log2_fmax, log2_fmax);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float y[4];
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      const float x0 = x[4 * w + j], x1 = x[4 * w + j + 1];
      const float2 r = fmul2(make_float2(x0, x1), RM);
      const float2 z = ffma2(K, make_float2(lg2_approx(fabsf(r.x)), lg2_approx(fabsf(r.y))), LF);
      y[j] = __uint_as_float(__float_as_uint(ex2_approx(z.x)) | (__float_as_uint(x0) & 0x80000000u));
      y[j + 1] =
          __uint_as_float(__float_as_uint(ex2_approx(z.y)) | (__float_as_uint(x1) & 0x80000000u));
    }
    out[w] = float4_to_fp8x4<F>(y[0], y[1], y[2], y[3]);
  }
}

// ---- correctly rounded inverse expansion, one element ---------------------------
// x = sign(d) RN32(|d|^(1/k)) * s with |d|^(1/k) = 2^(log2|d| * (1/k)) in
// binary64: log2|d| is the exponent of d plus log2(1 + i/8) from a binary64
// table (d has at most three significant mantissa bits).  The binary64
// result is within a few units of 2^-53, so its rounding to binary32 is the
// correctly rounded power except in vanishingly rare cases.  d == 0 or s == 0
// give +0; NaN codes give NaN.
__device__ __forceinline__ float dequant_exact(float d, float s, double rk, const double *tab8) {
  const float ad = fabsf(d);
  const uint32_t b = __float_as_uint(ad);
  const double L = static_cast<double>(static_cast<int>(b >> 23) - 127) + tab8[(b >> 20) & 7u];
  const float pw = static_cast<float>(exp2_d(L * rk));
  float x = __fmul_rn(pw, s);
  x = (ad > 0.0f && s != 0.0f) ? x : 0.0f;
  x = (d != d) ? d : x;
  return d < 0.0f ? -x : x;
}

// ---- per-group decode tables ---------------------------------------------------
// For a group with exponent k and scale s, entry c (c = 0..127: a code
// without its sign bit) holds RN32(RN32(RN32(|d_c|^(1/k)) * s) * beta): the
// decoded moment already multiplied by its beta, the first product of the
// moment update (beta = 1 gives the plain decode).  A lookup applies the
// code's sign.
//
// Layout: a table takes 512 bytes at a 512-byte-aligned offset of the
// kernel's dynamic shared memory; entry c sits at byte (4c) XOR swz, with
// swz = 32 (j & 3) for the warp's table j.  The XOR sends the simultaneous
// stores of the build (below) to distinct banks, while a lookup still forms
// its address with one bitwise operation: (4c) ^ (table offset | swz).
//
// Build: the L lanes of a table (L = 4, 8 or 16) own the normal codes
// c0 + 2L i and c0 + 2L i + 1, with c0 = first + 2t for lane t (first = 8 for
// E4M3, whose codes 8..127 are normal; 4 for E5M2, codes 4..123).  A normal
// code is (1 + f 2^-mb) 2^e, so |d|^(1/k) = 2^((e + log2(1 + f 2^-mb)) / k),
// and the values of one lane advance by the constant factor M = 2^(H/k), H
// the binades per step (L/4 for E4M3, L/2 for E5M2).  A lane evaluates its
// two starting powers and a = 2^(1/k) with the binary64 exp2 and steps them
// with binary64 products: after at most 15 steps each is within ~2^-47 of
// the exact power, so its rounding to binary32 is the correctly rounded
// power except in vanishingly rare cases.  Code 0, the subnormal codes and
// the inf / NaN codes are set from their own definitions by lanes 0..3.
constexpr int kTableBytes = 512;

// log2(1 + i/8), i = 0..7, binary64
__constant__ double c_log2_1p8th[8] = {
    0.0, 0x1.5c01a39fbd688p-3, 0x1.49a784bcd1b8bp-2, 0x1.d6753e032ea0fp-2,
    0x1.2b803473f7ad1p-1, 0x1.66a008e4788ccp-1, 0x1.9d5d9fd5010b3p-1, 0x1.d053f6d260896p-1};

// RN32(RN32(RN32(q) * s) * beta)
__device__ __forceinline__ float table_entry(double q, float s, float beta) {
  return __fmul_rn(__fmul_rn(static_cast<float>(q), s), beta);
}

__device__ __forceinline__ void st_shared_f32(unsigned char *smem, uint32_t off, float v) {
  *reinterpret_cast<float *>(smem + off) = v;
}

__device__ __forceinline__ void st_shared_f32x2(unsigned char *smem, uint32_t off, float2 v) {
  *reinterpret_cast<float2 *>(smem + off) = v;
}

// Lane t (0 <= t < L) of the L lanes that build one table.  key = the
// table's offset in `smem` (a multiple of 512) | swz.  kMixed: the lanes of
// the warp build tables of both formats (E4M3 first moments beside E5M2
// second moments), so e4 differs between them.  The caller synchronises the
// warp before the first lookup.
template <int L, bool kMixed>
__device__ __forceinline__ void build_table(unsigned char *smem, uint32_t key, int t, bool e4,
                                            float k, float s, float beta) {
  static_assert(L == 4 || L == 8 || L == 16, "lanes per table");
  const double rk = recip_d(static_cast<double>(k));
  // f = 0 (E4M3: 3 mantissa bits, bias 7) or 1 (E5M2: 2 bits, bias 15)
  const int f = e4 ? 0 : 1;
  const int c0 = 8 - 4 * f + 2 * t;
  const int ex = (c0 >> (3 - f)) - 7 - 8 * f;  // exponent of the lane's first binade
  const int i0 = (c0 & (7 >> f)) << f;         // log2(1 + i/8) index of its two codes
  const int i1 = i0 + 1 + f;
  const double ed = static_cast<double>(ex);
  double P0 = exp2_d((ed + c_log2_1p8th[i0]) * rk);
  double P1 = exp2_d((ed + c_log2_1p8th[i1]) * rk);
  const double a = exp2_d(rk);
  double M = a;
#pragma unroll
  for (int h = 4; h < L; h <<= 1) M *= M;  // a^(L/4)
  M = e4 ? M : M * M;                      // E5M2 steps twice as many binades
  const float nanv = s != 0.0f ? __int_as_float(0x7fc00000) : 0.0f;
  const float infv = s != 0.0f ? __int_as_float(0x7f800000) : 0.0f;

  // Code 0 and the subnormal codes, from the lane's starting power P0
  // (binade 1): E4M3 code w is w 2^-9, E5M2 code w is w 2^-16.  The inf
  // (E5M2 0x7C) and NaN codes hold inf / NaN (0 in an all-zero group).
  if (t < 4) {
    const double ai = recip_d(a);
    const double q1 = P0 * ai, q2 = q1 * ai, q3 = q2 * ai;
    const float v1 = table_entry(q1, s, beta), v2 = table_entry(q2, s, beta);
    const float v3 = table_entry(q3, s, beta);
    // E4M3: lane 0 (P0 = 2^(-6/k)): 0, 2^-9, 2^-8, 2^-7 at codes 0, 1, 2, 4;
    // lane 1 (1.25 2^-6): code 5; lane 2 (1.5 2^-6): codes 3, 6; lane 3 (1.75 2^-6): code 7.
    // E5M2: lane 0 (2^(-14/k)): 0, 2^-16, 2^-15 at codes 0, 1, 2; lane 1
    // (1.5 2^-14): code 3; lanes 2, 3: codes 124..127 (inf, NaN x 3).
    const int pc = t == 0 ? 0 : (t == 2 ? 124 : 126);
    const float2 pv = t == 0 ? make_float2(0.0f, e4 ? v3 : v2)
                             : make_float2(t == 2 ? infv : nanv, nanv);
    if constexpr (kMixed) {
      // the same three stores in every lane, without divergent branches: a
      // lane with less to store repeats one of its stores (same address,
      // same bits)
      const int sc = e4 ? (t == 0 ? 2 : (t == 1 ? 5 : (t == 2 ? 3 : 7)))
                        : (t == 0 ? 2 : (t == 1 ? 3 : pc));
      const float sv = e4 ? ((t & 1) ? v1 : v2) : (t < 2 ? v1 : pv.x);
      const bool two = e4 && !(t & 1);
      const int sb = two ? (t == 0 ? 4 : 6) : sc;
      const float svb = two ? v1 : sv;
      if (t == 0 || !e4) st_shared_f32x2(smem, (4u * pc) ^ key, pv);
      st_shared_f32(smem, (4u * sc) ^ key, sv);
      st_shared_f32(smem, (4u * sb) ^ key, svb);
    } else {
      if (t == 0 || (!e4 && t >= 2)) st_shared_f32x2(smem, (4u * pc) ^ key, pv);
      if (e4 || t < 2) {
        const int sc = e4 ? (t == 0 ? 2 : (t == 1 ? 5 : (t == 2 ? 3 : 7))) : (t == 0 ? 2 : 3);
        const float sv = (e4 && !(t & 1)) ? v2 : v1;
        st_shared_f32(smem, (4u * sc) ^ key, sv);
      }
      if (e4 && !(t & 1)) st_shared_f32(smem, (4u * (t == 0 ? 4 : 6)) ^ key, v1);
    }
  }

  // the normal codes
  constexpr int NI = (120 + 2 * L - 1) / (2 * L);
  const float2 S = make_float2(s, s), B = make_float2(beta, beta);
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int c = c0 + 2 * L * i;
    float2 v = fmul2(fmul2(make_float2(static_cast<float>(P0), static_cast<float>(P1)), S), B);
    if (i == NI - 1) {
      if (e4 && c == 126) v.y = nanv;  // E4M3 0x7F is NaN
      // with L = 4 the last pair of every lane lies within its format's 128 codes
      if (L == 4 || c < (e4 ? 128 : 124)) st_shared_f32x2(smem, (4u * c) ^ key, v);
    } else {
      st_shared_f32x2(smem, (4u * c) ^ key, v);
    }
    P0 *= M;
    P1 *= M;
  }
}

// x[i] = sign(code i) * entry(|code i|) for the 16 codes in w[0..3] (element
// 0 in the low byte of w[0]); key = table offset | swz.
__device__ __forceinline__ void lookup16(const unsigned char *smem, uint32_t key,
                                         const uint32_t *w, float *x) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t wd = w[q];
    const float e0 = *reinterpret_cast<const float *>(smem + (((wd << 2) & 0x1FCu) ^ key));
    const float e1 = *reinterpret_cast<const float *>(smem + (((wd >> 6) & 0x1FCu) ^ key));
    const float e2 = *reinterpret_cast<const float *>(smem + (((wd >> 14) & 0x1FCu) ^ key));
    const float e3 = *reinterpret_cast<const float *>(smem + (((wd >> 22) & 0x1FCu) ^ key));
    x[4 * q + 0] = __uint_as_float(__float_as_uint(e0) | ((wd << 24) & 0x80000000u));
    x[4 * q + 1] = __uint_as_float(__float_as_uint(e1) | ((wd << 16) & 0x80000000u));
    x[4 * q + 2] = __uint_as_float(__float_as_uint(e2) | ((wd << 8) & 0x80000000u));
    x[4 * q + 3] = __uint_as_float(__float_as_uint(e3) | (wd & 0x80000000u));
  }
}

}  // namespace coat
