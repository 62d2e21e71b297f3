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

// k = ln(R_target) / ln(M / mn) in binary64, rounded once, clamped to k_max;
// k = 1 when M == mn.  s = M * fmax^(-1/k) (binary32 through the exp2 unit;
// an IEEE quotient when k == 1).
__device__ __forceinline__ GroupQ group_params(float M, float mn, double ln_range, float fmax,
                                               float log2_fmax, float k_max, int force_k1) {
  GroupQ g;
  g.zero = !(M > 0.0f);
  float k = 1.0f;
  if (!g.zero && !force_k1 && M != mn) {
    const double ratio = static_cast<double>(M) * recip_d(static_cast<double>(mn));
    double kd = ln_range * recip_d(log(ratio));
    if (k_max > 0.0f && kd > static_cast<double>(k_max)) kd = static_cast<double>(k_max);
    k = static_cast<float>(kd);
  }
  g.k = k;
  float rk, rM;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rk) : "f"(k));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rM) : "f"(M));
  if (g.zero)
    g.s = 0.0f;
  else if (k == 1.0f)
    g.s = __fdiv_rn(M, fmax);
  else
    g.s = __fmul_rn(M, ex2_approx(-log2_fmax * rk));
  g.rM = g.zero ? 0.0f : rM;
  return g;
}

// ---- expansion + encode ---------------------------------------------------------
// y = fmax * (|x| / M)^k = 2^(k log2(|x| / M) + log2 fmax), carrying x's sign
// bit (+0 encodes as 0x00; -0, which the update can produce only from a
// negative-zero gradient on a zero moment, as the equal-valued 0x80).
__device__ __forceinline__ float expand_signed(float x, float rM, float k, float log2_fmax) {
  const float r = __fmul_rn(fabsf(x), rM);
  const float y = ex2_approx(__fmaf_rn(k, lg2_approx(r), log2_fmax));
  return __uint_as_float(__float_as_uint(y) | (__float_as_uint(x) & 0x80000000u));
}

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

// ---- per-group dequantization tables --------------------------------------------
// For a group with exponent k and scale s, entry c holds
// RN32(RN32(|d_c|^(1/k)) * s) with the sign of code c.  |d_c| = (1 + f/8) 2^e,
// so |d_c|^(1/k) = A(e) B(f) with A(e) = a^e, a = 2^(1/k), and
// B(f) = 2^(log2(1 + f/8) / k), all in binary64: a, 1/a and B(2..7) come from
// exp2_d, B(1) = B(4)^2 / a (since 1.5^2 = 2 * 1.125), and a^e from at most
// four squarings and four products, so every entry is within ~2^-48 of the
// exact power before the binary32 roundings of the definition.
//
// Every warp builds the tables of the groups its threads touch (with only
// warp-level synchronisation): 2 per group (m, v), 256 signed entries each
// (ENT == 256) or 128 magnitude entries plus a sign fix-up at lookup time
// (ENT == 128, used when a warp holds many small groups).
constexpr int kTabDoubles = 8;   // a, 1/a, B(2..7)

template <int ENT>
struct WarpTables {
  float *ent;    // [TW][ENT]
  double *D;     // [TW][8]: a, 1/a, B(2), ..., B(7)
  float *S;      // [TW] scale s
};

template <int ENT>
__host__ __device__ constexpr int warp_table_bytes(int TW) {
  return ((TW * (ENT * 4 + kTabDoubles * 8 + 4)) + 15) / 16 * 16;
}

template <int ENT>
__device__ __forceinline__ WarpTables<ENT> warp_tables(unsigned char *base, int TW) {
  WarpTables<ENT> v;
  v.ent = reinterpret_cast<float *>(base);
  v.D = reinterpret_cast<double *>(base + static_cast<size_t>(TW) * ENT * 4);
  v.S = reinterpret_cast<float *>(v.D + static_cast<size_t>(TW) * kTabDoubles);
  return v;
}

// b^|e| with b = a (e >= 0) or 1/a (e < 0), |e| < 2^BITS, by square-and-multiply.
template <int BITS>
__device__ __forceinline__ double ipow(double a, double ai, int e) {
  double base = e >= 0 ? a : ai;
  int n = e >= 0 ? e : -e;
  double r = 1.0;
#pragma unroll
  for (int bit = 0; bit < BITS; ++bit) {
    const double t = r * base;
    r = (n & 1) ? t : r;
    base *= base;
    n >>= 1;
  }
  return r;
}

__device__ __forceinline__ float entry_value(double A, double B, float s) {
  return __fmul_rn(static_cast<float>(A * B), s);
}

// The decode of a pair of codes, optionally scaled by the caller's factor:
// RN32(RN32(RN32(A B) * s) * beta), two lanes at a time (products only).
__device__ __forceinline__ float2 entry_pair(double A0, double B0, double A1, double B1, float2 S,
                                             float2 BETA) {
  const float2 p = make_float2(static_cast<float>(A0 * B0), static_cast<float>(A1 * B1));
  return fmul2(fmul2(p, S), BETA);
}

// Phase 1 for one job of a warp: table j, slot f (0 = a, 1 = 1/a, 2..7 =
// B(f)).  mult8 = {1, -1, log2(1 + f/8) for f = 2..7}.
template <int ENT>
__device__ __forceinline__ void table_slot(const WarpTables<ENT> &tw, int j, int f, float k,
                                           float s, const double *mult8) {
  const double rk = recip_d(static_cast<double>(k));
  tw.D[j * kTabDoubles + f] = exp2_d(mult8[f] * rk);
  if (f == 0) tw.S[j] = s;
}

// Phase 2 for one job: the sixteen codes 16q .. 16q+15 of table j, whose
// format is E4M3 (e4) or E5M2, each entry multiplied by beta (the table
// then holds beta * x, the first product of the moment update; beta = 1
// gives the plain decode).  Code 0 and the subnormal codes (q == 0) and the
// inf / NaN codes (q == 7) are set from their own definitions.
template <int ENT>
__device__ __forceinline__ void table_codes(const WarpTables<ENT> &tw, int j, int q, bool e4,
                                            float beta) {
  const double *D = tw.D + j * kTabDoubles;
  const float s = tw.S[j];
  const float2 S = make_float2(s, s), BETA = make_float2(beta, beta);
  const double2 aai = reinterpret_cast<const double2 *>(D)[0];
  const double2 b23 = reinterpret_cast<const double2 *>(D)[1];
  const double2 b45 = reinterpret_cast<const double2 *>(D)[2];
  const double2 b67 = reinterpret_cast<const double2 *>(D)[3];
  const double a = aai.x, ai = aai.y;
  const double B[8] = {1.0, b45.x * b45.x * ai, b23.x, b23.y, b45.x, b45.y, b67.x, b67.y};
  float r[16];
  const float nan = s != 0.0f ? __int_as_float(0x7fc00000) : 0.0f;
  if (e4) {
    // binades 2q, 2q+1: exponents 2q-7, 2q-6 (binade 0 holds the subnormals)
    const double A0 = ipow<3>(a, ai, 2 * q - 7);
    const double A1 = A0 * a;
#pragma unroll
    for (int f = 0; f < 8; f += 2) {
      const float2 lo = entry_pair(A0, B[f], A0, B[f + 1], S, BETA);
      const float2 hi = entry_pair(A1, B[f], A1, B[f + 1], S, BETA);
      r[f] = lo.x;
      r[f + 1] = lo.y;
      r[8 + f] = hi.x;
      r[9 + f] = hi.y;
    }
    if (q == 0) {
      // code w = w * 2^-9: 1 -> 2^-9, 2 -> 2^-8, 3 -> 1.5 2^-8, 4 -> 2^-7,
      // 5 -> 1.25 2^-7, 6 -> 1.5 2^-7, 7 -> 1.75 2^-7; A0 = A(-7)
      const double Am8 = A0 * ai, Am9 = Am8 * ai;
      const float2 e12 = entry_pair(Am9, 1.0, Am8, 1.0, S, BETA);
      const float2 e34 = entry_pair(Am8, B[4], A0, 1.0, S, BETA);
      const float2 e56 = entry_pair(A0, B[2], A0, B[4], S, BETA);
      const float2 e70 = entry_pair(A0, B[6], A0, B[6], S, BETA);
      r[0] = 0.0f;
      r[1] = e12.x;
      r[2] = e12.y;
      r[3] = e34.x;
      r[4] = e34.y;
      r[5] = e56.x;
      r[6] = e56.y;
      r[7] = e70.x;
    }
    if (q == 7) r[15] = nan;  // 0x7F
  } else {
    // binades 4q .. 4q+3: exponents 4q-15 .. 4q-12 (binade 0: subnormals,
    // binade 31: inf and NaN)
    double A = ipow<4>(a, ai, 4 * q - 15);
    const double A0 = A;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float2 lo = entry_pair(A, B[0], A, B[2], S, BETA);
      const float2 hi = entry_pair(A, B[4], A, B[6], S, BETA);
      r[4 * b] = lo.x;
      r[4 * b + 1] = lo.y;
      r[4 * b + 2] = hi.x;
      r[4 * b + 3] = hi.y;
      A *= a;
    }
    if (q == 0) {
      // code w = w * 2^-16: 1 -> 2^-16, 2 -> 2^-15, 3 -> 1.5 2^-15; A0 = A(-15)
      const float2 e12 = entry_pair(A0 * ai, 1.0, A0, 1.0, S, BETA);
      const float2 e33 = entry_pair(A0, B[4], A0, B[4], S, BETA);
      r[0] = 0.0f;
      r[1] = e12.x;
      r[2] = e12.y;
      r[3] = e33.x;
    }
    if (q == 7) {
      r[12] = s != 0.0f ? __int_as_float(0x7f800000) : 0.0f;  // 0x7C
      r[13] = nan;
      r[14] = nan;
      r[15] = nan;
    }
  }
  // the eight jobs of a table (q = 0..7) store their 64-byte runs in a
  // rotated chunk order, so that each store instruction of eight lanes
  // touches eight different 16-byte bank groups (no bank conflicts)
  float4 *pos = reinterpret_cast<float4 *>(tw.ent + j * ENT + 16 * q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = (i + (q >> 1)) & 3;
    const float4 v = c == 0   ? make_float4(r[0], r[1], r[2], r[3])
                     : c == 1 ? make_float4(r[4], r[5], r[6], r[7])
                     : c == 2 ? make_float4(r[8], r[9], r[10], r[11])
                              : make_float4(r[12], r[13], r[14], r[15]);
    pos[c] = v;
  }
  if constexpr (ENT == 256) {
    float4 *neg = reinterpret_cast<float4 *>(tw.ent + j * ENT + 128 + 16 * q);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      neg[i] = make_float4(-r[4 * i], -r[4 * i + 1], -r[4 * i + 2], -r[4 * i + 3]);
  }
}

// Table lookup for the 16 codes held in four words (element 0 in the low
// byte of w[0]).
template <int ENT>
__device__ __forceinline__ void lookup16(const float *ent, const uint32_t *w, float *x) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t word = w[i >> 2];
    const int sh = 8 * (i & 3);
    if constexpr (ENT == 256) {
      x[i] = ent[(word >> sh) & 0xFFu];
    } else {
      const uint32_t c = (word >> sh) & 0x7Fu;
      const uint32_t sign = (word << (24 - sh)) & 0x80000000u;
      x[i] = __uint_as_float(__float_as_uint(ent[c]) | sign);
    }
  }
}

}  // namespace coat
