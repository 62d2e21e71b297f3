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
    double kd = ln_range / log(static_cast<double>(M) / static_cast<double>(mn));
    if (k_max > 0.0f && kd > static_cast<double>(k_max)) kd = static_cast<double>(k_max);
    k = static_cast<float>(kd);
  }
  g.k = k;
  if (g.zero)
    g.s = 0.0f;
  else if (k == 1.0f)
    g.s = __fdiv_rn(M, fmax);
  else
    g.s = __fmul_rn(M, ex2_approx(-log2_fmax * __frcp_rn(k)));
  g.rM = g.zero ? 0.0f : __frcp_rn(M);
  return g;
}

// ---- expansion + encode ---------------------------------------------------------
// y = fmax * (|x| / M)^k = 2^(k log2(|x| / M) + log2 fmax), signed like x
// (zero stays +0, so x == 0 encodes as 0x00).
__device__ __forceinline__ float expand_signed(float x, float rM, float k, float log2_fmax) {
  const float r = __fmul_rn(fabsf(x), rM);
  const float y = ex2_approx(__fmaf_rn(k, lg2_approx(r), log2_fmax));
  return x < 0.0f ? -y : y;
}

template <int F>
__device__ __forceinline__ void encode16(const float *x, const GroupQ &g, float log2_fmax,
                                         uint32_t *out) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = expand_signed(x[4 * w + j], g.rM, g.k, log2_fmax);
    out[w] = g.zero ? 0u : float4_to_fp8x4<F>(y[0], y[1], y[2], y[3]);
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
// For a group with exponent k and scale s, entry c (c = 0..127, the code's
// magnitude bits) holds RN32(RN32(|d_c|^(1/k)) * s).  |d_c| = (1 + f/8) 2^e,
// so |d_c|^(1/k) = A(e) B(f) with A(e) = 2^(e/k) and B(f) = 2^(log2(1+f/8)/k),
// both in binary64 (A from powers of 2^(+-1/k)); one product per entry, then
// the two binary32 roundings the definition has.  Subnormal, zero, inf and
// NaN codes are patched afterwards.
constexpr int kTabEntries = 128;
constexpr int kAOff = 16;   // A(e) at index e + 16, e in [-16, 16]
constexpr int kASize = 33;
constexpr int kTableBytes = kTabEntries * 4 + kASize * 8 + 8 * 8;  // 840

struct TableView {
  float *ent;    // [T][128]
  double *A;     // [T][33]
  double *B;     // [T][8]
};

__device__ __forceinline__ TableView table_view(unsigned char *smem, int T) {
  TableView v;
  v.ent = reinterpret_cast<float *>(smem);
  v.A = reinterpret_cast<double *>(smem + static_cast<size_t>(T) * kTabEntries * 4);
  v.B = v.A + static_cast<size_t>(T) * kASize;
  return v;
}

// Phase 1: A(e) for e in [-16, 16] (jobs [0, T)) and B(f), f = 1..7
// (jobs [T, 8T)).  k_of(j) returns table j's k.
template <class KOf>
__device__ __forceinline__ void table_phase1(const TableView &tv, int T, const double *log2tab,
                                             KOf k_of) {
  for (int job = threadIdx.x; job < 8 * T; job += blockDim.x) {
    if (job < T) {
      const double rk = 1.0 / static_cast<double>(k_of(job));
      const double a = exp2_d(rk), ai = exp2_d(-rk);
      double *Aj = tv.A + job * kASize;
      Aj[kAOff] = 1.0;
      double up = 1.0, dn = 1.0;
#pragma unroll
      for (int e = 1; e <= 16; ++e) {
        up *= a;
        dn *= ai;
        Aj[kAOff + e] = up;
        Aj[kAOff - e] = dn;
      }
    } else {
      const int q = job - T;
      const int j = q / 7;
      const int f = q - 7 * j + 1;
      const double rk = 1.0 / static_cast<double>(k_of(j));
      tv.B[j * 8 + f] = exp2_d(log2tab[f] * rk);
      if (f == 1) tv.B[j * 8] = 1.0;
    }
  }
}

// Phase 2: the 128 entries of every table, eight codes per job.  Tables
// [0, T_m) hold E4M3 first moments; [T_m, T) the second moment in VF.
template <int VF, class SOf>
__device__ __forceinline__ void table_phase2(const TableView &tv, int T, int T_m, SOf s_of) {
  for (int job = threadIdx.x; job < 16 * T; job += blockDim.x) {
    const int j = job >> 4;
    const int c0 = (job & 15) << 3;
    const float s = s_of(j);
    const double *Aj = tv.A + j * kASize;
    const double *Bj = tv.B + j * 8;
    float r[8];
    if (VF == kE4M3 || j < T_m) {
      const double a = Aj[kAOff + (c0 >> 3) - 7];
#pragma unroll
      for (int f = 0; f < 8; ++f) r[f] = __fmul_rn(static_cast<float>(a * Bj[f]), s);
    } else {
      const int E = c0 >> 2;
      const double a0 = Aj[kAOff + E - 15], a1 = Aj[kAOff + E + 1 - 15];
#pragma unroll
      for (int f = 0; f < 4; ++f) {
        r[f] = __fmul_rn(static_cast<float>(a0 * Bj[2 * f]), s);
        r[4 + f] = __fmul_rn(static_cast<float>(a1 * Bj[2 * f]), s);
      }
    }
    float4 *dst = reinterpret_cast<float4 *>(tv.ent + j * kTabEntries + c0);
    dst[0] = make_float4(r[0], r[1], r[2], r[3]);
    dst[1] = make_float4(r[4], r[5], r[6], r[7]);
  }
}

// Phase 3: zero, subnormal, inf and NaN codes.
template <int VF, class SOf>
__device__ __forceinline__ void table_phase3(const TableView &tv, int T, int T_m, SOf s_of) {
  for (int job = threadIdx.x; job < 9 * T; job += blockDim.x) {
    const int j = job / 9;
    const int w = job - 9 * j;
    const float s = s_of(j);
    float *ent = tv.ent + j * kTabEntries;
    const double *Aj = tv.A + j * kASize;
    const double *Bj = tv.B + j * 8;
    const bool e4 = (VF == kE4M3 || j < T_m);
    const int nsub = e4 ? 7 : 3;          // subnormal codes 1..nsub
    const int emin = e4 ? -9 : -16;       // exponent of the smallest subnormal
    if (w == 0) {
      ent[0] = 0.0f;
    } else if (w <= nsub) {
      // code w is w * 2^emin = (1 + f/8) 2^(lz + emin), lz = floor(log2 w)
      const int lz = 31 - __clz(w);
      const int f = (w << (3 - lz)) & 7;
      ent[w] = __fmul_rn(static_cast<float>(Aj[kAOff + lz + emin] * Bj[f]), s);
    } else if (e4) {
      if (w == 8) ent[127] = s != 0.0f ? __int_as_float(0x7fc00000) : 0.0f;
    } else if (w >= 4 && w <= 7) {
      // E5M2: 0x7C = inf, 0x7D..0x7F = NaN
      const float special = w == 4 ? __int_as_float(0x7f800000) : __int_as_float(0x7fc00000);
      ent[120 + w] = s != 0.0f ? special : 0.0f;
    }
  }
}

// Table lookup for the 16 codes held in four words (element 0 in the low
// byte of w[0]): x = entry[c & 0x7F] with the code's sign bit.
__device__ __forceinline__ void lookup16(const float *ent, const uint32_t *w, float *x) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t word = w[i >> 2];
    const int sh = 8 * (i & 3);
    const uint32_t c = (word >> sh) & 0x7Fu;
    const uint32_t sign = (word << (24 - sh)) & 0x80000000u;
    x[i] = __uint_as_float(__float_as_uint(ent[c]) | sign);
  }
}

}  // namespace coat
