// Monitoring of one compressed optimizer state (FP8 codes with per-group k
// and s): how many groups are all zero or stored without expansion, the
// spread of k over the other groups, and how many codes sit at the format's
// largest magnitude, at zero, or on an inf/NaN pattern.  A separate call,
// run as often as the caller wants, so the step kernel carries none of it.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "coat.h"

namespace coat {

constexpr int kStatsThreads = 256;

struct StatsParams {
  const uint8_t *code;
  const float *k;
  const float *s;
  int64_t n, ngroups;
  uint32_t max_mag;    // largest finite magnitude code (0x7E E4M3, 0x7B E5M2)
  coat_state_stats_t *out;
};

__global__ void state_stats_init_kernel(coat_state_stats_t *out) {
  out->groups = 0;
  out->zero_groups = 0;
  out->k1_groups = 0;
  out->max_codes = 0;
  out->zero_codes = 0;
  out->nonfinite_codes = 0;
  out->k_sum = 0.0;
  out->k_min = __int_as_float(0x7f800000);   // +inf until a nonzero group is seen
  out->k_max = __int_as_float(0xff800000);   // -inf
}

// float min / max through compare-and-swap (any sign; NaN never wins)
__device__ __forceinline__ void atomic_min_f32(float *a, float v) {
  int *ai = reinterpret_cast<int *>(a);
  int old = *ai;
  while (v < __int_as_float(old)) {
    const int seen = atomicCAS(ai, old, __float_as_int(v));
    if (seen == old) break;
    old = seen;
  }
}

__device__ __forceinline__ void atomic_max_f32(float *a, float v) {
  int *ai = reinterpret_cast<int *>(a);
  int old = *ai;
  while (v > __int_as_float(old)) {
    const int seen = atomicCAS(ai, old, __float_as_int(v));
    if (seen == old) break;
    old = seen;
  }
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kStatsThreads) state_stats_kernel(const StatsParams p) {
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * kStatsThreads + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kStatsThreads;
  unsigned long long cmax = 0, czero = 0, cnf = 0;
  for (int64_t i = tid * 16; i < p.n; i += stride * 16) {
    uint32_t w[4];
    if (i + 16 <= p.n) {
      const uint4 v = *reinterpret_cast<const uint4 *>(p.code + i);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
      w[0] = w[1] = w[2] = w[3] = 0;
      for (int j = 0; j < 16 && i + j < p.n; ++j)
        w[j >> 2] |= static_cast<uint32_t>(p.code[i + j]) << (8 * (j & 3));
    }
    const int valid = p.n - i < 16 ? static_cast<int>(p.n - i) : 16;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t mag = (w[j >> 2] >> (8 * (j & 3))) & 0x7Fu;
      if (j < valid) {
        cmax += mag == p.max_mag;
        czero += mag == 0u;
        cnf += mag > p.max_mag;
      }
    }
  }
  unsigned long long gz = 0, gk1 = 0, gn = 0;
  float kmin = __int_as_float(0x7f800000), kmax = __int_as_float(0xff800000);
  double ksum = 0.0;
  for (int64_t g = tid; g < p.ngroups; g += stride) {
    ++gn;
    if (p.s[g] == 0.0f) {
      ++gz;
    } else {
      const float kk = p.k[g];
      gk1 += kk == 1.0f;
      kmin = fminf(kmin, kk);
      kmax = fmaxf(kmax, kk);
      ksum += static_cast<double>(kk);
    }
  }
  cmax = warp_sum_u64(cmax);
  czero = warp_sum_u64(czero);
  cnf = warp_sum_u64(cnf);
  gz = warp_sum_u64(gz);
  gk1 = warp_sum_u64(gk1);
  gn = warp_sum_u64(gn);
  for (int o = 16; o > 0; o >>= 1) {
    kmin = fminf(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    ksum += __shfl_xor_sync(0xffffffffu, ksum, o);
  }
  if ((threadIdx.x & 31) == 0) {
    coat_state_stats_t *o = p.out;
    if (cmax) atomicAdd(reinterpret_cast<unsigned long long *>(&o->max_codes), cmax);
    if (czero) atomicAdd(reinterpret_cast<unsigned long long *>(&o->zero_codes), czero);
    if (cnf) atomicAdd(reinterpret_cast<unsigned long long *>(&o->nonfinite_codes), cnf);
    if (gn) atomicAdd(reinterpret_cast<unsigned long long *>(&o->groups), gn);
    if (gz) atomicAdd(reinterpret_cast<unsigned long long *>(&o->zero_groups), gz);
    if (gk1) atomicAdd(reinterpret_cast<unsigned long long *>(&o->k1_groups), gk1);
    if (gn > gz) {
      atomicAdd(&o->k_sum, ksum);
      atomic_min_f32(&o->k_min, kmin);
      atomic_max_f32(&o->k_max, kmax);
    }
  }
}

}  // namespace coat
