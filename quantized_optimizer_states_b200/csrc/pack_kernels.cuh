// Multi-tensor packing between per-parameter tensors and the flat buffers of
// one parameter group (an optimizer step over a group is one
// coat_adamw_fp8_step over flat buffers).  One launch moves up to
// kPackTensors tensors: the pointer, size and offset tables travel in the
// kernel's parameter block, so nothing is allocated on the device.
//
// Work split: each tensor is cut into kPackChunk-element chunks, one chunk
// per block; block b finds its tensor by binary search over the prefix sums
// of chunks per tensor (the tables are the same for every thread, so those
// reads are uniform).  FP32 -> BF16 conversion rounds to nearest even, as a
// BF16 cast does.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace coat {

constexpr int kPackTensors = 128;   // tensors per launch (parameter block < 4 KB)
constexpr int kPackThreads = 256;
constexpr int kPackPerThread = 8;
constexpr int kPackChunk = kPackThreads * kPackPerThread;  // 2048 elements per block

struct PackParams {
  const void *ptr[kPackTensors];  // per-tensor pointer (source or destination)
  int64_t numel[kPackTensors];
  int64_t offset[kPackTensors];   // element offset in the flat buffer
  int32_t chunk0[kPackTensors + 1];  // prefix sums of chunks per tensor
  int32_t count;
  int32_t src_f32;                 // pack: sources are FP32 (else BF16 bits)
  void *flat;                      // pack: BF16 dst; unpack: FP32 src
};

__device__ __forceinline__ int pack_find(const PackParams &p, int b) {
  int lo = 0, hi = p.count - 1;
  while (lo < hi) {  // largest i with chunk0[i] <= b
    const int mid = (lo + hi + 1) >> 1;
    if (p.chunk0[mid] <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ uint16_t bf16_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// flat_bf16[offset[i] + j] = bf16(src_i[j]) (0 where src_i is NULL)
__global__ void __launch_bounds__(kPackThreads) pack_bf16_kernel(const PackParams p) {
  const int t = pack_find(p, blockIdx.x);
  const int64_t n = p.numel[t];
  const int64_t j0 = static_cast<int64_t>(blockIdx.x - p.chunk0[t]) * kPackChunk +
                     threadIdx.x * kPackPerThread;
  if (j0 >= n) return;
  uint16_t *dst = static_cast<uint16_t *>(p.flat) + p.offset[t] + j0;
  const void *src = p.ptr[t];
  uint16_t o[kPackPerThread];
  if (src == nullptr) {
#pragma unroll
    for (int i = 0; i < kPackPerThread; ++i) o[i] = 0;
  } else if (p.src_f32) {
    const float *s = static_cast<const float *>(src) + j0;
    if (j0 + kPackPerThread <= n && (reinterpret_cast<uintptr_t>(s) & 15u) == 0) {
      const float4 a = reinterpret_cast<const float4 *>(s)[0];
      const float4 b = reinterpret_cast<const float4 *>(s)[1];
      o[0] = bf16_rn(a.x); o[1] = bf16_rn(a.y); o[2] = bf16_rn(a.z); o[3] = bf16_rn(a.w);
      o[4] = bf16_rn(b.x); o[5] = bf16_rn(b.y); o[6] = bf16_rn(b.z); o[7] = bf16_rn(b.w);
    } else {
#pragma unroll
      for (int i = 0; i < kPackPerThread; ++i) o[i] = j0 + i < n ? bf16_rn(s[i]) : 0;
    }
  } else {
    const uint16_t *s = static_cast<const uint16_t *>(src) + j0;
    if (j0 + kPackPerThread <= n && (reinterpret_cast<uintptr_t>(s) & 15u) == 0) {
      const uint4 a = reinterpret_cast<const uint4 *>(s)[0];
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[2 * i] = static_cast<uint16_t>(w[i]);
        o[2 * i + 1] = static_cast<uint16_t>(w[i] >> 16);
      }
    } else {
#pragma unroll
      for (int i = 0; i < kPackPerThread; ++i) o[i] = j0 + i < n ? s[i] : 0;
    }
  }
  // destination slices start on 16-element boundaries (the flat layout pads
  // every tensor to a multiple of max(G, 16)); the caller checks this
  if (j0 + kPackPerThread <= n) {
    uint4 v;
    v.x = o[0] | (static_cast<uint32_t>(o[1]) << 16);
    v.y = o[2] | (static_cast<uint32_t>(o[3]) << 16);
    v.z = o[4] | (static_cast<uint32_t>(o[5]) << 16);
    v.w = o[6] | (static_cast<uint32_t>(o[7]) << 16);
    *reinterpret_cast<uint4 *>(dst) = v;
  } else {
    for (int i = 0; i < kPackPerThread && j0 + i < n; ++i) dst[i] = o[i];
  }
}

// dst_i[j] = bf16(flat_f32[offset[i] + j])
__global__ void __launch_bounds__(kPackThreads) unpack_bf16_kernel(const PackParams p) {
  const int t = pack_find(p, blockIdx.x);
  const int64_t n = p.numel[t];
  const int64_t j0 = static_cast<int64_t>(blockIdx.x - p.chunk0[t]) * kPackChunk +
                     threadIdx.x * kPackPerThread;
  if (j0 >= n) return;
  const float *s = static_cast<const float *>(p.flat) + p.offset[t] + j0;
  uint16_t *d = static_cast<uint16_t *>(const_cast<void *>(p.ptr[t])) + j0;
  if (j0 + kPackPerThread <= n && (reinterpret_cast<uintptr_t>(d) & 15u) == 0) {
    const float4 a = reinterpret_cast<const float4 *>(s)[0];
    const float4 b = reinterpret_cast<const float4 *>(s)[1];
    uint4 v;
    v.x = bf16_rn(a.x) | (static_cast<uint32_t>(bf16_rn(a.y)) << 16);
    v.y = bf16_rn(a.z) | (static_cast<uint32_t>(bf16_rn(a.w)) << 16);
    v.z = bf16_rn(b.x) | (static_cast<uint32_t>(bf16_rn(b.y)) << 16);
    v.w = bf16_rn(b.z) | (static_cast<uint32_t>(bf16_rn(b.w)) << 16);
    *reinterpret_cast<uint4 *>(d) = v;
  } else {
    for (int i = 0; i < kPackPerThread && j0 + i < n; ++i) d[i] = bf16_rn(s[i]);
  }
}

}  // namespace coat
