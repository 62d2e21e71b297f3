// Grid size of a persistent kernel: every SM filled to the occupancy the
// kernel allows, never more blocks than units of work.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

namespace coat {

// SMs x resident blocks is found once per device (the occupancy query costs
// microseconds of host time, as much as a small launch) and kept.
constexpr int kGridMaxDevices = 64;

template <auto K>
inline unsigned int resident_grid(int threads, size_t smem, int64_t units) {
  static std::atomic<int> slots[kGridMaxDevices];  // 0: not yet known
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kGridMaxDevices) dev = -1;
  int want = dev >= 0 ? slots[dev].load(std::memory_order_relaxed) : 0;
  if (want <= 0) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev < 0 ? 0 : dev) !=
            cudaSuccess ||
        sms <= 0)
      sms = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, K, threads, smem) !=
            cudaSuccess ||
        per_sm <= 0)
      per_sm = 1;
    want = sms * per_sm;
    if (dev >= 0) slots[dev].store(want, std::memory_order_relaxed);
  }
  return static_cast<unsigned int>(units < want ? units : want);
}

}  // namespace coat
