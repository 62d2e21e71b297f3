// Multi-stage global -> shared streaming for the activation-side kernels,
// built on the untiled bulk asynchronous copy (cp.async.bulk, the TMA
// engine's 1-D form) whose completion is counted on an mbarrier.
//
// A persistent block walks its tiles b, b + grid, b + 2 grid, ...; thread 0
// keeps kBulkStages tiles in flight, so each SM holds tens of kilobytes
// of outstanding reads with no registers spent on them.  Per tile:
//   1. every thread waits (bounded) for the stage's mbarrier phase,
//   2. reads its slice of the tile from shared memory into registers and
//      fences those (generic-proxy) reads against the asynchronous proxy,
//   3. one block barrier (which also combines the wait results),
//   4. thread 0 refills the stage with the tile kBulkStages ahead,
//   5. the threads compute and store their results to global memory.
// Without the fence of step 2 the refill's copy can overwrite a stage
// before reads that were issued ahead of the barrier have taken their data
// (measured: a few hundred of 8192 tiles decoded from the wrong codes).
// The copies here never use cluster multicast: every source is this GPU's
// own memory, and no code path runs across GPUs.
//
// Every wait is bounded.  A wait that runs out counts itself in
// g_bulk_wait_timeouts (read on the host through coat_bulk_wait_timeouts),
// and the block then waits, again with a bound, for its copies still in
// flight before it returns, so that no copy lands in shared memory that a
// later block owns -- as long as that second wait succeeds.  If it too
// runs out, a copy may still be in flight when the block leaves: the
// counter is nonzero either way, and a caller that sees it must treat the
// outputs as incomplete and the context as suspect.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

namespace coat {

// Two stages: measured against three and four (1xG quantizer, 33.5M and
// 134M elements), the shallowest pipeline is fastest -- deeper ones only
// queue more bytes in front of the DRAM, lengthening each kernel's fill and
// drain without raising its streaming rate.
constexpr int kBulkStages = 2;
// mbarrier polls before a wait gives up (each poll may itself suspend the
// thread for a short, hardware-chosen time): far longer than any copy
// takes, far shorter than a watchdog
constexpr uint32_t kBulkWaitPolls = 1u << 20;

__device__ unsigned int g_bulk_wait_timeouts;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// make barrier initialisation visible to the asynchronous (copy) proxy
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// one arrival that also announces `bytes` of copies to complete this phase
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "  selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// bounded wait for the phase with the given parity to complete
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint32_t polls = kBulkWaitPolls) {
  for (uint32_t i = 0; i < polls; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// a plain arrival (no transaction count)
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// orders this thread's earlier shared-memory reads before later writes by
// the asynchronous proxy (a bulk copy into the same stage)
__device__ __forceinline__ void fence_reads_before_async_writes() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// global -> shared bulk copy of `bytes` (a multiple of 16; both addresses
// 16-byte aligned), completing on `bar`
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :
      : "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// The stages of one block: kBulkStages buffers of kStageBytes in dynamic shared
// memory and one mbarrier each.  Local tile i (the block's i-th) lives in
// stage i % kBulkStages, and completes the barrier's phase i / kBulkStages.
template <int kStageBytes>
struct BulkPipe {
  unsigned char *buf;
  uint64_t *bar;

  __device__ unsigned char *stage(int i) const { return buf + (i % kBulkStages) * kStageBytes; }

  // thread 0; the caller synchronises the block afterwards
  __device__ void init() const {
    for (int s = 0; s < kBulkStages; ++s) mbar_init(&bar[s], 1);
    mbar_init_fence();
  }

  // thread 0: announce `bytes` for local tile i's stage; issue its copies
  // with copy() afterwards
  __device__ void expect(int i, uint32_t bytes) const {
    mbar_arrive_expect_tx(&bar[i % kBulkStages], bytes);
  }
  __device__ void copy(int i, uint32_t offset, const void *src, uint32_t bytes) const {
    bulk_load(stage(i) + offset, src, bytes, &bar[i % kBulkStages]);
  }

  __device__ bool wait(int i) const {
    return mbar_wait(&bar[i % kBulkStages], static_cast<uint32_t>(i / kBulkStages) & 1u);
  }

  // after a wait ran out at local tile i with `issued` tiles issued in all:
  // thread 0 counts the timeout and waits (bounded) for the tiles
  // i .. issued - 1 that may still be in flight
  __device__ void abandon(int i, int issued) const {
    if (threadIdx.x != 0) return;
    atomicAdd(&g_bulk_wait_timeouts, 1u);
    for (int j = i; j < issued; ++j) wait(j);
  }
};

// Self-test of the bounded wait: a barrier that needs two arrivals gets
// `arrivals` of them (2: the phase completes; 1: nothing ever completes
// it); every thread waits with the same bounded wait the streamed kernels
// use, the block combines the results as they do, and a wait that ran out
// is counted in g_wait_selftest_timeouts.  No copy is involved, so nothing
// is in flight when the block leaves.
__device__ unsigned int g_wait_selftest_timeouts;

__global__ void bounded_wait_selftest_kernel(uint32_t arrivals, uint32_t polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 2);
    mbar_init_fence();
  }
  __syncthreads();
  if (threadIdx.x < arrivals) mbar_arrive(&bar);
  const bool ok = mbar_wait(&bar, 0u, polls);
  if (!__syncthreads_and(ok) && threadIdx.x == 0) atomicAdd(&g_wait_selftest_timeouts, 1u);
}

// Blocks for a persistent streaming grid of kernel K: every SM filled to
// the occupancy K allows, never more blocks than tiles.  SMs x resident
// blocks is found once per device (the occupancy query costs microseconds
// of host time, as much as a small launch) and kept.
constexpr int kBulkMaxDevices = 64;

template <auto K>
inline unsigned int bulk_grid(int threads, size_t smem, int64_t tiles) {
  static std::atomic<int> slots[kBulkMaxDevices];  // 0: not yet known
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kBulkMaxDevices) dev = -1;
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
  return static_cast<unsigned int>(tiles < want ? tiles : want);
}

}  // namespace coat
