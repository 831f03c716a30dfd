// launch.cuh -- host-side launch helpers shared by the layer's kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include <atomic>

namespace moe {

// Largest dynamic shared memory a block may opt in to on sm_100a.
constexpr size_t kSmemOptInMax = 227 * 1024;

// Dynamic shared-memory opt-in of one kernel.  The attribute belongs to the
// kernel as loaded on one device, so it is set once per device the kernel is
// launched on (ordinals beyond the table are set on every launch).  Each call
// site passes one fixed size, the kernel's largest, so concurrent first
// launches from several host threads all set the same value.  A function-local
// static of this type is zero-initialised before any launch.
struct SmemOptIn {
  static constexpr int kDevices = 64;
  std::atomic<bool> done[kDevices];
};

template <typename Kernel>
cudaError_t opt_in_smem(Kernel kernel, size_t bytes, SmemOptIn &state) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool tracked = dev >= 0 && dev < SmemOptIn::kDevices;
  if (tracked && state.done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && tracked) state.done[dev].store(true, std::memory_order_release);
  return e;
}

}  // namespace moe
