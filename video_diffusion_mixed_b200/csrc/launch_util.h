// launch_util.h -- host helpers shared by the kernel launchers: per-device one-time kernel
// attributes and the current device's SM count.
//
// A kernel attribute (the dynamic shared-memory limit) is a property of the kernel on one device:
// it must be set once on every device the library launches on, and two host threads may launch
// for the first time at once. Each launcher keeps one bit per device in an atomic mask; setting
// the attribute twice (a race on the first launch) is harmless.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace sb {

inline int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  return dev;
}

// SM count of the current device (148 on a B200).
inline int device_sm_count() {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, current_device()) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

// Raises the kernel's dynamic shared-memory limit to `bytes` on the current device, once per
// device (devices 0..63 are remembered; others are set on every call).
template <class Kernel>
inline cudaError_t smem_attr_once(Kernel* kernel, int bytes, std::atomic<uint64_t>& done) {
  const int dev = current_device();
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

}  // namespace sb
