// Host-side helpers shared by the launchers: per-device, thread-safe one-time set-up.
//
// Function attributes (the dynamic shared-memory limit) and device properties (the SM
// count) belong to a device, and a process may launch on several devices from several
// host threads.  DeviceOnce runs a set-up function once per device, under
// std::call_once, and keeps its integer result for that device.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace gr {

constexpr int kMaxDevices = 64;

class DeviceOnce {
 public:
  // Runs init(dev) once for the current device dev and returns its (cached) result, or
  // kNoDevice when the current device cannot be read.
  static constexpr int kNoDevice = -(1 << 30);
  template <typename F>
  int run(F&& init) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return kNoDevice;
    std::call_once(flag_[dev], [&] { result_[dev] = init(dev); });
    return result_[dev];
  }

 private:
  std::once_flag flag_[kMaxDevices];
  int result_[kMaxDevices] = {};
};

// Number of SMs of the current device (148 on B200), looked up once per device; 0 if
// the query fails.
inline int sm_count_current() {
  static DeviceOnce once;
  const int n = once.run([](int dev) {
    int v = 0;
    return cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? v : 0;
  });
  return n > 0 ? n : 0;
}

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device, once
// per device and kernel (each kernel passes its own DeviceOnce).  True on success.
inline bool set_smem_limit_once(DeviceOnce& once, const void* kernel, int bytes) {
  return once.run([&](int) {
           return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       bytes) == cudaSuccess
                      ? 1
                      : 0;
         }) == 1;
}

}  // namespace gr
