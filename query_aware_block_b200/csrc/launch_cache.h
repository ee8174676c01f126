// launch_cache.h -- per-device, thread-safe records of the one-time set-up before a launch.
//
// cudaFuncSetAttribute and the occupancy answer both apply to the current device only, so a
// launcher keeps, for each kernel instance and each device: the largest dynamic shared
// memory size set so far, and the launch shapes (cluster size, shared memory) already found
// schedulable.  One mutex per record covers the attribute and occupancy calls; the launch
// itself runs outside it.  The attribute only ever grows, so a launch never sees a limit
// below the size it was checked with.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace lsa {

constexpr int kMaxDevices = 64;

inline cudaError_t current_device(int* dev) {
  const cudaError_t err = cudaGetDevice(dev);
  if (err != cudaSuccess) return err;
  if (*dev < 0 || *dev >= kMaxDevices) return cudaErrorInvalidDevice;
  return cudaSuccess;
}

struct LaunchRecord {
  static constexpr int kShapes = 16;
  std::mutex mu;
  int smem_set[kMaxDevices] = {};
  int n_ok[kMaxDevices] = {};
  long long ok[kMaxDevices][kShapes] = {};
  int sms[kMaxDevices] = {};

  // Caller holds mu.  Raises the kernel's dynamic shared memory limit on `dev` to at least
  // `smem`; `cluster` also allows non-portable cluster sizes (up to 16 CTAs).
  template <typename Kernel>
  cudaError_t ensure_smem(int dev, Kernel kernel, int smem, bool cluster) {
    if (smem <= smem_set[dev]) return cudaSuccess;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    if (cluster) {
      err = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (err != cudaSuccess) return err;
    }
    smem_set[dev] = smem;
    return cudaSuccess;
  }
  // Caller holds mu.  The number of SMs of `dev` (asked once).
  cudaError_t sm_count(int dev, int* n) {
    if (sms[dev] == 0) {
      const cudaError_t err = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
      if (err != cudaSuccess) return err;
    }
    *n = sms[dev];
    return cudaSuccess;
  }
  // Caller holds mu.  Whether (cl, smem) was found schedulable on `dev`.
  bool shape_ok(int dev, int cl, int smem) const {
    const long long key = ((long long)cl << 32) | (unsigned)smem;
    for (int i = 0; i < n_ok[dev]; ++i)
      if (ok[dev][i] == key) return true;
    return false;
  }
  // Caller holds mu.  Records (cl, smem) as schedulable on `dev` (the oldest entry makes
  // room when the list is full: it is only checked again).
  void remember_shape(int dev, int cl, int smem) {
    const long long key = ((long long)cl << 32) | (unsigned)smem;
    if (n_ok[dev] < kShapes) {
      ok[dev][n_ok[dev]++] = key;
    } else {
      for (int i = 1; i < kShapes; ++i) ok[dev][i - 1] = ok[dev][i];
      ok[dev][kShapes - 1] = key;
    }
  }
};

// A set-up step run once per device (the first launch on each device runs it; racing host
// threads wait for that one run).  Its error, if any, is returned to every later caller on
// that device.
struct DeviceOnce {
  std::once_flag flag[kMaxDevices];
  cudaError_t err[kMaxDevices] = {};

  template <typename F>
  cudaError_t run(F&& f) {
    int dev = 0;
    const cudaError_t e = current_device(&dev);
    if (e != cudaSuccess) return e;
    std::call_once(flag[dev], [&] { err[dev] = f(); });
    return err[dev];
  }
};

}  // namespace lsa
