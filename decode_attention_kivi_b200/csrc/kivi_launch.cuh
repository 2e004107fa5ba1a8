// kivi_launch.cuh - programmatic dependent launch (PDL) for the per-step kernels.
//
// append -> decode -> combine -> (next layer's) append run back to back on one
// stream.  Launching each with programmatic stream serialization lets the GPU
// schedule a kernel's CTAs while its predecessor drains; every kernel executes
// griddepcontrol.wait before it touches memory the predecessor may write, so
// the stream's ordering guarantees are unchanged.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <utility>

namespace kivi {

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Per-device, once-only launch set-up (function attributes such as the dynamic
// shared-memory limit are per device).  `init(int* value)` runs once for each
// device, with that device current, under a lock; later calls return the value
// it produced.  Every distinct `Init` type (one lambda per kernel
// instantiation) has its own table.
constexpr int kMaxDevices = 64;

template <typename Init>
cudaError_t per_device_setup(int device, int* value, Init init) {
  static std::mutex mu;
  static bool done[kMaxDevices] = {};
  static int values[kMaxDevices] = {};
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[device]) {
    int v = 0;
    const cudaError_t e = init(&v);
    if (e != cudaSuccess) return e;
    values[device] = v;
    done[device] = true;
  }
  *value = values[device];
  return cudaSuccess;
}

// Waits until the preceding kernel on the stream has completed and its writes
// are visible (a no-op when the launch was not programmatic).
__device__ __forceinline__ void wait_for_predecessor() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Allows the next kernel on the stream to begin launching its CTAs.
__device__ __forceinline__ void allow_successor() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace kivi
