// Per-device facts the launchers need, looked up once per device and kept
// for the life of the process: the SM count, the opt-in shared-memory limit
// per block, and which kernels already carry the attributes they launch with.
// A call then costs no attribute query and no attribute set after the first
// call on a device.
#include <mutex>
#include <unordered_set>

#include "internal.h"

namespace lrkv {

namespace {

constexpr int kMaxDevices = 64;

struct DeviceSlot {
  std::once_flag once;
  int status = LRKV_ERR_CUDA;
  DevInfo info = {0, 0};
  std::mutex mu;
  std::unordered_set<const void*> prepared;
};

DeviceSlot g_slots[kMaxDevices];

}  // namespace

int current_device_info(int& dev, DevInfo& info) {
  if (cudaGetDevice(&dev) != cudaSuccess) return LRKV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LRKV_ERR_UNSUPPORTED;
  DeviceSlot& s = g_slots[dev];
  std::call_once(s.once, [&s, dev] {
    int sms = 0, optin = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) ==
            cudaSuccess) {
      s.info.sms = sms;
      s.info.optin = optin;
      s.status = LRKV_OK;
    }
  });
  if (s.status != LRKV_OK) return s.status;
  info = s.info;
  return LRKV_OK;
}

int prepare_kernel(const void* fn, bool max_carveout) {
  int dev = 0;
  DevInfo info;
  const int rc = current_device_info(dev, info);
  if (rc != LRKV_OK) return rc;
  DeviceSlot& s = g_slots[dev];
  std::lock_guard<std::mutex> lock(s.mu);
  if (s.prepared.count(fn)) return LRKV_OK;
  // the opt-in limit covers static and dynamic shared memory together
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess ||
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           info.optin - (int)fa.sharedSizeBytes) != cudaSuccess ||
      (max_carveout &&
       cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                            (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)) {
    cudaGetLastError();  // leave no error behind for the caller's next check
    return LRKV_ERR_CUDA;
  }
  s.prepared.insert(fn);
  return LRKV_OK;
}

}  // namespace lrkv
