// Decode layer forward with its workspace in a fixed device array of this
// library, for callers that cannot hand the library a device buffer: a host
// that has no device allocator to draw from at the call site (a plugin
// interface that passes only the layer's input and output pointers), or one
// that must not allocate while it serves tokens, because an allocation can
// synchronise the device and the memory pool was sized once at start-up.
//
// The array is file-scope device memory, reserved when the library's device
// code is loaded on a device.  It is shared by every call on that device:
// nothing in it has to start at zero (each call writes every workspace word
// it later reads), but two calls whose work overlaps in time on the same
// device (different streams, or different host threads without ordering)
// overwrite each other's intermediate results.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moeq.h"

namespace {

constexpr size_t kStaticWsBytes = (size_t)8 << 20;

static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

// Device address of the array on the current device, looked up once per
// device (null if the lookup fails).
void* static_ws_ptr() {
  static std::mutex mu;
  static void* ptrs[moeq::kMaxDevices] = {nullptr};
  int dev;
  if (!moeq::current_device(dev)) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess) return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

}  // namespace

extern "C" __attribute__((visibility("default"))) size_t moeq_static_workspace_capacity(void) {
  return kStaticWsBytes;
}

extern "C" __attribute__((visibility("default"))) moeq_status moeq_layer_forward_static(
    const moeq_layer* L, const uint16_t* x, int32_t M, float* y, const float* residual,
    int32_t* idx_out, float* w_out, void* stream) {
  // the ordinary entry point's argument checks come first, so a call fails
  // with the same status as moeq_layer_forward would; then the capacity
  const moeq_status s = moeq::forward_arg_check(L, x, M, y, residual, MOEQ_MODE_DECODE);
  if (s != MOEQ_OK || M == 0) return s;
  const size_t need = moeq_workspace_bytes(L, M, MOEQ_MODE_DECODE);
  if (need == 0)  // beyond the decode path's limits: the ordinary entry point says which
    return moeq_layer_forward(L, x, M, y, residual, idx_out, w_out, nullptr, 0,
                              MOEQ_MODE_DECODE, stream);
  if (need > kStaticWsBytes) return MOEQ_ERR_WORKSPACE;
  void* ws = static_ws_ptr();
  if (!ws) return MOEQ_ERR_CUDA;
  return moeq_layer_forward(L, x, M, y, residual, idx_out, w_out, ws, kStaticWsBytes,
                            MOEQ_MODE_DECODE, stream);
}
