// signrot_calibrate_static: calibration for callers that cannot allocate device memory.
//
// signrot_calibrate needs an 8 * n byte per-channel workspace from its caller. Some callers have
// no way to provide one at the point where they calibrate: runtimes that reserve all device
// memory in one pool at start-up and forbid any later cudaMalloc, plugins whose host framework
// owns the device allocator and hands them only their inputs and outputs, and latency-bound code
// that must not risk the implicit device synchronisation a cudaMalloc/cudaFree can cause. This
// entry point keeps the workspace in a fixed array in the library's own device memory instead,
// so the caller passes only the activations and the two outputs.
//
// The array is a file-scope __device__ variable of SIGNROT_STATIC_SCRATCH_MAX_N keys (256 KB). It
// is part of the module's device image: every GPU that loads the library holds it until the
// process exits. Host code cannot use the array's name as a device address, so the first call on
// each device looks the address up with cudaGetSymbolAddress (with that device current) and
// caches it; later calls reuse the cached address. The cache is keyed by device ordinal and
// assumes the device's primary context lives as long as the process: after a cudaDeviceReset the
// module is loaded again, possibly at another address, and the cached one must not be used.
#include <cstdint>
#include <cstdio>
#include <mutex>

#include <cuda_runtime.h>

#include "signrot.h"
#include "signrot_internal.h"

static __device__ __align__(256) unsigned long long g_calib_scratch[SIGNROT_STATIC_SCRATCH_MAX_N];

namespace {

constexpr int kMaxDevices = 64;

// Device address of g_calib_scratch on the current device, looked up once per device.
signrot_status scratch_address(uint64_t** out) {
  static std::mutex mu;
  static uint64_t* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    signrot::set_last_error("signrot_calibrate_static: cudaGetDevice failed");
    return SIGNROT_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    signrot::set_last_error("signrot_calibrate_static: device ordinal out of range");
    return SIGNROT_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> guard(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_calib_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[160];
      std::snprintf(msg, sizeof(msg), "signrot_calibrate_static: cudaGetSymbolAddress failed: %s",
                    cudaGetErrorString(e));
      signrot::set_last_error(msg);
      return SIGNROT_ERR_CUDA;
    }
    addr[dev] = static_cast<uint64_t*>(p);
  }
  *out = addr[dev];
  return SIGNROT_OK;
}

}  // namespace

extern "C" signrot_status signrot_calibrate_static(const void* x, int32_t dtype, int64_t T, int32_t n,
                                                   int64_t ld, int64_t t_offset, int32_t accumulate,
                                                   int32_t* k_out, float* xk_out, void* stream) {
  // every argument is checked before any CUDA call, as for the workspace-taking entry point
  signrot_status st = signrot::check_calibrate_args(x, dtype, T, n, ld, t_offset, k_out, xk_out);
  if (st != SIGNROT_OK) return st;
  // The array covers every supported row length (the longest is 2^15), so this guard only fires
  // if the two ever drift apart; an unsupported n has already been refused above.
  static_assert(SIGNROT_STATIC_SCRATCH_MAX_N >= (1 << 15), "the static array must hold the longest row");
  if (n > SIGNROT_STATIC_SCRATCH_MAX_N) {
    char msg[160];
    std::snprintf(msg, sizeof(msg),
                  "signrot_calibrate_static: n = %d exceeds the static workspace (%d channels); "
                  "use signrot_calibrate with a caller workspace",
                  n, SIGNROT_STATIC_SCRATCH_MAX_N);
    signrot::set_last_error(msg);
    return SIGNROT_ERR_UNSUPPORTED_N;
  }
  uint64_t* ws = nullptr;
  st = scratch_address(&ws);
  if (st != SIGNROT_OK) return st;
  return signrot_calibrate(x, dtype, T, n, ld, t_offset, ws, accumulate, k_out, xk_out, stream);
}
