// Library-wide status: error names, version, and the device error-bit word
// that bounded waits set when they time out.
#include <string.h>

#include "common.cuh"

namespace {
// One word per device (each device that loads the library has its own copy).
__device__ int32_t g_error_bits;
constexpr int kMaxDevices = 64;
int32_t* g_error_ptr[kMaxDevices];
}  // namespace

namespace sep {
int32_t* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_error_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_bits) != cudaSuccess) return nullptr;
    g_error_ptr[dev] = static_cast<int32_t*>(p);
  }
  return g_error_ptr[dev];
}
}  // namespace sep

extern "C" const char* sep_strerror(int status) {
  switch (status) {
    case SEP_OK: return "ok";
    case SEP_EINVAL: return "invalid argument";
    case SEP_EDTYPE: return "unsupported dtype or head_dim";
    case SEP_EALIGN: return "pointer not 16-byte aligned";
    case SEP_ECUDA: return "CUDA launch or runtime error";
    case SEP_EDEVICE: return "a kernel reported an error";
    case SEP_ENULL: return "required pointer is NULL";
    case SEP_ETOOBIG: return "sizes exceed the no-allocation decode scratch";
    default: return "unknown status";
  }
}

extern "C" int sep_version(void) { return 100; }

extern "C" int sep_device_status(int32_t* host_bits, int clear, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* w = sep::device_error_word();
  if (!w) return SEP_ECUDA;
  int32_t bits = 0;
  if (cudaMemcpyAsync(&bits, w, sizeof bits, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SEP_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SEP_ECUDA;
  if (clear && bits) {
    if (cudaMemsetAsync(w, 0, sizeof(int32_t), st) != cudaSuccess) return SEP_ECUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SEP_ECUDA;
  }
  if (host_bits) *host_bits = bits;
  return bits ? SEP_EDEVICE : SEP_OK;
}
