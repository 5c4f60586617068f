// nvfp4_quantize_noalloc: the activation quantiser with a device-computed
// global scale for callers that cannot allocate device memory.
//
// The dynamic global scale needs a little device scratch (one amax partial
// per block of the first launch) between its two launches.  nvfp4_quantize
// takes that scratch from the caller's workspace; this entry point keeps it in
// a file-scope __device__ array of the library instead, so the caller passes
// only its inputs and outputs.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "internal.h"

namespace nvfp4 {
namespace na {

// Capacity of the static scratch (bytes).  One call needs
// nvfp4_quantize_workspace_bytes(1) bytes of it.
constexpr size_t kScratchBytes = NVFP4_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) float g_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device.  In host code the name
// g_scratch is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
cudaError_t scratch_address(int dev, float** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace na
}  // namespace nvfp4

extern "C" int nvfp4_quantize_noalloc(const void* x, int x_dtype, int64_t M, int64_t K, int64_t ld_x,
                                      float* g_out, uint8_t* codes, uint8_t* sf, void* stream) {
  int st = check_quant_args(x, x_dtype, M, K, ld_x, g_out, codes, sf);
  if (st != NVFP4_OK) return st;
  if (nvfp4_quantize_workspace_bytes(1) > nvfp4::na::kScratchBytes) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  st = check_device();
  if (st != NVFP4_OK) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  float* scratch = nullptr;
  e = nvfp4::na::scratch_address(dev, &scratch);
  if (e != cudaSuccess) return cuda_fail(e);
  nvfp4::RowSegments segs{};
  segs.n = 1;
  segs.begin[0] = 0;
  segs.begin[1] = M;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the amax launch overwrites every scratch word the quantise launch reads
  e = nvfp4::launch_quantize(x, x_dtype, M, K, ld_x, segs, nullptr, scratch, g_out, codes, sf, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}
