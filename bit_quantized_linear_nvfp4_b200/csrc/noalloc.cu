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

#include <cuda.h>
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
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context the address belongs to

// Unique id of the calling thread's current context (cuCtxGetId), 0 when the
// driver does not provide it.  A context that is destroyed and created again
// (cudaDeviceReset, a primary context released and retained) gets a new id,
// and with it a new copy of g_scratch at a possibly different address.
unsigned long long current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_scratch on the current device.  In host code the name
// g_scratch is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress while the device is current, once per device and
// context, and cached; a call made in a new context of the device (after a
// reset) looks it up again.
cudaError_t scratch_address(int dev, float** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
    // the lookup makes the device's context current if it was not yet
    g_scratch_ctx[dev] = ctx != 0 ? ctx : current_context_id();
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
