// absorb_static.cu -- ispa_absorb_static: the absorb with its scratch in a module-scope device array,
// for callers that cannot allocate device memory.
//
// The array below is sized for the largest width this entry point accepts (d <= 1536).  Every GPU
// that loads the library holds it (about 36.8 MiB) until the process exits.  Host code must not
// hand the array's name to a kernel: in host code it is only a stand-in for the symbol.  The device
// address is resolved once per device with cudaGetSymbolAddress, on the first call made while that
// device is current, and cached.
#include <mutex>

#include "../../include/ispa.h"
#include "internal.h"

namespace ispa {
namespace {

constexpr int kStaticMaxD = 1536;
// absorb_workspace_bytes(1536): four 1536 x 1536 fp32 matrices, twelve 128 x 128 inverted diagonal
// blocks, the reduction partials and scalars (each region 256-byte aligned).
constexpr size_t kStaticBytes = 4ull * 1536 * 1536 * 4 + 12ull * 128 * 128 * 4 + 16384 + 256;

static __device__ __align__(256) unsigned char g_absorb_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_absorb_scratch on the current device, resolved on first use.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_absorb_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace ispa

extern "C" ispa_status ispa_absorb_static(const float* G, const float* R, const float* S, int32_t dtype_w,
                                          const void* W, int32_t d, float lambda, uint32_t flags, float* dW,
                                          double* eps_out, void* w_new, void* stream) {
  using namespace ispa;
  if (d > kStaticMaxD) return ISPA_ERR_UNSUPPORTED;
  if (d < 16 || d % 16) return ISPA_ERR_INVALID_ARG;
  if (absorb_workspace_bytes(d, false) > kStaticBytes) return ISPA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) return ISPA_ERR_CUDA;
  // the same checks and kernels as ispa_absorb, on one stream (no library streams or events), over
  // the module-scope scratch
  return static_cast<ispa_status>(
      absorb_entry(G, R, S, dtype_w, W, d, lambda, flags, dW, eps_out, w_new, ws, kStaticBytes, stream, false));
}
