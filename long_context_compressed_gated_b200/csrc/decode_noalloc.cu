// decode_noalloc.cu - csa_decode for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: serving loops that forbid
// allocator traffic on the hot path, embedders that hand the library only the
// tensors they already own, and code running where an allocation is not
// allowed.  For them this file keeps the decode
// scratch (device status word, positions, the per-range top-k candidates and
// the selected indices) in one file-scope device array instead of a caller
// workspace.  Every GPU that loads the library holds the array until the
// process exits; calls on the same device share it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/csa.h"

namespace {

// Largest decode scratch this entry point serves (the size csa_decode_workspace_bytes
// reports for the call must fit): 8 MiB covers, e.g., B = 16 sequences with
// k = 1024 over caches of any length when H <= 64 at d = 128 (with H = 128 the
// split attention partials alone need 9.4 MB).
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device. Host code cannot
// use the array's name as a device address, so it is looked up once per device
// (with that device current) and cached for the life of the process.  The cache
// assumes the runtime's primary context of each device and no cudaDeviceReset
// (after a reset the module, and the array, would be loaded anew).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return CSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return CSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CSA_OK;
}

}  // namespace

extern "C" int csa_decode_noalloc(const void* q, const uint8_t* qI_codes, const uint8_t* qI_scales,
                                  const uint8_t* w_codes, const void* Kc, const void* Vc, const uint8_t* kI_codes,
                                  const uint8_t* kI_scales, const void* Kwin, const void* Vwin, const int64_t* pos,
                                  int B, int64_t Ncap, int H, int d, int HI, int dI, int m, int k, int W, float scale,
                                  void* O, float* lse, int32_t* idx, float* scores, int* status_out,
                                  csa_stream_t stream) {
  const size_t need = csa_decode_workspace_bytes(B, Ncap, H, d, HI, dI, k, W);
  if (need > kNoAllocScratchBytes) return CSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != CSA_OK) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  // the status word is the only part of the scratch that must start at zero
  if (cudaMemsetAsync(scratch, 0, sizeof(int), s) != cudaSuccess) return CSA_ERR_CUDA;
  rc = csa_decode(q, qI_codes, qI_scales, w_codes, Kc, Vc, kI_codes, kI_scales, Kwin, Vwin, pos, B, Ncap, H, d, HI,
                  dI, m, k, W, scale, O, CSA_BF16, lse, idx, scores, scratch, kNoAllocScratchBytes, stream);
  if (rc != CSA_OK) return rc;
  if (status_out != nullptr &&
      cudaMemcpyAsync(status_out, scratch, sizeof(int), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}
