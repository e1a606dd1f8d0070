// common.cuh - shared definitions of the CUDA kernels of libcsa (device side).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/csa.h"

namespace csa {

// Device status word: first 4 bytes of every workspace. The first error wins.
__device__ __forceinline__ void report(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Compressed entries visible to absolute position t: block j (tokens j*m..j*m+m-1)
// is visible iff j*m + m - 1 <= t.
__host__ __device__ __forceinline__ int64_t n_visible(int64_t t, int m) { return t < 0 ? 0 : (t + 1) / m; }

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Two floats -> packed bf16x2 (round to nearest even), low half = a.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Programmatic dependent launch.  A kernel launched with pdl = true may start
// (and run its setup) while the kernel before it in the stream is still running;
// griddep_wait() returns once that kernel has completed and its writes are
// visible, so every read of an earlier kernel's output comes after it, and
// griddep_launch_dependents() lets the next such kernel start early.  Only the
// second and later kernels of one library call are launched this way: the first
// waits for all earlier work of the stream in the ordinary way, so nothing a
// caller's own kernels write is ever read before its writer has finished.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... P, typename... A>
cudaError_t launch_kernel(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
                          A&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<A&&>(args)...);
}

// Decode positions (absolute position of each sequence's new token) travel
// inside the kernel arguments for up to kInlinePos sequences; more are first
// copied into the workspace by a small kernel.
constexpr int kInlinePos = 64;

// Workspace header: status word + padding to 256 bytes.
constexpr size_t kWorkspaceHeader = 256;

// Most key ranges one decode sequence's indexer search is split into (the
// block finalize that merges them keeps one prefix entry per range).
constexpr int kMaxKeyRanges = 63;

}  // namespace csa
