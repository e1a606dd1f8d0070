// peak.cu - tensor-pipe throughput of this GPU, measured by a plain loop of
// tcgen05.mma instructions: the roofline denominators of the indexer's MXFP4
// contraction (kind::mxf4) and, for calibration against a library GEMM, of the
// bf16 attention tiles (kind::f16).
//
// One CTA per SM keeps its operands resident in shared memory (pseudo-random
// bytes) and issues MMAs of shape M = 128 x N = 240 back to back from one
// elected thread, alternating between two TMEM accumulators (columns 0 and
// 240) so that consecutive instructions do not depend on each other; the scale
// factors of the mxf4 form sit in columns 480..495 (all 2^0):
//   kind::mxf4.block_scale.block32  K = 64 per instruction (E2M1 x E2M1)
//   kind::f16, bf16 inputs          K = 16 per instruction
// Work per instruction: 2 * 128 * 240 * K flops.  Nothing is loaded from global
// memory inside the loop, so this is the pipe's own ceiling, which a GEMM that
// streams its operands can approach but not pass.
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

namespace {

constexpr int kPeakThreads = 128;
constexpr int kPM = 128, kPN = 240;
constexpr uint32_t kAcc1 = 240, kSFA = 480, kSFB = 488;
// shared memory: A 128 rows, B 240 rows of up to 128 bytes (K-major)
constexpr int kRowB = 128;
constexpr int kABytes = kPM * kRowB, kBBytes = kPN * kRowB;

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352dU;
  x ^= x >> 15;
  x *= 0x846ca68bU;
  x ^= x >> 16;
  return x;
}

}  // namespace

// kind: 0 = bf16 (kind::f16), 1 = MXFP4 (kind::mxf4.block_scale.block32)
__global__ void __launch_bounds__(kPeakThreads, 1) peak_mma_kernel(int kind, long long iters, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_a = smem;
  uint8_t* s_b = smem + kABytes;
  uint64_t* fin = reinterpret_cast<uint64_t*>(smem + kABytes + kBBytes);
  uint32_t* s_tslot = reinterpret_cast<uint32_t*>(fin + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // operands: pseudo-random bytes; bf16 words keep a small exponent (finite values)
  for (int i = tid; i < (kABytes + kBBytes) / 4; i += kPeakThreads) {
    uint32_t v = mix32((uint32_t)i * 2654435761u + blockIdx.x);
    if (kind == 0) v = (v & 0x807F807Fu) | 0x3F003F00u;  // bf16 pairs with exponents near 2^0
    reinterpret_cast<uint32_t*>(smem)[i] = v;
  }
  if (tid == 0) {
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(s_tslot, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *s_tslot;
  // scale factors 2^0 (byte 127) in every lane of the scale columns
  {
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    tmem_st4(tbase + lane_base + kSFA, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    tmem_st4(tbase + lane_base + kSFB, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    tmem_st4(tbase + lane_base + kSFB + 4, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    const uint32_t sa = smem_u32(s_a), sb = smem_u32(s_b);
    if (elect_one()) {
      if (kind == 1) {
        // 64-byte rows (128 E2M1 codes) with the 64-byte swizzle, as the indexer's key tiles
        const uint32_t idesc0 = idesc_mxf4(kPM, kPN, 0, 0), idesc1 = idesc_mxf4(kPM, kPN, 2, 2);
        for (long long i = 0; i < iters; ++i) {
          const int kk = (int)(i >> 1) & 1;  // which 32-byte K half of the rows
          const uint32_t d = tbase + ((i & 1) ? kAcc1 : 0u);
          mma_mxf4_ss(d, make_sdesc(sa + kk * 32, 16, 512, kSwizzle64), make_sdesc(sb + kk * 32, 16, 512, kSwizzle64),
                      kk ? idesc1 : idesc0, (tbase + kSFA) | ((uint32_t)(2 * kk) << 30),
                      (tbase + kSFB) | ((uint32_t)(2 * kk) << 30), i >= 2);
        }
      } else {
        // 128-byte rows (64 bf16) with the 128-byte swizzle, as the attention tiles
        const uint32_t idesc = idesc_bf16(kPM, kPN, 0, 0);
        for (long long i = 0; i < iters; ++i) {
          const int kk = (int)(i >> 1) & 3;  // 32-byte K step within the rows
          const uint32_t d = tbase + ((i & 1) ? kAcc1 : 0u);
          mma_bf16_ss(d, make_sdesc(sa + kk * 32, 16, 1024, kSwizzle128), make_sdesc(sb + kk * 32, 16, 1024, kSwizzle128),
                      idesc, i >= 2);
        }
      }
      mma_commit(fin);
    }
    __syncwarp();
    mbar_wait(fin, 0, status, CSA_ERR_DEVICE_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

cudaError_t launch_peak_mma(int kind, long long iters, int ctas, int* status, cudaStream_t stream) {
  const size_t smem = kABytes + kBBytes + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(peak_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  peak_mma_kernel<<<ctas, kPeakThreads, smem, stream>>>(kind, iters, status);
  return cudaGetLastError();
}

double peak_mma_flops(int kind, long long iters, int ctas) {
  const double k = kind == 1 ? 64.0 : 16.0;
  return 2.0 * kPM * kPN * k * (double)iters * (double)ctas;
}

}  // namespace csa
