// quantize.cu - bf16 activations -> MXFP4, the operand format of the indexer's
// query-key contraction (m.youleyou.com/wenzhang/2906406.html section 1 and
// ferris-liu.github.io ... deepseek-v4 "engineering": the indexer's QK path
// runs in FP4).  The pages give no scale rule; this follows the OCP MX
// conversion: per block of 32 consecutive elements
//   X = floor(log2 max|x|) - 2,  scale byte = X + 127 (E8M0),
//   code = E2M1 nearest to x / 2^X, ties to the even code, |.| > 6 -> 6, sign kept.
// mode CSA_MX_INDEXER clamps X to [-2, 1] (scale bytes 125..128), the range in
// which the indexer's exact fixed-point head sum holds.
//
// HBM-bound: one thread per 32-element block reads its 64 bytes with four
// 16-byte loads and writes 16 bytes of codes and one scale byte.
#include "common.cuh"

namespace csa {

namespace {

// Two floats -> one byte of two E2M1 codes (round to nearest, ties to the even
// code, saturating at +-6), a in the low nibble.
__device__ __forceinline__ uint32_t e2m1x2(float a, float b) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b16 %0, {t, 0};\n\t}"
      : "=h"(r)
      : "f"(b), "f"(a));
  return r & 0xFFu;
}

// floor(log2 a) of a bf16 magnitude a > 0 given by its bits (sign cleared), from
// the format's fields: normal 1.m * 2^(E-127); subnormal m * 2^-133.
__device__ __forceinline__ int floor_log2_bf16(uint32_t bits) {
  const int E = (int)(bits >> 7);
  return E > 0 ? E - 127 : (31 - __clz(bits & 0x7Fu)) - 133;
}

// 2^-X as an fp32 value (X in [-127, 126]: a normal power of two), so that x * 2^-X
// is the correctly rounded scaling (exact unless the product is subnormal)
__device__ __forceinline__ float pow2_neg(int X) { return __uint_as_float((uint32_t)(127 - X) << 23); }

__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(const uint4* __restrict__ x, int64_t nblocks, int mode,
                                                             uint4* __restrict__ codes,
                                                             uint8_t* __restrict__ scales) {
  const int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk >= nblocks) return;
  uint32_t w[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = __ldg(x + blk * 4 + q);
    w[4 * q] = u.x;
    w[4 * q + 1] = u.y;
    w[4 * q + 2] = u.z;
    w[4 * q + 3] = u.w;
  }
  // max |x| over the block on the bf16 magnitude bits (an order-preserving
  // integer for finite values); an exponent field of all ones is Inf or NaN
  uint32_t amax_bits = 0;
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t lo = w[i] & 0x7FFFu, hi = (w[i] >> 16) & 0x7FFFu;
    finite &= (lo < 0x7F80u) & (hi < 0x7F80u);
    amax_bits = max(amax_bits, max(lo, hi));
  }
  if (!finite) {
    codes[blk] = make_uint4(0u, 0u, 0u, 0u);
    scales[blk] = 255;
    return;
  }
  int X = -127;
  if (amax_bits != 0) X = floor_log2_bf16(amax_bits) - 2;  // at most 125 (finite bf16)
  X = X < -127 ? -127 : X;
  if (mode == CSA_MX_INDEXER) X = X < -2 ? -2 : (X > 1 ? 1 : X);
  const float p = pow2_neg(X);
  uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    // elements 2i (low half of word i) and 2i+1: E2M1 of x / 2^X by the hardware
    // conversion (nearest, ties to the even code, saturating at +-6, sign kept),
    // the first element in the low nibble
    const float y0 = __fmul_rn(bf16_lo(w[i]), p), y1 = __fmul_rn(bf16_hi(w[i]), p);
    out[i >> 2] |= e2m1x2(y0, y1) << (8 * (i & 3));
  }
  codes[blk] = make_uint4(out[0], out[1], out[2], out[3]);
  scales[blk] = (uint8_t)(X + 127);
}

// Two floats -> two E4M3 bytes (round to nearest even, saturating at +-448), a in
// the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

// MXFP8 for the compressed K/V cache: per block of 32 elements X = floor(log2
// max|x|) - 8 (448 = 1.75 * 2^8 is E4M3's largest value), scale byte X + 127,
// codes E4M3(x / 2^X).  One thread per block: 64 bytes in, 32 + 1 out.
__global__ void __launch_bounds__(256) mxfp8_quantize_kernel(const uint4* __restrict__ x, int64_t nblocks,
                                                             uint4* __restrict__ codes,
                                                             uint8_t* __restrict__ scales) {
  const int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk >= nblocks) return;
  uint32_t w[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = __ldg(x + blk * 4 + q);
    w[4 * q] = u.x;
    w[4 * q + 1] = u.y;
    w[4 * q + 2] = u.z;
    w[4 * q + 3] = u.w;
  }
  uint32_t amax_bits = 0;
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t lo = w[i] & 0x7FFFu, hi = (w[i] >> 16) & 0x7FFFu;
    finite &= (lo < 0x7F80u) & (hi < 0x7F80u);
    amax_bits = max(amax_bits, max(lo, hi));
  }
  if (!finite) {
    codes[blk * 2] = make_uint4(0u, 0u, 0u, 0u);
    codes[blk * 2 + 1] = make_uint4(0u, 0u, 0u, 0u);
    scales[blk] = 255;
    return;
  }
  int X = -127;
  if (amax_bits != 0) X = floor_log2_bf16(amax_bits) - 8;  // at most 119 (finite bf16)
  X = X < -127 ? -127 : X;
  const float p = pow2_neg(X);
  uint32_t out[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    // elements 4q .. 4q+3 (words 2q, 2q+1)
    const float a0 = __fmul_rn(bf16_lo(w[2 * q]), p), a1 = __fmul_rn(bf16_hi(w[2 * q]), p);
    const float a2 = __fmul_rn(bf16_lo(w[2 * q + 1]), p), a3 = __fmul_rn(bf16_hi(w[2 * q + 1]), p);
    out[q] = e4m3x2(a0, a1) | (e4m3x2(a2, a3) << 16);
  }
  codes[blk * 2] = make_uint4(out[0], out[1], out[2], out[3]);
  codes[blk * 2 + 1] = make_uint4(out[4], out[5], out[6], out[7]);
  scales[blk] = (uint8_t)(X + 127);
}

}  // namespace

cudaError_t launch_mxfp8_quantize(const void* x, int64_t nblocks, uint8_t* codes, uint8_t* scales,
                                  cudaStream_t stream) {
  if (nblocks == 0) return cudaSuccess;
  const unsigned grid = (unsigned)ceil_div(nblocks, 256);
  mxfp8_quantize_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4*>(x), nblocks,
                                                  reinterpret_cast<uint4*>(codes), scales);
  return cudaGetLastError();
}

cudaError_t launch_mxfp4_quantize(const void* x, int64_t nblocks, int mode, uint8_t* codes, uint8_t* scales,
                                  cudaStream_t stream) {
  if (nblocks == 0) return cudaSuccess;
  const unsigned grid = (unsigned)ceil_div(nblocks, 256);
  mxfp4_quantize_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4*>(x), nblocks, mode,
                                                  reinterpret_cast<uint4*>(codes), scales);
  return cudaGetLastError();
}

}  // namespace csa
