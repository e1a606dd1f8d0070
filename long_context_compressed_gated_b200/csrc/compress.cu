// compress.cu - KV block compression: softmax-gated per-channel pooling.
//
// blog.nickys.cn/?p=150, "1. CSA": every m tokens' key/value entries become one
// entry.  Gate rule of the specification: for block j, channel c,
//   a_i = exp(Z[i,c] + B[i-j*m, c]) / sum_{i' in block} exp(Z[i',c] + B[i'-j*m, c])
//   Kc[j,c] = sum_i a_i K[i,c],  Vc[j,c] = sum_i a_i V[i,c].
//
// HBM-bound: every input byte is read once with 16-byte vector loads and every
// output byte written once.  One thread owns 8 channels (one 16-byte vector) of
// one block and a slice of L <= 8 consecutive rows, keeping a per-channel online
// softmax (running max, denominator, two weighted sums) in fp32.  When m > 8 the
// S = m/L slices of a block are merged through shared memory in slice order, so
// the result does not depend on scheduling.
#include "common.cuh"
#include "compress.cuh"

namespace csa {

// Thread layout inside one compressed block's group: [slice s][channel group cg];
// blockDim.x = (d/8 * S) * blocks_per_cta.
__global__ void __launch_bounds__(256) compress_kernel(const __nv_bfloat16* __restrict__ K,
                                                       const __nv_bfloat16* __restrict__ V,
                                                       const __nv_bfloat16* __restrict__ Z,
                                                       const float* __restrict__ Bias, int64_t nblocks, int d, int m,
                                                       int L, int S, __nv_bfloat16* __restrict__ Kc,
                                                       __nv_bfloat16* __restrict__ Vc) {
  extern __shared__ __align__(16) float smem_f[];
  const int CG = d / 8;
  const int tpb = CG * S;            // threads per compressed block
  const int bpc = blockDim.x / tpb;  // compressed blocks per CTA
  const int local = threadIdx.x / tpb;
  const int r = threadIdx.x % tpb;
  const int64_t j = (int64_t)blockIdx.x * bpc + local;
  const bool active = j < nblocks;
  const int64_t last = (j * m + m - 1) * d;
  pool_block(K + j * m * d, V + j * m * d, Z + j * m * d, K + last, V + last, Z + last, Bias, d, L, S, r, true, active,
             reinterpret_cast<Gate8*>(smem_f) + local * tpb, Kc + j * d, Vc + j * d);
}

// Host launcher (validated arguments).
cudaError_t launch_compress(const void* K, const void* V, const void* Z, const float* B, int64_t T, int d, int m,
                            void* Kc, void* Vc, cudaStream_t stream) {
  const int64_t nblocks = T / m;
  if (nblocks == 0) return cudaSuccess;
  int L, S;  // rows per thread; grow until one block fits in 256 threads
  pool_shape(d, m, &L, &S);
  const int tpb = (d / 8) * S;
  int bpc = 256 / tpb;
  if (bpc < 1) bpc = 1;
  const int threads = tpb * bpc;
  const size_t smem = S > 1 ? (size_t)threads * sizeof(float) * 32 : 0;
  const int64_t grid = ceil_div(nblocks, bpc);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(compress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  compress_kernel<<<(unsigned)grid, threads, smem, stream>>>(
      static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), static_cast<const __nv_bfloat16*>(Z),
      B, nblocks, d, m, L, S, static_cast<__nv_bfloat16*>(Kc), static_cast<__nv_bfloat16*>(Vc));
  return cudaGetLastError();
}

}  // namespace csa
