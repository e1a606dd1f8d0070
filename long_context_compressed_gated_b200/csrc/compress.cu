// compress.cu - KV block compression: softmax-gated per-channel pooling.
//
// blog.nickys.cn/?p=150, "1. CSA": every m tokens' key/value entries become one
// entry.  Gate rule of the specification: for block j, channel c,
//   a_i = exp(Z[i,c] + B[i-j*m, c]) / sum_{i' in block} exp(Z[i',c] + B[i'-j*m, c])
//   Kc[j,c] = sum_i a_i K[i,c],  Vc[j,c] = sum_i a_i V[i,c].
//
// HBM-bound: every input byte is read once and every output byte written once.
// A group of (d/4)*S threads pools one block (compress.cuh): the CTA first
// copies all rows of its blocks into shared memory with 16-byte cp.async (every
// load in flight at once, no registers held), each thread then pools 4
// channels of a slice of L rows, and the slices merge in a fixed pairwise tree,
// so the result does not depend on scheduling.  A CTA holds 512 threads (one group
// when the group is larger), capped at 64 registers so that two CTAs - 32
// warps, ~100 KB of loads in flight - share an SM (measured on the 131072-token
// HCA compression: 50 us with two CTAs per SM, 63 us with one).
#include "common.cuh"
#include "compress.cuh"

namespace csa {

namespace {

constexpr int kCtaThreads = 512;

// Thread layout: [block of the CTA][slice s][channel group cg]; blockDim.x =
// tpb * blocks_per_cta.  Shared memory: pool_smem_bytes (staged rows, then the
// merge slots).
template <bool kStaged>
__global__ void __launch_bounds__(kPoolMaxThreads, 2) compress_kernel(const __nv_bfloat16* __restrict__ K,
                                                                      const __nv_bfloat16* __restrict__ V,
                                                                      const __nv_bfloat16* __restrict__ Z,
                                                                      const float* __restrict__ Bias,
                                                                      int64_t nblocks, int d, int m, int L, int S,
                                                                      __nv_bfloat16* __restrict__ Kc,
                                                                      __nv_bfloat16* __restrict__ Vc) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  const int CG = d / kPoolChan;
  const int tpb = CG * S;            // threads per compressed block
  const int bpc = blockDim.x / tpb;  // compressed blocks per CTA
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int local = tid / tpb, r = tid % tpb;
  const int s = r / CG, c0 = (r % CG) * kPoolChan;
  const int64_t j0 = (int64_t)blockIdx.x * bpc;
  const int64_t j = j0 + local;
  const bool active = j < nblocks;
  Gate4 st;
  if (kStaged) {
    // the CTA's blocks are consecutive rows: one cooperative copy of all of them
    const int nb = (int)(nblocks - j0 < bpc ? nblocks - j0 : bpc);
    const int nrows = nb * m;
    __nv_bfloat16* sm = reinterpret_cast<__nv_bfloat16*>(sm_raw);
    const int64_t base = j0 * m * d;
    pool_stage_rows(K + base, V + base, Z + base, nullptr, nullptr, nullptr, -1, nrows, d, sm, tid, nthr);
    if (active)
      pool_slice_staged(st, sm + (size_t)local * m * d, (size_t)nrows * d, Bias, d, L, s, c0);
    else
      gate_init(st);
    if (S > 1) {
      __syncthreads();  // the merge slots reuse the staged rows
      gate_tree(st, reinterpret_cast<float*>(sm_raw), nthr, tid, s, CG, S, true);
    }
  } else {
    const int64_t base = active ? j * m * d : 0;
    if (active)
      pool_slice_direct<false>(st, K + base, V + base, Z + base, nullptr, nullptr, nullptr, Bias, d, m, L, s, c0);
    else
      gate_init(st);
    if (S > 1) gate_tree(st, reinterpret_cast<float*>(sm_raw), nthr, tid, s, CG, S, true);
  }
  if (active && s == 0) gate_store(st, Kc + j * d + c0, Vc + j * d + c0);
}

}  // namespace

// Host launcher (validated arguments).
cudaError_t launch_compress(const void* K, const void* V, const void* Z, const float* B, int64_t T, int d, int m,
                            void* Kc, void* Vc, cudaStream_t stream) {
  const int64_t nblocks = T / m;
  if (nblocks == 0) return cudaSuccess;
  int L, S;
  pool_shape(d, m, &L, &S);
  const int tpb = (d / kPoolChan) * S;
  int bpc = kCtaThreads / tpb;
  if (bpc < 1) bpc = 1;
  const int threads = tpb * bpc;
  const bool staged = L <= kPoolStageRows;
  const size_t smem = pool_smem_bytes(L, S, m, d, bpc, threads);
  const int64_t grid = ceil_div(nblocks, bpc);
  if (smem > 48 * 1024) {
    static bool attr_set[64] = {};  // opt in to the largest staging area once per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !attr_set[dev]) {
      e = cudaFuncSetAttribute(compress_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPoolMaxSmem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(compress_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPoolMaxSmem);
      if (e != cudaSuccess) return e;
      if (dev < 64) attr_set[dev] = true;
    }
  }
  auto kern = staged ? compress_kernel<true> : compress_kernel<false>;
  kern<<<(unsigned)grid, threads, smem, stream>>>(
      static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), static_cast<const __nv_bfloat16*>(Z),
      B, nblocks, d, m, L, S, static_cast<__nv_bfloat16*>(Kc), static_cast<__nv_bfloat16*>(Vc));
  return cudaGetLastError();
}

}  // namespace csa
