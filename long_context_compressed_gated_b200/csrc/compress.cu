// compress.cu - KV block compression: softmax-gated per-channel pooling.
//
// blog.nickys.cn/?p=150, "1. CSA": every m tokens' key/value entries become one
// entry.  Gate rule of the specification: for block j, channel c,
//   a_i = exp(Z[i,c] + B[i-j*m, c]) / sum_{i' in block} exp(Z[i',c] + B[i'-j*m, c])
//   Kc[j,c] = sum_i a_i K[i,c],  Vc[j,c] = sum_i a_i V[i,c].
//
// HBM-bound: every input byte is read once and every output byte written once.
// One CTA of 512 threads per SM (384 where 512 threads' staging and the bias
// table do not fit together), persistent.  The CTA's threads form groups of
// d/8 * S threads that each pool one block at a time with the layout of
// compress.cuh (8 channels of a slice of R = m/S rows per thread); block j goes
// to CTA j mod grid, so every SM gets the same number of blocks to within one,
// and a CTA's blocks go to its groups in turn.  Each thread streams its own
// rows: a two-stage ring of 2-row chunks in shared memory filled by 16-byte
// cp.async (three row pieces per row: Z, K, V), the next chunk's copies in
// flight while the current one is pooled, so no barrier of the CTA and no
// register holds a load in flight.  The bias table B [m, d] is copied into
// shared memory once per CTA when it is at most 64 KB (every chunk would
// otherwise wait on an L2 round trip for its rows of B).  A group's slices
// merge when its block's last chunk is pooled (warp shuffles, then the group's
// first warp).
#include "common.cuh"
#include "compress.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kStages = 2;
constexpr int kBiasSmemMax = 64 * 1024;  // bias tables up to this size are staged in shared memory
constexpr int kSmemMax = 232448;         // shared memory of one CTA on sm_100

// staged chunk rows: [stage][row][Z, K, V][thread] x 16 bytes
__host__ __device__ constexpr size_t stage_bytes(int nt) { return (size_t)kStages * kPoolChunk * 3 * nt * 16; }

// Shared memory: the staged rows, then the bias table [m][d] fp32 (kBiasSmem),
// then the merge scratch of the CTA's groups.
template <int NT, bool kBiasSmem>
__global__ void __launch_bounds__(NT, 1) compress_kernel(const __nv_bfloat16* __restrict__ K,
                                                         const __nv_bfloat16* __restrict__ V,
                                                         const __nv_bfloat16* __restrict__ Z,
                                                         const float* __restrict__ Bias, int64_t nblocks, int d, int m,
                                                         int S, __nv_bfloat16* __restrict__ Kc,
                                                         __nv_bfloat16* __restrict__ Vc) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  const int tid = threadIdx.x;
  const int CG = d / kPoolChan, gsize = CG * S, gpc = NT / gsize;
  const int g = tid / gsize, tg = tid % gsize, s = tg / CG, cg = tg % CG;
  const int R = m / S, nch = (R + kPoolChunk - 1) / kPoolChunk;
  float* bias_sm = reinterpret_cast<float*>(sm_raw + stage_bytes(NT));
  const size_t bias_floats = kBiasSmem ? (size_t)m * d : 0;
  if (kBiasSmem) {
    // the bias table, shared by every group of the CTA (all threads, before any leaves)
    for (int i = tid; i < m * d / 4; i += NT)
      reinterpret_cast<float4*>(bias_sm)[i] = __ldg(reinterpret_cast<const float4*>(Bias) + i);
    __syncthreads();
  }
  // blocks of this group: j = blockIdx.x + gridDim.x * (g + gpc * i), i = 0, 1, ...
  const int64_t j0 = blockIdx.x + (int64_t)gridDim.x * g, jstep = (int64_t)gridDim.x * gpc;
  if (g >= gpc || j0 >= nblocks) return;  // whole groups leave together
  const int64_t items = (nblocks - 1 - j0) / jstep + 1;
  const uint32_t stage0 = sm100::smem_u32(sm_raw) + (uint32_t)tid * 16u;
  const uint4* stage_ld = reinterpret_cast<const uint4*>(sm_raw) + tid;
  float* scratch = bias_sm + bias_floats + (size_t)g * gate_scratch_floats(gsize, CG);
  const float* bias_base = (kBiasSmem ? bias_sm : Bias) + (size_t)s * R * d + cg * kPoolChan;
  // the copy stream runs kStages chunks ahead of the pooling: offset of the
  // next chunk's first row piece (the thread's slice of its group's first block
  // to begin with), and the chunk and item it belongs to
  int64_t ioff = j0 * m * d + (int64_t)s * R * d + cg * kPoolChan;
  const int64_t item_skip = jstep * m * d - (int64_t)nch * kPoolChunk * d;
  int64_t ii = 0;
  int ic = 0;
  auto issue = [&](int stg) {
    if (ii < items) {
      const int n = min(kPoolChunk, R - ic * kPoolChunk);
#pragma unroll
      for (int q = 0; q < kPoolChunk; ++q) {
        if (q < n) {
          const uint32_t dst = stage0 + (uint32_t)((stg * kPoolChunk + q) * 3) * (NT * 16u);
          const int64_t off = ioff + (int64_t)q * d;
          sm100::cp_async16(dst, Z + off, 16u);
          sm100::cp_async16(dst + NT * 16u, K + off, 16u);
          sm100::cp_async16(dst + 2u * NT * 16u, V + off, 16u);
        }
      }
      ioff += (int64_t)kPoolChunk * d;
      if (++ic == nch) ic = 0, ++ii, ioff += item_skip;
    }
    sm100::cp_async_commit();  // possibly empty: one group per chunk slot keeps the count uniform
  };
#pragma unroll
  for (int stg = 0; stg < kStages; ++stg) issue(stg);

  int stg = 0;
  for (int64_t i = 0; i < items; ++i) {
    const int64_t j = j0 + jstep * i;
    Gate st;
    gate_init(st);
    for (int c = 0; c < nch; ++c) {
      const int r0 = c * kPoolChunk, n = min(kPoolChunk, R - r0);
      const float* bias = bias_base + (size_t)r0 * d;
      sm100::cp_async_wait<kStages - 1>();
      const uint4* sp = stage_ld + (size_t)stg * kPoolChunk * 3 * NT;
      float2 g2[kPoolChunk][4], nm[4];
      float2 cm[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) cm[p] = make_float2(-INFINITY, -INFINITY);
#pragma unroll
      for (int q = 0; q < kPoolChunk; ++q)
        if (q < n) {
          const float4* br = reinterpret_cast<const float4*>(bias + (size_t)q * d);
          if (kBiasSmem)
            gate_logits(sp[(q * 3) * NT], br[0], br[1], g2[q], cm);
          else
            gate_logits(sp[(q * 3) * NT], __ldg(br), __ldg(br + 1), g2[q], cm);
        }
      if (c == 0)
        gate_begin(st, cm, nm);
      else
        gate_rescale(st, cm, nm);
#pragma unroll
      for (int q = 0; q < kPoolChunk; ++q)
        if (q < n) gate_accum(st, g2[q], nm, sp[(q * 3 + 1) * NT], sp[(q * 3 + 2) * NT]);
      issue(stg);  // this thread's reads of the slot are done: refill it
      stg = stg + 1 == kStages ? 0 : stg + 1;
    }
    gate_group_merge(st, scratch, tg, CG, gsize, 1 + g);
    if (s == 0) gate_store(st, Kc + j * d + cg * kPoolChan, Vc + j * d + cg * kPoolChan);
  }
  sm100::cp_async_wait_all();
}

template <int NT, bool kBiasSmem>
size_t smem_bytes(int d, int m, int gsize) {
  return stage_bytes(NT) + (kBiasSmem ? (size_t)m * d * sizeof(float) : 0) +
         (size_t)(NT / gsize) * gate_scratch_floats(gsize, d / kPoolChan) * sizeof(float);
}

template <int NT, bool kBiasSmem>
cudaError_t launch_t(const void* K, const void* V, const void* Z, const float* B, int64_t nblocks, int d, int m, int S,
                     void* Kc, void* Vc, int sms, int dev, cudaStream_t stream) {
  static bool attr_set[64] = {};  // opt in to the largest shared memory once per device
  if (dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(compress_kernel<NT, kBiasSmem>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemMax);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  const int gsize = (d / kPoolChan) * S, gpc = NT / gsize;
  // enough CTAs that every group has a block, at most one per SM
  const int64_t need = ceil_div(nblocks, (int64_t)gpc);
  const int grid = (int)(need < sms ? need : sms);
  compress_kernel<NT, kBiasSmem><<<grid, NT, smem_bytes<NT, kBiasSmem>(d, m, gsize), stream>>>(
      static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), static_cast<const __nv_bfloat16*>(Z),
      B, nblocks, d, m, S, static_cast<__nv_bfloat16*>(Kc), static_cast<__nv_bfloat16*>(Vc));
  return cudaGetLastError();
}

}  // namespace

// Host launcher (validated arguments).  512 threads per CTA; when the bias
// table fits in shared memory it is staged there, with 384 threads if 512
// threads' rows and the table do not fit together.
cudaError_t launch_compress(const void* K, const void* V, const void* Z, const float* B, int64_t T, int d, int m,
                            void* Kc, void* Vc, cudaStream_t stream) {
  const int64_t nblocks = T / m;
  if (nblocks == 0) return cudaSuccess;
  const int S = pool_slices(d, m);
  const int gsize = (d / kPoolChan) * S;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if ((size_t)m * d * sizeof(float) <= (size_t)kBiasSmemMax) {
    if (smem_bytes<512, true>(d, m, gsize) <= (size_t)kSmemMax)
      return launch_t<512, true>(K, V, Z, B, nblocks, d, m, S, Kc, Vc, sms, dev, stream);
    if (384 % gsize == 0 && smem_bytes<384, true>(d, m, gsize) <= (size_t)kSmemMax)
      return launch_t<384, true>(K, V, Z, B, nblocks, d, m, S, Kc, Vc, sms, dev, stream);
  }
  return launch_t<512, false>(K, V, Z, B, nblocks, d, m, S, Kc, Vc, sms, dev, stream);
}

}  // namespace csa
