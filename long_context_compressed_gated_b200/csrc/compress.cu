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

namespace csa {

namespace {

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x);
  f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z);
  f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

// Online-softmax state of 8 channels.
struct Gate8 {
  float mx[8], den[8], k[8], v[8];
};

// Merge b into a (both normalised to their own running max).
__device__ __forceinline__ void merge(Gate8& a, const Gate8& b) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float m = fmaxf(a.mx[e], b.mx[e]);
    if (m == -INFINITY) continue;
    const float sa = expf(a.mx[e] - m), sb = expf(b.mx[e] - m);
    a.den[e] = a.den[e] * sa + b.den[e] * sb;
    a.k[e] = a.k[e] * sa + b.k[e] * sb;
    a.v[e] = a.v[e] * sa + b.v[e] * sb;
    a.mx[e] = m;
  }
}

}  // namespace

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
  const int s = r / CG, cg = r % CG;
  const int64_t j = (int64_t)blockIdx.x * bpc + local;
  const bool active = j < nblocks;
  const int c0 = cg * 8;

  Gate8 st;
#pragma unroll
  for (int e = 0; e < 8; ++e) st.mx[e] = -INFINITY, st.den[e] = st.k[e] = st.v[e] = 0.f;

  if (active) {
    for (int p = s * L; p < s * L + L; ++p) {
      const int64_t row = j * m + p;
      float z[8], kk[8], vv[8];
      load8(Z + row * d + c0, z);
      load8(K + row * d + c0, kk);
      load8(V + row * d + c0, vv);
      const float4 b0 = __ldg(reinterpret_cast<const float4*>(Bias + (int64_t)p * d + c0));
      const float4 b1 = __ldg(reinterpret_cast<const float4*>(Bias + (int64_t)p * d + c0 + 4));
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float g = z[e] + b[e];
        if (g > st.mx[e]) {  // rescale the running sums to the new maximum
          const float sc = expf(st.mx[e] - g);
          st.den[e] *= sc;
          st.k[e] *= sc;
          st.v[e] *= sc;
          st.mx[e] = g;
        }
        const float w = expf(g - st.mx[e]);
        st.den[e] += w;
        st.k[e] = fmaf(w, kk[e], st.k[e]);
        st.v[e] = fmaf(w, vv[e], st.v[e]);
      }
    }
  }

  if (S > 1) {
    // slices 1..S-1 publish their state; slice 0 merges in slice order.
    Gate8* sh = reinterpret_cast<Gate8*>(smem_f);
    if (s > 0) sh[threadIdx.x] = st;
    __syncthreads();
    if (s == 0) {
      for (int q = 1; q < S; ++q) merge(st, sh[threadIdx.x + q * CG]);
    }
  }
  if (active && s == 0) {
    uint4 ok, ov;
    float kf[8], vf[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float inv = 1.0f / st.den[e];
      kf[e] = st.k[e] * inv;
      vf[e] = st.v[e] * inv;
    }
    ok.x = pack_bf16x2(kf[0], kf[1]); ok.y = pack_bf16x2(kf[2], kf[3]);
    ok.z = pack_bf16x2(kf[4], kf[5]); ok.w = pack_bf16x2(kf[6], kf[7]);
    ov.x = pack_bf16x2(vf[0], vf[1]); ov.y = pack_bf16x2(vf[2], vf[3]);
    ov.z = pack_bf16x2(vf[4], vf[5]); ov.w = pack_bf16x2(vf[6], vf[7]);
    *reinterpret_cast<uint4*>(Kc + j * d + c0) = ok;
    *reinterpret_cast<uint4*>(Vc + j * d + c0) = ov;
  }
}

// Host launcher (validated arguments).
cudaError_t launch_compress(const void* K, const void* V, const void* Z, const float* B, int64_t T, int d, int m,
                            void* Kc, void* Vc, cudaStream_t stream) {
  const int64_t nblocks = T / m;
  if (nblocks == 0) return cudaSuccess;
  int L = m <= 8 ? m : 8;  // rows per thread; grow until one block fits in 256 threads
  while ((d / 8) * (m / L) > 256) L *= 2;
  const int S = m / L;
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
