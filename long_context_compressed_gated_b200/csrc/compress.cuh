// compress.cuh - the gated pooling of one block of m rows, shared by the prefill
// compression kernel and the decode append (so that an entry appended during
// decode is bit for bit the entry a prefill would have written).
//
// blog.nickys.cn/?p=150, "1. CSA": every m tokens' key/value entries become one
// entry.  Gate rule: for channel c of a block of rows p = 0..m-1,
//   a_p = exp(Z[p,c] + B[p,c]) / sum_p' exp(Z[p',c] + B[p',c]),
//   Kc[c] = sum_p a_p K[p,c],  Vc[c] = sum_p a_p V[p,c].
#pragma once
#include "common.cuh"

namespace csa {

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

// Gated pooling of one block by a group of (d/8)*S threads: thread r = s*(d/8)+cg
// owns channels 8cg..8cg+7 of rows s*L .. s*L+L-1 (rows at K/V/Z + p*d, bias row
// p at Bias + p*d) with an online softmax in fp32; slices s > 0 publish their
// state in sh[r] and slice 0 merges them in slice order (so the result does not
// depend on scheduling) and writes the 8 channels of Kc/Vc (round to nearest
// even).  Every thread of the CTA must call this when S > 1 (a CTA barrier);
// threads outside a group pass in_group = false, inactive groups active = false.
// The block's last row is read from (Klast, Vlast, Zlast), which a caller that
// has not stored it yet passes separately; otherwise it is row m-1 of K/V/Z.
__device__ __forceinline__ void pool_block(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                                           const __nv_bfloat16* __restrict__ Z, const __nv_bfloat16* __restrict__ Klast,
                                           const __nv_bfloat16* __restrict__ Vlast,
                                           const __nv_bfloat16* __restrict__ Zlast, const float* __restrict__ Bias,
                                           int d, int L, int S, int r, bool in_group, bool active, Gate8* sh,
                                           __nv_bfloat16* __restrict__ Kc, __nv_bfloat16* __restrict__ Vc) {
  const int m = L * S;
  const int CG = d / 8;
  const int s = r / CG, cg = r % CG;
  const int c0 = cg * 8;
  active = active && in_group;
  Gate8 st;
#pragma unroll
  for (int e = 0; e < 8; ++e) st.mx[e] = -INFINITY, st.den[e] = st.k[e] = st.v[e] = 0.f;

  if (active) {
    for (int p = s * L; p < s * L + L; ++p) {
      const bool last = p == m - 1;
      const int64_t row = p;
      float z[8], kk[8], vv[8];
      load8((last ? Zlast : Z + row * d) + c0, z);
      load8((last ? Klast : K + row * d) + c0, kk);
      load8((last ? Vlast : V + row * d) + c0, vv);
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
    if (in_group && s > 0) sh[r] = st;
    __syncthreads();
    if (in_group && s == 0) {
      for (int q = 1; q < S; ++q) merge(st, sh[r + q * CG]);
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
    *reinterpret_cast<uint4*>(Kc + c0) = ok;
    *reinterpret_cast<uint4*>(Vc + c0) = ov;
  }
}

// Rows per thread L and slices S = m / L of one block (d/8 * S <= 256 threads).
__host__ __device__ inline void pool_shape(int d, int m, int* L, int* S) {
  int l = m <= 8 ? m : 8;
  while ((d / 8) * (m / l) > 256) l *= 2;
  *L = l;
  *S = m / l;
}

}  // namespace csa
