// compress.cuh - the gated pooling of one block of m rows, shared by the prefill
// compression kernel and the decode append (so that an entry appended during
// decode is bit for bit the entry a prefill would have written).
//
// blog.nickys.cn/?p=150, "1. CSA": every m tokens' key/value entries become one
// entry.  Gate rule: for channel c of a block of rows p = 0..m-1,
//   a_p = exp(Z[p,c] + B[p,c]) / sum_p' exp(Z[p',c] + B[p',c]),
//   Kc[c] = sum_p a_p K[p,c],  Vc[c] = sum_p a_p V[p,c].
//
// Thread layout of one block: (d/4) * S threads, thread r = s*(d/4) + cg owns
// channels 4cg..4cg+3 (one 8-byte load per row and array, so a warp reads a
// whole 256-byte row) of the slice of L consecutive rows s*L .. s*L+L-1.  A
// slice is pooled in chunks of up to four rows: all of a chunk's loads are
// issued first, then the chunk's maximum logit per channel (a rescale of the
// running sums only when it grows), then one exp per element.  The S slices
// merge pairwise in a fixed tree through shared memory.  Every arithmetic
// step is an explicit IEEE operation (no contraction left to the compiler),
// so all callers produce the same bits for a block.
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kPoolChan = 4;          // channels per thread
constexpr int kPoolChunk = 4;         // rows per chunk of loads
constexpr int kPoolMaxThreads = 512;   // threads of one block's group
constexpr int kGateWords = 4 * kPoolChan;

// Online-softmax state of 4 channels: running max, denominator, two sums.
struct Gate4 {
  float mx[kPoolChan], den[kPoolChan], k[kPoolChan], v[kPoolChan];
};

__device__ __forceinline__ float& gate_word(Gate4& st, int w) {
  return w < 4 ? st.mx[w] : (w < 8 ? st.den[w - 4] : (w < 12 ? st.k[w - 8] : st.v[w - 12]));
}

__device__ __forceinline__ void bf16x4(const uint2 u, float (&f)[4]) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
}

// Merge b into a (both normalised to their own running max).
__device__ __forceinline__ void gate_merge(Gate4& a, const Gate4& b) {
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    const float m = fmaxf(a.mx[e], b.mx[e]);
    if (m == -INFINITY) continue;
    const float sa = expf(__fsub_rn(a.mx[e], m)), sb = expf(__fsub_rn(b.mx[e], m));
    a.den[e] = __fadd_rn(__fmul_rn(a.den[e], sa), __fmul_rn(b.den[e], sb));
    a.k[e] = __fadd_rn(__fmul_rn(a.k[e], sa), __fmul_rn(b.k[e], sb));
    a.v[e] = __fadd_rn(__fmul_rn(a.v[e], sa), __fmul_rn(b.v[e], sb));
    a.mx[e] = m;
  }
}

// Pools rows s*L .. s*L+L-1 of a block (rows at K/V/Z + p*d, bias row p at
// Bias + p*d), channels c0..c0+3.  With kSeparateLast the block's last row
// (p = m-1) is read from (Klast, Vlast, Zlast): a caller that has not stored it
// yet passes it separately.
template <bool kSeparateLast>
__device__ __forceinline__ void pool_slice(Gate4& st, const __nv_bfloat16* __restrict__ K,
                                           const __nv_bfloat16* __restrict__ V, const __nv_bfloat16* __restrict__ Z,
                                           const __nv_bfloat16* __restrict__ Klast,
                                           const __nv_bfloat16* __restrict__ Vlast,
                                           const __nv_bfloat16* __restrict__ Zlast, const float* __restrict__ Bias,
                                           int d, int m, int L, int s, int c0) {
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) st.mx[e] = -INFINITY, st.den[e] = st.k[e] = st.v[e] = 0.f;
  const int p_end = s * L + L;
#pragma unroll 1
  for (int p0 = s * L; p0 < p_end; p0 += kPoolChunk) {
    uint2 zr[kPoolChunk], kr[kPoolChunk], vr[kPoolChunk];
#pragma unroll
    for (int i = 0; i < kPoolChunk; ++i) {
      const int p = p0 + i;
      if (p < p_end) {
        const int64_t off = (int64_t)p * d + c0;
        const bool last = kSeparateLast && p == m - 1;
        zr[i] = __ldg(reinterpret_cast<const uint2*>(last ? Zlast + c0 : Z + off));
        kr[i] = __ldg(reinterpret_cast<const uint2*>(last ? Klast + c0 : K + off));
        vr[i] = __ldg(reinterpret_cast<const uint2*>(last ? Vlast + c0 : V + off));
      }
    }
    // the chunk's maximum logit per channel (the bias rows are shared by every
    // block: cache hits, read where used to keep the registers for the rows)
    float cm[kPoolChan] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < kPoolChunk; ++i) {
      if (p0 + i < p_end) {
        const float4 bb = __ldg(reinterpret_cast<const float4*>(Bias + (int64_t)(p0 + i) * d + c0));
        float z[4];
        bf16x4(zr[i], z);
        cm[0] = fmaxf(cm[0], __fadd_rn(z[0], bb.x));
        cm[1] = fmaxf(cm[1], __fadd_rn(z[1], bb.y));
        cm[2] = fmaxf(cm[2], __fadd_rn(z[2], bb.z));
        cm[3] = fmaxf(cm[3], __fadd_rn(z[3], bb.w));
      }
    }
#pragma unroll
    for (int e = 0; e < kPoolChan; ++e) {
      if (cm[e] > st.mx[e]) {  // rescale the running sums to the new maximum
        const float sc = expf(__fsub_rn(st.mx[e], cm[e]));
        st.den[e] = __fmul_rn(st.den[e], sc);
        st.k[e] = __fmul_rn(st.k[e], sc);
        st.v[e] = __fmul_rn(st.v[e], sc);
        st.mx[e] = cm[e];
      }
    }
#pragma unroll
    for (int i = 0; i < kPoolChunk; ++i) {
      if (p0 + i < p_end) {
        const float4 bb = __ldg(reinterpret_cast<const float4*>(Bias + (int64_t)(p0 + i) * d + c0));
        const float b[4] = {bb.x, bb.y, bb.z, bb.w};
        float z[4], kf[4], vf[4];
        bf16x4(zr[i], z);
        bf16x4(kr[i], kf);
        bf16x4(vr[i], vf);
#pragma unroll
        for (int e = 0; e < kPoolChan; ++e) {
          const float w = expf(__fsub_rn(__fadd_rn(z[e], b[e]), st.mx[e]));
          st.den[e] = __fadd_rn(st.den[e], w);
          st.k[e] = __fmaf_rn(w, kf[e], st.k[e]);
          st.v[e] = __fmaf_rn(w, vf[e], st.v[e]);
        }
      }
    }
  }
}

// Pairwise tree over the S slices of a block: at step 2^q slice s (s mod 2^(q+1)
// = 2^q) publishes its state and slice s - 2^q merges it; slice 0 ends with the
// block's state.  sh holds kGateWords floats per thread of the CTA, word w of
// thread t at sh[w * nthr + t] (consecutive threads, consecutive banks).  Every
// thread of the CTA calls this (CTA barriers); threads outside a group pass
// in_group = false.  A slot is read only in the step it is written, so one
// barrier per step suffices; a caller that calls this again with the same sh
// puts a CTA barrier in between.
__device__ __forceinline__ void gate_tree(Gate4& st, float* sh, int nthr, int tid, int s, int CG, int S,
                                          bool in_group) {
  for (int step = 1; step < S; step <<= 1) {
    const int pos = s & (2 * step - 1);
    if (in_group && pos == step) {
#pragma unroll
      for (int w = 0; w < kGateWords; ++w) sh[w * nthr + tid] = gate_word(st, w);
    }
    __syncthreads();
    if (in_group && pos == 0 && s + step < S) {
      Gate4 o;
      const int src = tid + step * CG;
#pragma unroll
      for (int w = 0; w < kGateWords; ++w) gate_word(o, w) = sh[w * nthr + src];
      gate_merge(st, o);
    }
  }
}

// Normalise and write 4 channels of Kc/Vc (round to nearest even).
__device__ __forceinline__ void gate_store(const Gate4& st, __nv_bfloat16* __restrict__ Kc,
                                           __nv_bfloat16* __restrict__ Vc) {
  float kf[4], vf[4];
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    const float inv = __fdiv_rn(1.0f, st.den[e]);
    kf[e] = __fmul_rn(st.k[e], inv);
    vf[e] = __fmul_rn(st.v[e], inv);
  }
  *reinterpret_cast<uint2*>(Kc) = make_uint2(pack_bf16x2(kf[0], kf[1]), pack_bf16x2(kf[2], kf[3]));
  *reinterpret_cast<uint2*>(Vc) = make_uint2(pack_bf16x2(vf[0], vf[1]), pack_bf16x2(vf[2], vf[3]));
}

// Gated pooling of one block by its group of (d/4)*S threads (r = this
// thread's index in the group, tid its index in the CTA, nthr the CTA's
// threads); kSeparateLast as for pool_slice (the same bits either way).  Every thread of the CTA must call this when S > 1; threads
// outside a group pass in_group = false, inactive groups active = false.
template <bool kSeparateLast>
__device__ __forceinline__ void pool_block(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                                           const __nv_bfloat16* __restrict__ Z, const __nv_bfloat16* __restrict__ Klast,
                                           const __nv_bfloat16* __restrict__ Vlast,
                                           const __nv_bfloat16* __restrict__ Zlast, const float* __restrict__ Bias,
                                           int d, int L, int S, int r, int tid, int nthr, bool in_group, bool active,
                                           float* sh, __nv_bfloat16* __restrict__ Kc, __nv_bfloat16* __restrict__ Vc) {
  const int m = L * S;
  const int CG = d / kPoolChan;
  const int s = r / CG, c0 = (r % CG) * kPoolChan;
  active = active && in_group;
  Gate4 st;
  if (active) {
    pool_slice<kSeparateLast>(st, K, V, Z, Klast, Vlast, Zlast, Bias, d, m, L, s, c0);
  } else {
#pragma unroll
    for (int e = 0; e < kPoolChan; ++e) st.mx[e] = -INFINITY, st.den[e] = st.k[e] = st.v[e] = 0.f;
  }
  if (S > 1) gate_tree(st, sh, nthr, tid, s, CG, S, in_group);
  if (active && s == 0) gate_store(st, Kc + c0, Vc + c0);
}

// Rows per thread L and slices S = m / L of one block: L = m up to 8 rows, else
// 4 (one chunk of loads per thread), doubled while the group would exceed 512
// threads.
__host__ __device__ inline void pool_shape(int d, int m, int* L, int* S) {
  int l = m <= 8 ? m : 4;
  while ((d / kPoolChan) * (m / l) > kPoolMaxThreads) l *= 2;
  *L = l;
  *S = m / l;
}

}  // namespace csa
