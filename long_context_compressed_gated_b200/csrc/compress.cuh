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
// channels 4cg..4cg+3 of the slice of L consecutive rows s*L .. s*L+L-1 (a
// warp covers whole 256-byte rows).  A slice is pooled in chunks of up to four
// rows: the chunk's base-2 logits g2 = (z + b) * log2(e) and their maximum per
// channel first (the running sums are rescaled only when it grows), then one
// exp2 per element, w = exp2(g2 - max) (exp2f: 2 ulp).  The S slices merge
// pairwise in a fixed tree through shared memory.  Every arithmetic step is an
// explicit IEEE operation (no contraction left to the compiler), so all
// callers produce the same bits for a block.
//
// Row sources: a CTA whose slices have at most kPoolStageRows rows first copies
// all of its rows into shared memory with 16-byte cp.async (every load of the
// CTA in flight at once, no registers held) and pools from there; longer
// slices load each chunk's rows from global memory into registers.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int kPoolChan = 4;           // channels per thread
constexpr int kPoolChunk = 4;          // rows per chunk
constexpr int kPoolMaxThreads = 512;   // threads of one block's group
constexpr int kGateWords = 4 * kPoolChan;
constexpr float kPoolLog2e = 1.44269504088896341f;  // log2(e), rounded to fp32
constexpr int kPoolStageRows = 8;      // slices of at most this many rows are staged
// rows of K, V, Z a CTA stages: 512 threads x 8 rows x 4 channels = 16384
// elements per array, 96 KB
constexpr int kPoolMaxSmem = 3 * kPoolMaxThreads * kPoolStageRows * kPoolChan * 2;

// Online-softmax state of 4 channels: running max (of base-2 logits),
// denominator, two sums.
struct Gate4 {
  float mx[kPoolChan], den[kPoolChan], k[kPoolChan], v[kPoolChan];
};

__device__ __forceinline__ float& gate_word(Gate4& st, int w) {
  return w < 4 ? st.mx[w] : (w < 8 ? st.den[w - 4] : (w < 12 ? st.k[w - 8] : st.v[w - 12]));
}

__device__ __forceinline__ void gate_init(Gate4& st) {
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) st.mx[e] = -INFINITY, st.den[e] = st.k[e] = st.v[e] = 0.f;
}

// Merge b into a (both normalised to their own running max).
__device__ __forceinline__ void gate_merge(Gate4& a, const Gate4& b) {
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    const float m = fmaxf(a.mx[e], b.mx[e]);
    if (m == -INFINITY) continue;
    const float sa = exp2f(__fsub_rn(a.mx[e], m)), sb = exp2f(__fsub_rn(b.mx[e], m));
    a.den[e] = __fadd_rn(__fmul_rn(a.den[e], sa), __fmul_rn(b.den[e], sb));
    a.k[e] = __fadd_rn(__fmul_rn(a.k[e], sa), __fmul_rn(b.k[e], sb));
    a.v[e] = __fadd_rn(__fmul_rn(a.v[e], sa), __fmul_rn(b.v[e], sb));
    a.mx[e] = m;
  }
}

// The arithmetic of one row, shared by both row sources: base-2 logits and the
// chunk maximum; the rescale of the running sums when the maximum grows; the
// weight exp2(g2 - max) accumulated into the denominator and the two sums.
__device__ __forceinline__ void gate_logits(const uint2 zr, const float4 bb, float (&g2)[kPoolChan],
                                            float (&cm)[kPoolChan]) {
  const float z[4] = {bf16_lo(zr.x), bf16_hi(zr.x), bf16_lo(zr.y), bf16_hi(zr.y)};
  const float b[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    g2[e] = __fmul_rn(__fadd_rn(z[e], b[e]), kPoolLog2e);
    cm[e] = fmaxf(cm[e], g2[e]);
  }
}
__device__ __forceinline__ void gate_rescale(Gate4& st, const float (&cm)[kPoolChan]) {
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    if (cm[e] > st.mx[e]) {
      const float sc = exp2f(__fsub_rn(st.mx[e], cm[e]));
      st.den[e] = __fmul_rn(st.den[e], sc);
      st.k[e] = __fmul_rn(st.k[e], sc);
      st.v[e] = __fmul_rn(st.v[e], sc);
      st.mx[e] = cm[e];
    }
  }
}
__device__ __forceinline__ void gate_accum(Gate4& st, const float (&g2)[kPoolChan], const uint2 kr, const uint2 vr) {
  const float kf[4] = {bf16_lo(kr.x), bf16_hi(kr.x), bf16_lo(kr.y), bf16_hi(kr.y)};
  const float vf[4] = {bf16_lo(vr.x), bf16_hi(vr.x), bf16_lo(vr.y), bf16_hi(vr.y)};
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    const float w = exp2f(__fsub_rn(g2[e], st.mx[e]));
    st.den[e] = __fadd_rn(st.den[e], w);
    st.k[e] = __fmaf_rn(w, kf[e], st.k[e]);
    st.v[e] = __fmaf_rn(w, vf[e], st.v[e]);
  }
}

// Copies rows [0, nrows) of Z, K, V (row r at X + r*d, rows contiguous; row
// `last_row` - or none when negative - from Zlast, Klast, Vlast instead) into
// shared memory as [Z, K, V][nrows][d] bf16, by all nthr threads of the CTA with
// 16-byte cp.async (a flat copy of each array), and makes them visible to every
// thread (CTA barrier: all threads call this).
__device__ __forceinline__ void pool_stage_rows(const __nv_bfloat16* __restrict__ K,
                                                const __nv_bfloat16* __restrict__ V,
                                                const __nv_bfloat16* __restrict__ Z,
                                                const __nv_bfloat16* __restrict__ Klast,
                                                const __nv_bfloat16* __restrict__ Vlast,
                                                const __nv_bfloat16* __restrict__ Zlast, int last_row, int nrows,
                                                int d, __nv_bfloat16* sm, int tid, int nthr) {
  const int per = nrows * d / 8;  // 16-byte chunks per array
  const int last_lo = last_row >= 0 ? last_row * d / 8 : per, last_hi = last_lo + d / 8;
#pragma unroll
  for (int arr = 0; arr < 3; ++arr) {
    const __nv_bfloat16* X = arr == 0 ? Z : (arr == 1 ? K : V);
    const __nv_bfloat16* Xl = arr == 0 ? Zlast : (arr == 1 ? Klast : Vlast);
    const uint32_t dst0 = sm100::smem_u32(sm + (size_t)arr * nrows * d);
#pragma unroll 4
    for (int c = tid; c < per; c += nthr) {
      const __nv_bfloat16* src = (c >= last_lo && c < last_hi) ? Xl + (c - last_lo) * 8 : X + (size_t)c * 8;
      sm100::cp_async16(dst0 + (uint32_t)c * 16u, src, 16u);
    }
  }
  sm100::cp_async_wait_all();
  __syncthreads();
}

// Pools rows s*L .. s*L+L-1 of a block, channels c0..c0+3, from global memory:
// rows at K/V/Z + p*d, the block's last row (p = m-1) from (Klast, Vlast,
// Zlast) when kSeparateLast.  Bias row p at Bias + p*d (the same rows for
// every block: cache hits).
template <bool kSeparateLast>
__device__ __forceinline__ void pool_slice_direct(Gate4& st, const __nv_bfloat16* __restrict__ K,
                                                  const __nv_bfloat16* __restrict__ V,
                                                  const __nv_bfloat16* __restrict__ Z,
                                                  const __nv_bfloat16* __restrict__ Klast,
                                                  const __nv_bfloat16* __restrict__ Vlast,
                                                  const __nv_bfloat16* __restrict__ Zlast,
                                                  const float* __restrict__ Bias, int d, int m, int L, int s, int c0) {
  gate_init(st);
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
    float g2[kPoolChunk][kPoolChan];
    float cm[kPoolChan] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < kPoolChunk; ++i)
      if (p0 + i < p_end)
        gate_logits(zr[i], __ldg(reinterpret_cast<const float4*>(Bias + (int64_t)(p0 + i) * d + c0)), g2[i], cm);
    gate_rescale(st, cm);
#pragma unroll
    for (int i = 0; i < kPoolChunk; ++i)
      if (p0 + i < p_end) gate_accum(st, g2[i], kr[i], vr[i]);
  }
}

// The same from rows staged in shared memory: row p of the block's Z at
// rowz + p*d, its K at + plane, its V at + 2*plane.
__device__ __forceinline__ void pool_slice_staged(Gate4& st, const __nv_bfloat16* rowz, size_t plane,
                                                  const float* __restrict__ Bias, int d, int L, int s, int c0) {
  gate_init(st);
  const int p_end = s * L + L;
#pragma unroll 1
  for (int p0 = s * L; p0 < p_end; p0 += kPoolChunk) {
    float g2[kPoolChunk][kPoolChan];
    float cm[kPoolChan] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < kPoolChunk; ++i)
      if (p0 + i < p_end)
        gate_logits(*reinterpret_cast<const uint2*>(rowz + (size_t)(p0 + i) * d + c0),
                    __ldg(reinterpret_cast<const float4*>(Bias + (int64_t)(p0 + i) * d + c0)), g2[i], cm);
    gate_rescale(st, cm);
#pragma unroll
    for (int i = 0; i < kPoolChunk; ++i)
      if (p0 + i < p_end) {
        const __nv_bfloat16* r = rowz + (size_t)(p0 + i) * d + c0;
        gate_accum(st, g2[i], *reinterpret_cast<const uint2*>(r + plane),
                   *reinterpret_cast<const uint2*>(r + 2 * plane));
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

// Rows per thread L and slices S = m / L of one block: L = m up to 8 rows, else
// 4, doubled while the group would exceed 512 threads.
__host__ __device__ inline void pool_shape(int d, int m, int* L, int* S) {
  int l = m <= 8 ? m : 4;
  while ((d / kPoolChan) * (m / l) > kPoolMaxThreads) l *= 2;
  *L = l;
  *S = m / l;
}

// Shared memory of a CTA of nthr threads pooling `blocks` blocks of m rows with
// (L, S): the staged rows (L <= kPoolStageRows) - the merge slots reuse them -
// else the merge slots only.  At most kPoolMaxSmem bytes.
__host__ __device__ inline size_t pool_smem_bytes(int L, int S, int m, int d, int blocks, int nthr) {
  const size_t stage = L <= kPoolStageRows ? (size_t)3 * blocks * m * d * 2 : 0;
  const size_t merge = S > 1 ? (size_t)kGateWords * nthr * 4 : 0;
  return stage > merge ? stage : merge;
}

}  // namespace csa
