// compress.cuh - the gated pooling of one block of m rows, shared by the prefill
// compression kernel and the decode append (so that an entry appended during
// decode is bit for bit the entry a prefill would have written).
//
// blog.nickys.cn/?p=150, "1. CSA": every m tokens' key/value entries become one
// entry.  Gate rule: for channel c of a block of rows p = 0..m-1,
//   a_p = exp(Z[p,c] + B[p,c]) / sum_p' exp(Z[p',c] + B[p',c]),
//   Kc[c] = sum_p a_p K[p,c],  Vc[c] = sum_p a_p V[p,c].
//
// Thread layout of one block (its "group"): S slices of R = m / S consecutive
// rows times d/8 channel groups; thread t = s*(d/8) + cg owns channels
// 8cg..8cg+7 (one 16-byte piece of a row) of slice s.  A slice is pooled in
// chunks of up to four rows: the chunk's base-2 logits g2 = (z + b) * log2(e)
// and their maximum per channel first, the running sums rescaled when that
// maximum grows, then one exp2 per element, w = exp2(g2 - max) (the SFU's
// ex2.approx.ftz: about 2 ulp; results below 2^-126 flush to zero).
// The slices merge in a fixed order: pairwise by warp shuffles inside a warp,
// then the first warp of the group takes the other warps' states in turn.
// Every arithmetic step is an explicit IEEE operation (no contraction left to
// the compiler) and a pairwise merge is symmetric in its operands, so every
// caller that follows this layout writes the same bits for a block.
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kPoolChan = 8;           // channels per thread: one 16-byte piece of a row
constexpr int kPoolChunk = 4;          // rows per chunk
constexpr int kPoolMaxThreads = 512;   // threads of one block's group at most
constexpr int kGateWords = 4 * kPoolChan;
constexpr float kPoolLog2e = 1.44269504088896341f;  // log2(e), rounded to fp32

// Slices of one block: S = 1 up to 16 rows, else the largest power of two with
// at least 16 rows per slice that divides m into slices of a multiple of 4
// rows and keeps the group of d/8 * S threads within 512 (m = 128: 8 slices of
// 16 rows; m = 512: 32 slices at d = 128).
__host__ __device__ inline int pool_slices(int d, int m) {
  int S = 1;
  while (2 * S <= m / 16 && m % (8 * S) == 0 && 2 * S * (d / kPoolChan) <= kPoolMaxThreads) S *= 2;
  return S;
}

// 2^x on the SFU (ex2.approx.ftz.f32, about 2 ulp; -inf -> +0; results below
// 2^-126 flush to 0: such a weight is below 2^-126 of the largest one of its
// block, whose weight is 1).
__device__ __forceinline__ float pool_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Online-softmax state of 8 channels: running max (of base-2 logits),
// denominator, two sums.
struct Gate {
  float mx[kPoolChan], den[kPoolChan], k[kPoolChan], v[kPoolChan];
};

__device__ __forceinline__ float& gate_word(Gate& st, int w) {
  return w < 8 ? st.mx[w] : (w < 16 ? st.den[w - 8] : (w < 24 ? st.k[w - 16] : st.v[w - 24]));
}

__device__ __forceinline__ void gate_init(Gate& st) {
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) st.mx[e] = -INFINITY, st.den[e] = st.k[e] = st.v[e] = 0.f;
}

// a <- merge(a, b), both normalised to their own running max.  Every operation
// is commutative in (a, b), so merge(a, b) and merge(b, a) are the same bits.
__device__ __forceinline__ void gate_merge(Gate& a, const Gate& b) {
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    const float m = fmaxf(a.mx[e], b.mx[e]);
    if (m == -INFINITY) continue;
    const float sa = pool_exp2(__fsub_rn(a.mx[e], m)), sb = pool_exp2(__fsub_rn(b.mx[e], m));
    a.den[e] = __fadd_rn(__fmul_rn(a.den[e], sa), __fmul_rn(b.den[e], sb));
    a.k[e] = __fadd_rn(__fmul_rn(a.k[e], sa), __fmul_rn(b.k[e], sb));
    a.v[e] = __fadd_rn(__fmul_rn(a.v[e], sa), __fmul_rn(b.v[e], sb));
    a.mx[e] = m;
  }
}

__device__ __forceinline__ void unpack8(const uint4 r, float (&f)[8]) {
  f[0] = bf16_lo(r.x), f[1] = bf16_hi(r.x), f[2] = bf16_lo(r.y), f[3] = bf16_hi(r.y);
  f[4] = bf16_lo(r.z), f[5] = bf16_hi(r.z), f[6] = bf16_lo(r.w), f[7] = bf16_hi(r.w);
}

// Base-2 logits of one row (8 channels) and the chunk maximum.
__device__ __forceinline__ void gate_logits(const uint4 zr, const float4 b0, const float4 b1, float (&g2)[kPoolChan],
                                            float (&cm)[kPoolChan]) {
  float z[8];
  unpack8(zr, z);
  const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    g2[e] = __fmul_rn(__fadd_rn(z[e], b[e]), kPoolLog2e);
    cm[e] = fmaxf(cm[e], g2[e]);
  }
}

// The running sums follow the chunk maximum when it grows (a multiply by
// exp2 of the rounded difference; by exactly 1 otherwise).
__device__ __forceinline__ void gate_rescale(Gate& st, const float (&cm)[kPoolChan]) {
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    const bool grow = cm[e] > st.mx[e];
    const float sc = grow ? pool_exp2(__fsub_rn(st.mx[e], cm[e])) : 1.0f;
    st.den[e] = __fmul_rn(st.den[e], sc);
    st.k[e] = __fmul_rn(st.k[e], sc);
    st.v[e] = __fmul_rn(st.v[e], sc);
    st.mx[e] = grow ? cm[e] : st.mx[e];
  }
}

__device__ __forceinline__ void gate_accum(Gate& st, const float (&g2)[kPoolChan], const uint4 kr, const uint4 vr) {
  float kf[8], vf[8];
  unpack8(kr, kf);
  unpack8(vr, vf);
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    const float w = pool_exp2(__fsub_rn(g2[e], st.mx[e]));
    st.den[e] = __fadd_rn(st.den[e], w);
    st.k[e] = __fmaf_rn(w, kf[e], st.k[e]);
    st.v[e] = __fmaf_rn(w, vf[e], st.v[e]);
  }
}

// Merges the S slice states of a block held by a group of gsize = CG * S
// threads (thread tg = s * CG + cg, group-relative; lane = tg % 32 when the
// group spans whole warps).  Afterwards threads with s == 0 hold the block's
// state for their channels.
//  1. inside a warp: pairs of slices at distance 1, 2, ... (lane masks CG, 2CG
//     .. 16) by shuffles, restricted to the group's lanes when it is smaller
//     than a warp;
//  2. across the nw = gsize/32 warps of a larger group: warps 1..nw-1 publish
//     their state (lanes cg < CG) in the group's `scratch` (gate_scratch_floats:
//     32 * CG floats per publishing warp), and warp 0 merges them in warp
//     order; two barriers `bar_id` of gsize threads (the second keeps the
//     scratch until it is read).
// Every thread of the group calls this with the same arguments.
__device__ __forceinline__ void gate_group_merge(Gate& st, float* scratch, int tg, int CG, int gsize, int bar_id) {
  const int lane = tg & 31;
  const unsigned gmask = gsize >= 32 ? 0xFFFFFFFFu : (((1u << gsize) - 1u) << (lane & ~(gsize - 1)));
  for (int mask = CG; mask < 32 && mask < gsize; mask <<= 1) {
    Gate o;
#pragma unroll
    for (int w = 0; w < kGateWords; ++w) gate_word(o, w) = __shfl_xor_sync(gmask, gate_word(st, w), mask);
    gate_merge(st, o);
  }
  if (gsize > 32) {
    const int wg = tg >> 5, nw = gsize >> 5;
    if (wg > 0 && lane < CG) {
#pragma unroll
      for (int w = 0; w < kGateWords; ++w) scratch[((wg - 1) * kGateWords + w) * CG + lane] = gate_word(st, w);
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(gsize) : "memory");
    if (wg == 0 && lane < CG) {
      for (int i = 1; i < nw; ++i) {
        Gate o;
#pragma unroll
        for (int w = 0; w < kGateWords; ++w) gate_word(o, w) = scratch[((i - 1) * kGateWords + w) * CG + lane];
        gate_merge(st, o);
      }
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(gsize) : "memory");
  }
}

// Scratch floats of gate_group_merge for one group of gsize threads.
__host__ __device__ inline int gate_scratch_floats(int gsize, int CG) {
  return gsize > 32 ? (gsize / 32 - 1) * kGateWords * CG : 0;
}

// Normalise and write 8 channels of Kc/Vc (round to nearest even).
__device__ __forceinline__ void gate_store(const Gate& st, __nv_bfloat16* __restrict__ Kc,
                                           __nv_bfloat16* __restrict__ Vc) {
  float kf[8], vf[8];
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    const float inv = __fdiv_rn(1.0f, st.den[e]);
    kf[e] = __fmul_rn(st.k[e], inv);
    vf[e] = __fmul_rn(st.v[e], inv);
  }
  *reinterpret_cast<uint4*>(Kc) = make_uint4(pack_bf16x2(kf[0], kf[1]), pack_bf16x2(kf[2], kf[3]),
                                             pack_bf16x2(kf[4], kf[5]), pack_bf16x2(kf[6], kf[7]));
  *reinterpret_cast<uint4*>(Vc) = make_uint4(pack_bf16x2(vf[0], vf[1]), pack_bf16x2(vf[2], vf[3]),
                                             pack_bf16x2(vf[4], vf[5]), pack_bf16x2(vf[6], vf[7]));
}

}  // namespace csa
