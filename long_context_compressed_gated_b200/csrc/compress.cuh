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
// chunks of up to two rows: the chunk's base-2 logits g2 = (z + b) * log2(e)
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
constexpr int kPoolChunk = 2;          // rows per chunk
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

// Online-softmax state of 8 channels as 4 channel pairs: running max (of
// base-2 logits), denominator, two sums.  The element-wise steps run on pairs
// (sm_100's packed fp32 add/mul/fma: per component the same IEEE operation,
// round to nearest even, as the scalar one).
struct Gate {
  float2 mx[4], den[4], k[4], v[4];
};

__device__ __forceinline__ float& pair_at(float2* a, int i) { return (i & 1) ? a[i >> 1].y : a[i >> 1].x; }

__device__ __forceinline__ float& gate_word(Gate& st, int w) {
  return w < 8 ? pair_at(st.mx, w) : (w < 16 ? pair_at(st.den, w - 8) : (w < 24 ? pair_at(st.k, w - 16) : pair_at(st.v, w - 24)));
}

__device__ __forceinline__ void gate_init(Gate& st) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    st.mx[p] = make_float2(-INFINITY, -INFINITY);
    st.den[p] = st.k[p] = st.v[p] = make_float2(0.f, 0.f);
  }
}

// a <- merge(a, b), both normalised to their own running max.  Every operation
// is commutative in (a, b), so merge(a, b) and merge(b, a) are the same bits.
__device__ __forceinline__ void gate_merge(Gate& a, Gate& b) {
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    float &amx = pair_at(a.mx, e), &aden = pair_at(a.den, e), &ak = pair_at(a.k, e), &av = pair_at(a.v, e);
    const float bmx = pair_at(b.mx, e), bden = pair_at(b.den, e), bk = pair_at(b.k, e), bv = pair_at(b.v, e);
    const float m = fmaxf(amx, bmx);
    if (m == -INFINITY) continue;
    const float sa = pool_exp2(__fsub_rn(amx, m)), sb = pool_exp2(__fsub_rn(bmx, m));
    aden = __fadd_rn(__fmul_rn(aden, sa), __fmul_rn(bden, sb));
    ak = __fadd_rn(__fmul_rn(ak, sa), __fmul_rn(bk, sb));
    av = __fadd_rn(__fmul_rn(av, sa), __fmul_rn(bv, sb));
    amx = m;
  }
}

// bf16 pair (low half first) -> two floats, exactly.
__device__ __forceinline__ float2 bf16x2_f2(uint32_t w) { return make_float2(bf16_lo(w), bf16_hi(w)); }

// Base-2 logits of one row (8 channels) and the chunk maximum.
__device__ __forceinline__ void gate_logits(const uint4 zr, const float4 b0, const float4 b1, float2 (&g2)[4],
                                            float2 (&cm)[4]) {
  const float2 z[4] = {bf16x2_f2(zr.x), bf16x2_f2(zr.y), bf16x2_f2(zr.z), bf16x2_f2(zr.w)};
  const float2 b[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                       make_float2(b1.z, b1.w)};
  const float2 l2e = make_float2(kPoolLog2e, kPoolLog2e);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    g2[p] = __fmul2_rn(__fadd2_rn(z[p], b[p]), l2e);
    cm[p].x = fmaxf(cm[p].x, g2[p].x);
    cm[p].y = fmaxf(cm[p].y, g2[p].y);
  }
}

// The running sums follow the chunk maximum when it grows (a multiply by
// exp2 of the rounded difference; by exactly 1 otherwise); nm receives the
// negated running maxima for gate_accum.
__device__ __forceinline__ void gate_rescale(Gate& st, const float2 (&cm)[4], float2 (&nm)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const bool gx = cm[p].x > st.mx[p].x, gy = cm[p].y > st.mx[p].y;
    const float2 sc = make_float2(gx ? pool_exp2(__fsub_rn(st.mx[p].x, cm[p].x)) : 1.0f,
                                  gy ? pool_exp2(__fsub_rn(st.mx[p].y, cm[p].y)) : 1.0f);
    st.den[p] = __fmul2_rn(st.den[p], sc);
    st.k[p] = __fmul2_rn(st.k[p], sc);
    st.v[p] = __fmul2_rn(st.v[p], sc);
    st.mx[p] = make_float2(gx ? cm[p].x : st.mx[p].x, gy ? cm[p].y : st.mx[p].y);
    nm[p] = make_float2(-st.mx[p].x, -st.mx[p].y);
  }
}

// gate_rescale on a state fresh from gate_init (the slice's first chunk): the
// sums are +0 and stay +0 (+0 * exp2(-inf) = +0), so only the maximum moves.
__device__ __forceinline__ void gate_begin(Gate& st, const float2 (&cm)[4], float2 (&nm)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    st.mx[p] = cm[p];
    nm[p] = make_float2(-cm[p].x, -cm[p].y);
  }
}

// One row: w = exp2(g2 - max) (the difference as g2 + (-max): the same
// rounding), den += w, k += w * K, v += w * V.
__device__ __forceinline__ void gate_accum(Gate& st, const float2 (&g2)[4], const float2 (&nm)[4], const uint4 kr,
                                           const uint4 vr) {
  const float2 kf[4] = {bf16x2_f2(kr.x), bf16x2_f2(kr.y), bf16x2_f2(kr.z), bf16x2_f2(kr.w)};
  const float2 vf[4] = {bf16x2_f2(vr.x), bf16x2_f2(vr.y), bf16x2_f2(vr.z), bf16x2_f2(vr.w)};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 dd = __fadd2_rn(g2[p], nm[p]);
    const float2 w = make_float2(pool_exp2(dd.x), pool_exp2(dd.y));
    st.den[p] = __fadd2_rn(st.den[p], w);
    st.k[p] = __ffma2_rn(w, kf[p], st.k[p]);
    st.v[p] = __ffma2_rn(w, vf[p], st.v[p]);
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
__device__ __forceinline__ void gate_store(Gate& st, __nv_bfloat16* __restrict__ Kc, __nv_bfloat16* __restrict__ Vc) {
  float kf[8], vf[8];
#pragma unroll
  for (int e = 0; e < kPoolChan; ++e) {
    const float inv = __fdiv_rn(1.0f, pair_at(st.den, e));
    kf[e] = __fmul_rn(pair_at(st.k, e), inv);
    vf[e] = __fmul_rn(pair_at(st.v, e), inv);
  }
  *reinterpret_cast<uint4*>(Kc) = make_uint4(pack_bf16x2(kf[0], kf[1]), pack_bf16x2(kf[2], kf[3]),
                                             pack_bf16x2(kf[4], kf[5]), pack_bf16x2(kf[6], kf[7]));
  *reinterpret_cast<uint4*>(Vc) = make_uint4(pack_bf16x2(vf[0], vf[1]), pack_bf16x2(vf[2], vf[3]),
                                             pack_bf16x2(vf[4], vf[5]), pack_bf16x2(vf[6], vf[7]));
}

}  // namespace csa
