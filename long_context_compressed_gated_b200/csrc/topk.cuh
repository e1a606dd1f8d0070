// topk.cuh - block-cooperative selection primitives on unique 64-bit keys.
//
// The indexer's selection rule (k largest scores, ties toward the smaller block
// index j) is a total order once a candidate is encoded as
//     key = (uint64(score_bits ^ 0x80000000) << 32) | (0xFFFFFFFF - j)
// (score as a two's-complement integer in units of 2^-7): a larger key ranks
// higher, keys are unique, and 0 never occurs for a real candidate.
//
// All functions are called by NT threads (thread index `tid` in [0, NT)) that
// synchronise with a named barrier `bar_id`.
#pragma once
#include <cstdint>

namespace csa {
namespace topk {

__device__ __forceinline__ void named_sync(int bar_id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint64_t make_key(int32_t score_units, uint32_t j) {
  return ((uint64_t)((uint32_t)score_units ^ 0x80000000u) << 32) | (uint64_t)(0xFFFFFFFFu - j);
}
__device__ __forceinline__ uint32_t key_index(uint64_t key) { return 0xFFFFFFFFu - (uint32_t)key; }
__device__ __forceinline__ int32_t key_score(uint64_t key) {
  return (int32_t)((uint32_t)(key >> 32) ^ 0x80000000u);
}

// Smallest threshold `thr` such that exactly min(keep, cnt) of buf[0..cnt) satisfy
// key >= thr (radix select, 8-bit digits from the top, early exit as soon as the
// selected digit bucket is taken whole).  hist: 256 ints, sh: 4 ints of shared
// scratch.  Returns 0 when cnt <= keep (everything is kept).
template <int NT>
__device__ uint64_t radix_threshold(const uint64_t* buf, int cnt, int keep, int* hist, int* sh, int tid,
                                    int bar_id) {
  if (cnt <= keep) return 0;
  uint64_t prefix = 0, pmask = 0;
  int need = keep;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    named_sync(bar_id, NT);
    for (int i = tid; i < cnt; i += NT) {
      const uint64_t key = buf[i];
      if ((key & pmask) == prefix) atomicAdd(&hist[(int)(key >> shift) & 255], 1);
    }
    named_sync(bar_id, NT);
    if (tid < 32) {
      // lane l owns digits 255-8l .. 248-8l (descending): exclusive scan across lanes
      int c[8], tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = hist[255 - (tid * 8 + e)];
        tot += c[e];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += v;
      }
      const int excl = incl - tot;
      if (excl < need && need <= incl) {
        int cum = excl;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (cum + c[e] >= need) {
            sh[0] = 255 - (tid * 8 + e);
            sh[1] = cum;
            sh[2] = c[e];
            break;
          }
          cum += c[e];
        }
      }
    }
    named_sync(bar_id, NT);
    const int d = sh[0], cum_gt = sh[1], hd = sh[2];
    named_sync(bar_id, NT);  // everyone has read sh before it is rewritten
    need -= cum_gt;
    prefix |= (uint64_t)d << shift;
    pmask |= (uint64_t)255 << shift;
    if (hd == need) break;
  }
  return prefix;
}

// Keep the keys >= thr of buf[0..cnt) (compacted to the front, any order).
// Returns the new count. MAXPER bounds the keys per thread (cnt <= NT*MAXPER).
template <int NT, int MAXPER>
__device__ int compact_ge(uint64_t* buf, int cnt, uint64_t thr, int* counter, int tid, int bar_id) {
  uint64_t v[MAXPER];
#pragma unroll
  for (int e = 0; e < MAXPER; ++e) {
    const int i = tid + e * NT;
    v[e] = i < cnt ? buf[i] : 0;
  }
  if (tid == 0) *counter = 0;
  named_sync(bar_id, NT);
#pragma unroll
  for (int e = 0; e < MAXPER; ++e) {
    if (v[e] != 0 && v[e] >= thr) {
      const int p = atomicAdd(counter, 1);
      buf[p] = v[e];
    }
  }
  named_sync(bar_id, NT);
  const int n = *counter;
  named_sync(bar_id, NT);
  return n;
}

// Sort buf[0..P) descending (P a power of two; pad with zeros beforehand).
template <int NT>
__device__ void bitonic_desc(uint64_t* buf, int P, int tid, int bar_id) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < (P >> 1); i += NT) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t a = buf[lo], b = buf[hi];
        if ((a < b) == desc) {
          buf[lo] = b;
          buf[hi] = a;
        }
      }
      named_sync(bar_id, NT);
    }
  }
}

__host__ __device__ constexpr int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

}  // namespace topk
}  // namespace csa
