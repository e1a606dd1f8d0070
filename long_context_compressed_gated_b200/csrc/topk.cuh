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

// ------------------------------------------------------------------ warp-level selection
// One warp owns one token's candidate buffer in shared memory; only __syncwarp
// is needed.  `hist` is a per-warp shared-memory array of kWarpBins ints.
constexpr int kWarpBins = 1024;

__device__ __forceinline__ uint64_t warp_min_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w < v ? w : v;
  }
  return v;
}
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// Order-preserving in-place compaction of buf[0..cnt) to the keys >= thr.
__device__ __forceinline__ int warp_compact_ge(uint64_t* buf, int cnt, uint64_t thr, int lane) {
  int out = 0;
  for (int base = 0; base < cnt; base += 32) {
    const int i = base + lane;
    const uint64_t v = i < cnt ? buf[i] : 0;
    const bool keep = i < cnt && v >= thr;
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    __syncwarp();
    if (keep) buf[out + __popc(bal & ((1u << lane) - 1u))] = v;
    out += __popc(bal);
    __syncwarp();
  }
  return out;
}

// Given a histogram of kWarpBins counts (bin index increasing with the key),
// the highest bin b such that count(bins >= b) >= need, and that count.
__device__ __forceinline__ void warp_hist_cut(const int* hist, int need, int lane, int* bin_out, int* kept_out) {
  // lane l sums bins [kWarpBins - 32(l+1), kWarpBins - 32l): descending order across lanes
  constexpr int PER = kWarpBins / 32;
  const int hi_bin = kWarpBins - PER * lane;  // exclusive
  int tot = 0;
#pragma unroll 8
  for (int e = 1; e <= PER; ++e) tot += hist[hi_bin - e];
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int excl = incl - tot;
  int bin = -1, kept = 0;
  if (excl < need && need <= incl) {
    int cum = excl;
    for (int e = 1; e <= PER; ++e) {
      cum += hist[hi_bin - e];
      if (cum >= need) {
        bin = hi_bin - e;
        kept = cum;
        break;
      }
    }
  }
  const uint32_t who = __ballot_sync(0xffffffffu, bin >= 0);
  const int src = who ? __ffs(who) - 1 : 0;
  *bin_out = __shfl_sync(0xffffffffu, bin, src);
  *kept_out = __shfl_sync(0xffffffffu, kept, src);
}

// Threshold t such that exactly min(keep, cnt) keys of buf[0..cnt) are >= t:
// radix select over the bits where the keys differ, kWarpBins-ary digits.
__device__ uint64_t warp_exact_threshold(const uint64_t* buf, int cnt, int keep, int* hist, int lane) {
  if (cnt <= keep) return 0;
  uint64_t lo = ~0ull, hi = 0;
  for (int i = lane; i < cnt; i += 32) {
    const uint64_t v = buf[i];
    lo = v < lo ? v : lo;
    hi = v > hi ? v : hi;
  }
  lo = warp_min_u64(lo);
  hi = warp_max_u64(hi);
  // bits below `top` are undetermined; the prefix above is common to all keys
  int top = 64 - __clzll(lo ^ hi);  // number of differing low bits (keys unique => top >= 1)
  uint64_t prefix = lo & ~((top >= 64) ? ~0ull : ((1ull << top) - 1));
  int need = keep;
  while (top > 0) {
    const int w = top >= 10 ? 10 : top;  // digit width (kWarpBins = 1024 bins)
    const int shift = top - w;
    const uint64_t pmask = (top >= 64) ? 0ull : ~((1ull << top) - 1);
    for (int b = lane; b < kWarpBins; b += 32) hist[b] = 0;
    __syncwarp();
    for (int i = lane; i < cnt; i += 32) {
      const uint64_t v = buf[i];
      if ((v & pmask) == prefix) atomicAdd(&hist[(int)((v >> shift) & ((1ull << w) - 1))], 1);
    }
    __syncwarp();
    int bin, kept;
    warp_hist_cut(hist, need, lane, &bin, &kept);
    __syncwarp();
    const int in_bin = hist[bin];
    need -= kept - in_bin;  // keys in higher bins are all kept
    prefix |= (uint64_t)bin << shift;
    top = shift;
    __syncwarp();
    if (in_bin == need) break;  // the whole bin is kept
  }
  return prefix;
}

// One-pass approximate cut: a score threshold keeping at least `keep` keys (all
// keys of the threshold bin are kept).  Returns the number kept through *kept.
// Falls back to the exact threshold when ties would keep more than `room`.
__device__ uint64_t warp_approx_threshold(const uint64_t* buf, int cnt, int keep, int room, int* hist, int lane,
                                          int* kept_out) {
  if (cnt <= keep) {
    *kept_out = cnt;
    return 0;
  }
  uint32_t lo = 0xFFFFFFFFu, hi = 0;
  for (int i = lane; i < cnt; i += 32) {
    const uint32_t sc = (uint32_t)(buf[i] >> 32);
    lo = sc < lo ? sc : lo;
    hi = sc > hi ? sc : hi;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const uint32_t range = hi - lo;
  if (range > 0) {
    const int bits = 32 - __clz(range);
    const int shift = bits > 10 ? bits - 10 : 0;
    for (int b = lane; b < kWarpBins; b += 32) hist[b] = 0;
    __syncwarp();
    for (int i = lane; i < cnt; i += 32) atomicAdd(&hist[((uint32_t)(buf[i] >> 32) - lo) >> shift], 1);
    __syncwarp();
    int bin, kept;
    warp_hist_cut(hist, keep, lane, &bin, &kept);
    __syncwarp();
    if (kept <= room) {
      *kept_out = kept;
      return (uint64_t)(lo + ((uint32_t)bin << shift)) << 32;
    }
  }
  *kept_out = keep;
  return warp_exact_threshold(buf, cnt, keep, hist, lane);
}

// Sort buf[0..P) descending (P a power of two, padding zeros), one warp.
__device__ void warp_bitonic_desc(uint64_t* buf, int P, int lane) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < (P >> 1); i += 32) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t x = buf[lo], y = buf[hi];
        if ((x < y) == desc) {
          buf[lo] = y;
          buf[hi] = x;
        }
      }
      __syncwarp();
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
