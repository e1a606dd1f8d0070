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
// is needed.  `hist` is a per-warp shared-memory array of kWarpBins ints (16-byte
// aligned).  Every pass over a buffer loads kBatch keys per lane before using
// any of them, so a pass costs about one shared-memory latency per 32*kBatch keys.
constexpr int kWarpBins = 1024;
constexpr int kBatch = 8;

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

// Bitonic sort of one key per lane across the warp, descending by lane.
__device__ __forceinline__ uint64_t warp_sort32_desc(uint64_t x, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t y = __shfl_xor_sync(0xffffffffu, x, stride);
      const bool lower = (lane & stride) == 0;
      const bool desc = (lane & size) == 0;
      x = (lower == desc) ? (x > y ? x : y) : (x < y ? x : y);
    }
  }
  return x;
}

__device__ __forceinline__ void warp_clear_hist(int* hist, int lane) {
#pragma unroll
  for (int b = 4 * lane; b < kWarpBins; b += 128) *reinterpret_cast<int4*>(hist + b) = make_int4(0, 0, 0, 0);
}

// Range of the score field (upper 32 bits) over buf[0..cnt), cnt > 0.
__device__ __forceinline__ void warp_score_range(const uint64_t* buf, int cnt, int lane, uint32_t* lo_out,
                                                 uint32_t* hi_out) {
  uint32_t lo = 0xFFFFFFFFu, hi = 0;
  for (int base = 0; base < cnt; base += 32 * kBatch) {
    uint32_t v[kBatch];
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      const int i = base + 32 * t + lane;
      v[t] = (uint32_t)(buf[i < cnt ? i : 0] >> 32);  // buf[0] is a member: neutral for min and max
    }
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      lo = v[t] < lo ? v[t] : lo;
      hi = v[t] > hi ? v[t] : hi;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  *lo_out = lo;
  *hi_out = hi;
}

// Histogram of bin(key) = ((score - lo) >> shift) over buf[0..cnt) (bins < kWarpBins).
__device__ __forceinline__ void warp_score_hist(const uint64_t* buf, int cnt, uint32_t lo, int shift, int* hist,
                                                int lane) {
  warp_clear_hist(hist, lane);
  __syncwarp();
  for (int base = 0; base < cnt; base += 32 * kBatch) {
    uint32_t v[kBatch];
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      const int i = base + 32 * t + lane;
      v[t] = (uint32_t)(buf[i < cnt ? i : 0] >> 32);
    }
#pragma unroll
    for (int t = 0; t < kBatch; ++t)
      if (base + 32 * t + lane < cnt) atomicAdd(&hist[(v[t] - lo) >> shift], 1);
  }
  __syncwarp();
}

// Order-preserving in-place compaction of buf[0..cnt) to the keys >= thr.
__device__ __forceinline__ int warp_compact_ge(uint64_t* buf, int cnt, uint64_t thr, int lane) {
  int out = 0;
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = 0; base < cnt; base += 32 * kBatch) {
    uint64_t v[kBatch];
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      const int i = base + 32 * t + lane;
      v[t] = i < cnt ? buf[i] : 0;  // 0 is below every threshold of a real key set
    }
    __syncwarp();  // stores below only reach positions already loaded
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      const bool keep = v[t] >= thr && v[t] != 0;
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      if (keep) buf[out + __popc(bal & lt)] = v[t];
      out += __popc(bal);
    }
    __syncwarp();
  }
  return out;
}

// Given a histogram of kWarpBins counts (bin index increasing with the key),
// the highest bin b such that count(bins >= b) >= need, and that count.
__device__ __forceinline__ void warp_hist_cut(const int* hist, int need, int lane, int* bin_out, int* kept_out) {
  constexpr int PER = kWarpBins / 32;  // lane l holds bins [kWarpBins - PER(l+1), kWarpBins - PER l)
  const int lo_bin = kWarpBins - PER * (lane + 1);
  int c[PER];
#pragma unroll
  for (int q = 0; q < PER / 4; ++q) {
    const int4 x = *reinterpret_cast<const int4*>(hist + lo_bin + 4 * q);
    c[4 * q] = x.x;
    c[4 * q + 1] = x.y;
    c[4 * q + 2] = x.z;
    c[4 * q + 3] = x.w;
  }
  int tot = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) tot += c[e];
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
#pragma unroll
    for (int e = PER - 1; e >= 0; --e) {
      cum += c[e];
      if (bin < 0 && cum >= need) {
        bin = lo_bin + e;
        kept = cum;
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
// General fallback of warp_select_threshold (heavy score ties).
__device__ uint64_t warp_exact_threshold(const uint64_t* buf, int cnt, int keep, int* hist, int lane) {
  if (cnt <= keep) return 0;
  uint64_t lo = ~0ull, hi = 0;
  for (int base = 0; base < cnt; base += 32 * kBatch) {
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      const int i = base + 32 * t + lane;
      const uint64_t v = buf[i < cnt ? i : 0];
      lo = v < lo ? v : lo;
      hi = v > hi ? v : hi;
    }
  }
  lo = warp_min_u64(lo);
  hi = warp_max_u64(hi);
  // bits below `top` are undetermined; the prefix above is common to all keys
  int top = 64 - __clzll(lo ^ hi);  // keys unique and cnt >= 2 => top >= 1
  uint64_t prefix = lo & ~((top >= 64) ? ~0ull : ((1ull << top) - 1));
  int need = keep;
  while (top > 0) {
    const int w = top >= 10 ? 10 : top;  // digit width (kWarpBins = 1024 bins)
    const int shift = top - w;
    const uint64_t pmask = (top >= 64) ? 0ull : ~((1ull << top) - 1);
    warp_clear_hist(hist, lane);
    __syncwarp();
    for (int base = 0; base < cnt; base += 32 * kBatch) {
      uint64_t v[kBatch];
#pragma unroll
      for (int t = 0; t < kBatch; ++t) {
        const int i = base + 32 * t + lane;
        v[t] = buf[i < cnt ? i : 0];
      }
#pragma unroll
      for (int t = 0; t < kBatch; ++t)
        if (base + 32 * t + lane < cnt && (v[t] & pmask) == prefix)
          atomicAdd(&hist[(int)((v[t] >> shift) & ((1ull << w) - 1))], 1);
    }
    __syncwarp();
    int bin, kept;
    warp_hist_cut(hist, need, lane, &bin, &kept);
    const int in_bin = hist[bin];
    __syncwarp();
    need -= kept - in_bin;  // keys in higher bins are all kept
    prefix |= (uint64_t)bin << shift;
    top = shift;
    if (in_bin == need) break;  // the whole bin is kept
  }
  return prefix;
}

// Exact threshold (as warp_exact_threshold) in one histogram pass over the
// score range plus, when the boundary bin must be split, one gather of that
// bin's keys (at most 32) and an in-register sort.
__device__ uint64_t warp_select_threshold(const uint64_t* buf, int cnt, int keep, int* hist, int lane) {
  if (cnt <= keep) return 0;
  uint32_t lo, hi;
  warp_score_range(buf, cnt, lane, &lo, &hi);
  if (hi > lo) {
    const int bits = 32 - __clz(hi - lo);
    const int shift = bits > 10 ? bits - 10 : 0;
    warp_score_hist(buf, cnt, lo, shift, hist, lane);
    int bin, kept;
    warp_hist_cut(hist, keep, lane, &bin, &kept);
    const int in_bin = hist[bin];
    const int need = keep - (kept - in_bin);  // 1 <= need <= in_bin
    if (need == in_bin) return (uint64_t)(lo + ((uint32_t)bin << shift)) << 32;
    if (in_bin <= 32) {
      __syncwarp();
      uint64_t* sc = reinterpret_cast<uint64_t*>(hist);  // 32 keys of scratch
      int n = 0;
      for (int base = 0; base < cnt; base += 32 * kBatch) {
        uint64_t v[kBatch];
#pragma unroll
        for (int t = 0; t < kBatch; ++t) {
          const int i = base + 32 * t + lane;
          v[t] = buf[i < cnt ? i : 0];
        }
#pragma unroll
        for (int t = 0; t < kBatch; ++t) {
          const bool in = base + 32 * t + lane < cnt && (int)(((uint32_t)(v[t] >> 32) - lo) >> shift) == bin;
          const uint32_t bal = __ballot_sync(0xffffffffu, in);
          if (in) sc[n + __popc(bal & ((1u << lane) - 1u))] = v[t];
          n += __popc(bal);
        }
      }
      __syncwarp();
      uint64_t x = lane < in_bin ? sc[lane] : 0;
      __syncwarp();
      x = warp_sort32_desc(x, lane);
      return __shfl_sync(0xffffffffu, x, need - 1);
    }
    __syncwarp();
  }
  return warp_exact_threshold(buf, cnt, keep, hist, lane);
}

// Sort buf[0..P) descending (P a power of two, padding zeros), one warp.  Each
// compare-exchange stage loads a batch of pairs per lane before swapping them.
__device__ void warp_bitonic_desc(uint64_t* buf, int P, int lane) {
  if (P <= 32) {
    uint64_t x = lane < P ? buf[lane] : 0;
    __syncwarp();
    x = warp_sort32_desc(x, lane);
    if (lane < P) buf[lane] = x;
    __syncwarp();
    return;
  }
  const int half = P >> 1;
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int base = 0; base < half; base += 32 * kBatch) {
        uint64_t x[kBatch], y[kBatch];
        int lo[kBatch];
#pragma unroll
        for (int t = 0; t < kBatch; ++t) {
          const int i = base + 32 * t + lane;
          const int ii = i < half ? i : 0;
          lo[t] = 2 * ii - (ii & (stride - 1));
          x[t] = buf[lo[t]];
          y[t] = buf[lo[t] + stride];
        }
#pragma unroll
        for (int t = 0; t < kBatch; ++t) {
          const bool desc = (lo[t] & size) == 0;
          if (base + 32 * t + lane < half && (x[t] < y[t]) == desc) {
            buf[lo[t]] = y[t];
            buf[lo[t] + stride] = x[t];
          }
        }
      }
      __syncwarp();
    }
  }
}

// ------------------------------------------------------------------ group-cooperative selection
// NT threads (gt in [0, NT), whole warps) that meet on named barrier `bar` work
// on one buffer.  `hist` is a shared array of kWarpBins ints, `scr` shared ints
// (at least 2 * NT/32 + 8).  All threads get the same results.

// Threshold t such that at least `keep` keys of buf[0..cnt) are >= t.  exact:
// exactly min(keep, cnt) keys.  Approximate (exact = false): all keys of the
// boundary histogram bin are kept, unless that keeps more than `room`.
template <int NT>
__device__ uint64_t group_threshold(const uint64_t* buf, int cnt, int keep, int room, bool exact, int* hist,
                                    int* scr, int gt, int bar, bool span_known = false, uint32_t span_lo = 0,
                                    uint32_t span_hi = 0) {
  constexpr int NW = NT / 32;
  const int warp = gt >> 5, lane = gt & 31;
  if (cnt <= keep) return 0;
  uint64_t* s_thr64 = reinterpret_cast<uint64_t*>(scr + 2 * NW + 4);  // 8-byte aligned slot
  // score range (span_known: each thread brings the range of the scores it wrote)
  uint32_t lo = span_known ? span_lo : 0xFFFFFFFFu, hi = span_known ? span_hi : 0;
  for (int i = gt; i < cnt && !span_known; i += NT) {
    const uint32_t sc = (uint32_t)(buf[i] >> 32);
    lo = sc < lo ? sc : lo;
    hi = sc > hi ? sc : hi;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    scr[warp] = (int)lo;
    scr[NW + warp] = (int)hi;
  }
  named_sync(bar, NT);
  lo = (uint32_t)scr[0];
  hi = (uint32_t)scr[NW];
  for (int w = 1; w < NW; ++w) {
    lo = min(lo, (uint32_t)scr[w]);
    hi = max(hi, (uint32_t)scr[NW + w]);
  }
  const int bits = hi > lo ? 32 - __clz(hi - lo) : 0;
  const int shift = bits > 10 ? bits - 10 : 0;
  named_sync(bar, NT);  // scr reused below
  if (hi > lo) {
    for (int b = gt; b < kWarpBins; b += NT) hist[b] = 0;
    named_sync(bar, NT);
    for (int i = gt; i < cnt; i += NT) atomicAdd(&hist[((uint32_t)(buf[i] >> 32) - lo) >> shift], 1);
    named_sync(bar, NT);
    if (warp == 0) {
      int bin, kept;
      warp_hist_cut(hist, keep, lane, &bin, &kept);
      if (lane == 0) {
        scr[0] = bin;
        scr[1] = kept;
        scr[2] = hist[bin];
      }
    }
    named_sync(bar, NT);
    const int bin = scr[0], kept = scr[1], in_bin = scr[2];
    const uint64_t bin_lo = (uint64_t)(lo + ((uint32_t)bin << shift)) << 32;
    const int need = keep - (kept - in_bin);
    if ((!exact && kept <= room) || need == in_bin) {
      named_sync(bar, NT);
      return bin_lo;
    }
    if (in_bin <= 32) {
      // the boundary bin's keys into shared scratch (the histogram is done with), sorted in registers
      uint64_t* sc = reinterpret_cast<uint64_t*>(hist);
      if (gt == 0) scr[3] = 0;
      named_sync(bar, NT);
      for (int i = gt; i < cnt; i += NT) {
        const uint64_t v = buf[i];
        if ((int)(((uint32_t)(v >> 32) - lo) >> shift) == bin) sc[atomicAdd(&scr[3], 1)] = v;
      }
      named_sync(bar, NT);
      if (warp == 0) {
        uint64_t x = lane < in_bin ? sc[lane] : 0;
        x = warp_sort32_desc(x, lane);
        const uint64_t t = __shfl_sync(0xffffffffu, x, need - 1);
        if (lane == 0) *s_thr64 = t;
      }
      named_sync(bar, NT);
      const uint64_t t = *s_thr64;
      named_sync(bar, NT);
      return t;
    }
  }
  // heavy ties: exact radix select by one warp
  if (warp == 0) {
    const uint64_t t = warp_exact_threshold(buf, cnt, keep, hist, lane);
    if (lane == 0) *s_thr64 = t;
  }
  named_sync(bar, NT);
  const uint64_t t = *s_thr64;
  named_sync(bar, NT);
  return t;
}

// In-place compaction of buf[0..cnt) to the keys >= thr (order not kept).  Rounds
// of U*NT keys: every thread loads its keys of the round before any survivor is
// written, and survivors only land below the round's end, so nothing unread is
// overwritten.  Returns the survivor count.
template <int NT>
__device__ int group_compact_ge(uint64_t* buf, int cnt, uint64_t thr, int* scr, int gt, int bar) {
  constexpr int NW = NT / 32, U = 4;
  const int warp = gt >> 5, lane = gt & 31;
  const uint32_t lt = (1u << lane) - 1u;
  int out = 0;
  for (int base = 0; base < cnt; base += U * NT) {
    uint64_t v[U];
    uint32_t bal[U];
    int mine = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * NT + gt;
      v[u] = i < cnt ? buf[i] : 0;
      bal[u] = __ballot_sync(0xffffffffu, i < cnt && v[u] >= thr);
      mine += __popc(bal[u]);
    }
    if (lane == 0) scr[warp] = mine;
    named_sync(bar, NT);
    int woff = out, total = out;
    for (int w = 0; w < NW; ++w) {
      const int c = scr[w];
      woff += w < warp ? c : 0;
      total += c;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if ((bal[u] >> lane) & 1u) buf[woff + __popc(bal[u] & lt)] = v[u];
      woff += __popc(bal[u]);
    }
    named_sync(bar, NT);
    out = total;
  }
  return out;
}

// The keys of buf[0..cnt) >= thr written to out[0..), in an order fixed by their
// positions; returns how many.  Rounds of U*NT keys: every thread loads its keys
// of the round, a per-warp count places them; the counts are double-buffered by
// round parity, so one barrier per round suffices.  scr: 2*NT/32 ints.
template <int NT>
__device__ int group_emit_ge(const uint64_t* buf, int cnt, uint64_t thr, uint64_t* out, int* scr, int gt, int bar) {
  constexpr int NW = NT / 32, U = 4;
  const int warp = gt >> 5, lane = gt & 31;
  const uint32_t lt = (1u << lane) - 1u;
  int done = 0;
  for (int base = 0, round = 0; base < cnt; base += U * NT, ++round) {
    int* cnts = scr + (round & 1) * NW;
    uint64_t v[U];
    uint32_t bal[U];
    int mine = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * NT + gt;
      v[u] = i < cnt ? buf[i] : 0;
      bal[u] = __ballot_sync(0xffffffffu, i < cnt && v[u] >= thr);
      mine += __popc(bal[u]);
    }
    if (lane == 0) cnts[warp] = mine;
    named_sync(bar, NT);
    int woff = done, total = done;
    for (int w = 0; w < NW; ++w) {
      const int c = cnts[w];
      woff += w < warp ? c : 0;
      total += c;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if ((bal[u] >> lane) & 1u) out[woff + __popc(bal[u] & lt)] = v[u];
      woff += __popc(bal[u]);
    }
    done = total;
  }
  named_sync(bar, NT);  // the counts are read before the caller reuses scr
  return done;
}

// Lane-major register bitonic sort of 32*R keys, descending: element e = lane*R + r
// lives in v[r] of lane `lane`.  Strides below R compare registers of one lane
// (plain ALU), strides of R and more exchange between lanes by shuffles: for
// R = 16, 15 of the 45 stages shuffle.
template <int R>
__device__ __forceinline__ void lm_within_lane(uint64_t (&v)[R], int j, int size, int lane) {
#define CSA_LM_CASE(J)                                                    \
  case J:                                                                 \
    _Pragma("unroll") for (int r = 0; r < R; ++r) {                       \
      if ((r & J) == 0 && (r | J) < R) {                                  \
        const bool desc = ((lane * R + r) & size) == 0;                   \
        const uint64_t x = v[r], y = v[r | J];                            \
        const bool sw = (x < y) == desc;                                  \
        v[r] = sw ? y : x;                                                \
        v[r | J] = sw ? x : y;                                            \
      }                                                                   \
    }                                                                     \
    break;
  switch (j) {
    CSA_LM_CASE(1)
    CSA_LM_CASE(2)
    CSA_LM_CASE(4)
    CSA_LM_CASE(8)
    CSA_LM_CASE(16)
    CSA_LM_CASE(32)
    default: break;
  }
#undef CSA_LM_CASE
}

template <int R>
__device__ __forceinline__ void warp_sort_lm_desc(uint64_t (&v)[R], int lane) {
  constexpr int P = 32 * R;
#pragma unroll 1
  for (int size = 2; size <= P; size <<= 1) {
#pragma unroll 1
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride < R) {
        lm_within_lane<R>(v, stride, size, lane);
      } else {
        const int ls = stride / R;  // lane distance
        const bool lower = (lane & ls) == 0;
        uint64_t y[R];
#pragma unroll
        for (int r = 0; r < R; ++r) y[r] = __shfl_xor_sync(0xffffffffu, v[r], ls);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const bool desc = ((lane * R + r) & size) == 0;
          const bool keep_max = lower == desc;
          v[r] = ((v[r] > y[r]) == keep_max) ? v[r] : y[r];
        }
      }
    }
  }
}

// One stage (size, stride) of a bitonic sort, descending overall, on a warp's
// lane-major chunk of 32*R keys whose first key has index `base` in the whole
// array (the direction of a pair depends on its global index).  stride < 32*R.
template <int R>
__device__ __forceinline__ void lm_stage_at(uint64_t (&v)[R], int size, int stride, int base, int lane) {
  if (stride < R) {
    // compile-time register indices per stride (a runtime index would put v in local memory)
#define CSA_LMA_CASE(J)                                          \
  case J:                                                        \
    _Pragma("unroll") for (int r = 0; r < R; ++r) {              \
      if ((r & J) == 0 && (r | J) < R) {                         \
        const bool desc = ((base + lane * R + r) & size) == 0;   \
        const uint64_t x = v[r], y = v[r | J];                   \
        const bool sw = (x < y) == desc;                         \
        v[r] = sw ? y : x;                                       \
        v[r | J] = sw ? x : y;                                   \
      }                                                          \
    }                                                            \
    break;
    switch (stride) {
      CSA_LMA_CASE(1)
      CSA_LMA_CASE(2)
      CSA_LMA_CASE(4)
      CSA_LMA_CASE(8)
      CSA_LMA_CASE(16)
      default: break;
    }
#undef CSA_LMA_CASE
  } else {
    const int ls = stride / R;
    const bool lower = (lane & ls) == 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint64_t y = __shfl_xor_sync(0xffffffffu, v[r], ls);
      const bool desc = ((base + lane * R + r) & size) == 0;
      const bool keep_max = lower == desc;
      v[r] = ((v[r] > y) == keep_max) ? v[r] : y;
    }
  }
}

// Block bitonic sort, descending, of buf[0 .. NT*R) (NT threads, R keys per
// lane).  Each warp sorts its chunk of 32*R keys in registers; every larger
// merge runs its strides of 32*R and more as shared-memory compare-exchanges
// (one barrier each) and its smaller strides in registers again: for 256
// threads x 4 keys that is 10 barriers instead of one per stage (55).
template <int NT, int R>
__device__ void block_sort_desc(uint64_t* buf, int tid) {
  constexpr int C = 32 * R, P = NT * R;
  const int lane = tid & 31, base = (tid >> 5) * C;
  uint64_t v[R];
#pragma unroll
  for (int r = 0; r < R; ++r) v[r] = buf[base + lane * R + r];
#pragma unroll 1
  for (int size = 2; size <= C; size <<= 1)
#pragma unroll 1
    for (int stride = size >> 1; stride > 0; stride >>= 1) lm_stage_at<R>(v, size, stride, base, lane);
#pragma unroll
  for (int r = 0; r < R; ++r) buf[base + lane * R + r] = v[r];
  __syncthreads();
#pragma unroll 1
  for (int size = 2 * C; size <= P; size <<= 1) {
#pragma unroll 1
    for (int stride = size >> 1; stride >= C; stride >>= 1) {
      for (int i = tid; i < P / 2; i += NT) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t a = buf[lo], b = buf[hi];
        if ((a < b) == desc) {
          buf[lo] = b;
          buf[hi] = a;
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < R; ++r) v[r] = buf[base + lane * R + r];
#pragma unroll 1
    for (int stride = C >> 1; stride > 0; stride >>= 1) lm_stage_at<R>(v, size, stride, base, lane);
#pragma unroll
    for (int r = 0; r < R; ++r) buf[base + lane * R + r] = v[r];
    __syncthreads();
  }
}

__host__ __device__ constexpr int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

}  // namespace topk
}  // namespace csa
