// attention.cu - CSA sparse + window attention and HCA dense + window attention.
//
// blog.nickys.cn/?p=150, "1. CSA": each query attends only to its k selected
// compressed entries plus a few sliding-window (uncompressed) entries; "2. HCA":
// dense attention over every compressed entry.  Window branch in both: ifanr
// repost (sz-guanghua.com.cn), attention section.  One joint softmax over the
// whole key set (the specification's reading); MQA: all heads share K/V.
//
// One CTA = 128 query rows = GQ = 128/H consecutive tokens x H heads.  The CTA
// walks a list of key tiles (<= 128 keys each, width a multiple of 16):
//   SEG(g)  : up to 128 of token g's selected compressed entries (CSA)
//   HCA(j0) : compressed entries j0 .. j0+127 (HCA)
//   WIN(w0) : raw tokens at positions w0 .. w0+127 (window union of the group)
// and every row sees, per tile, one contiguous range of its columns (its own
// segment / the visible prefix / its window), so masking needs no per-key data.
//
// Per tile: S = Q K^T (tcgen05 kind::f16, M=128, N=width, fp32 in TMEM), online
// softmax, P (bf16) to shared memory, O += P V (tcgen05, V as an MN-major
// operand).  The two halves of a tile's keys (columns 0..63 and 64..127) are
// softmaxed by different warps, each with its own running maximum and fp32 row
// sum, and accumulate into their own output accumulators O_A / O_B in TMEM; the
// halves combine once after the last tile (O = (O_A 2^(mA-m) + O_B 2^(mB-m)) / l),
// so no warp waits for the other half inside the tile loop.  Warp roles:
//   warps 0..7   softmax: two warps per TMEM lane quarter, one per key half;
//   warps 8..11  loaders: 16-byte cp.async gathers of selected rows into
//                128B-swizzled tiles (MXFP8 rows dequantised on the way);
//                contiguous tiles (HCA, window) and Q come in whole 128-row
//                boxes by TMA;
//   warp 12      TMEM allocation and MMA issue.
// K and V have separate double-buffered rings, so S of tile i+2 can start while
// PV of tile i still reads V.
#include <cuda.h>

#include <cuda_fp16.h>

#include "attention.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

namespace {

constexpr int kRows = 128;
constexpr int kTileKeys = 128;
// Selected-entry (SEG) tiles of one CTA are listed in shared memory (4 bytes
// each); dense (HCA) and window tiles are computed from their index, so their
// number is not limited by the list.
constexpr int kMaxSegTiles = 512;
constexpr int kSoftmaxWarps = 8, kLoaderWarps = 4;
constexpr int kLoaderThreads = kLoaderWarps * 32;
constexpr int kMmaWarp = kSoftmaxWarps + kLoaderWarps;
constexpr int kSchedWarp = kMmaWarp + 1;  // builds the next work item's tile list
constexpr int kThreads = (kSchedWarp + 1) * 32;
constexpr int kRoleWarps = kSchedWarp;    // warps that consume work items (all but the scheduler)
constexpr float kRescaleSlack = 8.0f;  // raise the running max only when it grows by > 2^8
constexpr int kSoftmaxBar = 1;         // named barrier of the softmax warps (end of kernel)
// V ring depth (K has 2): 3 when P lives in tensor memory (V of tile i+3 loads
// while PV of tile i runs), 2 when P is staged in shared memory
constexpr int kMaxVStages = 3;

enum TileType : int { kSeg = 0, kHca = 1, kWin = 2 };

struct Tile {
  int type, owner, width, valid;  // valid: keys of the tile that exist (<= width)
  int64_t base;                   // SEG: offset in the token's list; HCA: j0; WIN: w0
};

// A CTA's tile list: nseg listed SEG tiles, then nhca dense tiles of the visible
// prefix (nv_hca entries), then nwin window tiles from position win_lo; the CTA
// works on tiles [first, first + count) of that list.
struct TileList {
  int nseg, nhca, nwin, first, count, pad;
  int64_t nv_hca, win_lo, win_hi;  // win_hi: last window position (inclusive)
};

__device__ __forceinline__ Tile tile_at(const TileList& L, const uint32_t* seg, int i) {
  i += L.first;
  if (i < L.nseg) {
    const uint32_t p = seg[i];
    return Tile{kSeg, (int)(p & 0xFFu), (int)((p >> 16) & 0xFFu), (int)(p >> 24), (int64_t)((p >> 8) & 0xFFu) * kTileKeys};
  }
  i -= L.nseg;
  if (i < L.nhca) {
    const int64_t j0 = (int64_t)i * kTileKeys;
    const int v = (int)(L.nv_hca - j0 < kTileKeys ? L.nv_hca - j0 : kTileKeys);
    return Tile{kHca, 0, (v + 15) & ~15, v, j0};
  }
  i -= L.nhca;
  const int64_t w0 = L.win_lo + (int64_t)i * kTileKeys;
  const int v = (int)(L.win_hi - w0 + 1 < kTileKeys ? L.win_hi - w0 + 1 : kTileKeys);
  return Tile{kWin, 0, (v + 15) & ~15, v, w0};
}

// 2^x with the SFU (ex2.approx, ~2 ulp; -inf -> +0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32x2 add.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long x, y, z;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b.x), "f"(b.y));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(x), "l"(y));
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(z));
  return r;
}

// (a*c - m, b*c - m) with one packed fp32x2 fma.
__device__ __forceinline__ float2 scale_sub2(float a, float b, float c, float m) {
  unsigned long long x, y;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a), "f"(b));
  asm("{\n\t.reg .b64 cc, mm;\n\t"
      "mov.b64 cc, {%2, %2};\n\t"
      "mov.b64 mm, {%3, %3};\n\t"
      "fma.rn.f32x2 %0, %1, cc, mm;\n\t}"
      : "=l"(y)
      : "l"(x), "f"(c), "f"(-m));
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(y));
  return r;
}

// Eight E4M3 codes times the block scale 2^(sbyte-127) as eight bf16 values (exact:
// an E4M3 value has 4 significant bits and the scale is a power of two).
__device__ __forceinline__ uint4 dequant_e4m3x8(uint2 c, uint32_t sbyte) {
  const float s = __uint_as_float(sbyte == 0 ? 0x00400000u : ((sbyte & 0xFFu) << 23));  // 2^(sbyte-127)
  uint32_t r[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint16_t pair = (uint16_t)(((q < 2 ? c.x : c.y) >> (16 * (q & 1))) & 0xFFFFu);
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
    r[q] = pack_bf16x2(f.x * s, f.y * s);
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

}  // namespace

// TMA descriptors of one launch: 128-row boxes (64-column halves, 128B swizzle).
struct alignas(64) AttnMaps {
  CUtensorMap q, kc, vc, kr, vr;
};

// One work item: GQ consecutive query tokens (prefill) or one sequence's share of
// key tiles (decode), with its tile list.  Built by the scheduler warp into one of
// two slots while the other roles still work on the previous item.
struct ItemInfo {
  int64_t row_tok0, t_first, t_last, raw_lo, b;
  TileList tl;
  int ntok, ntiles, valid, split;
};

// P (the bf16 weights of a tile) goes either back into tensor memory, into the
// tile's S columns, and PV reads A from there (TMEM_P: the softmax never waits for
// PV; the S buffer is released by PV), or into a shared-memory tile (the softmax
// waits for the previous PV before writing it; the S buffer is released as soon
// as it has been read).  Measured: the first is faster for dense (HCA) tiles,
// the second for selected-entry (CSA) tiles.
template <int D, bool TMEM_P>
struct AttnSmem {
  static constexpr int kHalf = kRows * 128;                // one 64-column half of a 128-row tile
  static constexpr int kTileBytes = (D / 64) * kHalf;      // 128 rows x D bf16
  static constexpr int kVS = TMEM_P ? 3 : 2;               // V stages
  static constexpr size_t off_q = 0;
  static constexpr size_t off_k = off_q + kTileBytes;      // 2 stages
  static constexpr size_t off_v = off_k + 2 * kTileBytes;  // kVS stages
  static constexpr size_t off_p = off_v + kVS * kTileBytes;  // 128 x 128 bf16 (shared-memory P)
  static constexpr size_t off_info = off_p + (TMEM_P ? 0 : 2 * kHalf);  // [2] ItemInfo
  static constexpr size_t off_tiles = off_info + 2 * 128;  // [2][kMaxSegTiles] SEG tiles, packed
  static constexpr size_t off_bar = off_tiles + 2 * kMaxSegTiles * 4;
  static constexpr size_t off_misc = off_bar + 32 * 8;
  static constexpr size_t off_cnt = off_misc + 256;        // [2][32] selected entries per token
  static constexpr size_t off_red = off_cnt + 2 * 32 * 4;  // [2][2][128][4] (max, sums) of the two halves
  static constexpr size_t off_idx = off_red + 2 * 4096;    // [slots][idx_entries]
  static size_t bytes(int idx_entries, int slots) { return off_idx + (size_t)slots * idx_entries * 4 + 1024; }
};

template <int D, bool WANT_LSE, bool TMEM_P>
__global__ void __launch_bounds__(kThreads, 1) attention_kernel(const __grid_constant__ AttnArgs a,
                                                                const __grid_constant__ AttnMaps maps) {
  using L = AttnSmem<D, TMEM_P>;
  constexpr int kVStages = L::kVS;
  constexpr int KSTEPS_QK = D / 16;
  constexpr int HALVES = D / 64;
  constexpr uint32_t kHalfBytes = kRows * 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_q = smem + L::off_q;
  uint8_t* s_k = smem + L::off_k;
  uint8_t* s_v = smem + L::off_v;
  uint8_t* s_p = smem + L::off_p;
  uint8_t* s_info = smem + L::off_info;  // [2] ItemInfo, 128 bytes apart
  uint32_t* s_seg_all = reinterpret_cast<uint32_t*>(smem + L::off_tiles);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* q_full = bar + 0;
  uint64_t* k_full = bar + 1;     // [2]
  uint64_t* k_empty = bar + 3;    // [2]
  uint64_t* v_full = bar + 5;     // [kVStages] (kMaxVStages reserved)
  uint64_t* v_empty = bar + 8;    // [kVStages]
  uint64_t* s_full = bar + 11;    // [2]
  uint64_t* s_free = bar + 13;    // [2] S buffer (and the P it then holds) consumed by PV
  // [2] P of a tile written, by tile parity: a softmax warp may finish tile i+1
  // before another has finished tile i (nothing makes it wait for PV any more)
  uint64_t* p_full = bar + 15;
  uint64_t* pv_done = bar + 17;
  uint64_t* mma_fin = bar + 18;   // every issued MMA complete (before TMEM is freed)
  uint64_t* q_free = bar + 19;    // the QK products of an item complete: Q may be reloaded
  // the output of an item with tiles read out of TMEM: the next such item's PV may
  // start (an item without tiles leaves TMEM alone and takes no part: its epilogue
  // waits for nothing, so it could otherwise run two phases ahead of the MMA warp)
  uint64_t* o_free = bar + 20;
  uint64_t* list_full = bar + 21;  // [2] an item's description is ready in its slot
  uint64_t* list_free = bar + 23;  // [2] every role is done with the slot
  int* misc = reinterpret_cast<int*>(smem + L::off_misc);  // [1] tmem
  volatile int* s_abort = misc + 48;  // set by the first wait that timed out; every role then stops
  int* s_cnt_all = reinterpret_cast<int*>(smem + L::off_cnt);
  float* s_red_all = reinterpret_cast<float*>(smem + L::off_red);
  int* s_idx_all = reinterpret_cast<int*>(smem + L::off_idx);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int GQ = kRows / H;
  const bool decode = a.pos != nullptr;
  const int slots = a.slots;
  const int idx_entries = a.idx ? GQ * a.k : 0;
  // work items of this CTA: decode one (sequence blockIdx.x, split blockIdx.y);
  // prefill the token groups blockIdx.x, + gridDim.x, ..., heaviest (latest) first
  auto item_of = [&](int n) -> int64_t {
    if (decode) return n == 0 ? (int64_t)blockIdx.x : -1;
    const int64_t r = (int64_t)blockIdx.x + (int64_t)n * gridDim.x;
    return r < a.nitems ? a.nitems - 1 - r : -1;
  };

  // ---- setup: barriers, TMEM
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], kLoaderThreads + 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], TMEM_P ? 1 : kSoftmaxWarps);
      mbar_init(&p_full[i], kSoftmaxWarps);
      mbar_init(&list_full[i], 32);
      mbar_init(&list_free[i], kRoleWarps);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&v_full[i], kLoaderThreads + 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(pv_done, 1);
    mbar_init(mma_fin, 1);
    mbar_init(q_free, 1);
    mbar_init(o_free, kSoftmaxWarps);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(reinterpret_cast<uint32_t*>(&misc[1]), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = (uint32_t)misc[1];
  // Bounded wait that also stops once any role of this CTA has given up.
  auto wait = [&](uint64_t* b_, uint32_t ph) -> bool {
    if (*s_abort) return false;
    if (mbar_wait(b_, ph, a.status, CSA_ERR_DEVICE_TIMEOUT)) return true;
    *s_abort = 1;
    return false;
  };
  // the next item's description (read in place: its slot is not rewritten before
  // every role has released it), or null at the end
  auto next_item = [&](int n) -> const ItemInfo* {
    const int slot = n % slots;
    if (!wait(&list_full[slot], (uint32_t)((n / slots) & 1))) return nullptr;
    const ItemInfo* inf = reinterpret_cast<const ItemInfo*>(s_info + slot * 128);
    return inf->valid ? inf : nullptr;
  };
  auto release_item = [&](int n) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&list_free[n % slots]);
  };
  // TMEM columns: S double buffer, then the two halves' output accumulators
  constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemOA = 256, kTmemOB = 256 + D;

  if (warp == kSchedWarp) {
    // =========================== scheduler: item n's token range, compacted selections, tile list
    // (the positions and selections may come from the kernel before: read once it completed)
    griddep_wait();
    griddep_launch_dependents();
    for (int n = 0;; ++n) {
      const int slot = n % slots;
      const int use = n / slots;
      if (use > 0 && !wait(&list_free[slot], (uint32_t)((use - 1) & 1))) break;
      const int64_t item = item_of(n);
      ItemInfo inf{};
      inf.valid = item >= 0 ? 1 : 0;
      uint32_t* s_seg = s_seg_all + slot * kMaxSegTiles;
      int* s_idx = s_idx_all + (size_t)slot * idx_entries;
      int* s_cnt = s_cnt_all + slot * 32;
      if (item >= 0) {
        // read now, used at the end: the load overlaps the list's construction
        const int status_now = *reinterpret_cast<volatile int*>(a.status);
        inf.b = decode ? item : 0;
        inf.split = decode ? (int)blockIdx.y : 0;
        inf.row_tok0 = decode ? 0 : item * GQ;
        const int64_t T = decode ? 1 : a.T;
        inf.ntok = (int)((T - inf.row_tok0) < GQ ? (T - inf.row_tok0) : GQ);
        const int64_t pos_b = decode ? a.pos_at(inf.b) : 0;
        inf.raw_lo = decode ? pos_b - a.W + 1 : a.raw_lo;  // absolute position of raw row 0
        inf.t_first = decode ? pos_b : a.t0 + inf.row_tok0;
        inf.t_last = decode ? pos_b : a.t0 + inf.row_tok0 + inf.ntok - 1;
        // compact each token's selected list (drop -1 / out-of-range); 32 loads per
        // lane are in flight before any is used (one memory round trip for k <= 1024)
        if (a.idx != nullptr) {
          const int32_t* idx = a.idx + inf.b * (decode ? (int64_t)a.k : 0);
          for (int g = 0; g < inf.ntok; ++g) {
            const int32_t* src = idx + (inf.row_tok0 + g) * a.k;
            int nsel = 0;
            for (int base = 0; base < a.k; base += 1024) {
              int32_t jv[32];
#pragma unroll
              for (int u = 0; u < 32; ++u) {
                const int q = base + 32 * u + lane;
                jv[u] = q < a.k ? __ldg(src + q) : -1;
              }
#pragma unroll
              for (int u = 0; u < 32; ++u) {
                const int64_t jl = (int64_t)jv[u] - a.idx_base;  // row of this (slice of the) cache
                const bool ok = jv[u] >= 0 && jl >= 0 && jl < a.Nc;
                const uint32_t bal = __ballot_sync(0xffffffffu, ok);
                if (ok) s_idx[g * a.k + nsel + __popc(bal & ((1u << lane) - 1u))] = (int)jl;
                nsel += __popc(bal);
              }
            }
            if (lane == 0) s_cnt[g] = nsel;
          }
          __syncwarp();
        }
        if (lane == 0) {
          TileList tl{};
          int nseg = 0;
          if (a.idx != nullptr) {
            // the tokens' selected-entry tiles alternate, so that consecutive tiles (in
            // the two S buffers) keep the softmax warps of both tokens busy
            int nmax = 0;
            for (int g = 0; g < inf.ntok; ++g) nmax = s_cnt[g] > nmax ? s_cnt[g] : nmax;
            for (int off = 0; off < nmax; off += kTileKeys) {
              for (int g = 0; g < inf.ntok && nseg < kMaxSegTiles; ++g) {
                const int nsel = s_cnt[g];
                if (off >= nsel) continue;
                const int v = nsel - off < kTileKeys ? nsel - off : kTileKeys;
                s_seg[nseg++] = (uint32_t)g | ((uint32_t)(off / kTileKeys) << 8) | ((uint32_t)((v + 15) & ~15) << 16) |
                                ((uint32_t)v << 24);
              }
            }
          } else {
            int64_t nv = n_visible(inf.t_last, a.m);
            if (nv > a.Nc) nv = a.Nc;
            tl.nv_hca = nv > 0 ? nv : 0;
            tl.nhca = (int)ceil_div(tl.nv_hca, kTileKeys);
          }
          tl.nseg = nseg;
          if (a.W > 0 && inf.ntok > 0) {
            int64_t w_lo = inf.t_first - a.W + 1;
            if (w_lo < inf.raw_lo) w_lo = inf.raw_lo;
            if (w_lo < 0) w_lo = 0;
            tl.win_lo = w_lo;
            tl.win_hi = inf.t_last;
            tl.nwin = inf.t_last >= w_lo ? (int)ceil_div(inf.t_last - w_lo + 1, kTileKeys) : 0;
          }
          int nt = tl.nseg + tl.nhca + tl.nwin;
          tl.first = 0;
          if (a.nsplit > 1) {
            // this CTA's share of the sequence's tiles
            const int tps = (nt + a.nsplit - 1) / a.nsplit;
            const int first = inf.split * tps;
            int cnt = nt - first;
            if (cnt > tps) cnt = tps;
            if (cnt < 0) cnt = 0;
            tl.first = first < nt ? first : 0;
            nt = cnt;
          }
          // a bounded wait of an earlier CTA (or kernel on this workspace) gave up:
          // skip the work instead of waiting out every deadline again
          if (status_now == CSA_ERR_DEVICE_TIMEOUT) nt = 0;
          tl.count = nt;
          inf.tl = tl;
          inf.ntiles = nt;
        }
      }
      if (lane == 0) *reinterpret_cast<ItemInfo*>(s_info + slot * 128) = inf;
      __syncwarp();
      mbar_arrive(&list_full[slot]);  // every lane: its smem writes are released
      if (item < 0) break;
    }
  } else if (warp >= kSoftmaxWarps && warp < kMmaWarp) {
    // =========================== loaders: Q and contiguous tiles by TMA, selected rows by cp.async
    const int lt = tid - kSoftmaxWarps * 32;                 // 0..127
    // cp.async mapping: thread lt copies 16-byte chunk c of rows r0, r0 + RSTEP, ...; the
    // 128B swizzle term (chunk ^ row%8) is the same for all of them.
    constexpr int CH = D / 8;
    constexpr int RSTEP = kLoaderThreads / CH;
    const int c = lt % CH, r0 = lt / CH;
    const uint32_t dst_lane = (uint32_t)((c >> 3) * kHalfBytes + r0 * 128 + (((c & 7) ^ (r0 & 7)) << 4));
    // TMA loads this thread has armed and not yet seen consumed: [K/V][stage] parity
    int armed[2][kMaxVStages] = {{-1, -1, -1}, {-1, -1, -1}};
    int q_armed = -1;  // parity of the last Q load issued
    bool live = true;
    int gbase = 0;  // tiles of the earlier items (ring stages and phases run on)
    // Q of the first item right away: its rows are known from the item number,
    // so the load overlaps the scheduler's work on the item's tile list
    auto load_q = [&](int n, int64_t item) {
      mbar_arrive_expect_tx(q_full, HALVES * kHalfBytes);
      const int qrow = (int)(decode ? item * H : item * GQ * H);
      for (int hf = 0; hf < HALVES; ++hf) tma_load_2d(s_q + hf * kHalfBytes, &maps.q, q_full, hf * 64, qrow);
      q_armed = n & 1;
    };
    if (lt == 0) {
      const int64_t item0 = item_of(0);
      if (item0 >= 0) {
        prefetch_tmap(&maps.q);
        load_q(0, item0);
      }
    }
    for (int n = 0; live; ++n) {
      const ItemInfo* infp = next_item(n);
      if (infp == nullptr) break;
      const ItemInfo& inf = *infp;
      const int64_t b = inf.b;
      const int64_t kc_base = decode ? b * a.Nc : 0;           // first compressed row of this sequence
      const int64_t raw_base = decode ? b * (int64_t)a.W : 0;  // first raw row of this sequence
      const __nv_bfloat16* Kc = a.Kc + b * a.kc_batch_stride;
      const __nv_bfloat16* Vc = a.Vc + b * a.kc_batch_stride;
      const uint32_t* s_seg = s_seg_all + (n % slots) * kMaxSegTiles;
      const int* s_idx = s_idx_all + (size_t)(n % slots) * idx_entries;
      if (lt == 0 && n > 0) {
        // Q of this item, once the previous item's QK products are complete
        if (!wait(q_free, (uint32_t)((n - 1) & 1))) live = false;
        if (live) load_q(n, decode ? b : inf.row_tok0 / GQ);
      }
      for (int i = 0; i < inf.ntiles && live; ++i) {
        const Tile tl = tile_at(inf.tl, s_seg, i);
        const int gi = gbase + i;
        for (int which = 0; which < 2; ++which) {  // 0: K (2 stages), 1: V (kVStages)
          const int st = which ? gi % kVStages : (gi & 1);
          const uint32_t ph = (uint32_t)((which ? gi / kVStages : gi >> 1) & 1);
          uint64_t* empty = which ? &v_empty[st] : &k_empty[st];
          uint64_t* fullb = which ? &v_full[st] : &k_full[st];
          uint8_t* dst = (which ? s_v : s_k) + (size_t)st * L::kTileBytes;
          if (!wait(empty, ph ^ 1)) {
            live = false;
            break;
          }
          armed[which][st] = -1;  // the stage's previous load was consumed
          if (tl.type == kSeg && a.kc8 != nullptr) {
            // MXFP8 entries: 8 codes + their block scale per thread and row, dequantised
            const int* sel = s_idx + tl.owner * a.k + (int)tl.base;
            const uint8_t* codes = (which ? a.vc8 : a.kc8) + kc_base * D + c * 8;
            const uint8_t* scl = (which ? a.vc8_scales : a.kc8_scales) + kc_base * (D / 32) + c / 4;
            const uint32_t d0 = smem_u32(dst) + dst_lane;
            // eight rows' loads are in flight before any of them is converted
            for (int x0 = r0; x0 < tl.width; x0 += 8 * RSTEP) {
              uint2 cw[8];
              uint32_t sb[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int x = x0 + u * RSTEP;
                cw[u] = make_uint2(0u, 0u);
                sb[u] = 0u;
                if (x < tl.valid) {
                  const int j = sel[x];
                  cw[u] = __ldg(reinterpret_cast<const uint2*>(codes + (int64_t)j * D));
                  sb[u] = __ldg(scl + (int64_t)j * (D / 32));
                }
              }
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int x = x0 + u * RSTEP;
                if (x < tl.width) {
                  const uint4 v = x < tl.valid ? dequant_e4m3x8(cw[u], sb[u]) : make_uint4(0u, 0u, 0u, 0u);
                  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(d0 + (uint32_t)(x - r0) * 128),
                               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                               : "memory");
                }
              }
            }
            fence_proxy_async_smem();  // generic-proxy stores -> tcgen05 (async proxy) reads
            mbar_arrive(fullb);
            if (lt == 0) mbar_arrive(fullb);
          } else if (tl.type == kSeg) {
            const int* sel = s_idx + tl.owner * a.k + (int)tl.base;
            const __nv_bfloat16* src0 = (which ? Vc : Kc) + c * 8;
            const uint32_t d0 = smem_u32(dst) + dst_lane;
            for (int x = r0; x < tl.width; x += RSTEP) {
              const bool ok = x < tl.valid;
              const int j = ok ? sel[x] : 0;
              cp_async16(d0 + (uint32_t)(x - r0) * 128, src0 + (int64_t)j * D, ok ? 16u : 0u);
            }
            cp_async_arrive(fullb);
            if (lt == 0) mbar_arrive(fullb);
          } else {
            if (lt == 0) {
              const CUtensorMap* m = tl.type == kHca ? (which ? &maps.vc : &maps.kc) : (which ? &maps.vr : &maps.kr);
              const int row = (int)(tl.type == kHca ? kc_base + tl.base : raw_base + (tl.base - inf.raw_lo));
              mbar_arrive_expect_tx(fullb, HALVES * kHalfBytes);
              for (int hf = 0; hf < HALVES; ++hf) tma_load_2d(dst + hf * kHalfBytes, m, fullb, hf * 64, row);
              armed[which][st] = (int)ph;
            }
            mbar_arrive(fullb);
          }
        }
      }
      gbase += inf.ntiles;
      release_item(n);
    }
    cp_async_wait_all();
    // after an abort, wait (bounded) for the TMA loads still landing in shared memory
    if (lt == 0) {
      for (int w = 0; w < 2; ++w)
        for (int st = 0; st < (w ? kVStages : 2); ++st)
          if (armed[w][st] >= 0) mbar_wait(w ? &v_full[st] : &k_full[st], (uint32_t)armed[w][st]);
      if (q_armed >= 0) mbar_wait(q_full, (uint32_t)q_armed);
    }
  } else if (warp == kMmaWarp) {
    // =========================== MMA issuer
    const uint32_t sq = smem_u32(s_q), sp = smem_u32(s_p);
    bool live = true;
    int gbase = 0;
    int o_items = 0;  // items with tiles so far (o_free completions to wait for)
    for (int n = 0; live; ++n) {
      const ItemInfo* infp = next_item(n);
      if (infp == nullptr) break;
      const ItemInfo& inf = *infp;
      const uint32_t* s_seg = s_seg_all + (n % slots) * kMaxSegTiles;
      const int ntiles = inf.ntiles;
      if (!wait(q_full, (uint32_t)(n & 1))) break;
      tc_fence_after();
      // S = Q K^T of the item's tile i; after the item's last one, q_free
      auto issue_s = [&](int i) -> bool {
        const int gi = gbase + i;
        const int st = (int)(gi & 1);
        const uint32_t ph = (uint32_t)((gi >> 1) & 1);
        if (!wait(&k_full[st], ph) || !wait(&s_free[st], ph ^ 1)) return false;
        fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tcgen05 (async proxy) reads
        tc_fence_after();
        if (elect_one()) {  // converged-warp issue
          const int width = tile_at(inf.tl, s_seg, i).width;
          const uint32_t sk = smem_u32(s_k + (size_t)st * L::kTileBytes);
          const uint32_t d = tbase + (st ? kTmemS1 : kTmemS0);
#pragma unroll
          for (int kk = 0; kk < KSTEPS_QK; ++kk) {
            const uint32_t off = (uint32_t)((kk >> 2) * kHalfBytes + (kk & 3) * 32);
            mma_bf16_ss(d, make_sdesc(sq + off, 16, 1024, kSwizzle128), make_sdesc(sk + off, 16, 1024, kSwizzle128),
                        idesc_bf16(128, width, 0, 0), kk > 0);
          }
          mma_commit(&s_full[st]);
          mma_commit(&k_empty[st]);
          if (i == ntiles - 1) mma_commit(q_free);
        }
        __syncwarp();
        return true;
      };
      if (ntiles == 0) {
        if (elect_one()) mma_commit(q_free);
        __syncwarp();
      }
      if (live && ntiles > 0) live = issue_s(0);
      if (live && ntiles > 1) live = issue_s(1);
      // the previous item's output must be read out of TMEM before this item's first PV
      if (live && ntiles > 0) {
        if (o_items > 0 && !wait(o_free, (uint32_t)((o_items - 1) & 1))) live = false;
        ++o_items;
      }
      tc_fence_after();
      bool o_written[2] = {false, false};  // O_A / O_B hold data (else the first PV MMA initialises)
      for (int i = 0; i < ntiles && live; ++i) {
        const int gi = gbase + i;
        const int st = (int)(gi & 1), vs = gi % kVStages;
        if (!wait(&p_full[st], (uint32_t)((gi >> 1) & 1)) || !wait(&v_full[vs], (uint32_t)((gi / kVStages) & 1))) {
          live = false;
          break;
        }
        fence_proxy_async_smem();
        tc_fence_after();
        const int width = tile_at(inf.tl, s_seg, i).width;
        if (elect_one()) {
          const uint32_t sv = smem_u32(s_v + (size_t)vs * L::kTileBytes);
          const uint32_t pcol = tbase + (st ? kTmemS1 : kTmemS0);
          for (int ks = 0; ks < width / 16; ++ks) {
            const int hf = ks >> 2;  // key half: 0 -> O_A, 1 -> O_B
            const uint32_t acc = (o_written[hf] || (ks & 3) > 0) ? 1u : 0u;
            const uint64_t vdesc = make_sdesc(sv + ks * 2048, kHalfBytes, 1024, kSwizzle128);
            if constexpr (TMEM_P) {
              // P (bf16 pairs) in the S buffer's columns: key half hf at columns
              // 64*hf .. 64*hf+31 of the buffer
              mma_bf16_ts(tbase + (hf ? kTmemOB : kTmemOA), pcol + (uint32_t)(64 * hf + 8 * (ks & 3)), vdesc,
                          idesc_bf16(128, D, 0, 1), acc);
            } else {
              const uint32_t aoff = (uint32_t)(hf * kHalfBytes + (ks & 3) * 32);
              mma_bf16_ss(tbase + (hf ? kTmemOB : kTmemOA), make_sdesc(sp + aoff, 16, 1024, kSwizzle128), vdesc,
                          idesc_bf16(128, D, 0, 1), acc);
            }
          }
          mma_commit(pv_done);
          mma_commit(&v_empty[vs]);
          if constexpr (TMEM_P) mma_commit(&s_free[st]);  // S buffer and its P consumed
        }
        __syncwarp();
        o_written[0] = true;
        if (width > 64) o_written[1] = true;
        if (i + 2 < ntiles && !issue_s(i + 2)) {
          live = false;
          break;
        }
      }
      gbase += ntiles;
      release_item(n);
    }
    // every MMA this warp issued has completed before TMEM is freed
    if (elect_one()) mma_commit(mma_fin);
    __syncwarp();
    mbar_wait(mma_fin, 0);
  } else {
    // =========================== softmax (warps 0..7): row = TMEM lane, key columns [64*half, +64)
    // Each half keeps its own running maximum, its own fp32 row sum and its own
    // output accumulator (O_A for keys 0..63 of every tile, O_B for 64..127), so
    // the two halves never wait for each other inside the tile loop; they combine
    // once, after the item's last tile.
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const int g = row / H, h = row % H;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float c = a.scale_log2;  // > 0: max of raw logits * c = max of scaled logits
    const int my0 = half * 64;     // first key column of this half
    const uint32_t o_mine = tbase + lane_base + (half ? kTmemOB : kTmemOA);
    bool live = true;
    int gbase = 0;
    for (int n = 0; live; ++n) {
      const ItemInfo* infp = next_item(n);
      if (infp == nullptr) break;
      const ItemInfo& inf = *infp;
      const uint32_t* s_seg = s_seg_all + (n % slots) * kMaxSegTiles;
      const int ntiles = inf.ntiles;
      const int64_t t = g < inf.ntok ? (decode ? inf.t_first : a.t0 + inf.row_tok0 + g) : -1;
      int64_t nvis = n_visible(t, a.m);
      if (nvis > a.Nc) nvis = a.Nc;
      float m_run = -INFINITY;
      // last PV this warp has waited for: a parity wait may be issued only for the
      // barrier's next phase, never again for one it has already seen complete
      int pv_waited = gbase - 1;
      float2 l2 = make_float2(0.f, 0.f);  // running row sum of the bf16 weights (two partial sums)
      float2 u2 = make_float2(0.f, 0.f);  // the same of the unrounded weights (for the log-sum-exp)
      for (int i = 0; i < ntiles; ++i) {
        const int gi = gbase + i;
        const int st = (int)(gi & 1);
        const Tile tl = tile_at(inf.tl, s_seg, i);
        int lo = 0, hi = 0;
        if (t >= 0) {
          if (tl.type == kSeg) {
            if (tl.owner == g) hi = tl.valid;
          } else if (tl.type == kHca) {
            const int64_t e = nvis - tl.base;
            hi = (int)(e < 0 ? 0 : (e > tl.valid ? tl.valid : e));
          } else {
            int64_t l0 = t - a.W + 1 - tl.base, h0 = t - tl.base + 1;
            if (l0 < 0) l0 = 0;
            if (h0 > tl.valid) h0 = tl.valid;
            lo = (int)l0;
            hi = (int)(h0 > l0 ? h0 : l0);
          }
        }
        // this half's part of the visible range
        lo = lo > my0 ? lo : my0;
        hi = hi < my0 + 64 ? hi : my0 + 64;
        const int width = tl.width;
        const bool warp_any = my0 < width && __any_sync(0xffffffffu, hi > lo);
        const bool warp_full = __all_sync(0xffffffffu, lo == my0 && hi == my0 + 64);
        if (!wait(&s_full[st], (uint32_t)((gi >> 1) & 1))) {
          live = false;
          break;
        }
        tc_fence_after();
        const uint32_t scol = tbase + lane_base + (st ? kTmemS1 : kTmemS0) + my0;
        // pass 1: maximum of this half's visible raw logits
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (warp_any) {
#pragma unroll
          for (int b0 = 0; b0 < 64; b0 += 32) {
            if (my0 + b0 < width) {
              uint32_t v[32];
              tmem_ld32p(scol + b0, v);
              tmem_wait_ld();
              if (warp_full) {
#pragma unroll
                for (int e = 0; e < 32; ++e) mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(v[e]));
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                  if (my0 + b0 + e >= lo && my0 + b0 + e < hi) mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(v[e]));
              }
            }
          }
        }
        const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
        const bool raise = mt > m_run + kRescaleSlack || (m_run == -INFINITY && mt > -INFINITY);
        const float m_new = raise ? mt : m_run;
        const float alpha = raise ? exp2f(m_run - m_new) : 1.0f;  // exp2(-inf) = 0 on the first raise
        // pass 2: p = 2^(s*c - m) over this half's 64 columns, packed to bf16 pairs
        uint32_t pk[32];
        float2 ps = make_float2(0.f, 0.f), pu = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 32; ++q) pk[q] = 0u;
        if (warp_any) {
#pragma unroll
          for (int b0 = 0; b0 < 64; b0 += 32) {
            if (my0 + b0 < width) {
              uint32_t v[32];
              tmem_ld32p(scol + b0, v);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                if (my0 + b0 + 16 * q < width) {
#pragma unroll
                  for (int e = 16 * q; e < 16 * q + 16; e += 2) {
                    const float2 z = scale_sub2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]), c, m_new);
                    float p0 = fast_exp2(z.x), p1 = fast_exp2(z.y);
                    if (!warp_full) {
                      const int x = my0 + b0 + e;
                      p0 = (x >= lo && x < hi) ? p0 : 0.f;
                      p1 = (x + 1 >= lo && x + 1 < hi) ? p1 : 0.f;
                    }
                    const uint32_t pw = pack_bf16x2(p0, p1);
                    pk[(b0 + e) / 2] = pw;
                    // the row sum of the same bf16 weights the PV product uses, so that
                    // numerator and denominator see identical P
                    ps = add2(ps, make_float2(bf16_lo(pw), bf16_hi(pw)));
                    if (WANT_LSE) pu = add2(pu, make_float2(p0, p1));
                  }
                }
              }
            }
          }
        }
        if constexpr (!TMEM_P) {
          // S read: its buffer may take the next QK; then PV of the previous tile
          // must have finished (the P tile is free, O stable)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[st]);
          if (i > 0) {
            if (!wait(pv_done, (uint32_t)((gi - 1) & 1))) {
              live = false;
              break;
            }
            pv_waited = gi - 1;
            tc_fence_after();
          }
        }
        if (__any_sync(0xffffffffu, raise && i > 0 && alpha != 1.0f)) {
          // rescale this half's output accumulator (all D columns), once PV of the
          // previous tile has finished with it
          if constexpr (TMEM_P) {
            if (!wait(pv_done, (uint32_t)((gi - 1) & 1))) {
              live = false;
              break;
            }
            pv_waited = gi - 1;
            tc_fence_after();
          }
          const float sc = (raise && i > 0) ? alpha : 1.0f;
#pragma unroll 1
          for (int b0 = 0; b0 < D; b0 += 32) {
            uint32_t v[32];
            tmem_ld32p(o_mine + b0, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * sc);
            tmem_st32p(o_mine + b0, v);
          }
          tmem_wait_st();
        }
        l2 = make_float2(l2.x * alpha + ps.x, l2.y * alpha + ps.y);
        if (WANT_LSE) u2 = make_float2(u2.x * alpha + pu.x, u2.y * alpha + pu.y);
        m_run = m_new;
        if constexpr (TMEM_P) {
          // this half's P row (bf16 pairs) into the first 32 columns of its own S
          // columns, which this warp has read: PV takes A from tensor memory
          if (my0 < width) {
            tmem_st32p(scol, pk);
            tmem_wait_st();
          }
        } else {
          // this half's P row into the shared-memory tile (K-major, 128B swizzle)
          const uint32_t prow = smem_u32(s_p) + (uint32_t)(half * kHalfBytes + row * 128);
          if (my0 < width) {
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              if (my0 + cc * 8 < width) {
                const uint32_t off = (uint32_t)(((cc ^ (row & 7)) << 4));
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + off), "r"(pk[cc * 4]),
                             "r"(pk[cc * 4 + 1]), "r"(pk[cc * 4 + 2]), "r"(pk[cc * 4 + 3])
                             : "memory");
              }
            }
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[st]);
      }
      // epilogue: the two halves' (max, sum) meet once; O = (O_A f_A + O_B f_B) / l
      float* s_red = s_red_all + (n & 1) * (2 * kRows * 4);
      const int64_t b = inf.b;
      // PV of the last tile.  A parity wait must be for the barrier's next phase:
      // a warp that has not waited for PV of the tile before (it may be two PVs
      // behind the last one) waits for that first; one that has already seen it
      // complete must not wait for it again
      bool have_o = ntiles > 0 && live;
      const int last = gbase + ntiles - 1;
      for (int j = pv_waited + 1 > last - 1 ? pv_waited + 1 : last - 1; have_o && j <= last; ++j)
        have_o = wait(pv_done, (uint32_t)(j & 1));
      if (have_o) tc_fence_after();
      const float l_mine = have_o ? l2.x + l2.y : 0.f;
      *reinterpret_cast<float4*>(s_red + 4 * (half * kRows + row)) =
          make_float4(m_run, l_mine, have_o ? u2.x + u2.y : 0.f, 0.f);
      asm volatile("bar.sync %0, %1;" ::"r"(kSoftmaxBar), "r"(kSoftmaxWarps * 32) : "memory");
      const float4 ra = *reinterpret_cast<const float4*>(s_red + 4 * row);
      const float4 rb = *reinterpret_cast<const float4*>(s_red + 4 * (kRows + row));
      const float mA = ra.x, lA = ra.y, mB = rb.x, lB = rb.y;
      const float mm = fmaxf(mA, mB);
      const float fA = lA > 0.f ? exp2f(mA - mm) : 0.f, fB = lB > 0.f ? exp2f(mB - mm) : 0.f;
      const float l_all = lA * fA + lB * fB;
      const float inv = l_all > 0.f ? 1.0f / l_all : 0.f;
      const float wA = fA * inv, wB = fB * inv;
      const bool part = a.nsplit > 1;
      __nv_bfloat16* orow = nullptr;
      float* part_row = nullptr;  // fp32 rows: a split's partial output, or O itself when o_f32
      const int64_t o_off = b * a.o_batch_stride + ((inf.row_tok0 + g) * H + h) * (int64_t)D;
      if (t >= 0 && !part && !a.o_f32) orow = static_cast<__nv_bfloat16*>(a.O) + o_off;
      if (t >= 0 && !part && a.o_f32) part_row = static_cast<float*>(a.O) + o_off;
      if (t >= 0 && part) part_row = a.o_part + ((b * a.nsplit + inf.split) * H + h) * (int64_t)D;
#pragma unroll 1
      for (int b0 = 0; b0 < 64; b0 += 16) {
        if (my0 >= D) break;  // d = 64: half 1 has no output columns
        float o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) o[e] = 0.f;
        if (have_o) {
          uint32_t va[16], vb[16];
          tmem_ld16p(tbase + lane_base + kTmemOA + my0 + b0, va);
          tmem_ld16p(tbase + lane_base + kTmemOB + my0 + b0, vb);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            // an accumulator that never received a key holds no data: weight 0 exactly
            const float x = wA != 0.f ? __uint_as_float(va[e]) * wA : 0.f;
            o[e] = wB != 0.f ? fmaf(__uint_as_float(vb[e]), wB, x) : x;
          }
        }
        if (part_row) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(part_row + my0 + b0 + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        }
        if (orow) {
#pragma unroll
          for (int e = 0; e < 16; e += 8) {
            uint4 ov;
            ov.x = pack_bf16x2(o[e], o[e + 1]);
            ov.y = pack_bf16x2(o[e + 2], o[e + 3]);
            ov.z = pack_bf16x2(o[e + 4], o[e + 5]);
            ov.w = pack_bf16x2(o[e + 6], o[e + 7]);
            *reinterpret_cast<uint4*>(orow + my0 + b0 + e) = ov;
          }
        }
      }
      if (WANT_LSE && half == 0 && t >= 0 && (a.lse || part)) {
        // the log-sum-exp of the unrounded weights
        const float u_all = ra.z * fA + rb.z * fB;
        const float lse = u_all > 0.f ? (mm + log2f(u_all)) * 0.69314718055994531f : -INFINITY;
        if (part) a.lse_part[(b * a.nsplit + inf.split) * H + h] = lse;
        else a.lse[b * (decode ? H : 0) + (inf.row_tok0 + g) * H + h] = lse;
      }
      // O of this item is out of TMEM: the next item's PV may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ntiles > 0) mbar_arrive(o_free);
      gbase += ntiles;
      release_item(n);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------------ host side

size_t attention_smem_bytes(int d, bool tmem_p, int idx_entries, int slots) {
  if (tmem_p)
    return d == 128 ? AttnSmem<128, true>::bytes(idx_entries, slots) : AttnSmem<64, true>::bytes(idx_entries, slots);
  return d == 128 ? AttnSmem<128, false>::bytes(idx_entries, slots) : AttnSmem<64, false>::bytes(idx_entries, slots);
}
static_assert(sizeof(ItemInfo) <= 128, "item slot");

int attention_max_seg_tiles() { return kMaxSegTiles; }

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeFn get_encode_fn();

// bf16 matrix [rows, d] with 128B-swizzled boxes of 64 columns x box_rows rows
static bool bf16_map(CUtensorMap* m, const void* base, int64_t rows, int d, int box_rows) {
  EncodeFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool L, bool TP>
static cudaError_t launch_t(const AttnArgs& a, const AttnMaps& maps, unsigned grid, size_t smem,
                            cudaStream_t stream) {
  cudaError_t e =
      cudaFuncSetAttribute(attention_kernel<D, L, TP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(attention_kernel<D, L, TP>, dim3(grid, a.nsplit > 1 ? a.nsplit : 1), dim3(kThreads), smem,
                       stream, a.pdl != 0, a, maps);
}

template <int D>
static cudaError_t launch_d(const AttnArgs& a, const AttnMaps& maps, unsigned grid, size_t smem, bool lse, bool tp,
                            cudaStream_t stream) {
  if (tp) return lse ? launch_t<D, true, true>(a, maps, grid, smem, stream) : launch_t<D, false, true>(a, maps, grid, smem, stream);
  return lse ? launch_t<D, true, false>(a, maps, grid, smem, stream) : launch_t<D, false, false>(a, maps, grid, smem, stream);
}

// Merge the split partial outputs: one warp per (sequence, head), lane c owning
// dims 4c..4c+3; every partial is loaded before any is combined.
constexpr int kCombineSplits = 16;

// Partial s of sequence b is at row (b * sb + s * ss) of the partials ([B, nsplit]
// order: sb = nsplit, ss = 1; [nsplit, B] order: sb = 1, ss = B).
template <int D>
__global__ void __launch_bounds__(256) attention_combine_kernel(const float* __restrict__ o_part,
                                                                const float* __restrict__ lse_part, int nsplit, int H,
                                                                int64_t rows, void* __restrict__ O, int o_f32,
                                                                int64_t o_batch_stride, float* __restrict__ lse,
                                                                int64_t sb, int64_t ss) {
  griddep_wait();  // the partials come from the attention kernel before
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // (b, h)
  if (w >= rows) return;
  const int64_t b = w / H;
  const int h = (int)(w % H);
  constexpr int V = D / 4;
  float ls[kCombineSplits];
  float mx = -INFINITY;
#pragma unroll
  for (int s = 0; s < kCombineSplits; ++s) {
    ls[s] = s < nsplit ? lse_part[(b * sb + s * ss) * H + h] : -INFINITY;
    mx = fmaxf(mx, ls[s]);
  }
  if (lane >= V) return;
  float4 o[kCombineSplits];
#pragma unroll
  for (int s = 0; s < kCombineSplits; ++s)
    o[s] = (s < nsplit && ls[s] > -INFINITY)
               ? reinterpret_cast<const float4*>(o_part + ((b * sb + s * ss) * H + h) * (int64_t)D)[lane]
               : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float sum = 0.f;
  if (mx > -INFINITY) {
#pragma unroll
    for (int s = 0; s < kCombineSplits; ++s) {
      const float wt = ls[s] > -INFINITY ? __expf(ls[s] - mx) : 0.f;
      acc.x += wt * o[s].x;
      acc.y += wt * o[s].y;
      acc.z += wt * o[s].z;
      acc.w += wt * o[s].w;
      sum += wt;
    }
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  const int64_t off = b * o_batch_stride + (int64_t)h * D + 4 * lane;
  if (o_f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(O) + off) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  } else {
    uint2 packed;
    packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(O) + off) = packed;
  }
  if (lse && lane == 0) lse[b * H + h] = sum > 0.f ? mx + __logf(sum) : -INFINITY;
}

cudaError_t launch_combine(const float* o_part, const float* lse_part, int nsplit, int B, int H, int d, void* O,
                           int o_f32, int64_t o_batch_stride, float* lse, int64_t sb, int64_t ss,
                           cudaStream_t stream, bool pdl) {
  if (nsplit > kCombineSplits) return cudaErrorInvalidConfiguration;
  const int64_t rows = (int64_t)B * H;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (rows == 0) return cudaSuccess;
  auto kern = d == 128 ? attention_combine_kernel<128> : attention_combine_kernel<64>;
  return launch_kernel(kern, dim3(grid), dim3(256), 0, stream, pdl, o_part, lse_part, nsplit, H, rows, O, o_f32,
                       o_batch_stride, lse, sb, ss);
}

cudaError_t launch_attention_combine(const AttnArgs& a, int B, int d, cudaStream_t stream) {
  return launch_combine(a.o_part, a.lse_part, a.nsplit, B, a.H, d, a.O, a.o_f32, a.o_batch_stride, a.lse, a.nsplit, 1,
                        stream, true);
}

int sm_count();

// grid: the number of work items (prefill: token groups; decode: sequences, each
// split over a.nsplit CTAs).  Prefill runs persistent CTAs, one per SM, that
// take the items in turn (heaviest first); the next item's tile list is built
// while the current one runs when two item slots fit in shared memory.
cudaError_t launch_attention(const AttnArgs& a_in, int d, unsigned grid, cudaStream_t stream) {
  AttnArgs a = a_in;
  const int GQ = kRows / a.H;
  const int idx_entries = a.idx ? GQ * a.k : 0;
  const bool tp = a.idx == nullptr;  // P in tensor memory for dense (HCA) tiles
  a.slots = attention_smem_bytes(d, tp, idx_entries, 2) <= 227 * 1024 ? 2 : 1;
  const size_t smem = attention_smem_bytes(d, tp, idx_entries, a.slots);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  a.nitems = grid;
  if (a.pos == nullptr) {
    const unsigned sms = (unsigned)sm_count();
    grid = grid < sms ? grid : sms;
  }
  if (grid == 0) return cudaSuccess;
  AttnMaps maps;
  if (!bf16_map(&maps.q, a.Q, a.q_rows, d, 128) || !bf16_map(&maps.kc, a.Kc, a.kc_rows, d, 128) ||
      !bf16_map(&maps.vc, a.Vc, a.kc_rows, d, 128) || !bf16_map(&maps.kr, a.Kr, a.raw_rows, d, 128) ||
      !bf16_map(&maps.vr, a.Vr, a.raw_rows, d, 128))
    return cudaErrorInvalidValue;
  const bool lse = a.lse != nullptr || a.nsplit > 1;
  if (d == 128) return launch_d<128>(a, maps, grid, smem, lse, tp, stream);
  return launch_d<64>(a, maps, grid, smem, lse, tp, stream);
}

}  // namespace csa
