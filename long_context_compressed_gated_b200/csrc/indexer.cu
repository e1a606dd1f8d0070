// indexer.cu - lightning indexer on MXFP4 fused with the causal top-k.
//
// ifanr repost (sz-guanghua.com.cn), attention section: the indexer scores every
// query token against every compressed block in FP4 and keeps the top-k blocks;
// m.youleyou.com/wenzhang/2906406.html section 1: MXFP4 on the indexer QK path.
// Score of the specification:  I[t,j] = sum_h w[t,h] * ReLU(qI[t,h] . kI[j]),
// visible when j*m + m - 1 <= t, ties toward the smaller j.
//
// Design (one CTA = G query tokens x one range of compressed entries):
//  * tcgen05.mma kind::mxf4 (packed E2M1 x E2M1, UE8M0 scale per 32 elements):
//    A = 128 compressed keys (TMEM lanes), B = the G*HI (token, head) rows of
//    the query group (TMEM columns), K = dI.  A third MMA with constant
//    operands (all 1.0 x all 6.0 * 2^9) adds 196608 = 1.5*2^17 to every
//    accumulator, which pins the fp32 exponent so the raw bit pattern of the
//    accumulator minus that of 196608 is the exact dot product in units of
//    2^-6 (valid while every scale exponent lies in [-2, 1]).
//  * Epilogue (8 warps, two per TMEM lane quarter): per key lane, per token,
//        acc += w2[h] * max(bits, bits(196608))          (int32, exact)
//    then I*2^7 = acc - bits(196608)*sum_h w2[h] (mod 2^32), with w2 = 2*w.
//    Ranking uses the exact integer; no floating-point head sum.
//  * Streaming top-k per token: candidates whose 64-bit key (score, -j) clears
//    the token's running threshold are appended to a shared-memory buffer; when
//    the buffer could overflow on the next tile it is cut back to the k best by
//    radix select, which also raises the threshold.  At the end the k best are
//    bitonic-sorted (score desc, j asc) and written out.
//  * Warp roles: warp 0 TMA producer (key codes) + scale-factor staging, warp 1
//    TMEM allocation and MMA issue (scales copied to TMEM with tcgen05.cp),
//    warps 2..9 epilogue + selection.  Key tiles are 4-stage pipelined;
//    accumulators double-buffered in TMEM.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"
#include "topk.cuh"

namespace csa {

using namespace sm100;

namespace {

constexpr int kMaxCols = 224;       // N of the MMA: G*HI rounded up to 16
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;
constexpr uint32_t kMagicBits = 0x48400000u;  // bit pattern of 196608.0f
constexpr int kCheckWarp = 6;                // epilogue warp that range-checks the key scales
constexpr int kHalfBar0 = 1;                  // named barriers 1, 2: the four warps of each half
constexpr size_t kSmemLimit = 227 * 1024;

// TMEM column map (512 allocated): D[0] at 0, D[1] at 256; scale factors at 224..
constexpr uint32_t kTmemD1 = 256;
constexpr uint32_t kTmemSFA0 = 224;   // 4 columns per buffer (x2)
constexpr uint32_t kTmemSFB = 232;    // 8 columns
constexpr uint32_t kTmemMagicSFA = 240;
constexpr uint32_t kTmemMagicSFB = 244;  // 8 columns

template <int HI>
struct Geometry {
  static constexpr int G = kMaxCols / HI < 8 ? kMaxCols / HI : 8;  // tokens per CTA (prefill)
};

__device__ __forceinline__ int e2m1_times2(uint32_t code) {
  // 2 * E2M1 value as an integer: magnitudes {0,1,2,3,4,6,8,12}
  const uint32_t e = (code >> 1) & 3u, mb = code & 1u;
  const int mag = e == 0 ? (int)mb : (int)((2u + mb) << (e - 1));
  return (code & 8u) ? -mag : mag;
}

}  // namespace

// Head sums of this thread's key lane for the tokens of one half of the group:
// acc[g] += w2[h] * max(bits(D[g*HI+h]), bits(196608)) over the half's columns,
// loading up to 64 TMEM columns per wait.  NP partial sums per token break the
// dependent multiply-add chain when a token has many heads.
template <int HI, int G, int HALF>
__device__ __forceinline__ void head_sums(uint32_t dcol, const int* s_w2, uint32_t (&acc)[G]) {
  constexpr int G0 = (G + 1) / 2;
  constexpr int c_lo = (HALF ? G0 : 0) * HI;
  constexpr int c_hi = (HALF ? G : G0) * HI;
  constexpr int NP = HI >= 32 ? 4 : 1;
  uint32_t part[G][NP];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int p = 0; p < NP; ++p) part[g][p] = 0u;
#pragma unroll
  for (int b0 = c_lo; b0 < c_hi; b0 += 64) {
    uint32_t v[64];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (b0 + 16 * q < c_hi) tmem_ld16p(dcol + b0 + 16 * q, v + 16 * q);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 64; i += 4) {
      if (b0 + i < c_hi) {
        const int4 w = *reinterpret_cast<const int4*>(s_w2 + b0 + i);
        const int ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = b0 + i + q;
          part[col / HI][col % NP] += (uint32_t)ww[q] * (uint32_t)max((int)v[i + q], (int)kMagicBits);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int p = 0; p < NP; ++p) acc[g] += part[g][p];
}

struct IndexerArgs {
  const uint8_t* q_scales;  // [rows, HI, dI/32]
  const uint8_t* w_codes;   // [rows, HI]
  const uint8_t* k_scales;  // [key_rows, dI/32]
  int64_t rows;             // query rows (prefill T, decode B)
  int64_t t0;               // prefill: absolute position of row 0
  const int64_t* pos;       // decode: absolute position per row (device), else null
  int64_t Nc;               // prefill: entries in the cache; decode: Ncap per sequence
  int64_t key_rows;         // rows of the kI tensor (bounds for scale loads)
  int m, k;
  int cap;                  // candidate buffer capacity per token
  int check;                // tiles between buffer cut-backs (cap >= k + 128 * check)
  int nsplit;               // key ranges per query group
  int64_t split_tiles;      // 128-key tiles per range
  int32_t* idx;             // [rows, k]      (nsplit == 1)
  float* scores;            // [rows, k]      (nsplit == 1, nullable)
  uint64_t* cand;           // [rows, nsplit, k] keys (nsplit > 1)
  int* status;
};

template <int HI, int DI, int G>
struct IndexerSmem {
  static constexpr int N = ((G * HI + 15) / 16) * 16;
  static constexpr int kStages = (G == 1) ? 8 : 4;
  static constexpr int kRowBytes = DI / 2;
  static constexpr int kQBytes = ((N * kRowBytes + 1023) / 1024) * 1024;
  static constexpr int kABytes = 128 * kRowBytes;  // multiple of 1024
  static constexpr size_t off_q = 0;
  static constexpr size_t off_a = off_q + kQBytes;
  static constexpr size_t off_sf = off_a + (size_t)kStages * kABytes;  // key scales, tcgen05.cp layout
  static constexpr size_t off_ma = off_sf + (size_t)kStages * 512;
  static constexpr size_t off_mb = off_ma + 4096;
  static constexpr size_t off_w2 = off_mb + (size_t)N * 32;
  static constexpr size_t off_sumw = off_w2 + (size_t)N * 4;
  static constexpr size_t off_cnt = off_sumw + 64 * 4;
  static constexpr size_t off_thr = off_cnt + 64 * 4;
  static constexpr size_t off_hist = off_thr + 64 * 8;               // per epilogue warp, kWarpBins ints
  static constexpr size_t off_sh = off_hist + (size_t)kEpiWarps * topk::kWarpBins * 4;
  static constexpr size_t off_bar = off_sh + 64;
  static constexpr size_t off_tslot = off_bar + (2 * kStages + 5) * 8;
  static constexpr size_t off_cand = ((off_tslot + 16 + 15) / 16) * 16;
  static size_t bytes(int cap) { return off_cand + (size_t)G * cap * 8 + 1024; }
};

// Sort a token's final candidates (cnt <= 32*R) in registers and write idx /
// scores in rank order, padding with -1 / -inf up to k.
template <int R>
__device__ __forceinline__ void write_sorted(const uint64_t* buf, int cnt, const IndexerArgs& a, int64_t r, int lane) {
  uint64_t v[R];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int e = i * 32 + lane;
    v[i] = e < cnt ? buf[e] : 0;
  }
  topk::warp_sort_regs_desc<R>(v, lane);
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int q = i * 32 + lane;
    if (q < a.k) {
      int32_t id = -1;
      float sc = -INFINITY;
      if (q < cnt) {
        id = (int32_t)topk::key_index(v[i]);
        sc = (float)topk::key_score(v[i]) * (1.0f / 128.0f);
      }
      a.idx[r * a.k + q] = id;
      if (a.scores) a.scores[r * a.k + q] = sc;
    }
  }
  // rows beyond 32*R (k > 32*R with cnt <= 32*R) are padding
  for (int q = 32 * R + lane; q < a.k; q += 32) {
    a.idx[r * a.k + q] = -1;
    if (a.scores) a.scores[r * a.k + q] = -INFINITY;
  }
}

template <int HI, int DI, int G>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_topk_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                        const IndexerArgs a) {
  using L = IndexerSmem<HI, DI, G>;
  constexpr int N = L::N;
  constexpr int NST = L::kStages;
  constexpr int KB = DI / 64;  // MMAs of K=64 per tile
  static_assert(N <= kMaxCols, "N too large");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_q = smem + L::off_q;
  uint8_t* s_a = smem + L::off_a;
  uint8_t* s_sf = smem + L::off_sf;
  uint8_t* s_ma = smem + L::off_ma;
  uint8_t* s_mb = smem + L::off_mb;
  int* s_w2 = reinterpret_cast<int*>(smem + L::off_w2);
  int* s_sumw = reinterpret_cast<int*>(smem + L::off_sumw);
  int* s_cnt = reinterpret_cast<int*>(smem + L::off_cnt);
  uint64_t* s_thr = reinterpret_cast<uint64_t*>(smem + L::off_thr);
  int* s_hist = reinterpret_cast<int*>(smem + L::off_hist);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* full = bar;                 // [NST] producer -> MMA
  uint64_t* empty = bar + NST;          // [NST] MMA -> producer
  uint64_t* dfull = bar + 2 * NST;      // [2]   MMA -> epilogue
  uint64_t* dempty = bar + 2 * NST + 2; // [2]   epilogue -> MMA
  uint64_t* ready = bar + 2 * NST + 4;  //       epilogue (TMEM scales written) + q tile -> MMA
  uint32_t* s_tslot = reinterpret_cast<uint32_t*>(smem + L::off_tslot);
  uint64_t* s_cand = reinterpret_cast<uint64_t*>(smem + L::off_cand);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cap = a.cap;
  const bool decode = a.pos != nullptr;

  // ---- which tokens and which key range
  const int64_t grp = decode ? blockIdx.x : (int64_t)(gridDim.x - 1 - blockIdx.x);  // heavy groups first
  const int64_t row0 = grp * G;
  const int split = blockIdx.y;
  int64_t tnvis[G];  // entries visible to each token of the group (0 for rows past the end)
  int64_t nvis_max = 0;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int64_t r = row0 + g;
    int64_t t = -1;
    if (r < a.rows) t = decode ? a.pos[r] : a.t0 + r;
    int64_t nv = n_visible(t, a.m);
    if (nv > a.Nc) nv = a.Nc;
    tnvis[g] = nv;
    if (nv > nvis_max) nvis_max = nv;
  }
  const int64_t key_row_base = decode ? row0 * a.Nc : 0;  // per-sequence cache (decode)
  const int64_t j_begin = (int64_t)split * a.split_tiles * 128;
  int64_t j_end = j_begin + a.split_tiles * 128;
  if (j_end > nvis_max) j_end = nvis_max;
  const int ntiles = j_end > j_begin ? (int)ceil_div(j_end - j_begin, 128) : 0;

  // ---- setup
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1 + 32);  // TMA transaction arrival + one per producer lane (scales)
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&dfull[b], 1);
      mbar_init(&dempty[b], kEpiWarps);
    }
    mbar_init(ready, kEpiWarps + 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tslot, 512);
    tmem_relinquish();
  }
  // constant-offset operands: A all 1.0 (code 2), B all 6.0 (code 7)
  for (int i = tid; i < 4096 / 16; i += kThreads)
    reinterpret_cast<uint4*>(s_ma)[i] = make_uint4(0x22222222u, 0x22222222u, 0x22222222u, 0x22222222u);
  for (int i = tid; i < N * 32 / 16; i += kThreads)
    reinterpret_cast<uint4*>(s_mb)[i] = make_uint4(0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u);
  for (int c = tid; c < N; c += kThreads) {
    const int g = c / HI, h = c % HI;
    const int64_t r = row0 + g;
    int w2 = 0;
    if (g < G && r < a.rows) w2 = e2m1_times2(a.w_codes[r * HI + h] & 15u);
    s_w2[c] = w2;
  }
  if (tid < G) {
    int sw = 0;
    const int64_t r = row0 + tid;
    if (r < a.rows)
      for (int h = 0; h < HI; ++h) sw += e2m1_times2(a.w_codes[r * HI + h] & 15u);
    s_sumw[tid] = sw;
    s_cnt[tid] = 0;
    s_thr[tid] = 0;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *s_tslot;

  if (warp == 0) {
    // =========================== producer
    if (lane == 0 && ntiles > 0) {
      prefetch_tmap(&qmap);
      prefetch_tmap(&kmap);
      mbar_arrive_expect_tx(ready, N * L::kRowBytes);
      tma_load_2d(s_q, &qmap, ready, 0, (int)(row0 * HI));
    }
    for (int it = 0; it < ntiles; ++it) {
      const int s = it % NST;
      const uint32_t ph = (it / NST) & 1;
      if (!mbar_wait(&empty[s], ph ^ 1, a.status, CSA_ERR_DEVICE_TIMEOUT)) break;
      const int64_t j0 = j_begin + (int64_t)it * 128;
      const int64_t row0k = key_row_base + j0;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], L::kABytes);
        tma_load_2d(s_a + (size_t)s * L::kABytes, &kmap, &full[s], 0, (int)row0k);
      }
      // key scales straight into the tcgen05.cp 32x128b layout: lane l holds the
      // scale words of rows l, l+32, l+64, l+96 (rows past the tensor read as 0)
      const uint32_t sdst = smem_u32(s_sf + (size_t)s * 512) + lane * 16;
      if (DI == 128) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t row = row0k + lane + 32 * c;
          const bool in = row < a.key_rows;
          cp_async4(sdst + 4 * c, a.k_scales + (in ? row : 0) * 4, in ? 4u : 0u);
        }
        cp_async_arrive(&full[s]);
      } else {
        // two scale bytes per row: plain loads, padded to the 4-byte word
        uint32_t wv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t row = row0k + lane + 32 * c;
          wv[c] = row < a.key_rows ? (uint32_t)*reinterpret_cast<const uint16_t*>(a.k_scales + row * 2) | 0x7F7F0000u
                                   : 0x7F7F7F7Fu;
        }
        *reinterpret_cast<uint4*>(s_sf + (size_t)s * 512 + lane * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        fence_proxy_async_smem();  // generic-proxy writes -> tcgen05.cp
        mbar_arrive(&full[s]);
      }
    }
    cp_async_wait_all();
  } else if (warp == 1) {
    // =========================== MMA issuer
    if (ntiles > 0) {
      mbar_wait(ready, 0, a.status, CSA_ERR_DEVICE_TIMEOUT);
      tc_fence_after();
    }
    const uint32_t sq = smem_u32(s_q);
    const uint32_t layout = DI == 128 ? kSwizzle64 : kSwizzle32;
    const uint32_t sbo = 8 * L::kRowBytes;
    for (int it = 0; it < ntiles; ++it) {
      const int s = it % NST;
      const uint32_t ph = (it / NST) & 1;
      const int b = it & 1;
      const uint32_t dph = (it >> 1) & 1;
      if (!mbar_wait(&dempty[b], dph ^ 1, a.status, CSA_ERR_DEVICE_TIMEOUT)) break;
      if (!mbar_wait(&full[s], ph, a.status, CSA_ERR_DEVICE_TIMEOUT)) break;
      fence_proxy_async_smem();  // cp.async-written scales -> tcgen05.cp (async proxy)
      tc_fence_after();
      if (elect_one()) {  // issue from a converged warp (much cheaper than a lane-0 branch)
        const uint32_t d = tbase + (b ? kTmemD1 : 0u);
        const uint32_t sfa = tbase + kTmemSFA0 + 4 * b;
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(sfa),
                     "l"(make_sdesc(smem_u32(s_sf + (size_t)s * 512), 16, 128, kSwizzleNone))
                     : "memory");
        const uint32_t sa = smem_u32(s_a + (size_t)s * L::kABytes);
#pragma unroll
        for (int kk = 0; kk < KB; ++kk) {
          mma_mxf4_ss(d, make_sdesc(sa + kk * 32, 16, sbo, layout), make_sdesc(sq + kk * 32, 16, sbo, layout),
                      idesc_mxf4(128, N, 2 * kk, 2 * kk), sfa | ((uint32_t)(2 * kk) << 30),
                      (tbase + kTmemSFB) | ((uint32_t)(2 * kk) << 30), kk > 0);
        }
        mma_mxf4_ss(d, make_sdesc(smem_u32(s_ma), 128, 256, kSwizzleNone),
                    make_sdesc(smem_u32(s_mb), 128, 256, kSwizzleNone), idesc_mxf4(128, N, 0, 0),
                    tbase + kTmemMagicSFA, tbase + kTmemMagicSFB, 1);
        mma_commit(&empty[s]);
        mma_commit(&dfull[b]);
      }
      __syncwarp();
    }
  } else {
    // =========================== epilogue + selection (warps 2..9)
    const int quarter = warp & 3;       // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;   // which half of the token group
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    // scale factors of the query rows and the constant-offset operands (replicated layout)
    if (half == 0) {
      uint32_t w[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int rr = lane + 32 * c;  // row (g*HI + h) of the B operand
        const int g = rr / HI, h = rr % HI;
        const int64_t r = row0 + g;
        uint32_t v = 0x7F7F7F7Fu;
        if (rr < G * HI && r < a.rows) {
          const uint8_t* p = a.q_scales + (r * HI + h) * (DI / 32);
          v = DI == 128 ? *reinterpret_cast<const uint32_t*>(p)
                        : ((uint32_t)*reinterpret_cast<const uint16_t*>(p) | 0x7F7F0000u);
          bool bad = false;
#pragma unroll
          for (int b = 0; b < DI / 32; ++b) {
            const uint32_t e = (v >> (8 * b)) & 255u;
            bad |= (e < 125u) | (e > 128u);
          }
          if (bad) report(a.status, CSA_ERR_RANGE);
        }
        w[c] = v;
      }
      tmem_st4(tbase + lane_base + kTmemSFB, w[0], w[1], w[2], w[3]);
      tmem_st4(tbase + lane_base + kTmemSFB + 4, w[4], w[5], w[6], w[7]);
      tmem_st4(tbase + lane_base + kTmemMagicSFA, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
      tmem_st4(tbase + lane_base + kTmemMagicSFB, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
      tmem_st4(tbase + lane_base + kTmemMagicSFB + 4, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(ready);

    // token range of this half (compile-time per instantiation)
    constexpr int G0 = (G + 1) / 2;
    static_assert(G == 1 || (G0 * HI) % 16 == 0, "halves must split on a 16-column chunk");
    const int g_lo = half == 0 ? 0 : G0;
    const int g_hi = half == 0 ? G0 : G;
    static_assert(G0 <= 4, "one token per warp of a half");
    const int my_g = g_lo + quarter;  // token whose buffer this warp maintains
    int* my_hist = s_hist + (warp - 2) * topk::kWarpBins;

    for (int it = 0; it < ntiles; ++it) {
      const int b = it & 1;
      const uint32_t dph = (it >> 1) & 1;
      if (!mbar_wait(&dfull[b], dph, a.status, CSA_ERR_DEVICE_TIMEOUT)) break;
      tc_fence_after();
      if (warp == kCheckWarp) {
        // exactness precondition on this tile's key scales (rows below j_end), read
        // back from the replicated TMEM copy the MMA used
        uint32_t sw[4];
        tmem_ld4(tbase + lane_base + kTmemSFA0 + 4 * b, sw);
        tmem_wait_ld();
        const int64_t j0 = j_begin + (int64_t)it * 128;
        bool bad = false;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (j0 + lane + 32 * c < j_end) {
#pragma unroll
            for (int q = 0; q < DI / 32; ++q) bad |= ((sw[c] >> (8 * q)) & 255u) - 125u > 3u;
          }
        if (bad) report(a.status, CSA_ERR_RANGE);
      }
      const uint32_t dcol = tbase + lane_base + (b ? kTmemD1 : 0u);
      uint32_t acc[G];  // arithmetic mod 2^32: the true head sum fits in int32
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = 0u;
      if (half == 0) head_sums<HI, G, 0>(dcol, s_w2, acc);
      else head_sums<HI, G, 1>(dcol, s_w2, acc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[b]);

      // insert candidates
      const int64_t j = j_begin + (int64_t)it * 128 + quarter * 32 + lane;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (g < g_lo || g >= g_hi) continue;
        const int64_t nv = tnvis[g];
        const int32_t units = (int32_t)(acc[g] - kMagicBits * (uint32_t)s_sumw[g]);
        const uint64_t key = topk::make_key(units, (uint32_t)j);
        const bool take = (j < nv) && (j < j_end) && (key >= s_thr[g]);
        const uint32_t bal = __ballot_sync(0xffffffffu, take);
        if (bal) {
          int base = 0;
          if (lane == 0) base = atomicAdd(&s_cnt[g], __popc(bal));
          base = __shfl_sync(0xffffffffu, base, 0);
          if (take) s_cand[(size_t)g * cap + base + __popc(bal & ((1u << lane) - 1u))] = key;
        }
      }
      // every `check` tiles (and after the last one) the half's warps meet; warp
      // `quarter` then cuts back token g_lo + quarter's buffer if the next `check`
      // tiles could overflow it (one-pass histogram threshold that keeps >= k)
      if ((it + 1) % a.check != 0 && it + 1 != ntiles) continue;
      topk::named_sync(kHalfBar0 + half, kEpiThreads / 2);
      if (my_g < g_hi) {
        uint64_t* buf = s_cand + (size_t)my_g * cap;
        const int cnt = s_cnt[my_g];
        if (cnt > cap - 128 * a.check) {
          int kept;
          const uint64_t thr = topk::warp_approx_threshold(buf, cnt, a.k, cap - 128 * a.check, my_hist, lane, &kept);
          const int n = topk::warp_compact_ge(buf, cnt, thr, lane);
          if (lane == 0) {
            s_cnt[my_g] = n;
            s_thr[my_g] = thr;
          }
        }
      }
      topk::named_sync(kHalfBar0 + half, kEpiThreads / 2);
    }

    // final exact selection and sort: one warp per token, all tokens in parallel
    if (my_g < g_hi && row0 + my_g < a.rows) {
      const int64_t r = row0 + my_g;
      uint64_t* buf = s_cand + (size_t)my_g * cap;
      int cnt = s_cnt[my_g];
      if (cnt > a.k) {
        const uint64_t thr = topk::warp_select_threshold(buf, cnt, a.k, my_hist, lane);
        cnt = topk::warp_compact_ge(buf, cnt, thr, lane);
      }
      if (a.nsplit == 1) {
        // final order: descending key (the per-range lists of a split search are
        // merged and sorted by topk_merge_kernel instead)
        if (cnt <= 512) write_sorted<16>(buf, cnt, a, r, lane);
        else if (cnt <= 1024) write_sorted<32>(buf, cnt, a, r, lane);
        else {
          const int P = topk::next_pow2(cnt);
          for (int i = cnt + lane; i < P; i += 32) buf[i] = 0;
          __syncwarp();
          topk::warp_bitonic_desc(buf, P, lane);
          for (int q = lane; q < a.k; q += 32) {
            int32_t id = -1;
            float sc = -INFINITY;
            if (q < cnt) {
              const uint64_t key = buf[q];
              id = (int32_t)topk::key_index(key);
              sc = (float)topk::key_score(key) * (1.0f / 128.0f);
            }
            a.idx[r * a.k + q] = id;
            if (a.scores) a.scores[r * a.k + q] = sc;
          }
        }
      } else {
        uint64_t* out = a.cand + ((size_t)r * a.nsplit + split) * a.k;
        for (int q = lane; q < a.k; q += 32) out[q] = q < cnt ? buf[q] : 0;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// Merge the per-range candidate lists of every query row into its final top-k
// (radix select to k, compaction, bitonic sort).  nsplit*k <= 256*kMergePer.
constexpr int kMergePer = 40;

__global__ void __launch_bounds__(256) topk_merge_kernel(const uint64_t* __restrict__ cand, int nsplit, int k,
                                                         int32_t* __restrict__ idx, float* __restrict__ scores,
                                                         uint64_t* __restrict__ keys_out) {
  extern __shared__ __align__(16) uint8_t msmem[];
  const int total = nsplit * k;
  const int P = topk::next_pow2(total);
  uint64_t* buf = reinterpret_cast<uint64_t*>(msmem);
  int* hist = reinterpret_cast<int*>(buf + P);
  int* sh = hist + 256;
  const int64_t r = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid == 0) sh[8] = 0;
  __syncthreads();
  for (int i = tid; i < total; i += 256) {
    const uint64_t key = cand[(size_t)r * total + i];
    if (key != 0) buf[atomicAdd(&sh[8], 1)] = key;
  }
  __syncthreads();
  int cnt = sh[8];
  __syncthreads();
  if (cnt > k) {
    const uint64_t thr = topk::radix_threshold<256>(buf, cnt, k, hist, sh, tid, 1);
    cnt = topk::compact_ge<256, kMergePer>(buf, cnt, thr, sh + 4, tid, 1);
  }
  const int Pk = topk::next_pow2(cnt > 1 ? cnt : 1);
  for (int i = cnt + tid; i < Pk; i += 256) buf[i] = 0;
  __syncthreads();
  topk::bitonic_desc<256>(buf, Pk, tid, 1);
  for (int q = tid; q < k; q += 256) {
    int32_t id = -1;
    float sc = -INFINITY;
    uint64_t key = 0;
    if (q < cnt) {
      key = buf[q];
      id = (int32_t)topk::key_index(key);
      sc = (float)topk::key_score(key) * (1.0f / 128.0f);
    }
    if (idx) idx[r * k + q] = id;
    if (scores) scores[r * k + q] = sc;
    if (keys_out) keys_out[r * k + q] = key;
  }
}

// ------------------------------------------------------------------ host side

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeFn get_encode_fn();

static bool make_u8_map(CUtensorMap* m, const void* base, int64_t rows, int row_bytes, int box_rows) {
  EncodeFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapSwizzle sw = row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Candidate capacity per token: whatever shared memory is left (cut-backs are
// rarer the larger it is), at least k + 128*check and a power of two >= k.
template <int HI, int DI, int G>
static bool choose_cap(int k, int* cap, int* check) {
  using L = IndexerSmem<HI, DI, G>;
  const size_t base = L::bytes(0);
  const int budget = base < kSmemLimit ? (int)((kSmemLimit - base) / (8 * (size_t)G)) & ~127 : 0;
  const int p = topk::next_pow2(k);
  for (int c = 4; c >= 1; c >>= 1) {
    const int need = k + 128 * c > p ? k + 128 * c : p;
    if (budget >= need) {
      int want = 4 * k + 128 * c;  // cut-backs rare: room for several k between them
      if (want < 4096) want = 4096;
      if (want < need) want = need;
      *cap = (want < budget ? want : budget) & ~127;
      if (*cap < need) *cap = ((need + 127) / 128) * 128;
      *check = c;
      return true;
    }
  }
  return false;
}

template <int HI, int DI, int G>
static cudaError_t launch_one(const uint8_t* q_codes, const uint8_t* k_codes, IndexerArgs a, dim3 grid,
                              cudaStream_t stream) {
  using L = IndexerSmem<HI, DI, G>;
  CUtensorMap qmap, kmap;
  if (!make_u8_map(&qmap, q_codes, a.rows * HI, DI / 2, L::N)) return cudaErrorInvalidValue;
  if (!make_u8_map(&kmap, k_codes, a.key_rows, DI / 2, 128)) return cudaErrorInvalidValue;
  if (!choose_cap<HI, DI, G>(a.k, &a.cap, &a.check)) return cudaErrorInvalidConfiguration;
  const size_t smem = L::bytes(a.cap);
  if (smem > kSmemLimit) return cudaErrorInvalidConfiguration;
  auto kern = indexer_topk_kernel<HI, DI, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(qmap, kmap, a);
  return cudaGetLastError();
}

template <int HI, int DI>
static cudaError_t dispatch_g(bool decode, const uint8_t* q_codes, const uint8_t* k_codes, IndexerArgs a,
                              dim3 grid, cudaStream_t stream) {
  if (decode) return launch_one<HI, DI, 1>(q_codes, k_codes, a, grid, stream);
  return launch_one<HI, DI, Geometry<HI>::G>(q_codes, k_codes, a, grid, stream);
}

template <int DI>
static cudaError_t dispatch_hi(int HI, bool decode, const uint8_t* q_codes, const uint8_t* k_codes, IndexerArgs a,
                               dim3 grid, cudaStream_t stream) {
  switch (HI) {
    case 4: return dispatch_g<4, DI>(decode, q_codes, k_codes, a, grid, stream);
    case 8: return dispatch_g<8, DI>(decode, q_codes, k_codes, a, grid, stream);
    case 16: return dispatch_g<16, DI>(decode, q_codes, k_codes, a, grid, stream);
    case 32: return dispatch_g<32, DI>(decode, q_codes, k_codes, a, grid, stream);
    case 64: return dispatch_g<64, DI>(decode, q_codes, k_codes, a, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

int indexer_tokens_per_cta(int HI) {
  switch (HI) {
    case 4: return Geometry<4>::G;
    case 8: return Geometry<8>::G;
    case 16: return Geometry<16>::G;
    case 32: return Geometry<32>::G;
    default: return Geometry<64>::G;
  }
}


// Prefill: rows = T, one range per group (direct output).
cudaError_t launch_indexer_prefill(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* w_codes,
                                   const uint8_t* k_codes, const uint8_t* k_scales, int64_t T, int64_t t0, int64_t Nc,
                                   int HI, int DI, int m, int k, int32_t* idx, float* scores, int* status,
                                   cudaStream_t stream) {
  const int G = indexer_tokens_per_cta(HI);
  IndexerArgs a{};
  a.q_scales = q_scales;
  a.w_codes = w_codes;
  a.k_scales = k_scales;
  a.rows = T;
  a.t0 = t0;
  a.pos = nullptr;
  a.Nc = Nc;
  a.key_rows = Nc > 0 ? Nc : 1;
  a.m = m;
  a.k = k;
  a.nsplit = 1;
  a.split_tiles = ceil_div(Nc > 0 ? Nc : 1, 128);
  a.idx = idx;
  a.scores = scores;
  a.cand = nullptr;
  a.status = status;
  dim3 grid((unsigned)ceil_div(T, G), 1);
  const uint8_t* kc = Nc > 0 ? k_codes : q_codes;  // any valid mapping when the cache is empty
  return DI == 128 ? dispatch_hi<128>(HI, false, q_codes, kc, a, grid, stream)
                   : dispatch_hi<64>(HI, false, q_codes, kc, a, grid, stream);
}

// Decode: rows = B sequences, each with its own cache of Ncap entries and position
// pos[b] (device), key range split `nsplit` ways; candidates merged afterwards.
cudaError_t launch_indexer_decode(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* w_codes,
                                  const uint8_t* k_codes, const uint8_t* k_scales, int B, const int64_t* pos_dev,
                                  int64_t nvis_max, int64_t Ncap, int HI, int DI, int m, int k, int nsplit,
                                  uint64_t* cand, int32_t* idx, float* scores, uint64_t* keys_out, int* status,
                                  cudaStream_t stream) {
  IndexerArgs a{};
  a.q_scales = q_scales;
  a.w_codes = w_codes;
  a.k_scales = k_scales;
  a.rows = B;
  a.t0 = 0;
  a.pos = pos_dev;
  a.Nc = Ncap;
  a.key_rows = (int64_t)B * Ncap;
  a.m = m;
  a.k = k;
  a.nsplit = nsplit;
  a.split_tiles = ceil_div(ceil_div(nvis_max > 0 ? nvis_max : 1, nsplit), 128);
  a.idx = nullptr;
  a.scores = nullptr;
  a.cand = cand;
  a.status = status;
  dim3 grid((unsigned)B, (unsigned)nsplit);
  cudaError_t e = DI == 128 ? dispatch_hi<128>(HI, true, q_codes, k_codes, a, grid, stream)
                            : dispatch_hi<64>(HI, true, q_codes, k_codes, a, grid, stream);
  if (e != cudaSuccess) return e;
  const int total = nsplit * k;
  const int P = topk::next_pow2(total);
  const size_t smem = (size_t)P * 8 + 256 * 4 + 64 * 4;
  e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_merge_kernel<<<B, 256, smem, stream>>>(cand, nsplit, k, idx, scores, keys_out);
  return cudaGetLastError();
}

}  // namespace csa
