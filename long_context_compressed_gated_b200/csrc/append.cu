// append.cu - decode cache maintenance: one new token per sequence enters the
// sliding window, the staging buffer of the block it belongs to, and, when it
// completes a block of m tokens, the compressed cache (and the entry's indexer
// key).  blog.nickys.cn/?p=150 "1. CSA" / "2. HCA": every m (m') tokens become
// one compressed entry; the window keeps the most recent raw tokens;
// ferris-liu.github.io ... deepseek-v4 section 3: the compressed cache of a
// 1M-token context.
//
// One CTA per sequence:
//  1. window [W, d] (newest last): shifted up by one row in place, in rounds of
//     rows that are all read before any is written, then the token's K/V become
//     row W-1;
//  2. if the token completes block j = (pos+1)/m - 1: the gated pooling of the
//     staged rows 0..m-2 and the token's own row (read from the inputs: it was
//     not stored yet) writes Kc/Vc[j] with the arithmetic of the prefill
//     compression (the same device function and thread layout, so the entry is
//     bit for bit the one csa_compress writes); the caller's indexer key of the
//     entry is copied to kI[j];
//  3. otherwise the token's K/V/Z are staged in slot pos % m.
#include "common.cuh"
#include "compress.cuh"

namespace csa {

namespace {

constexpr int kMinThreads = 256;      // at least; more when the pooling group of a block is larger
constexpr int kChunksPerThread = 4;   // 16-byte chunks each thread holds per shift round
constexpr int kMaxSeqPerLaunch = 64;

struct AppendPos {
  int64_t v[kMaxSeqPerLaunch];
};

struct AppendArgs {
  const __nv_bfloat16 *Kn, *Vn, *Zn;  // [B, d] the new tokens
  const float* Bias;                  // [m, d]
  const uint8_t *kIc_new, *kIs_new;   // [B, dI/2], [B, dI/32] or null
  int d, m, W, dI, S;
  int64_t Ncap;
  __nv_bfloat16 *Kwin, *Vwin;         // [B, W, d]
  __nv_bfloat16 *Kblk, *Vblk, *Zblk;  // [B, m, d]
  __nv_bfloat16 *Kc, *Vc;             // [B, Ncap, d]
  uint8_t *kIc, *kIs;                 // [B, Ncap, dI/2], [B, Ncap, dI/32] or null
};

// blockDim.x = max(256, the pooling group of a block); shared memory: the
// merge scratch of that group (gate_scratch_floats).
__global__ void __launch_bounds__(kPoolMaxThreads) decode_append_kernel(const AppendArgs a, const AppendPos P,
                                                                        int b0) {
  extern __shared__ __align__(16) float sh_gate[];
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int64_t b = b0 + blockIdx.x;
  const int64_t pos = P.v[blockIdx.x];
  const int d = a.d, CH = d / 8;  // 16-byte chunks per row
  const __nv_bfloat16* kn = a.Kn + b * d;
  const __nv_bfloat16* vn = a.Vn + b * d;
  const __nv_bfloat16* zn = a.Zn + b * d;

  // 1. window shift (rows r -> r-1), K and V together, in rounds of R rows
  if (a.W > 0) {
    uint4* kw = reinterpret_cast<uint4*>(a.Kwin + b * (int64_t)a.W * d);
    uint4* vw = reinterpret_cast<uint4*>(a.Vwin + b * (int64_t)a.W * d);
    const int R = nthr * kChunksPerThread / (2 * CH);  // rows per round
    for (int r0 = 1; r0 < a.W; r0 += R) {
      uint4 v[kChunksPerThread];
#pragma unroll
      for (int u = 0; u < kChunksPerThread; ++u) {
        const int c = u * nthr + tid;  // chunk of the round: [matrix][row][chunk]
        const int mat = c / (R * CH), rr = (c / CH) % R, ch = c % CH;
        const int row = r0 + rr;
        if (row < a.W) v[u] = (mat ? vw : kw)[(int64_t)row * CH + ch];
      }
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kChunksPerThread; ++u) {
        const int c = u * nthr + tid;
        const int mat = c / (R * CH), rr = (c / CH) % R, ch = c % CH;
        const int row = r0 + rr;
        if (row < a.W) (mat ? vw : kw)[(int64_t)(row - 1) * CH + ch] = v[u];
      }
      __syncthreads();
    }
    if (tid < 2 * CH) {
      const int mat = tid / CH, ch = tid % CH;
      (mat ? vw : kw)[(int64_t)(a.W - 1) * CH + ch] = reinterpret_cast<const uint4*>(mat ? vn : kn)[ch];
    }
  }

  // 2./3. block staging and, on completion, the compressed entry
  const int slot = (int)(pos % a.m);
  const int64_t blk_base = b * (int64_t)a.m * d;
  if (slot == a.m - 1) {
    const int64_t j = (pos + 1) / a.m - 1;
    // the pooling of the prefill compression (same thread layout, same
    // arithmetic, same merge order): the staged rows 0..m-2 and the token's
    // own row m-1, read straight from global memory
    const int CG = d / kPoolChan, gsize = CG * a.S, R = a.m / a.S;
    if (tid < gsize) {
      const int s = tid / CG, cg = tid % CG;
      const int64_t col = (int64_t)cg * kPoolChan;
      Gate st;
      gate_init(st);
      for (int r0 = 0; r0 < R; r0 += kPoolChunk) {
        const int n = min(kPoolChunk, R - r0);
        float2 g2[kPoolChunk][4], nm[4];
        float2 cm[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) cm[e] = make_float2(-INFINITY, -INFINITY);
#pragma unroll
        for (int q = 0; q < kPoolChunk; ++q)
          if (q < n) {
            const int p = s * R + r0 + q;
            const __nv_bfloat16* zr = p == a.m - 1 ? zn + col : a.Zblk + blk_base + (int64_t)p * d + col;
            const float4* br = reinterpret_cast<const float4*>(a.Bias + (int64_t)p * d + col);
            gate_logits(*reinterpret_cast<const uint4*>(zr), br[0], br[1], g2[q], cm);
          }
        if (r0 == 0)
          gate_begin(st, cm, nm);
        else
          gate_rescale(st, cm, nm);
#pragma unroll
        for (int q = 0; q < kPoolChunk; ++q)
          if (q < n) {
            const int p = s * R + r0 + q;
            const bool last = p == a.m - 1;
            const __nv_bfloat16* kr = last ? kn + col : a.Kblk + blk_base + (int64_t)p * d + col;
            const __nv_bfloat16* vr = last ? vn + col : a.Vblk + blk_base + (int64_t)p * d + col;
            gate_accum(st, g2[q], nm, *reinterpret_cast<const uint4*>(kr), *reinterpret_cast<const uint4*>(vr));
          }
      }
      gate_group_merge(st, sh_gate, tid, CG, gsize, 1);
      if (s == 0) gate_store(st, a.Kc + (b * a.Ncap + j) * d + col, a.Vc + (b * a.Ncap + j) * d + col);
    }
    if (a.kIc != nullptr) {
      const int cb = a.dI / 2, sb = a.dI / 32;
      if (tid < cb / 4)
        reinterpret_cast<uint32_t*>(a.kIc + (b * a.Ncap + j) * cb)[tid] =
            reinterpret_cast<const uint32_t*>(a.kIc_new + b * cb)[tid];
      if (tid < sb) a.kIs[(b * a.Ncap + j) * sb + tid] = a.kIs_new[b * sb + tid];
    }
  } else if (tid < 3 * CH) {
    const int mat = tid / CH, ch = tid % CH;
    const __nv_bfloat16* src = mat == 0 ? kn : (mat == 1 ? vn : zn);
    __nv_bfloat16* dst = (mat == 0 ? a.Kblk : (mat == 1 ? a.Vblk : a.Zblk)) + blk_base + (int64_t)slot * d;
    reinterpret_cast<uint4*>(dst)[ch] = reinterpret_cast<const uint4*>(src)[ch];
  }
}

}  // namespace

cudaError_t launch_decode_append(const void* Kn, const void* Vn, const void* Zn, const float* Bias,
                                 const uint8_t* kIc_new, const uint8_t* kIs_new, const int64_t* pos, int B,
                                 int64_t Ncap, int d, int dI, int m, int W, void* Kwin, void* Vwin, void* Kblk,
                                 void* Vblk, void* Zblk, void* Kc, void* Vc, uint8_t* kIc, uint8_t* kIs,
                                 cudaStream_t stream) {
  AppendArgs a{};
  a.Kn = static_cast<const __nv_bfloat16*>(Kn);
  a.Vn = static_cast<const __nv_bfloat16*>(Vn);
  a.Zn = static_cast<const __nv_bfloat16*>(Zn);
  a.Bias = Bias;
  a.kIc_new = kIc_new;
  a.kIs_new = kIs_new;
  a.d = d;
  a.m = m;
  a.W = W;
  a.dI = dI;
  a.S = pool_slices(d, m);
  a.Ncap = Ncap;
  a.Kwin = static_cast<__nv_bfloat16*>(Kwin);
  a.Vwin = static_cast<__nv_bfloat16*>(Vwin);
  a.Kblk = static_cast<__nv_bfloat16*>(Kblk);
  a.Vblk = static_cast<__nv_bfloat16*>(Vblk);
  a.Zblk = static_cast<__nv_bfloat16*>(Zblk);
  a.Kc = static_cast<__nv_bfloat16*>(Kc);
  a.Vc = static_cast<__nv_bfloat16*>(Vc);
  a.kIc = kIc;
  a.kIs = kIs;
  const int gsize = (d / kPoolChan) * a.S;
  const int threads = gsize > kMinThreads ? gsize : kMinThreads;
  const size_t smem = (size_t)gate_scratch_floats(gsize, d / kPoolChan) * sizeof(float);
  for (int b0 = 0; b0 < B; b0 += kMaxSeqPerLaunch) {
    AppendPos P{};
    const int n = B - b0 < kMaxSeqPerLaunch ? B - b0 : kMaxSeqPerLaunch;
    for (int i = 0; i < n; ++i) P.v[i] = pos[b0 + i];
    decode_append_kernel<<<n, threads, smem, stream>>>(a, P, b0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace csa
