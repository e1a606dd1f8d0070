// api.cu - the C ABI of libcsa.so (declared in include/csa.h): host-side
// argument validation, workspace layout, status word, launch orchestration.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "attention.cuh"
#include "common.cuh"
#include "compress.cuh"

namespace csa {

// ---- kernels' host launchers (defined in the other translation units)
cudaError_t launch_compress(const void* K, const void* V, const void* Z, const float* B, int64_t T, int d, int m,
                            void* Kc, void* Vc, cudaStream_t stream);
cudaError_t launch_indexer_prefill(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* w_codes,
                                   const uint8_t* k_codes, const uint8_t* k_scales, int64_t T, int64_t t0, int64_t Nc,
                                   int HI, int DI, int m, int k, int32_t* idx, float* scores, uint64_t* cand,
                                   int* cand_cnt, int* status, cudaStream_t stream);
cudaError_t launch_indexer_decode(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* w_codes,
                                  const uint8_t* k_codes, const uint8_t* k_scales, int B, const int64_t* pos_dev,
                                  const int64_t* pos_in, bool pdl, int64_t nvis_max, int64_t Ncap, int HI, int DI,
                                  int m, int k, int nsplit, uint64_t* cand, int* cand_cnt, int32_t* idx, float* scores,
                                  uint64_t* keys_out, int* status, cudaStream_t stream, int64_t j_base);
cudaError_t launch_topk_merge(const uint64_t* keys, int rows, int lists, int k, int* cnt, int32_t* idx,
                              float* scores, uint64_t* keys_out, cudaStream_t stream);
int inject_fault(int code);
cudaError_t launch_decode_append(const void* Kn, const void* Vn, const void* Zn, const float* Bias,
                                 const uint8_t* kIc_new, const uint8_t* kIs_new, const int64_t* pos, int B,
                                 int64_t Ncap, int d, int dI, int m, int W, void* Kwin, void* Vwin, void* Kblk,
                                 void* Vblk, void* Zblk, void* Kc, void* Vc, uint8_t* kIc, uint8_t* kIs,
                                 cudaStream_t stream);
cudaError_t launch_mxfp4_quantize(const void* x, int64_t nblocks, int mode, uint8_t* codes, uint8_t* scales,
                                  cudaStream_t stream);
cudaError_t launch_mxfp8_quantize(const void* x, int64_t nblocks, uint8_t* codes, uint8_t* scales,
                                  cudaStream_t stream);
cudaError_t launch_peak_mma(int kind, long long iters, int ctas, int* status, cudaStream_t stream);
double peak_mma_flops(int kind, long long iters, int ctas);

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// Streaming multiprocessors of the current device (queried once per device).
int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cached[dev] = n;
  return n;
}

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  if (e == cudaErrorInvalidConfiguration) return CSA_ERR_UNSUPPORTED_SHAPE;
  return CSA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename... P>
int check_ptrs(P... ps) {
  const void* arr[] = {static_cast<const void*>(ps)...};
  for (const void* p : arr) {
    if (p == nullptr) return CSA_ERR_INVALID_ARG;
    if (!aligned16(p)) return CSA_ERR_MISALIGNED;
  }
  return CSA_OK;
}

int check_opt(const void* p) { return (p != nullptr && !aligned16(p)) ? CSA_ERR_MISALIGNED : CSA_OK; }

bool valid_H(int H) { return H == 4 || H == 8 || H == 16 || H == 32 || H == 64 || H == 128; }
bool valid_HI(int HI) { return HI == 4 || HI == 8 || HI == 16 || HI == 32 || HI == 64; }

int check_ws(void* ws, size_t bytes, size_t need) {
  if (ws == nullptr || bytes < need) return CSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return CSA_ERR_MISALIGNED;
  return CSA_OK;
}

int* status_word(void* ws) { return static_cast<int*>(ws); }

// window tiles a CTA of gq consecutive tokens may need
int64_t window_tiles(int W, int gq) { return W > 0 ? ceil_div((int64_t)W + gq - 1, 128) : 0; }

struct PosBlock {
  int64_t v[64];
};

__global__ void fill_i64_kernel(int64_t* dst, PosBlock blk, int n) {
  griddep_launch_dependents();  // the next kernel's setup may overlap this copy
  if ((int)threadIdx.x < n) dst[threadIdx.x] = blk.v[threadIdx.x];
}

cudaError_t upload_positions(int64_t* dst, const int64_t* host, int B, cudaStream_t stream) {
  for (int b0 = 0; b0 < B; b0 += 64) {
    PosBlock blk{};
    const int n = B - b0 < 64 ? B - b0 : 64;
    for (int i = 0; i < n; ++i) blk.v[i] = host[b0 + i];
    fill_i64_kernel<<<1, 64, 0, stream>>>(dst + b0, blk, n);
  }
  return cudaGetLastError();
}

// Decode positions: up to kInlinePos ride in the kernel arguments (nothing is
// launched); more are copied to the workspace first.  *copied: a copy kernel is
// the call's first kernel (the ones after it may then start during it).
cudaError_t stage_positions(int64_t* dst, const int64_t* host, int B, cudaStream_t stream, bool* copied) {
  *copied = B > kInlinePos;
  return *copied ? upload_positions(dst, host, B, stream) : cudaSuccess;
}

void inline_positions(AttnArgs& a, const int64_t* host, int B) {
  if (B > kInlinePos) return;
  for (int b = 0; b < B; ++b) a.pos_in[b] = host[b];
  a.npos_in = B;
}


bool valid_odtype(int t) { return t == CSA_BF16 || t == CSA_F32; }

// decode workspace: [header][pos B*8][idx B*k*4][cand B*nsplit*k*8]
// Key ranges per decode row: as many as fill the GPU in one wave of
// one-CTA-per-SM indexer blocks (a second partial wave would double the time).
int decode_nsplit(int B, int64_t Ncap, int k) {
  const int sms = sm_count();
  int ns = B > 0 ? sms / B : 1;
  const int64_t tiles = ceil_div(Ncap > 0 ? Ncap : 1, 128);
  if (ns > tiles) ns = (int)tiles;
  const int lim = 256 * 40 / k;  // merge capacity
  if (ns > lim) ns = lim;
  if (ns > kMaxKeyRanges) ns = kMaxKeyRanges;
  return ns < 1 ? 1 : ns;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Attention CTAs per decode sequence: enough to fill the GPU, at most one per
// key tile of the sequence; with more than one, partial outputs go through the
// workspace and a combine pass.
int decode_attn_splits(int B, int64_t tiles) {
  int ns = B > 0 ? sm_count() / B : 1;
  if (ns > 16) ns = 16;  // the combine pass merges at most 16 partials
  if (ns > tiles) ns = (int)tiles;
  return ns < 1 ? 1 : ns;
}
size_t attn_part_bytes(int B, int ns, int H, int d) {
  return ns > 1 ? align256((size_t)B * ns * H * d * 4) + align256((size_t)B * ns * H * 4) : 0;
}

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" {

const char* csa_status_string(int status) {
  switch (status) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case CSA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case CSA_ERR_CUDA: return "CUDA error (see csa_last_cuda_error)";
    case CSA_ERR_WORKSPACE: return "workspace missing or too small";
    case CSA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
    case CSA_ERR_RANGE: return "MXFP4 scale byte outside [125, 128]";
    default: return "unknown status";
  }
}

int csa_last_cuda_error(void) { return g_last_cuda_error; }

int csa_version(void) { return 200; }

int csa_peak_mma(int kind, int64_t iters, int ctas, void* workspace, size_t workspace_bytes, double* flops,
                 csa_stream_t stream) {
  if ((kind != CSA_PEAK_BF16 && kind != CSA_PEAK_MXF4) || iters < 2 || ctas < 1) return CSA_ERR_INVALID_ARG;
  int rc = check_ws(workspace, workspace_bytes, kWorkspaceHeader);
  if (rc) return rc;
  if (flops) *flops = peak_mma_flops(kind, iters, ctas);
  cudaError_t e = launch_peak_mma(kind, iters, ctas, status_word(workspace), (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

int csa_debug_inject(int code) {
  if (code != CSA_FAULT_NONE && code != CSA_FAULT_INDEXER_STALL) return CSA_ERR_INVALID_ARG;
  return inject_fault(code);
}

int csa_check_status(void* workspace, csa_stream_t stream) {
  if (workspace == nullptr) return CSA_ERR_WORKSPACE;
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(int), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return v;
}

int csa_compress(const void* K, const void* V, const void* Z, const float* B, int64_t T, int d, int m, void* Kc,
                 void* Vc, csa_stream_t stream) {
  if (T < 0 || m < 1) return CSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return CSA_ERR_UNSUPPORTED_SHAPE;
  // m <= 8 or a multiple of 8 up to 512: the pooling's slices then tile a block
  if (m > 512 || (m > 8 && m % 8 != 0)) return CSA_ERR_UNSUPPORTED_SHAPE;
  if (T / m == 0) return CSA_OK;
  int rc = check_ptrs(K, V, Z, B, Kc, Vc);
  if (rc) return rc;
  cudaError_t e = launch_compress(K, V, Z, B, T, d, m, Kc, Vc, (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

int csa_mxfp4_quantize(const void* x, int64_t rows, int n, int mode, uint8_t* codes, uint8_t* scales,
                       csa_stream_t stream) {
  if (rows < 0 || n <= 0 || n % 32 != 0 || (mode != CSA_MX_OCP && mode != CSA_MX_INDEXER)) return CSA_ERR_INVALID_ARG;
  if (rows == 0) return CSA_OK;
  int rc = check_ptrs(x, codes, scales);
  if (rc) return rc;
  cudaError_t e = launch_mxfp4_quantize(x, rows * (n / 32), mode, codes, scales, (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

int csa_mxfp8_quantize(const void* x, int64_t rows, int n, uint8_t* codes, uint8_t* scales, csa_stream_t stream) {
  if (rows < 0 || n <= 0 || n % 32 != 0) return CSA_ERR_INVALID_ARG;
  if (rows == 0) return CSA_OK;
  int rc = check_ptrs(x, codes, scales);
  if (rc) return rc;
  cudaError_t e = launch_mxfp8_quantize(x, rows * (n / 32), codes, scales, (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

// Indexer workspace: status header, then per query row the k selected keys
// (uint64) and their count, which the finalize pass sorts into idx / scores.
size_t csa_indexer_topk_workspace_bytes(int64_t T, int64_t, int, int, int k) {
  if (T <= 0 || k <= 0) return kWorkspaceHeader;
  return kWorkspaceHeader + align256((size_t)T * k * 8) + align256((size_t)T * 4);
}

int csa_indexer_topk(const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
                     const uint8_t* kI_codes, const uint8_t* kI_scales, int64_t T, int64_t t0, int64_t Nc, int HI,
                     int dI, int m, int k, int32_t* idx, float* scores, void* workspace, size_t workspace_bytes,
                     csa_stream_t stream) {
  if (T < 0 || t0 < 0 || Nc < 0 || m < 1 || k < 1 || k > 2048) return CSA_ERR_INVALID_ARG;
  if (!valid_HI(HI) || (dI != 64 && dI != 128)) return CSA_ERR_UNSUPPORTED_SHAPE;
  int rc = check_ws(workspace, workspace_bytes, csa_indexer_topk_workspace_bytes(T, Nc, HI, dI, k));
  if (rc) return rc;
  if (T == 0) return CSA_OK;
  rc = check_ptrs(qI_codes, qI_scales, w_codes, idx);
  if (rc) return rc;
  if (Nc > 0 && (rc = check_ptrs(kI_codes, kI_scales))) return rc;
  if ((rc = check_opt(scores))) return rc;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint64_t* cand = reinterpret_cast<uint64_t*>(w + kWorkspaceHeader);
  int* cand_cnt = reinterpret_cast<int*>(w + kWorkspaceHeader + align256((size_t)T * k * 8));
  cudaError_t e = launch_indexer_prefill(qI_codes, qI_scales, w_codes, kI_codes, kI_scales, T, t0, Nc, HI, dI, m, k,
                                         idx, scores, cand, cand_cnt, status_word(workspace), (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

size_t csa_sparse_attn_workspace_bytes(int64_t, int, int, int, int) { return kWorkspaceHeader; }

int csa_sparse_attn(const void* Q, const void* Kc, const void* Vc, const int32_t* idx, const void* Kraw,
                    const void* Vraw, int64_t T, int64_t t0, int64_t Nc, int H, int d, int k, int W, float scale,
                    void* O, int o_dtype, float* lse, void* workspace, size_t workspace_bytes, csa_stream_t stream) {
  if (T < 0 || t0 < 0 || Nc < 0 || k < 1 || k > 2048 || W < 0 || W > 1024 || !(std::isfinite(scale) && scale > 0.f) ||
      !valid_odtype(o_dtype))
    return CSA_ERR_INVALID_ARG;
  if (!valid_H(H) || (d != 64 && d != 128)) return CSA_ERR_UNSUPPORTED_SHAPE;
  const int gq = 128 / H;
  if (gq * ceil_div(k, 128) > attention_max_seg_tiles()) return CSA_ERR_UNSUPPORTED_SHAPE;
  int rc = check_ws(workspace, workspace_bytes, kWorkspaceHeader);
  if (rc) return rc;
  if (T == 0) return CSA_OK;
  rc = check_ptrs(Q, idx, O);
  if (rc) return rc;
  if (Nc > 0 && (rc = check_ptrs(Kc, Vc))) return rc;
  if (W > 0 && (rc = check_ptrs(Kraw, Vraw))) return rc;
  if ((rc = check_opt(lse))) return rc;
  AttnArgs a{};
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.Kc = static_cast<const __nv_bfloat16*>(Nc > 0 ? Kc : Q);
  a.Vc = static_cast<const __nv_bfloat16*>(Nc > 0 ? Vc : Q);
  a.idx = idx;
  a.Kr = static_cast<const __nv_bfloat16*>(W > 0 ? Kraw : Q);
  a.Vr = static_cast<const __nv_bfloat16*>(W > 0 ? Vraw : Q);
  a.T = T;
  a.t0 = t0;
  a.Nc = Nc;
  a.raw_lo = 0;
  a.H = H;
  a.k = k;
  a.m = 1;
  a.W = W;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.O = O;
  a.o_f32 = o_dtype == CSA_F32;
  a.lse = lse;
  a.status = status_word(workspace);
  a.q_rows = T * H;
  a.kc_rows = Nc > 0 ? Nc : 1;
  a.raw_rows = W > 0 ? t0 + T : 1;
  cudaError_t e = launch_attention(a, d, (unsigned)ceil_div(T, gq), (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

size_t hca_attn_workspace_bytes(int64_t, int, int, int) { return kWorkspaceHeader; }

int hca_attn(const void* Q, const void* Kc, const void* Vc, const void* Kraw, const void* Vraw, int64_t T, int64_t t0,
             int64_t Nc, int H, int d, int m, int W, float scale, void* O, int o_dtype, float* lse, void* workspace,
             size_t workspace_bytes, csa_stream_t stream) {
  if (T < 0 || t0 < 0 || Nc < 0 || m < 1 || W < 0 || W > 1024 || !(std::isfinite(scale) && scale > 0.f) ||
      !valid_odtype(o_dtype))
    return CSA_ERR_INVALID_ARG;
  if (!valid_H(H) || (d != 64 && d != 128)) return CSA_ERR_UNSUPPORTED_SHAPE;
  const int gq = 128 / H;
  int rc = check_ws(workspace, workspace_bytes, kWorkspaceHeader);
  if (rc) return rc;
  if (T == 0) return CSA_OK;
  rc = check_ptrs(Q, O);
  if (rc) return rc;
  if (Nc > 0 && (rc = check_ptrs(Kc, Vc))) return rc;
  if (W > 0 && (rc = check_ptrs(Kraw, Vraw))) return rc;
  if ((rc = check_opt(lse))) return rc;
  AttnArgs a{};
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.Kc = static_cast<const __nv_bfloat16*>(Nc > 0 ? Kc : Q);
  a.Vc = static_cast<const __nv_bfloat16*>(Nc > 0 ? Vc : Q);
  a.idx = nullptr;
  a.Kr = static_cast<const __nv_bfloat16*>(W > 0 ? Kraw : Q);
  a.Vr = static_cast<const __nv_bfloat16*>(W > 0 ? Vraw : Q);
  a.T = T;
  a.t0 = t0;
  a.Nc = Nc;
  a.raw_lo = 0;
  a.H = H;
  a.k = 0;
  a.m = m;
  a.W = W;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.O = O;
  a.o_f32 = o_dtype == CSA_F32;
  a.lse = lse;
  a.status = status_word(workspace);
  a.q_rows = T * H;
  a.kc_rows = Nc > 0 ? Nc : 1;
  a.raw_rows = W > 0 ? t0 + T : 1;
  cudaError_t e = launch_attention(a, d, (unsigned)ceil_div(T, gq), (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

size_t csa_decode_workspace_bytes(int B, int64_t Ncap, int H, int d, int, int, int k, int W) {
  if (B <= 0 || k <= 0) return kWorkspaceHeader;
  const int ns = decode_nsplit(B, Ncap, k);
  const int nsa = decode_attn_splits(B, ceil_div(k, 128) + window_tiles(W, 1));
  return kWorkspaceHeader + align256((size_t)B * 8) + align256((size_t)B * k * 4) +
         align256((size_t)B * ns * k * 8) + align256((size_t)B * ns * 4) + attn_part_bytes(B, nsa, H, d);
}

static int decode_impl(const void* q, const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
                       const void* Kc, const void* Vc, const uint8_t* kc8, const uint8_t* kc8s, const uint8_t* vc8,
                       const uint8_t* vc8s, const uint8_t* kI_codes, const uint8_t* kI_scales, const void* Kwin,
                       const void* Vwin, const int64_t* pos, int B, int64_t Ncap, int H, int d, int HI, int dI, int m,
                       int k, int W, float scale, void* O, int o_dtype, float* lse, int32_t* idx, float* scores,
                       void* workspace, size_t workspace_bytes, csa_stream_t stream) {
  const bool fp8 = kc8 != nullptr;
  if (B < 0 || Ncap < 0 || m < 1 || k < 1 || k > 2048 || W < 0 || W > 1024 || !(std::isfinite(scale) && scale > 0.f) ||
      !valid_odtype(o_dtype))
    return CSA_ERR_INVALID_ARG;
  if (!valid_H(H) || (d != 64 && d != 128) || !valid_HI(HI) || (dI != 64 && dI != 128))
    return CSA_ERR_UNSUPPORTED_SHAPE;
  int rc = check_ws(workspace, workspace_bytes, csa_decode_workspace_bytes(B, Ncap, H, d, HI, dI, k, W));
  if (rc) return rc;
  if (B == 0) return CSA_OK;
  if (pos == nullptr) return CSA_ERR_INVALID_ARG;
  int64_t nvis_max = 0;
  for (int b = 0; b < B; ++b) {
    if (pos[b] < 0) return CSA_ERR_INVALID_ARG;
    int64_t nv = n_visible(pos[b], m);
    if (nv > Ncap) nv = Ncap;
    if (nv > nvis_max) nvis_max = nv;
  }
  rc = check_ptrs(q, qI_codes, qI_scales, w_codes, O);
  if (rc) return rc;
  if (Ncap > 0 && (rc = check_ptrs(kI_codes, kI_scales))) return rc;
  if (Ncap > 0 && !fp8 && (rc = check_ptrs(Kc, Vc))) return rc;
  if (Ncap > 0 && fp8 && (rc = check_ptrs(kc8, kc8s, vc8, vc8s))) return rc;
  if (W > 0 && (rc = check_ptrs(Kwin, Vwin))) return rc;
  if ((rc = check_opt(lse)) || (rc = check_opt(idx)) || (rc = check_opt(scores))) return rc;
  const int ns = decode_nsplit(B, Ncap, k);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  int64_t* pos_dev = reinterpret_cast<int64_t*>(w + kWorkspaceHeader);
  int32_t* idx_ws = reinterpret_cast<int32_t*>(w + kWorkspaceHeader + align256((size_t)B * 8));
  uint64_t* cand = reinterpret_cast<uint64_t*>(w + kWorkspaceHeader + align256((size_t)B * 8) +
                                               align256((size_t)B * k * 4));
  int* cand_cnt = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(cand) + align256((size_t)B * ns * k * 8));
  const int nsa = decode_attn_splits(B, ceil_div(k, 128) + window_tiles(W, 1));
  float* o_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(cand_cnt) + align256((size_t)B * ns * 4));
  float* lse_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(o_part) + align256((size_t)B * nsa * H * d * 4));
  cudaStream_t s = (cudaStream_t)stream;
  bool copied = false;
  cudaError_t e = stage_positions(pos_dev, pos, B, s, &copied);
  if (e != cudaSuccess) return cuda_fail(e);
  int32_t* sel = idx ? idx : idx_ws;
  if (Ncap > 0) {
    e = launch_indexer_decode(qI_codes, qI_scales, w_codes, kI_codes, kI_scales, B, pos_dev, pos, copied, nvis_max,
                              Ncap, HI, dI, m, k, ns, cand, cand_cnt, sel, scores, nullptr, status_word(workspace), s,
                              0);
    if (e != cudaSuccess) return cuda_fail(e);
  } else {
    e = cudaMemsetAsync(sel, 0xFF, (size_t)B * k * 4, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  AttnArgs a{};
  a.Q = static_cast<const __nv_bfloat16*>(q);
  a.Kc = static_cast<const __nv_bfloat16*>(Ncap > 0 && !fp8 ? Kc : q);  // (FP8: the maps are unused)
  a.Vc = static_cast<const __nv_bfloat16*>(Ncap > 0 && !fp8 ? Vc : q);
  if (fp8 && Ncap > 0) {
    a.kc8 = kc8;
    a.kc8_scales = kc8s;
    a.vc8 = vc8;
    a.vc8_scales = vc8s;
  }
  a.idx = sel;
  a.Kr = static_cast<const __nv_bfloat16*>(W > 0 ? Kwin : q);
  a.Vr = static_cast<const __nv_bfloat16*>(W > 0 ? Vwin : q);
  a.T = 1;
  a.t0 = 0;
  a.Nc = Ncap;
  a.H = H;
  a.k = k;
  a.m = m;
  a.W = W;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.O = O;
  a.o_f32 = o_dtype == CSA_F32;
  a.lse = lse;
  a.status = status_word(workspace);
  a.q_batch_stride = (int64_t)H * d;
  a.kc_batch_stride = Ncap * d;
  a.raw_batch_stride = (int64_t)W * d;
  a.o_batch_stride = (int64_t)H * d;
  a.pos = pos_dev;
  inline_positions(a, pos, B);
  a.pdl = Ncap > 0 || copied;  // the search (or the position copy) of this call runs just before
  a.q_rows = (int64_t)B * H;
  a.kc_rows = Ncap > 0 && !fp8 ? (int64_t)B * Ncap : 1;
  a.raw_rows = W > 0 ? (int64_t)B * W : 1;
  a.nsplit = nsa;
  a.o_part = o_part;
  a.lse_part = lse_part;
  e = launch_attention(a, d, (unsigned)B, s);
  if (e == cudaSuccess && nsa > 1) e = launch_attention_combine(a, B, d, s);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

int csa_decode(const void* q, const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
               const void* Kc, const void* Vc, const uint8_t* kI_codes, const uint8_t* kI_scales, const void* Kwin,
               const void* Vwin, const int64_t* pos, int B, int64_t Ncap, int H, int d, int HI, int dI, int m, int k,
               int W, float scale, void* O, int o_dtype, float* lse, int32_t* idx, float* scores, void* workspace,
               size_t workspace_bytes, csa_stream_t stream) {
  return decode_impl(q, qI_codes, qI_scales, w_codes, Kc, Vc, nullptr, nullptr, nullptr, nullptr, kI_codes, kI_scales,
                     Kwin, Vwin, pos, B, Ncap, H, d, HI, dI, m, k, W, scale, O, o_dtype, lse, idx, scores, workspace,
                     workspace_bytes, stream);
}

int csa_decode_fp8(const void* q, const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
                   const uint8_t* Kc_codes, const uint8_t* Kc_scales, const uint8_t* Vc_codes, const uint8_t* Vc_scales,
                   const uint8_t* kI_codes, const uint8_t* kI_scales, const void* Kwin, const void* Vwin,
                   const int64_t* pos, int B, int64_t Ncap, int H, int d, int HI, int dI, int m, int k, int W,
                   float scale, void* O, int o_dtype, float* lse, int32_t* idx, float* scores, void* workspace,
                   size_t workspace_bytes, csa_stream_t stream) {
  if (Ncap > 0 && (Kc_codes == nullptr || Kc_scales == nullptr || Vc_codes == nullptr || Vc_scales == nullptr))
    return CSA_ERR_INVALID_ARG;
  static const uint8_t kNone = 0;  // marks the MXFP8 path when the cache is empty
  return decode_impl(q, qI_codes, qI_scales, w_codes, nullptr, nullptr, Kc_codes ? Kc_codes : &kNone, Kc_scales,
                     Vc_codes, Vc_scales, kI_codes, kI_scales, Kwin, Vwin, pos, B, Ncap, H, d, HI, dI, m, k, W, scale,
                     O, o_dtype, lse, idx, scores, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- split-cache decode pieces
size_t csa_decode_search_workspace_bytes(int B, int64_t Nloc, int k) {
  if (B <= 0 || k <= 0) return kWorkspaceHeader;
  const int ns = decode_nsplit(B, Nloc, k);
  return kWorkspaceHeader + align256((size_t)B * 8) + align256((size_t)B * k * 4) + align256((size_t)B * ns * k * 8) +
         align256((size_t)B * ns * 4);
}

int csa_decode_search(const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
                      const uint8_t* kI_codes, const uint8_t* kI_scales, const int64_t* pos, int B, int64_t Nloc,
                      int64_t j_base, int HI, int dI, int m, int k, uint64_t* keys, void* workspace,
                      size_t workspace_bytes, csa_stream_t stream) {
  if (B < 0 || Nloc < 0 || j_base < 0 || m < 1 || k < 1 || k > 2048) return CSA_ERR_INVALID_ARG;
  if (!valid_HI(HI) || (dI != 64 && dI != 128)) return CSA_ERR_UNSUPPORTED_SHAPE;
  int rc = check_ws(workspace, workspace_bytes, csa_decode_search_workspace_bytes(B, Nloc, k));
  if (rc) return rc;
  if (B == 0) return CSA_OK;
  if (pos == nullptr) return CSA_ERR_INVALID_ARG;
  int64_t nvis_max = 0;
  for (int b = 0; b < B; ++b) {
    if (pos[b] < 0) return CSA_ERR_INVALID_ARG;
    int64_t nv = n_visible(pos[b], m) - j_base;
    if (nv > Nloc) nv = Nloc;
    if (nv > nvis_max) nvis_max = nv;
  }
  rc = check_ptrs(qI_codes, qI_scales, w_codes, keys);
  if (rc) return rc;
  if (Nloc > 0 && (rc = check_ptrs(kI_codes, kI_scales))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  if (Nloc == 0 || nvis_max <= 0) {
    cudaError_t e = cudaMemsetAsync(keys, 0, (size_t)B * k * 8, s);
    return e == cudaSuccess ? CSA_OK : cuda_fail(e);
  }
  const int ns = decode_nsplit(B, Nloc, k);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  int64_t* pos_dev = reinterpret_cast<int64_t*>(w + kWorkspaceHeader);
  uint64_t* cand = reinterpret_cast<uint64_t*>(w + kWorkspaceHeader + align256((size_t)B * 8) +
                                               align256((size_t)B * k * 4));
  int* cand_cnt = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(cand) + align256((size_t)B * ns * k * 8));
  bool copied = false;
  cudaError_t e = stage_positions(pos_dev, pos, B, s, &copied);
  if (e == cudaSuccess)
    e = launch_indexer_decode(qI_codes, qI_scales, w_codes, kI_codes, kI_scales, B, pos_dev, pos, copied, nvis_max,
                              Nloc, HI, dI, m, k, ns, cand, cand_cnt, nullptr, nullptr, keys, status_word(workspace),
                              s, j_base);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

size_t csa_topk_merge_workspace_bytes(int B, int L) {
  return kWorkspaceHeader + align256((size_t)(B > 0 ? B : 0) * (L > 0 ? L : 0) * 4);
}

int csa_topk_merge(const uint64_t* keys, int B, int L, int k, int32_t* idx, float* scores, uint64_t* keys_out,
                   void* workspace, size_t workspace_bytes, csa_stream_t stream) {
  if (B < 0 || L < 1 || L > kMaxKeyRanges || k < 1 || k > 2048) return CSA_ERR_INVALID_ARG;
  int rc = check_ws(workspace, workspace_bytes, csa_topk_merge_workspace_bytes(B, L));
  if (rc) return rc;
  if (B == 0) return CSA_OK;
  if ((rc = check_ptrs(keys, idx))) return rc;
  if ((rc = check_opt(scores)) || (rc = check_opt(keys_out))) return rc;
  int* cnt = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeader);
  cudaError_t e = launch_topk_merge(keys, B, L, k, cnt, idx, scores, keys_out, (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

int csa_decode_attend(const void* q, const void* Kc, const void* Vc, const int32_t* idx, int64_t j_base,
                      const void* Kwin, const void* Vwin, const int64_t* pos, int B, int64_t Nloc, int H, int d, int m,
                      int k, int W, float scale, void* O, int o_dtype, float* lse, void* workspace,
                      size_t workspace_bytes, csa_stream_t stream) {
  if (B < 0 || Nloc < 0 || j_base < 0 || m < 1 || k < 1 || k > 2048 || W < 0 || W > 1024 ||
      !(std::isfinite(scale) && scale > 0.f) || !valid_odtype(o_dtype))
    return CSA_ERR_INVALID_ARG;
  if (!valid_H(H) || (d != 64 && d != 128)) return CSA_ERR_UNSUPPORTED_SHAPE;
  int rc = check_ws(workspace, workspace_bytes, csa_decode_workspace_bytes(B, Nloc, H, d, 16, 128, k, W));
  if (rc) return rc;
  if (B == 0) return CSA_OK;
  if (pos == nullptr) return CSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (pos[b] < 0) return CSA_ERR_INVALID_ARG;
  if ((rc = check_ptrs(q, idx, O))) return rc;
  if (Nloc > 0 && (rc = check_ptrs(Kc, Vc))) return rc;
  if (W > 0 && (rc = check_ptrs(Kwin, Vwin))) return rc;
  if ((rc = check_opt(lse))) return rc;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  int64_t* pos_dev = reinterpret_cast<int64_t*>(w + kWorkspaceHeader);
  const int ns = decode_nsplit(B, Nloc, k);
  uint8_t* part_base = w + kWorkspaceHeader + align256((size_t)B * 8) + align256((size_t)B * k * 4) +
                       align256((size_t)B * ns * k * 8) + align256((size_t)B * ns * 4);
  const int nsa = decode_attn_splits(B, ceil_div(k, 128) + window_tiles(W, 1));
  cudaStream_t s = (cudaStream_t)stream;
  bool copied = false;
  cudaError_t e = stage_positions(pos_dev, pos, B, s, &copied);
  if (e != cudaSuccess) return cuda_fail(e);
  AttnArgs a{};
  a.Q = static_cast<const __nv_bfloat16*>(q);
  a.Kc = static_cast<const __nv_bfloat16*>(Nloc > 0 ? Kc : q);
  a.Vc = static_cast<const __nv_bfloat16*>(Nloc > 0 ? Vc : q);
  a.idx = idx;
  a.idx_base = j_base;
  a.Kr = static_cast<const __nv_bfloat16*>(W > 0 ? Kwin : q);
  a.Vr = static_cast<const __nv_bfloat16*>(W > 0 ? Vwin : q);
  a.T = 1;
  a.Nc = Nloc;
  a.H = H;
  a.k = k;
  a.m = m;
  a.W = W;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.O = O;
  a.o_f32 = o_dtype == CSA_F32;
  a.lse = lse;
  a.status = status_word(workspace);
  a.q_batch_stride = (int64_t)H * d;
  a.kc_batch_stride = Nloc * d;
  a.raw_batch_stride = (int64_t)W * d;
  a.o_batch_stride = (int64_t)H * d;
  a.pos = pos_dev;
  inline_positions(a, pos, B);
  a.pdl = copied;  // the position copy of this call runs just before
  a.q_rows = (int64_t)B * H;
  a.kc_rows = Nloc > 0 ? (int64_t)B * Nloc : 1;
  a.raw_rows = W > 0 ? (int64_t)B * W : 1;
  a.nsplit = nsa;
  a.o_part = reinterpret_cast<float*>(part_base);
  a.lse_part = reinterpret_cast<float*>(part_base + align256((size_t)B * nsa * H * d * 4));
  e = launch_attention(a, d, (unsigned)B, s);
  if (e == cudaSuccess && nsa > 1) e = launch_attention_combine(a, B, d, s);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

int csa_attn_combine(const float* O_parts, const float* lse_parts, int L, int B, int H, int d, void* O, int o_dtype,
                     float* lse, csa_stream_t stream) {
  if (L < 1 || L > kMaxCombineParts || B < 0 || !valid_odtype(o_dtype)) return CSA_ERR_INVALID_ARG;
  if (!valid_H(H) || (d != 64 && d != 128)) return CSA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return CSA_OK;
  int rc = check_ptrs(O_parts, lse_parts, O);
  if (rc) return rc;
  if ((rc = check_opt(lse))) return rc;
  cudaError_t e = launch_combine(O_parts, lse_parts, L, B, H, d, O, o_dtype == CSA_F32, (int64_t)H * d, lse, 1, B,
                                 (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

int csa_decode_append(const void* K_new, const void* V_new, const void* Z_new, const float* Bias,
                      const uint8_t* kI_codes_new, const uint8_t* kI_scales_new, const int64_t* pos, int B,
                      int64_t Ncap, int d, int dI, int m, int W, void* Kwin, void* Vwin, void* Kblk, void* Vblk,
                      void* Zblk, void* Kc, void* Vc, uint8_t* kI_codes, uint8_t* kI_scales, csa_stream_t stream) {
  if (B < 0 || Ncap < 0 || m < 1 || m > 4096 || W < 0 || W > 1024) return CSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return CSA_ERR_UNSUPPORTED_SHAPE;
  if (m > 8 && m % 8 != 0) return CSA_ERR_UNSUPPORTED_SHAPE;
  const bool with_ki = kI_codes_new || kI_scales_new || kI_codes || kI_scales;
  if (with_ki && (dI != 64 && dI != 128)) return CSA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return CSA_OK;
  if (pos == nullptr) return CSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b) {
    if (pos[b] < 0) return CSA_ERR_INVALID_ARG;
    if ((pos[b] + 1) % m == 0 && (pos[b] + 1) / m > Ncap) return CSA_ERR_INVALID_ARG;  // no slot for the entry
  }
  int rc = check_ptrs(K_new, V_new, Z_new, Bias, Kblk, Vblk, Zblk);
  if (rc) return rc;
  if (Ncap > 0 && (rc = check_ptrs(Kc, Vc))) return rc;
  if (W > 0 && (rc = check_ptrs(Kwin, Vwin))) return rc;
  if (with_ki && (rc = check_ptrs(kI_codes_new, kI_scales_new, kI_codes, kI_scales))) return rc;
  cudaError_t e = launch_decode_append(K_new, V_new, Z_new, Bias, with_ki ? kI_codes_new : nullptr,
                                       with_ki ? kI_scales_new : nullptr, pos, B, Ncap, d, dI, m, W, Kwin, Vwin, Kblk,
                                       Vblk, Zblk, Kc, Vc, with_ki ? kI_codes : nullptr,
                                       with_ki ? kI_scales : nullptr, (cudaStream_t)stream);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

int hca_decode_append(const void* K_new, const void* V_new, const void* Z_new, const float* Bias, const int64_t* pos,
                      int B, int64_t Ncap, int d, int m, int W, void* Kwin, void* Vwin, void* Kblk, void* Vblk,
                      void* Zblk, void* Kc, void* Vc, csa_stream_t stream) {
  return csa_decode_append(K_new, V_new, Z_new, Bias, nullptr, nullptr, pos, B, Ncap, d, 0, m, W, Kwin, Vwin, Kblk,
                           Vblk, Zblk, Kc, Vc, nullptr, nullptr, stream);
}

size_t hca_decode_workspace_bytes(int B, int64_t Ncap, int H, int d, int W) {
  if (B <= 0) return kWorkspaceHeader;
  const int nsa = decode_attn_splits(B, ceil_div(Ncap, 128) + window_tiles(W, 1));
  return kWorkspaceHeader + align256((size_t)B * 8) + attn_part_bytes(B, nsa, H, d);
}

int hca_decode(const void* q, const void* Kc, const void* Vc, const void* Kwin, const void* Vwin, const int64_t* pos,
               int B, int64_t Ncap, int H, int d, int m, int W, float scale, void* O, int o_dtype, float* lse,
               void* workspace, size_t workspace_bytes, csa_stream_t stream) {
  if (B < 0 || Ncap < 0 || m < 1 || W < 0 || W > 1024 || !(std::isfinite(scale) && scale > 0.f) ||
      !valid_odtype(o_dtype))
    return CSA_ERR_INVALID_ARG;
  if (!valid_H(H) || (d != 64 && d != 128)) return CSA_ERR_UNSUPPORTED_SHAPE;
  int rc = check_ws(workspace, workspace_bytes, hca_decode_workspace_bytes(B, Ncap, H, d, W));
  if (rc) return rc;
  if (B == 0) return CSA_OK;
  if (pos == nullptr) return CSA_ERR_INVALID_ARG;
  int64_t nvis_max = 0;
  for (int b = 0; b < B; ++b) {
    if (pos[b] < 0) return CSA_ERR_INVALID_ARG;
    int64_t nv = n_visible(pos[b], m);
    if (nv > Ncap) nv = Ncap;
    if (nv > nvis_max) nvis_max = nv;
  }
  rc = check_ptrs(q, O);
  if (rc) return rc;
  if (Ncap > 0 && (rc = check_ptrs(Kc, Vc))) return rc;
  if (W > 0 && (rc = check_ptrs(Kwin, Vwin))) return rc;
  if ((rc = check_opt(lse))) return rc;
  int64_t* pos_dev = reinterpret_cast<int64_t*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeader);
  cudaStream_t s = (cudaStream_t)stream;
  bool copied = false;
  cudaError_t e = stage_positions(pos_dev, pos, B, s, &copied);
  if (e != cudaSuccess) return cuda_fail(e);
  AttnArgs a{};
  a.Q = static_cast<const __nv_bfloat16*>(q);
  a.Kc = static_cast<const __nv_bfloat16*>(Ncap > 0 ? Kc : q);
  a.Vc = static_cast<const __nv_bfloat16*>(Ncap > 0 ? Vc : q);
  a.idx = nullptr;
  a.Kr = static_cast<const __nv_bfloat16*>(W > 0 ? Kwin : q);
  a.Vr = static_cast<const __nv_bfloat16*>(W > 0 ? Vwin : q);
  a.T = 1;
  a.Nc = Ncap;
  a.H = H;
  a.m = m;
  a.W = W;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.O = O;
  a.o_f32 = o_dtype == CSA_F32;
  a.lse = lse;
  a.status = status_word(workspace);
  a.q_batch_stride = (int64_t)H * d;
  a.kc_batch_stride = Ncap * d;
  a.raw_batch_stride = (int64_t)W * d;
  a.o_batch_stride = (int64_t)H * d;
  a.pos = pos_dev;
  inline_positions(a, pos, B);
  a.pdl = copied;  // the position copy of this call runs just before
  a.q_rows = (int64_t)B * H;
  a.kc_rows = Ncap > 0 ? (int64_t)B * Ncap : 1;
  a.raw_rows = W > 0 ? (int64_t)B * W : 1;
  a.nsplit = decode_attn_splits(B, ceil_div(Ncap, 128) + window_tiles(W, 1));
  a.o_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeader + align256((size_t)B * 8));
  a.lse_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.o_part) +
                                        align256((size_t)B * a.nsplit * H * d * 4));
  e = launch_attention(a, d, (unsigned)B, s);
  if (e == cudaSuccess && a.nsplit > 1) e = launch_attention_combine(a, B, d, s);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e);
}

}  // extern "C"
