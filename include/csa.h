/*
 * csa.h -- C ABI of libcsa.so: the DeepSeek-V4 hybrid-attention hot path
 * (CSA: Compressed Sparse Attention, HCA: Heavily Compressed Attention) as
 * hand-written CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * The method (DeepSeek-V4 pages):
 *   - blog.nickys.cn/?p=150, "1. CSA": every m tokens' key/value entries are
 *     compressed into one entry (sequence length -> 1/m); a lightning indexer
 *     selects the k compressed entries most relevant to each query; attention
 *     runs over those plus a few sliding-window (uncompressed) entries.
 *     "2. HCA": compression ratio m' >> m, no selection, dense attention over
 *     every compressed entry.
 *   - sz-guanghua.com.cn ifanr repost, attention section: the indexer scores
 *     query/block relevance in FP4 and keeps the top-k blocks; both CSA and HCA
 *     carry the sliding-window branch.
 *   - m.youleyou.com/wenzhang/2906406.html, section 1: MXFP4 on the indexer's
 *     query-key path.
 * Where the pages leave a formula open, this library computes:
 *   compression   a_i = exp(Z[i,c]+B[i mod m,c]) / sum_{block} exp(...),
 *                 Kc[j,c] = sum_i a_i K[i,c], Vc[j,c] = sum_i a_i V[i,c]
 *   indexer       I[t,j] = sum_h w[t,h] * ReLU(qI[t,h] . kI[j]) on MXFP4
 *   visibility    block j (tokens j*m .. j*m+m-1) is visible to token t iff
 *                 j*m+m-1 <= t, i.e. j < n_vis(t) = floor((t+1)/m)
 *   top-k         k largest visible I[t,j]; ties -> smaller j
 *   attention     one joint softmax over {selected (CSA) / all visible (HCA)
 *                 compressed entries} U {raw tokens max(0,t-W+1) .. t}
 *
 * Conventions for every entry point
 *   - All tensor arguments are DEVICE pointers to caller-owned memory, dense
 *     row-major (last index fastest), 16-byte aligned.  bf16 tensors are passed
 *     as `const void*` holding IEEE bfloat16 values.
 *   - MXFP4 tensors: `*_codes` hold two E2M1 codes per byte (element 2i in the
 *     low nibble of byte i); `*_scales` hold one E8M0 byte (2^(e-127)) per 32
 *     consecutive elements.  Head weights w are one E2M1 code per byte (low
 *     nibble).  Exactness precondition: every scale byte lies in [125, 128]
 *     (2^-2 .. 2^1); a kernel that sees a byte outside it reports
 *     CSA_ERR_RANGE through the status word and its scores are then unspecified.
 *   - Work is enqueued on `stream` (0 = legacy default stream); no entry point
 *     synchronises, allocates device memory or frees it.  Scratch memory is the
 *     caller's `workspace`, sized by the matching *_workspace_bytes() query.
 *   - Arguments are validated on the host before anything is enqueued; on any
 *     error nothing is enqueued and a negative csa_status_t is returned.
 *   - Device-side failures (a bounded wait that timed out, a scale byte outside
 *     the exact range) are recorded in a 32-bit status word at the start of the
 *     workspace; read it with csa_check_status() after the stream completes.
 *   - Kernels are deterministic: no floating-point atomics, fixed reduction order.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa_stream_t; /* == cudaStream_t */

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = -1,       /* null pointer, negative size, k/W out of range */
  CSA_ERR_MISALIGNED = -2,        /* a pointer is not 16-byte aligned */
  CSA_ERR_UNSUPPORTED_SHAPE = -3, /* d, H, HI, dI or m outside the supported set */
  CSA_ERR_CUDA = -4,              /* a CUDA call failed; see csa_last_cuda_error() */
  CSA_ERR_WORKSPACE = -5,         /* workspace null or smaller than required */
  CSA_ERR_DEVICE_TIMEOUT = -6,    /* (status word) a bounded device wait gave up */
  CSA_ERR_RANGE = -7              /* (status word) MXFP4 scale outside [125,128] */
} csa_status_t;

/* Element type of an attention output O (the o_dtype argument). */
typedef enum {
  CSA_BF16 = 0, /* IEEE bfloat16, round to nearest even of the fp32 result */
  CSA_F32 = 1   /* the fp32 result itself (no output rounding; 2x the bytes) */
} csa_dtype_t;

/* Human-readable text of a status code (static storage). */
const char* csa_status_string(int status);
/* The cudaError_t of the last CSA_ERR_CUDA on this host thread (0 if none). */
int csa_last_cuda_error(void);
/* Library version, major*10000 + minor*100 + patch. */
int csa_version(void);

/* Reads the device status word at the start of `workspace` (synchronously on
 * `stream`) and clears it.  Returns CSA_OK or the first device-side error.
 * While the word holds CSA_ERR_DEVICE_TIMEOUT, kernels given that workspace
 * skip their work (their outputs are then unspecified) instead of waiting out
 * every deadline again: clear it before reusing the workspace. */
int csa_check_status(void* workspace, csa_stream_t stream);

/* Test hook for the device-side timeout path (no counterpart on the pages).
 * Every wait of a kernel on another part of the same kernel is bounded
 * (~0.14 s of SM clock); when a wait runs out, the kernel records
 * CSA_ERR_DEVICE_TIMEOUT in the status word, lets the copies it already
 * started land, frees its tensor memory and returns, so the context stays
 * usable.  csa_debug_inject(CSA_FAULT_INDEXER_STALL) makes the NEXT indexer
 * launch in this process (csa_indexer_topk or the indexer of csa_decode) skip
 * its first key-tile copy, so its MMA and epilogue waits run out; the launch
 * then reports CSA_ERR_DEVICE_TIMEOUT through csa_check_status.  No memory is
 * touched out of bounds.  The code is consumed by that launch.  Returns CSA_OK,
 * or CSA_ERR_INVALID_ARG for an unknown code. */
enum { CSA_FAULT_NONE = 0, CSA_FAULT_INDEXER_STALL = 1 };
int csa_debug_inject(int code);

/* ---------------------------------------------------------------- measurement
 * Tensor-pipe ceiling of this GPU, the roofline denominator of the indexer's
 * MXFP4 contraction (m.youleyou.com/wenzhang/2906406.html section 1 puts the
 * indexer's query-key path on MXFP4) and, for calibration against a library
 * GEMM, of bf16.  Enqueues `ctas` CTAs (one per SM: pass the SM count) that each
 * issue `iters` back-to-back tcgen05.mma instructions of shape 128 x 240 on
 * operands resident in shared memory (kind::mxf4.block_scale.block32 with K = 64
 * for CSA_PEAK_MXF4, kind::f16 on bf16 with K = 16 for CSA_PEAK_BF16).  *flops
 * (nullable) receives the work of the launch, 2*128*240*K*iters*ctas; time it
 * with events on `stream`.  workspace: >= 256 bytes for the status word.
 * iters >= 2, ctas >= 1. */
enum { CSA_PEAK_BF16 = 0, CSA_PEAK_MXF4 = 1 };
int csa_peak_mma(int kind, int64_t iters, int ctas, void* workspace, size_t workspace_bytes, double* flops,
                 csa_stream_t stream);

/* ---------------------------------------------------------------- compress
 * Softmax-gated per-channel pooling of every complete block of m tokens
 * (blog.nickys.cn/?p=150 "1. CSA"; gate weights exp(Z[i]+B[i mod m])).
 *   K, V, Z : [T, d] bf16      B : [m, d] float32 (bias by position in block)
 *   Kc, Vc  : [T/m, d] bf16 outputs (round-to-nearest-even of an fp32 result)
 * The trailing T % m tokens are not compressed.  d in {64, 128}; 1 <= m <= 512
 * with m <= 8 or m % 8 == 0.  For chunked prefill pass the chunk's rows (the
 * chunk must start at a multiple of m) and the matching rows of Kc/Vc.
 * No workspace. */
int csa_compress(const void* K, const void* V, const void* Z, const float* B, int64_t T, int d, int m, void* Kc,
                 void* Vc, csa_stream_t stream);

/* ---------------------------------------------------------------- MXFP4 quantiser
 * bf16 -> MXFP4, the operand format of the indexer's query-key path
 * (m.youleyou.com/wenzhang/2906406.html section 1: MXFP4 on the indexer's QK
 * path; ferris-liu.github.io ... deepseek-v4, engineering layer: FP4 on the
 * indexer).  The pages give no scale rule; this is the OCP MX conversion.  For
 * every block of 32 consecutive elements of a row of x [rows, n] bf16:
 *   X = floor(log2 max|x|) - 2 (an all-zero block: X = -127), clamped to
 *   [-127, 127]; with mode CSA_MX_INDEXER clamped to [-2, 1] instead, so that
 *   the scale bytes meet the indexer's exact range 125..128 (blocks with
 *   max|x| >= 12 then saturate, small ones round more coarsely);
 *   scales[r, b] = X + 127; codes: E2M1 nearest to x / 2^X, ties to the even
 *   code, magnitudes above 6 saturate to 6, the sign is kept (-0 is code 8);
 *   element 2i in the low nibble of byte i of codes [rows, n/2].
 * A block holding an Inf or NaN gets scale byte 255 and zero codes.
 * n % 32 == 0.  Deterministic; no workspace. */
enum { CSA_MX_OCP = 0, CSA_MX_INDEXER = 1 };
int csa_mxfp4_quantize(const void* x, int64_t rows, int n, int mode, uint8_t* codes, uint8_t* scales,
                       csa_stream_t stream);

/* MXFP8 for the compressed K/V cache (ferris-liu.github.io ... deepseek-v4,
 * engineering layer: the KV cache mixes BF16 and FP8 storage; read here as the
 * compressed entries in FP8 and the raw window in BF16).  For every block of 32
 * consecutive elements of a row of x [rows, n] bf16: X = floor(log2 max|x|) - 8
 * (an all-zero block: -127), clamped to [-127, 127]; scales[r, b] = X + 127
 * (E8M0); codes[r, i] = E4M3 (OCP: bias 7, no infinity) nearest to x / 2^X, ties
 * to even, saturating at +-448, sign kept.  An Inf/NaN block gets scale 255 and
 * zero codes.  codes [rows, n] u8, scales [rows, n/32] u8; n % 32 == 0.  Every
 * code times its scale is exactly a bf16 value (4 significant bits). */
int csa_mxfp8_quantize(const void* x, int64_t rows, int n, uint8_t* codes, uint8_t* scales, csa_stream_t stream);

/* ---------------------------------------------------------------- indexer + top-k
 * Lightning indexer on MXFP4 fused with the causal top-k (ifanr repost,
 * attention section; blog.nickys.cn/?p=150 "1. CSA").
 * For query rows r in [0, T) at absolute positions t = t0 + r:
 *   qI_codes [T, HI, dI/2] u8, qI_scales [T, HI, dI/32] u8, w_codes [T, HI] u8
 *   kI_codes [Nc, dI/2] u8, kI_scales [Nc, dI/32] u8  (entries 0..Nc-1 of the
 *            compressed cache; entry j covers tokens j*m .. j*m+m-1)
 * Outputs, per row, in rank order (score descending, then j ascending):
 *   idx    [T, k] int32  -- selected entries; -1 when fewer than k are visible
 *   scores [T, k] float  -- I[t, idx] rounded to nearest float (-inf padding);
 *                           may be NULL.
 * HI in {4, 8, 16, 32, 64}, dI in {64, 128}, 1 <= k <= 2048, m >= 1.
 * Scores are computed exactly (integer head sum), so idx is bit-exact. */
size_t csa_indexer_topk_workspace_bytes(int64_t T, int64_t Nc, int HI, int dI, int k);
int csa_indexer_topk(const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
                     const uint8_t* kI_codes, const uint8_t* kI_scales, int64_t T, int64_t t0, int64_t Nc, int HI,
                     int dI, int m, int k, int32_t* idx, float* scores, void* workspace, size_t workspace_bytes,
                     csa_stream_t stream);

/* ---------------------------------------------------------------- CSA attention
 * Sparse + sliding-window attention (blog.nickys.cn/?p=150 "1. CSA"; window
 * branch: ifanr repost, attention section).  MQA: one shared K/V head.
 *   Q      [T, H, d] bf16 (rows at absolute positions t = t0 + r)
 *   Kc, Vc [Nc, d] bf16 compressed entries; idx [T, k] int32 (-1 = none)
 *   Kraw, Vraw : raw K/V rows indexed by ABSOLUTE position (row s at
 *          Kraw + s*d); rows max(0, t0-W+1) .. t0+T-1 must be readable.
 *   O      [T, H, d] output of element type o_dtype (CSA_BF16 or CSA_F32; any
 *          other value is CSA_ERR_INVALID_ARG); lse [T, H] float natural-log sum
 *          of exp of the scaled logits (may be NULL).
 * One joint softmax over the selected entries and the window; scale is the
 * logit multiplier (> 0; 1/sqrt(d) for the usual reading).  A row with an empty key
 * set gets O = 0, lse = -inf.  H in {4, 8, 16, 32, 64, 128}, d in {64, 128},
 * 1 <= k <= 2048, 0 <= W <= 1024, and (128/H) * ceil(k/128) <= 512 (the
 * selected-entry tiles of one 128-row block; shared memory may bind first for
 * small H with large k, reported as CSA_ERR_UNSUPPORTED_SHAPE). */
size_t csa_sparse_attn_workspace_bytes(int64_t T, int H, int d, int k, int W);
int csa_sparse_attn(const void* Q, const void* Kc, const void* Vc, const int32_t* idx, const void* Kraw,
                    const void* Vraw, int64_t T, int64_t t0, int64_t Nc, int H, int d, int k, int W, float scale,
                    void* O, int o_dtype, float* lse, void* workspace, size_t workspace_bytes,
                    csa_stream_t stream);

/* ---------------------------------------------------------------- HCA attention
 * Dense attention over every visible compressed entry plus the window
 * (blog.nickys.cn/?p=150 "2. HCA").  Same layouts as csa_sparse_attn without
 * idx; entries j < min(Nc, floor((t+1)/m)) are visible to position t.  The
 * number of visible entries is not limited (dense tiles are generated, not
 * listed). */
size_t hca_attn_workspace_bytes(int64_t T, int H, int d, int W);
int hca_attn(const void* Q, const void* Kc, const void* Vc, const void* Kraw, const void* Vraw, int64_t T, int64_t t0,
             int64_t Nc, int H, int d, int m, int W, float scale, void* O, int o_dtype, float* lse,
             void* workspace, size_t workspace_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------- decode
 * One new token per sequence against a compressed KV cache (the decode case of
 * the same method; ferris-liu.github.io ... deepseek-v4 section 3 gives the
 * 1M-token cache sizes).  For sequence b in [0, B) the new token sits at
 * absolute position pos[b] (host array), and:
 *   q        [B, H, d] bf16           qI_codes [B, HI, dI/2], qI_scales [B, HI, dI/32]
 *   w_codes  [B, HI]                  Kc, Vc [B, Ncap, d] bf16 compressed cache
 *   kI_codes [B, Ncap, dI/2]          kI_scales [B, Ncap, dI/32]
 *   Kwin, Vwin [B, W, d] bf16: raw K/V of positions pos[b]-W+1 .. pos[b]
 *            (newest last; rows for negative positions are ignored)
 *   O [B, H, d] of element type o_dtype; lse [B, H] float (nullable); idx [B, k] int32 and
 *   scores [B, k] float (both nullable) receive the selection.
 * Entries j < min(Ncap, floor((pos[b]+1)/m)) are visible. */
size_t csa_decode_workspace_bytes(int B, int64_t Ncap, int H, int d, int HI, int dI, int k, int W);
int csa_decode(const void* q, const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
               const void* Kc, const void* Vc, const uint8_t* kI_codes, const uint8_t* kI_scales, const void* Kwin,
               const void* Vwin, const int64_t* pos, int B, int64_t Ncap, int H, int d, int HI, int dI, int m, int k,
               int W, float scale, void* O, int o_dtype, float* lse, int32_t* idx, float* scores, void* workspace,
               size_t workspace_bytes, csa_stream_t stream);

/* csa_decode over a compressed cache stored in MXFP8 (ferris-liu.github.io ...
 * deepseek-v4, engineering layer: the KV cache mixes BF16 and FP8 storage; here
 * the compressed entries are FP8 and the window BF16).  Kc_codes / Vc_codes
 * [B, Ncap, d] E4M3 bytes and Kc_scales / Vc_scales [B, Ncap, d/32] E8M0 bytes,
 * as csa_mxfp8_quantize writes them; every other argument as csa_decode.  The
 * selected entries are dequantised exactly to bf16 as they are gathered, so the
 * result equals csa_decode over the dequantised cache bit for bit; the gathered
 * bytes halve.  Workspace: csa_decode_workspace_bytes(). */
int csa_decode_fp8(const void* q, const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
                   const uint8_t* Kc_codes, const uint8_t* Kc_scales, const uint8_t* Vc_codes, const uint8_t* Vc_scales,
                   const uint8_t* kI_codes, const uint8_t* kI_scales, const void* Kwin, const void* Vwin,
                   const int64_t* pos, int B, int64_t Ncap, int H, int d, int HI, int dI, int m, int k, int W,
                   float scale, void* O, int o_dtype, float* lse, int32_t* idx, float* scores, void* workspace,
                   size_t workspace_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------- split-cache decode
 * One sequence's compressed cache split over several GPUs by entry ranges (the
 * decode case of blog.nickys.cn/?p=150 "1. CSA": the indexer's top-k over all
 * visible entries, then attention over the selection plus the window).  Rank r
 * holds entries [j_base, j_base + Nloc) of each sequence and runs:
 *   1. csa_decode_search: its slice's k best as exact 64-bit keys, keys [B, k]
 *      u64 (score << 32 | ~j, j the GLOBAL entry) in rank order (score desc,
 *      j asc; 0 = none, after the valid ones), over the visible entries
 *      j < floor((pos+1)/m);
 *   2. (all-gather of the keys; every rank then holds [B, L, k])
 *   3. csa_topk_merge: the exact top-k of the L lists per sequence (each list
 *      in rank order, as csa_decode_search writes it), in rank order (score
 *      desc, j asc), idx [B, k] int32 (global, -1 padding),
 *      scores [B, k] f32 (nullable), keys_out [B, k] (nullable); identical on
 *      every rank;
 *   4. csa_decode_attend: attention over the selected entries that lie in its
 *      slice (others are skipped) plus the window (pass W = 0 except on the
 *      rank holding the newest tokens), O (o_dtype; pass CSA_F32 for merging)
 *      and lse [B, H] (required for merging);
 *   5. (all-gather of O and lse) csa_attn_combine: O = sum_r exp(lse_r - lse) O_r.
 * Layouts as csa_decode, with Kc/Vc/kI the rank's slice [B, Nloc, .].  The result
 * equals csa_decode on the whole cache: idx/scores bit for bit, O within the
 * attention tolerance (fp32 partials merged in a different order).
 * Workspaces: csa_decode_search_workspace_bytes(B, Nloc, k),
 * csa_topk_merge_workspace_bytes(B, L), and for csa_decode_attend
 * csa_decode_workspace_bytes(B, Nloc, H, d, HI, dI, k, W).  1 <= L <= 63 lists,
 * L <= 16 partials. */
size_t csa_decode_search_workspace_bytes(int B, int64_t Nloc, int k);
int csa_decode_search(const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
                      const uint8_t* kI_codes, const uint8_t* kI_scales, const int64_t* pos, int B, int64_t Nloc,
                      int64_t j_base, int HI, int dI, int m, int k, uint64_t* keys, void* workspace,
                      size_t workspace_bytes, csa_stream_t stream);
size_t csa_topk_merge_workspace_bytes(int B, int L);
int csa_topk_merge(const uint64_t* keys, int B, int L, int k, int32_t* idx, float* scores, uint64_t* keys_out,
                   void* workspace, size_t workspace_bytes, csa_stream_t stream);
int csa_decode_attend(const void* q, const void* Kc, const void* Vc, const int32_t* idx, int64_t j_base,
                      const void* Kwin, const void* Vwin, const int64_t* pos, int B, int64_t Nloc, int H, int d, int m,
                      int k, int W, float scale, void* O, int o_dtype, float* lse, void* workspace,
                      size_t workspace_bytes, csa_stream_t stream);
int csa_attn_combine(const float* O_parts, const float* lse_parts, int L, int B, int H, int d, void* O, int o_dtype,
                     float* lse, csa_stream_t stream);

/* HCA decode: dense over every visible cached entry plus the window. */
size_t hca_decode_workspace_bytes(int B, int64_t Ncap, int H, int d, int W);
int hca_decode(const void* q, const void* Kc, const void* Vc, const void* Kwin, const void* Vwin, const int64_t* pos,
               int B, int64_t Ncap, int H, int d, int m, int W, float scale, void* O, int o_dtype, float* lse,
               void* workspace, size_t workspace_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------- decode cache maintenance
 * One new token per sequence enters the decode state that csa_decode /
 * hca_decode read (blog.nickys.cn/?p=150 "1. CSA" / "2. HCA": every m tokens
 * become one compressed entry, and the sliding window keeps the latest raw
 * tokens; ferris-liu.github.io ... deepseek-v4 section 3: the compressed cache
 * of a 1M-token context).  For sequence b, the token at absolute position
 * pos[b] (host array) with raw K_new[b], V_new[b] and gate logits Z_new[b]
 * ([B, d] bf16 each):
 *   - the window Kwin/Vwin [B, W, d] (newest last) moves up one row and the
 *     token becomes row W-1, so after the call it holds pos-W+1 .. pos;
 *   - if the token ends a block ((pos+1) % m == 0), entry j = (pos+1)/m - 1 of
 *     Kc/Vc [B, Ncap, d] is written by the gated pooling of the block's m
 *     tokens with bias Bias [m, d] f32 -- bit for bit the entry csa_compress
 *     computes from the same tokens -- and the caller's indexer key of that
 *     entry, kI_codes_new [B, dI/2] / kI_scales_new [B, dI/32], is copied to
 *     kI_codes [B, Ncap, dI/2] / kI_scales [B, Ncap, dI/32] (how an entry's
 *     indexer key is derived from its tokens is not on the pages);
 *   - otherwise the token's K/V/Z are staged in slot pos % m of Kblk/Vblk/Zblk
 *     [B, m, d] bf16 (the caller's buffers; a block's earlier tokens must have
 *     been appended by earlier calls, or staged by the caller).
 * Call it before csa_decode for the same position.  The four kI pointers are
 * all given or all NULL (hca_decode_append passes NULL).  A sequence whose
 * block completes at j >= Ncap is CSA_ERR_INVALID_ARG.  d in {64, 128};
 * m <= 4096 with m <= 8 or m % 8 == 0; 0 <= W <= 1024.  No workspace. */
int csa_decode_append(const void* K_new, const void* V_new, const void* Z_new, const float* Bias,
                      const uint8_t* kI_codes_new, const uint8_t* kI_scales_new, const int64_t* pos, int B,
                      int64_t Ncap, int d, int dI, int m, int W, void* Kwin, void* Vwin, void* Kblk, void* Vblk,
                      void* Zblk, void* Kc, void* Vc, uint8_t* kI_codes, uint8_t* kI_scales, csa_stream_t stream);
int hca_decode_append(const void* K_new, const void* V_new, const void* Z_new, const float* Bias, const int64_t* pos,
                      int B, int64_t Ncap, int d, int m, int W, void* Kwin, void* Vwin, void* Kblk, void* Vblk,
                      void* Zblk, void* Kc, void* Vc, csa_stream_t stream);

/* ---------------------------------------------------------------- decode without allocation
 * csa_decode for callers that cannot allocate device memory: serving loops
 * that forbid allocator calls once they are running, embedders that own every
 * buffer and hand the library nothing else, and code running where a
 * cudaMalloc is not allowed.  The pages describe no such interface; it exists
 * only for these callers.
 * Same arguments and results as csa_decode (O in bf16), minus the workspace:
 * the scratch lives in one static 8 MiB device array inside libcsa.so that
 * every GPU loading the library keeps until the process exits.  Calls whose
 * csa_decode_workspace_bytes() exceeds 8 MiB are rejected with
 * CSA_ERR_WORKSPACE; with H <= 64 at d = 128, B = 16 sequences with k = 1024
 * fit for any cache length (at H = 128 the split attention partials alone need
 * more).
 * The positions pos[] are read on the host during the call, like csa_decode.
 * The first call on a device looks up the array's device address (a runtime
 * query, once per device, with that device current) and keeps it for the life
 * of the process: it assumes the runtime's primary context of that device and
 * no cudaDeviceReset in between.  All calls on a device share the array, so
 * calls that can overlap on the GPU (different streams, no ordering between
 * them) race with each other; issue them on one stream or order them.  The
 * call clears the array's status word itself.  status_out (device int,
 * nullable) receives the device status word of the call (CSA_OK, or
 * CSA_ERR_DEVICE_TIMEOUT / CSA_ERR_RANGE) in stream order.
 * Allocates nothing: no cudaMalloc/cudaFree, no allocating library routine. */
int csa_decode_noalloc(const void* q, const uint8_t* qI_codes, const uint8_t* qI_scales, const uint8_t* w_codes,
                       const void* Kc, const void* Vc, const uint8_t* kI_codes, const uint8_t* kI_scales,
                       const void* Kwin, const void* Vwin, const int64_t* pos, int B, int64_t Ncap, int H, int d,
                       int HI, int dI, int m, int k, int W, float scale, void* O, float* lse, int32_t* idx,
                       float* scores, int* status_out, csa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H_ */
