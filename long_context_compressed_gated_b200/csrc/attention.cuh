// attention.cuh - arguments of the attention kernel (CSA sparse / HCA dense,
// prefill and decode) shared by its launcher and the C ABI.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace csa {

struct AttnArgs {
  const __nv_bfloat16* Q;   // [T, H, d] (decode: [B, H, d])
  const __nv_bfloat16* Kc;  // [Nc, d] compressed keys (decode: per-sequence cache)
  const __nv_bfloat16* Vc;
  const int32_t* idx;       // [T, k] selected entries (CSA) or null (HCA)
  int64_t idx_base;         // idx holds global entry numbers; Kc row r is entry idx_base + r
  const __nv_bfloat16* Kr;  // raw K rows, row 0 at absolute position raw_lo
  const __nv_bfloat16* Vr;
  int64_t T, t0, Nc, raw_lo;
  int H, k, m, W;
  float scale_log2;         // softmax scale * log2(e)
  void* O;                  // [T, H, d] bf16, or fp32 when o_f32
  int o_f32;                // 1: O is written as fp32 (no bf16 rounding of the result)
  float* lse;               // [T, H] natural-log normaliser, nullable
  int* status;              // device status word
  // decode (pos != null): one sequence per CTA, batch strides in elements
  int64_t q_batch_stride, kc_batch_stride, raw_batch_stride, o_batch_stride;
  const int64_t* pos;       // device, absolute position of each sequence's new token
  int64_t pos_in[kInlinePos];  // the same positions, when npos_in = B (<= kInlinePos)
  int npos_in;
  // extents (rows) of the tensors, for the TMA descriptors
  int64_t q_rows, kc_rows, raw_rows;
  // decode with the key tiles of a sequence spread over nsplit CTAs (grid.y):
  // each writes its normalised fp32 output and log-sum-exp, merged by
  // launch_attention_combine.  nsplit = 1: direct bf16 output.
  int nsplit;
  float* o_part;    // [B, nsplit, H, d]
  float* lse_part;  // [B, nsplit, H]
  // compressed entries in MXFP8 (decode): E4M3 codes [rows, d] and E8M0 scales
  // [rows, d/32]; when set, the selected rows are dequantised (exactly) into the
  // bf16 tiles instead of copied from Kc / Vc
  const uint8_t *kc8, *kc8_scales, *vc8, *vc8_scales;
  // set by launch_attention: work items (prefill token groups) and the number of
  // item descriptions kept in shared memory (2: the next one is built ahead)
  int64_t nitems;
  int slots;
  // 1: a kernel of the same library call runs just before this one (the launch may
  // overlap it; the scheduler reads positions and selections only once it completed)
  int pdl;
  __device__ __forceinline__ int64_t pos_at(int64_t b) const { return b < npos_in ? pos_in[b] : pos[b]; }
};

cudaError_t launch_attention(const AttnArgs& a, int d, unsigned grid, cudaStream_t stream);
// O[b,h] = sum_s exp(lse_s - lse) O_s with lse = log sum_s exp(lse_s), as bf16 (+ lse)
cudaError_t launch_attention_combine(const AttnArgs& a, int B, int d, cudaStream_t stream);
int attention_max_seg_tiles();
// Merge nsplit normalised fp32 partial outputs with their log-sum-exps (partial s
// of sequence b at row b*sb + s*ss): O = sum_s exp(lse_s - lse) O_s, lse = log sum exp.
cudaError_t launch_combine(const float* o_part, const float* lse_part, int nsplit, int B, int H, int d, void* O,
                           int o_f32, int64_t o_batch_stride, float* lse, int64_t sb, int64_t ss,
                           cudaStream_t stream, bool pdl = false);
constexpr int kMaxCombineParts = 16;

}  // namespace csa
