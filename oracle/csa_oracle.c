/*
 * csa_oracle.c -- slow, plain, obviously-correct CPU reference for the
 * DeepSeek-V4 hybrid-attention hot path (CSA / HCA).  TEST INFRASTRUCTURE ONLY:
 * the tests, the package smoke check and the benchmark's CPU-baseline leg are
 * the only callers.  It shares no code, header or table with the CUDA library.
 *
 * Arithmetic is IEEE fp64 throughout (exp from libm).  Inputs arrive as raw
 * storage words: bf16 as uint16 bit patterns, MXFP4 as packed E2M1 nibbles plus
 * one E8M0 scale byte per 32 elements, head weights as one E2M1 code per byte.
 *
 * Sources (DeepSeek-V4 pages):
 *  - blog.nickys.cn/?p=150, section "1. CSA": every m tokens' KV are compressed
 *    into one entry; a lightning indexer picks the k most relevant compressed
 *    entries per query; attention runs only on those plus a few sliding-window
 *    entries.  Section "2. HCA": ratio m' >> m, no selection, dense attention
 *    over every compressed entry.
 *  - sz-guanghua.com.cn ifanr repost, attention section: the indexer computes
 *    query/compressed-block relevance in FP4 and keeps the top-k blocks; both
 *    CSA and HCA add a sliding-window branch over the most recent tokens.
 *  - m.youleyou.com/wenzhang/2906406.html, section 1: MXFP4 is used on the
 *    indexer's query-key path.
 *  The formulas the pages leave open (gated pooling weights exp(Z+B[i mod m]),
 *  I[t,j] = sum_h w[t,h] ReLU(qI[t,h].kI[j]), visibility j*m+m-1 <= t, one
 *  joint softmax over compressed and window keys, ties toward smaller j) are
 *  the method's specification and are restated at each function.
 *
 * Exactness: E2M1 x E2M1 products and their sums are exact in fp64 as long as
 * all scale exponents lie within a window of ~25 binades (the test inputs use
 * 2^-2..2^1), so oracle_indexer returns the exact real score.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ decoding */

/* bf16 storage word -> value (bf16 is the top half of an IEEE binary32). */
static double bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* OCP MX E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.
 * exponent field 0 is subnormal: 0 or 0.5. Decoded from the bit fields. */
double oracle_e2m1_value(int code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, mbit = code & 1;
  double mag = (e == 0) ? 0.5 * mbit : ldexp(1.0 + 0.5 * mbit, e - 1);
  return s ? -mag : mag;
}

/* OCP MX E8M0 scale: 2^(byte-127); 255 is NaN. */
double oracle_e8m0_value(int byte) {
  if (byte == 255) return NAN;
  return ldexp(1.0, byte - 127);
}

/* element c of a packed row: element 2i in the low nibble of byte i. */
static int fp4_code(const uint8_t* row, int c) { return (row[c >> 1] >> ((c & 1) * 4)) & 15; }

/* ------------------------------------------------------------------ threads */

typedef void (*row_fn)(void* ctx, long i);
typedef struct {
  row_fn fn;
  void* ctx;
  long n, next;
  pthread_mutex_t mu;
} pool_t;

static void* pool_worker(void* arg) {
  pool_t* p = (pool_t*)arg;
  for (;;) {
    pthread_mutex_lock(&p->mu);
    long i = p->next++;
    pthread_mutex_unlock(&p->mu);
    if (i >= p->n) break;
    p->fn(p->ctx, i);
  }
  return NULL;
}

static void parallel_rows(row_fn fn, void* ctx, long n, int nthreads) {
  if (nthreads <= 1 || n <= 1) {
    for (long i = 0; i < n; ++i) fn(ctx, i);
    return;
  }
  if (nthreads > 256) nthreads = 256;
  pool_t p;
  p.fn = fn;
  p.ctx = ctx;
  p.n = n;
  p.next = 0;
  pthread_mutex_init(&p.mu, NULL);
  pthread_t th[256];
  for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, pool_worker, &p);
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&p.mu);
}

/* ------------------------------------------------------------------ compress
 * Block j covers tokens i = j*m .. j*m+m-1.  For every channel c:
 *   a_i = exp(Z[i,c] + B[i-j*m, c]) / sum_{i' in block} exp(Z[i',c] + B[i'-j*m, c])
 *   Kc[j,c] = sum_i a_i K[i,c],  Vc[j,c] = sum_i a_i V[i,c]
 * (per-channel softmax-gated pooling; the gate bias is indexed by the position
 * inside the block, i mod m).  The trailing partial block (T % m tokens) is not
 * compressed: it is not complete yet.  Layouts: K,V,Z [T,d] bf16, B [m,d] f32,
 * Kc,Vc [T/m, d] f64.
 */
typedef struct {
  const uint16_t *K, *V, *Z;
  const float* B;
  int d, m;
  double *Kc, *Vc;
} compress_ctx;

static void compress_row(void* vctx, long j) {
  compress_ctx* x = (compress_ctx*)vctx;
  int d = x->d, m = x->m;
  for (int c = 0; c < d; ++c) {
    double mx = -INFINITY;
    for (int p = 0; p < m; ++p) {
      long i = j * m + p;
      double g = bf16_value(x->Z[i * d + c]) + (double)x->B[p * d + c];
      if (g > mx) mx = g;
    }
    double den = 0, nk = 0, nv = 0;
    for (int p = 0; p < m; ++p) {
      long i = j * m + p;
      double e = exp(bf16_value(x->Z[i * d + c]) + (double)x->B[p * d + c] - mx);
      den += e;
      nk += e * bf16_value(x->K[i * d + c]);
      nv += e * bf16_value(x->V[i * d + c]);
    }
    x->Kc[j * d + c] = nk / den;
    x->Vc[j * d + c] = nv / den;
  }
}

int oracle_compress(const uint16_t* K, const uint16_t* V, const uint16_t* Z, const float* B, long T, int d, int m,
                    double* Kc, double* Vc, int nthreads) {
  if (!K || !V || !Z || !B || !Kc || !Vc || T < 0 || d <= 0 || m <= 0) return -1;
  compress_ctx x = {K, V, Z, B, d, m, Kc, Vc};
  parallel_rows(compress_row, &x, T / m, nthreads);
  return 0;
}

/* ------------------------------------------------------------------ indexer
 * For query row r (absolute position t = t0 + rows[i]) and compressed entry j:
 *   dot_h = sum_c qI[t,h,c] * kI[j,c]   (MXFP4 values: E2M1 * 2^(scale-127), one
 *                                       scale per 32 consecutive c)
 *   I[t,j] = sum_h w[t,h] * max(dot_h, 0)       (w: one E2M1 code per (t,h))
 * defined for j < min(Nc, n_vis(t)) with n_vis(t) = floor((t+1)/m) -- block j
 * is visible when it ends at or before t.  Invisible entries get -inf.
 * Layouts: q_codes [T,HI,dI/2], q_scales [T,HI,dI/32], w_codes [T,HI],
 * k_codes [Nc,dI/2], k_scales [Nc,dI/32]; out I [nrows, Nc].
 */
typedef struct {
  const uint8_t *qc, *qs, *wc, *kc, *ks;
  long t0, Nc;
  int HI, dI, m;
  const long* rows;
  double* I;
} indexer_ctx;

static void indexer_row(void* vctx, long i) {
  indexer_ctx* x = (indexer_ctx*)vctx;
  long r = x->rows[i], t = x->t0 + r;
  long nvis = (t + 1) / x->m;
  if (nvis > x->Nc) nvis = x->Nc;
  int HI = x->HI, dI = x->dI;
  double* out = x->I + i * x->Nc;
  /* decode this token's query heads once */
  double* q = (double*)malloc(sizeof(double) * HI * dI);
  double* w = (double*)malloc(sizeof(double) * HI);
  for (int h = 0; h < HI; ++h) {
    const uint8_t* row = x->qc + (r * HI + h) * (dI / 2);
    const uint8_t* sc = x->qs + (r * HI + h) * (dI / 32);
    for (int c = 0; c < dI; ++c) q[h * dI + c] = oracle_e2m1_value(fp4_code(row, c)) * oracle_e8m0_value(sc[c / 32]);
    w[h] = oracle_e2m1_value(x->wc[r * HI + h] & 15);
  }
  double* kv = (double*)malloc(sizeof(double) * dI);
  for (long j = 0; j < x->Nc; ++j) {
    if (j >= nvis) {
      out[j] = -INFINITY;
      continue;
    }
    const uint8_t* krow = x->kc + j * (dI / 2);
    const uint8_t* ksc = x->ks + j * (dI / 32);
    for (int c = 0; c < dI; ++c) kv[c] = oracle_e2m1_value(fp4_code(krow, c)) * oracle_e8m0_value(ksc[c / 32]);
    double s = 0;
    for (int h = 0; h < HI; ++h) {
      double dot = 0;
      for (int c = 0; c < dI; ++c) dot += q[h * dI + c] * kv[c];
      s += w[h] * (dot > 0 ? dot : 0.0);
    }
    out[j] = s;
  }
  free(kv);
  free(w);
  free(q);
}

int oracle_indexer(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* w_codes, const uint8_t* k_codes,
                   const uint8_t* k_scales, long t0, long Nc, int HI, int dI, int m, const long* rows, long nrows,
                   double* I, int nthreads) {
  if (!q_codes || !q_scales || !w_codes || !rows || !I || HI <= 0 || dI <= 0 || dI % 32 || m <= 0) return -1;
  if (Nc > 0 && (!k_codes || !k_scales)) return -1;
  indexer_ctx x = {q_codes, q_scales, w_codes, k_codes, k_scales, t0, Nc, HI, dI, m, rows, I};
  parallel_rows(indexer_row, &x, nrows, nthreads);
  return 0;
}

/* ------------------------------------------------------------------ top-k
 * For each row: among entries j < nvis[i], the k with the largest score; ties
 * go to the smaller j.  Output in rank order (score descending, then j
 * ascending); when fewer than k entries are visible the tail is idx = -1,
 * score = -inf.  A plain selection sort over the candidates: O(k * nvis).
 */
typedef struct {
  const double* S;
  long Nc;
  const long* nvis;
  int k;
  int32_t* idx;
  double* top;
} topk_ctx;

static void topk_row(void* vctx, long i) {
  topk_ctx* x = (topk_ctx*)vctx;
  const double* s = x->S + i * x->Nc;
  long n = x->nvis[i];
  if (n > x->Nc) n = x->Nc;
  unsigned char* taken = (unsigned char*)calloc(n > 0 ? n : 1, 1);
  for (int r = 0; r < x->k; ++r) {
    long best = -1;
    for (long j = 0; j < n; ++j) {
      if (taken[j]) continue;
      if (best < 0 || s[j] > s[best]) best = j; /* strict '>' keeps the smaller j on ties */
    }
    if (best >= 0) {
      taken[best] = 1;
      x->idx[i * x->k + r] = (int32_t)best;
      x->top[i * x->k + r] = s[best];
    } else {
      x->idx[i * x->k + r] = -1;
      x->top[i * x->k + r] = -INFINITY;
    }
  }
  free(taken);
}

int oracle_topk(const double* S, long nrows, long Nc, const long* nvis, int k, int32_t* idx, double* top,
                int nthreads) {
  if (!S || !nvis || !idx || !top || k < 0) return -1;
  topk_ctx x = {S, Nc, nvis, k, idx, top};
  parallel_rows(topk_row, &x, nrows, nthreads);
  return 0;
}

/* ------------------------------------------------------------------ attention
 * For query row r (t = t0 + rows[i]) and head h, the key set is
 *   S(t) = {compressed entry j : j listed in sel[i] (j >= 0), or, when sel is
 *           NULL, every j < min(Nc, n_vis(t))}
 *        U {raw token s : max(0, t-W+1) <= s <= t}
 * and, with one joint softmax over S(t),
 *   O[t,h] = sum_{x in S} exp(scale*q.k_x - M) v_x / sum_{x in S} exp(scale*q.k_x - M)
 *   lse[t,h] = M + log(sum_x exp(scale*q.k_x - M))
 * A token inside a selected block that is also in the window counts twice (once
 * inside the compressed entry, once raw).  Raw rows are addressed by absolute
 * position s as Kraw[(s - raw_pos0)*d].  Empty S gives O = 0, lse = -inf.
 * Layouts: Q [*, H, d] indexed by rows[i]; Kc,Vc [Nc,d]; sel [nrows, nsel];
 * O [nrows, H, d] f64; lse [nrows, H] f64.
 */
typedef struct {
  const uint16_t *Q, *Kc, *Vc, *Kr, *Vr;
  const int32_t* sel;
  int nsel, H, d, m;
  long Nc, W, t0, raw_pos0;
  double scale;
  const long* rows;
  double *O, *lse;
} attn_ctx;

static void attn_row(void* vctx, long i) {
  attn_ctx* x = (attn_ctx*)vctx;
  int H = x->H, d = x->d;
  long r = x->rows[i], t = x->t0 + r;
  /* gather the key/value rows of S(t) */
  long ncomp = 0;
  long nv = (t + 1) / x->m;
  if (nv > x->Nc) nv = x->Nc;
  long cap = (x->sel ? x->nsel : nv) + (x->W > 0 ? x->W : 0);
  const uint16_t** kr = (const uint16_t**)malloc(sizeof(void*) * (cap > 0 ? cap : 1));
  const uint16_t** vr = (const uint16_t**)malloc(sizeof(void*) * (cap > 0 ? cap : 1));
  long n = 0;
  if (x->sel) {
    for (int q = 0; q < x->nsel; ++q) {
      int32_t j = x->sel[i * x->nsel + q];
      if (j < 0) continue;
      kr[n] = x->Kc + (long)j * d;
      vr[n] = x->Vc + (long)j * d;
      ++n;
    }
  } else {
    for (long j = 0; j < nv; ++j) {
      kr[n] = x->Kc + j * d;
      vr[n] = x->Vc + j * d;
      ++n;
    }
  }
  ncomp = n;
  (void)ncomp;
  long s0 = t - x->W + 1;
  if (s0 < 0) s0 = 0;
  for (long s = s0; s <= t && x->W > 0; ++s) {
    kr[n] = x->Kr + (s - x->raw_pos0) * d;
    vr[n] = x->Vr + (s - x->raw_pos0) * d;
    ++n;
  }
  double* logit = (double*)malloc(sizeof(double) * (n > 0 ? n : 1));
  for (int h = 0; h < H; ++h) {
    const uint16_t* q = x->Q + (r * H + h) * d;
    double* o = x->O + (i * H + h) * d;
    double mx = -INFINITY;
    for (long a = 0; a < n; ++a) {
      double dot = 0;
      for (int c = 0; c < d; ++c) dot += bf16_value(q[c]) * bf16_value(kr[a][c]);
      logit[a] = x->scale * dot;
      if (logit[a] > mx) mx = logit[a];
    }
    for (int c = 0; c < d; ++c) o[c] = 0;
    if (n == 0) {
      if (x->lse) x->lse[i * H + h] = -INFINITY;
      continue;
    }
    double den = 0;
    for (long a = 0; a < n; ++a) {
      double e = exp(logit[a] - mx);
      den += e;
      for (int c = 0; c < d; ++c) o[c] += e * bf16_value(vr[a][c]);
    }
    for (int c = 0; c < d; ++c) o[c] /= den;
    if (x->lse) x->lse[i * H + h] = mx + log(den);
  }
  free(logit);
  free(vr);
  free(kr);
}

int oracle_attention(const uint16_t* Q, int H, int d, const uint16_t* Kc, const uint16_t* Vc, long Nc, int m,
                     const int32_t* sel, int nsel, const uint16_t* Kraw, const uint16_t* Vraw, long raw_pos0, long W,
                     long t0, const long* rows, long nrows, double scale, double* O, double* lse, int nthreads) {
  if (!Q || !rows || !O || H <= 0 || d <= 0 || m <= 0 || W < 0) return -1;
  if (W > 0 && (!Kraw || !Vraw)) return -1;
  attn_ctx x = {Q, Kc, Vc, Kraw, Vraw, sel, nsel, H, d, m, Nc, W, t0, raw_pos0, scale, rows, O, lse};
  parallel_rows(attn_row, &x, nrows, nthreads);
  return 0;
}

/* ------------------------------------------------------------------ MXFP4 quantiser
 * bf16 activations -> MXFP4 (the indexer's query-key operands; the pages put
 * the indexer's QK path on MXFP4 but give no scale rule).  Reading taken, the
 * OCP MX conversion: for every block of 32 consecutive elements of a row,
 *   X = floor(log2(max_i |x_i|)) - 2        (2 = exponent of E2M1's largest
 *                                            value 6 = 1.5 * 2^2)
 *   scale byte = X + 127 (E8M0), code_i = E2M1 nearest to x_i / 2^X, ties to
 *   the even code, magnitudes above 6 saturated to 6, sign kept (-0 allowed).
 * Mode 0 keeps X in the E8M0 range [-127, 127] (an all-zero block gets X =
 * -127); mode 1 clamps X to [-2, 1] (scale bytes 125..128, the range in which
 * the GPU indexer's exact fixed-point head sum holds), which saturates blocks
 * with max |x| >= 12 and flushes small ones more coarsely.  A block holding a
 * NaN or an infinity gets scale byte 255 (NaN) and zero codes.
 * Layouts: x [rows, n] bf16 (n % 32 == 0) -> codes [rows, n/2] (element 2i in
 * the low nibble of byte i), scales [rows, n/32].
 */
static int e2m1_round_magnitude(double y) {
  /* nearest of the eight E2M1 magnitudes (decoded from the bit fields), ties to
   * the even code; y >= 6 saturates to 6 */
  if (y >= 6.0) return 7;
  int best = 0;
  double bestd = fabs(y - oracle_e2m1_value(0));
  for (int c = 1; c < 8; ++c) {
    double dd = fabs(y - oracle_e2m1_value(c));
    if (dd < bestd || (dd == bestd && (c & 1) == 0)) {
      best = c;
      bestd = dd;
    }
  }
  return best;
}

int oracle_mxfp4_quantize(const uint16_t* x, long rows, int n, int mode, uint8_t* codes, uint8_t* scales) {
  if (!x || !codes || !scales || rows < 0 || n <= 0 || n % 32 || (mode != 0 && mode != 1)) return -1;
  for (long r = 0; r < rows; ++r) {
    for (int b = 0; b < n / 32; ++b) {
      const uint16_t* blk = x + r * n + b * 32;
      double amax = 0;
      int finite = 1;
      for (int i = 0; i < 32; ++i) {
        double v = bf16_value(blk[i]);
        if (!isfinite(v)) finite = 0;
        else if (fabs(v) > amax) amax = fabs(v);
      }
      uint8_t* crow = codes + r * (n / 2) + b * 16;
      if (!finite) {
        scales[r * (n / 32) + b] = 255;
        memset(crow, 0, 16);
        continue;
      }
      int X;
      if (amax == 0) {
        X = -127;
      } else {
        int e;
        frexp(amax, &e); /* amax = f * 2^e, f in [0.5, 1): floor(log2 amax) = e - 1 */
        X = (e - 1) - 2;
      }
      if (X < -127) X = -127;
      if (X > 127) X = 127;
      if (mode == 1) X = X < -2 ? -2 : (X > 1 ? 1 : X);
      scales[r * (n / 32) + b] = (uint8_t)(X + 127);
      for (int i = 0; i < 32; ++i) {
        double v = bf16_value(blk[i]);
        int sign = signbit(v) ? 8 : 0;
        int code = sign | e2m1_round_magnitude(fabs(v) / ldexp(1.0, X));
        if (i % 2 == 0) crow[i / 2] = (uint8_t)code;
        else crow[i / 2] |= (uint8_t)(code << 4);
      }
    }
  }
  return 0;
}

/* ------------------------------------------------------------------ MXFP8 (E4M3) cache quantiser
 * The compressed K/V cache in FP8 (ferris-liu.github.io ... deepseek-v4,
 * engineering layer: the KV cache mixes BF16 and FP8 storage).  Reading taken:
 * compressed entries in E4M3 with one E8M0 scale per 32 channels (OCP MX), the
 * raw window in bf16.  Per block of 32 elements:
 *   X = floor(log2 max|x|) - 8      (8 = exponent of E4M3's largest value
 *                                    448 = 1.75 * 2^8), clamped to [-127, 127];
 *   scale byte = X + 127; code = E4M3 nearest to x / 2^X, ties to the even
 *   code, magnitudes above 448 saturated to 448, sign kept.
 * An all-zero block gets X = -127; a block with Inf/NaN gets scale byte 255 and
 * zero codes.  E4M3 (OCP): sign, 4 exponent bits (bias 7), 3 mantissa bits;
 * exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN (never
 * produced), so the largest magnitude is 1.75 * 2^8.
 */
double oracle_e4m3_value(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, mbits = code & 7;
  if (e == 15 && mbits == 7) return NAN;
  double mag = (e == 0) ? ldexp(mbits / 8.0, -6) : ldexp(1.0 + mbits / 8.0, e - 7);
  return s ? -mag : mag;
}

static int e4m3_round_magnitude(double y) {
  /* nearest of the 127 finite non-negative E4M3 magnitudes (codes 0..126),
   * ties to the even code; y above 448 saturates to 448 (code 126) */
  if (y >= 448.0) return 126;
  int best = 0;
  double bestd = fabs(y - oracle_e4m3_value(0));
  for (int c = 1; c < 127; ++c) {
    double dd = fabs(y - oracle_e4m3_value(c));
    if (dd < bestd || (dd == bestd && (c & 1) == 0)) {
      best = c;
      bestd = dd;
    }
  }
  return best;
}

int oracle_mxfp8_quantize(const uint16_t* x, long rows, int n, uint8_t* codes, uint8_t* scales) {
  if (!x || !codes || !scales || rows < 0 || n <= 0 || n % 32) return -1;
  for (long r = 0; r < rows; ++r) {
    for (int b = 0; b < n / 32; ++b) {
      const uint16_t* blk = x + r * n + b * 32;
      double amax = 0;
      int finite = 1;
      for (int i = 0; i < 32; ++i) {
        double v = bf16_value(blk[i]);
        if (!isfinite(v)) finite = 0;
        else if (fabs(v) > amax) amax = fabs(v);
      }
      uint8_t* crow = codes + r * n + b * 32;
      if (!finite) {
        scales[r * (n / 32) + b] = 255;
        memset(crow, 0, 32);
        continue;
      }
      int X = -127;
      if (amax > 0) {
        int e;
        frexp(amax, &e);
        X = (e - 1) - 8;
      }
      if (X < -127) X = -127;
      if (X > 127) X = 127;
      scales[r * (n / 32) + b] = (uint8_t)(X + 127);
      for (int i = 0; i < 32; ++i) {
        double v = bf16_value(blk[i]);
        crow[i] = (uint8_t)((signbit(v) ? 0x80 : 0) | e4m3_round_magnitude(fabs(v) / ldexp(1.0, X)));
      }
    }
  }
  return 0;
}
