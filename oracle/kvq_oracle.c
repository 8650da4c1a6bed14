/*
 * kvq_oracle.c - plain, slow CPU statement of the rotated-INT4 paged KV cache.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * CPU-baseline leg of the benchmark may load this library. It shares no code,
 * header, table or constant with the CUDA path.
 *
 * What it follows (web pages, cited by title and section):
 *  [SAW]   "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World
 *          LLM Serving", Abstract: token-wise INT4 quantization with a
 *          block-diagonal Hadamard rotation, stored in a paged KV cache, read
 *          back by fused attention.
 *  [OSCAR] "OScaR: Occam's Razor for Extreme KV Cache Quantization in LLMs",
 *          section "The OScaR Framework": V^ = Quant(S.(R.V)) - rotate the
 *          cache, apply the per-token scaling, then quantize.
 *
 * Readings where the pages are silent (each is a choice of this library):
 *  - R = diag(H_b/sqrt(b), ...) over contiguous b-channel blocks, H_b the
 *    Sylvester Hadamard matrix in natural order, no random signs; b = 0 = I.
 *  - one (s, z) pair per row = (token, kv head, K or V) over all D channels.
 *  - z = largest fp16 <= min(y); s = smallest fp16 >= 0 with 15 s + z >= max(y).
 *  - code = round-half-even(fp32(y - z) * fp32(1/s)); s = 0 gives code 0.
 *    (The pages fix no rounding rule for this step; with bf16 inputs the
 *    exact quotient often lands exactly on a half-integer, where the rule
 *    decides, so the rule is stated here and computed in fp64 from those
 *    two fp32 operands.)
 *  - byte j of a packed row = code[2j] | code[2j+1] << 4.
 *  - cache [page][Hkv][2][16][D/2], scales/zeros [page][Hkv][2][16].
 *  - attention: softmax_scale defaults to 1/sqrt(D); out = R sum_t p_t v^_t.
 *
 * Everything here is a direct definition: a dense Hadamard matrix, fp64 sums,
 * scalar quantize/dequantize, brute-force softmax. Built with
 *   gcc -O2 -fopenmp -shared -fPIC kvq_oracle.c -o libkvq_oracle.so -lm
 * (build() in oracle/__init__.py does this).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_PAGE 16

/* ------------------------------------------------------------------------- */
/* Number formats, from the IEEE-754 binary16 and bfloat16 bit layouts.      */
/* ------------------------------------------------------------------------- */

/* bfloat16 is the top 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 31;
  int m = h & 1023;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
  } else if (e == 31) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* Non-negative binary16 patterns 0x0000..0x7C00 (0 .. +inf) are ordered like
 * their values; the roundings below search that ordered set. */
static uint16_t smallest_half_at_least(double x) { /* x >= 0 */
  uint16_t lo = 0, hi = 0x7C00;
  while (lo < hi) {
    uint16_t mid = (uint16_t)((lo + hi) / 2);
    if (oracle_half_to_double(mid) >= x) hi = mid; else lo = (uint16_t)(mid + 1);
  }
  return lo;
}

static uint16_t largest_half_at_most(double x) { /* x >= 0 */
  uint16_t lo = 0, hi = 0x7C00;
  while (lo < hi) {
    uint16_t mid = (uint16_t)((lo + hi + 1) / 2);
    if (oracle_half_to_double(mid) <= x) lo = mid; else hi = (uint16_t)(mid - 1);
  }
  return lo;
}

/* Round toward -inf to binary16. */
uint16_t oracle_half_round_down(double x) {
  if (!signbit(x)) return largest_half_at_most(x);
  uint16_t m = smallest_half_at_least(-x);
  return (uint16_t)(m | 0x8000);
}

/* Round toward +inf to binary16. */
uint16_t oracle_half_round_up(double x) {
  if (!signbit(x)) {
    uint16_t r = smallest_half_at_least(x);
    return r;
  }
  uint16_t m = largest_half_at_most(-x);
  return (uint16_t)(m | 0x8000);
}

/* Round to nearest, ties to even, to binary16 (overflow at >= 65520). */
uint16_t oracle_half_round_nearest(double x) {
  double a = fabs(x);
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  uint16_t d = largest_half_at_most(a);
  double dv = oracle_half_to_double(d);
  if (dv == a) return (uint16_t)(d | sign);
  /* the next value above 65504 counts as 65536 when judging nearness */
  double uv = (d == 0x7BFF) ? 65536.0 : oracle_half_to_double((uint16_t)(d + 1));
  uint16_t u = (uint16_t)(d + 1);
  uint16_t r;
  if (a - dv < uv - a) r = d;
  else if (a - dv > uv - a) r = u;
  else r = (d & 1) ? u : d;
  return (uint16_t)(r | sign);
}

/* ------------------------------------------------------------------------- */
/* Rotation: block-diagonal Hadamard ([SAW] Abstract; [OSCAR] R.V).          */
/* ------------------------------------------------------------------------- */

static int popcount_u32(uint32_t v) {
  int c = 0;
  while (v) { c += (int)(v & 1u); v >>= 1; }
  return c;
}

/* Dense Sylvester Hadamard matrix of order b (a power of two), natural order:
 * H[i*b + j] = (-1)^popcount(i & j). */
void oracle_hadamard(int b, int8_t* H) {
  for (int i = 0; i < b; ++i)
    for (int j = 0; j < b; ++j)
      H[i * b + j] = (popcount_u32((uint32_t)(i & j)) & 1) ? -1 : 1;
}

static int valid_block(int D, int b) {
  if (b == 0) return 1;
  if (b != 32 && b != 64 && b != 128) return 0;
  return (D % b) == 0;
}

/* The +-1 of channel c under a sign mask (NULL: all +1): bit c of
 * signs[c / 32] set means -1. Randomized Hadamard: R = (1/sqrt(b)) H_b
 * diag(sigma) per block, orthogonal for any signs, R^T = diag(sigma) H_b /
 * sqrt(b) (H_b is symmetric). */
static double sign_of(const uint32_t* signs, int c) {
  return (signs && ((signs[c >> 5] >> (c & 31)) & 1u)) ? -1.0 : 1.0;
}

/* y = R x in fp64 for an fp64 row: with x' = sigma * x (elementwise),
 * y[blk + i] = (1/sqrt(b)) sum_j H[i][j] x'[blk + j]. b = 0 copies x (signs
 * must then be NULL or zero). */
int oracle_rotate_f64_signed(const double* x, int D, int b, const uint32_t* signs, double* y) {
  if (!valid_block(D, b)) return -1;
  if (b == 0) {
    for (int c = 0; c < D; ++c) y[c] = x[c];
    return 0;
  }
  int8_t* H = (int8_t*)malloc((size_t)b * b);
  oracle_hadamard(b, H);
  double norm = 1.0 / sqrt((double)b);
  for (int blk = 0; blk < D; blk += b) {
    for (int i = 0; i < b; ++i) {
      double acc = 0.0;
      for (int j = 0; j < b; ++j) acc += (double)H[i * b + j] * (sign_of(signs, blk + j) * x[blk + j]);
      y[blk + i] = acc * norm;
    }
  }
  free(H);
  return 0;
}

int oracle_rotate_f64(const double* x, int D, int b, double* y) {
  return oracle_rotate_f64_signed(x, D, b, NULL, y);
}

/* y = R^T x = sigma * ((1/sqrt(b)) H_b x) (elementwise sign after the
 * transform); with no signs R^T = R. */
int oracle_unrotate_f64_signed(const double* x, int D, int b, const uint32_t* signs, double* y) {
  if (oracle_rotate_f64_signed(x, D, b, NULL, y) != 0) return -1;
  if (b > 0)
    for (int c = 0; c < D; ++c) y[c] *= sign_of(signs, c);
  return 0;
}

/* The rotated bf16 row, rounded once to fp32 (the precision the kernels keep
 * between rotation and quantization). */
int oracle_rotate_row_signed(const uint16_t* x_bf16, int D, int b, const uint32_t* signs, float* y) {
  double xd[256], yd[256];
  if (D <= 0 || D > 256) return -1;
  for (int c = 0; c < D; ++c) xd[c] = oracle_bf16_to_double(x_bf16[c]);
  if (oracle_rotate_f64_signed(xd, D, b, signs, yd) != 0) return -1;
  for (int c = 0; c < D; ++c) y[c] = (float)yd[c];
  return 0;
}

int oracle_rotate_row(const uint16_t* x_bf16, int D, int b, float* y) {
  return oracle_rotate_row_signed(x_bf16, D, b, NULL, y);
}

/* ------------------------------------------------------------------------- */
/* Asymmetric INT4 quantization, one scale per token ([SAW] Abstract;       */
/* [OSCAR] Quant(.) after the rotation).                                     */
/* ------------------------------------------------------------------------- */

/* z = largest fp16 <= mn; s = smallest fp16 >= 0 with 15 s + z >= mx.
 * 15 s + z is exact in fp64 (both are binary16 values), so the test is exact. */
/* z = largest fp16 <= mn; s = smallest fp16 >= 0 with top * s + z >= mx,
 * top the largest code (15 for INT4, 3 for INT2). */
void oracle_scale_zero_levels(float mn, float mx, int top, uint16_t* s_out, uint16_t* z_out) {
  uint16_t z = oracle_half_round_down((double)mn);
  double zd = oracle_half_to_double(z);
  double need = ((double)mx - zd) / (double)top;
  uint16_t s = (need <= 0.0) ? 0 : oracle_half_round_up(need);
  /* settle the candidate on the exact condition, in either direction */
  while (s < 0x7C00 && top * oracle_half_to_double(s) + zd < (double)mx) s = (uint16_t)(s + 1);
  while (s > 0 && top * oracle_half_to_double((uint16_t)(s - 1)) + zd >= (double)mx) s = (uint16_t)(s - 1);
  *s_out = s;
  *z_out = z;
}

void oracle_scale_zero(float mn, float mx, uint16_t* s_out, uint16_t* z_out) {
  oracle_scale_zero_levels(mn, mx, 15, s_out, z_out);
}

/* Codes of a row for a given (s, z): code = round-half-even(t * inv) with
 * t = fp32(y - z) and inv = fp32(1/s); the product of two fp32 values is
 * exact in fp64, so rint() on it is the one rounding. Clamped to [0, 15]. */
void oracle_quantize_given(const float* y, int D, uint16_t s, uint16_t z, uint8_t* codes) {
  float sf = (float)oracle_half_to_double(s);
  float zf = (float)oracle_half_to_double(z);
  float inv = (sf > 0.0f) ? 1.0f / sf : 0.0f;
  for (int c = 0; c < D; ++c) {
    float t = y[c] - zf;
    double q = (double)t * (double)inv;
    double r = nearbyint(q); /* default rounding mode: ties to even */
    if (r < 0) r = 0;
    if (r > 15) r = 15;
    codes[c] = (uint8_t)r;
  }
}

/* The quotient fp32(y - z) * fp32(1/s) itself, for classifying elements that
 * sit next to a rounding boundary. */
void oracle_quotient_given(const float* y, int D, uint16_t s, uint16_t z, double* qout) {
  float sf = (float)oracle_half_to_double(s);
  float zf = (float)oracle_half_to_double(z);
  float inv = (sf > 0.0f) ? 1.0f / sf : 0.0f;
  for (int c = 0; c < D; ++c) {
    float t = y[c] - zf;
    qout[c] = (double)t * (double)inv;
  }
}

void oracle_quantize_row(const float* y, int D, uint8_t* codes, uint16_t* s, uint16_t* z) {
  float mn = y[0], mx = y[0];
  for (int c = 1; c < D; ++c) {
    if (y[c] < mn) mn = y[c];
    if (y[c] > mx) mx = y[c];
  }
  oracle_scale_zero(mn, mx, s, z);
  oracle_quantize_given(y, D, *s, *z, codes);
}

/* byte j = code[2j] | code[2j+1] << 4 */
void oracle_pack_row(const uint8_t* codes, int D, uint8_t* packed) {
  for (int j = 0; j < D / 2; ++j)
    packed[j] = (uint8_t)((codes[2 * j] & 15) | ((codes[2 * j + 1] & 15) << 4));
}

void oracle_unpack_row(const uint8_t* packed, int D, uint8_t* codes) {
  for (int j = 0; j < D / 2; ++j) {
    codes[2 * j] = (uint8_t)(packed[j] & 15);
    codes[2 * j + 1] = (uint8_t)(packed[j] >> 4);
  }
}

/* x^ = code * s + z, exact in fp64. */
void oracle_dequant_row(const uint8_t* packed, int D, uint16_t s, uint16_t z, double* xhat) {
  double sd = oracle_half_to_double(s), zd = oracle_half_to_double(z);
  for (int j = 0; j < D / 2; ++j) {
    xhat[2 * j] = (double)(packed[j] & 15) * sd + zd;
    xhat[2 * j + 1] = (double)(packed[j] >> 4) * sd + zd;
  }
}

/* ------------------------------------------------------------------------- */
/* Paged placement ([SAW] Abstract: the quantized rows are stored straight   */
/* into the paged cache).                                                     */
/* ------------------------------------------------------------------------- */

static size_t row_index(int64_t page, int Hkv, int h, int kv, int off) {
  return (((size_t)page * (size_t)Hkv + (size_t)h) * 2 + (size_t)kv) * ORACLE_PAGE + (size_t)off;
}

/* Byte offset of a packed row inside the cache. */
size_t oracle_cache_row_offset(int64_t page, int Hkv, int D, int h, int kv, int off) {
  return row_index(page, Hkv, h, kv, off) * (size_t)(D / 2);
}

/* Element offset of a row's s (or z) inside scales (or zeros). */
size_t oracle_scale_offset(int64_t page, int Hkv, int h, int kv, int off) {
  return row_index(page, Hkv, h, kv, off);
}

/*
 * Rotate, quantize and place every (token, kv head, K|V) row.
 * k, v: bf16 bits [T][Hkv][D]. y_out (optional, may be NULL): the rotated fp32
 * rows [T][Hkv][2][D]. Rows with slot -1 are skipped (and get no y_out change).
 * Returns 0, -1 on bad shapes, -2 if a slot lies outside [0, num_pages*16).
 */
int oracle_quant_write(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping,
                       int T, int Hkv, int D, int b, const uint32_t* signs, int64_t num_pages,
                       uint8_t* cache, uint16_t* scales, uint16_t* zeros, float* y_out) {
  if (D != 64 && D != 128) return -1;
  if (!valid_block(D, b)) return -1;
  for (int t = 0; t < T; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot == -1) continue;
    if (slot < 0 || slot >= num_pages * ORACLE_PAGE) return -2;
  }
  int bad = 0;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot == -1) continue;
    int64_t page = slot / ORACLE_PAGE;
    int off = (int)(slot % ORACLE_PAGE);
    for (int h = 0; h < Hkv; ++h) {
      for (int kv = 0; kv < 2; ++kv) {
        const uint16_t* x = (kv == 0 ? k : v) + ((size_t)t * Hkv + h) * D;
        float y[128];
        uint8_t codes[128];
        uint16_t s, z;
        if (oracle_rotate_row_signed(x, D, b, signs, y) != 0) { bad = 1; continue; }
        oracle_quantize_row(y, D, codes, &s, &z);
        oracle_pack_row(codes, D, cache + oracle_cache_row_offset(page, Hkv, D, h, kv, off));
        scales[oracle_scale_offset(page, Hkv, h, kv, off)] = s;
        zeros[oracle_scale_offset(page, Hkv, h, kv, off)] = z;
        if (y_out) memcpy(y_out + (((size_t)t * Hkv + h) * 2 + kv) * D, y, sizeof(float) * D);
      }
    }
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------- */
/* Attention over the quantized cache ([SAW] Abstract: fused attention over  */
/* the paged INT4 cache). R is orthogonal, so q.k = (Rq).(Rk), and R^T = R.   */
/* ------------------------------------------------------------------------- */

/* Brute-force softmax attention for one query over n rotated rows:
 * qr = R q; logit_t = scale * qr . Krot[t]; p = softmax(logit);
 * out = R^T (sum_t p_t Vrot[t]). n = 0 gives out = 0. All fp64. */
int oracle_attn_rows(const double* q, const double* Krot, const double* Vrot, int n,
                     int D, int b, const uint32_t* signs, double scale, double* out) {
  double qr[256], orot[256];
  if (D > 256 || !valid_block(D, b)) return -1;
  if (n == 0) {
    for (int c = 0; c < D; ++c) out[c] = 0.0;
    return 0;
  }
  oracle_rotate_f64_signed(q, D, b, signs, qr);
  double* logit = (double*)malloc(sizeof(double) * (size_t)n);
  double m = -INFINITY;
  for (int t = 0; t < n; ++t) {
    double acc = 0.0;
    for (int c = 0; c < D; ++c) acc += qr[c] * Krot[(size_t)t * D + c];
    logit[t] = scale * acc;
    if (logit[t] > m) m = logit[t];
  }
  double l = 0.0;
  for (int c = 0; c < D; ++c) orot[c] = 0.0;
  for (int t = 0; t < n; ++t) {
    double p = exp(logit[t] - m);
    l += p;
    for (int c = 0; c < D; ++c) orot[c] += p * Vrot[(size_t)t * D + c];
  }
  for (int c = 0; c < D; ++c) orot[c] /= l;
  oracle_unrotate_f64_signed(orot, D, b, signs, out);
  free(logit);
  return 0;
}

/* One (sequence, query head): gather the context's rows through the page
 * table, dequantize them, and run oracle_attn_rows. Returns -2 if a page id
 * or the context length falls outside the pool or the table. */
int oracle_decode_one(const uint16_t* q_bf16, const uint8_t* cache, const uint16_t* scales,
                      const uint16_t* zeros, const int32_t* page_table, const int32_t* context_lens,
                      int n, int hq, int Hq, int Hkv, int D, int b, const uint32_t* signs, int max_pages,
                      int64_t num_pages, double softmax_scale, double* out) {
  if (Hkv <= 0 || Hq % Hkv != 0) return -1;
  int G = Hq / Hkv;
  int h = hq / G;
  int ctx = context_lens[n];
  if (ctx < 0 || ctx > max_pages * ORACLE_PAGE) return -2;
  double scale = (softmax_scale == 0.0) ? 1.0 / sqrt((double)D) : softmax_scale;
  double q[256];
  for (int c = 0; c < D; ++c) q[c] = oracle_bf16_to_double(q_bf16[((size_t)n * Hq + hq) * D + c]);
  double* K = (double*)malloc(sizeof(double) * (size_t)(ctx > 0 ? ctx : 1) * D);
  double* V = (double*)malloc(sizeof(double) * (size_t)(ctx > 0 ? ctx : 1) * D);
  int rc = 0;
  for (int t = 0; t < ctx; ++t) {
    int64_t page = page_table[(size_t)n * max_pages + t / ORACLE_PAGE];
    int off = t % ORACLE_PAGE;
    if (page < 0 || page >= num_pages) { rc = -2; break; }
    for (int kv = 0; kv < 2; ++kv) {
      size_t si = oracle_scale_offset(page, Hkv, h, kv, off);
      oracle_dequant_row(cache + oracle_cache_row_offset(page, Hkv, D, h, kv, off), D,
                         scales[si], zeros[si], (kv == 0 ? K : V) + (size_t)t * D);
    }
  }
  if (rc == 0) rc = oracle_attn_rows(q, K, V, ctx, D, b, signs, scale, out);
  free(K);
  free(V);
  return rc;
}

/* All sequences and query heads; out is fp64 [B][Hq][D]. */
int oracle_decode_attn(const uint16_t* q_bf16, const uint8_t* cache, const uint16_t* scales,
                       const uint16_t* zeros, const int32_t* page_table, const int32_t* context_lens,
                       int B, int Hq, int Hkv, int D, int b, const uint32_t* signs, int max_pages,
                       int64_t num_pages, double softmax_scale, double* out) {
  if (D != 64 && D != 128) return -1;
  if (!valid_block(D, b)) return -1;
  if (Hkv <= 0 || Hq % Hkv != 0) return -1;
  int rc = 0;
#pragma omp parallel for schedule(dynamic) collapse(2)
  for (int n = 0; n < B; ++n)
    for (int hq = 0; hq < Hq; ++hq) {
      int r = oracle_decode_one(q_bf16, cache, scales, zeros, page_table, context_lens, n, hq,
                                Hq, Hkv, D, b, signs, max_pages, num_pages, softmax_scale,
                                out + ((size_t)n * Hq + hq) * D);
      if (r != 0) {
#pragma omp critical
        rc = r;
      }
    }
  return rc;
}

/* Threads OpenMP will use (1 when built without it). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads of the oracle's parallel loops from now on (timing legs). */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------------- */
/* OScaR (forum summary, "The OScaR Framework": V^ = Quant(S (R V)); the     */
/* OScaR abstract: per-channel quantization of K, Token Norm Imbalance, INT2) */
/* Readings: R the same block Hadamard; S the per-token factor 1 / ||R k||_2  */
/* (the norm kept as fp16, so K^ = n * dequant); K quantized per channel over */
/* the 16 tokens of a page; V token-wise (S cancels there); codes 0..3, four  */
/* per byte, lowest channel in the lowest bits; a page is quantized whole.    */
/* ------------------------------------------------------------------------- */

#define OSCAR_TOP 3

static size_t oscar_code_row(int64_t page, int Hkv, int D, int h, int kv, int t) {
  return ((((size_t)page * Hkv + h) * 2 + kv) * ORACLE_PAGE + t) * (size_t)(D / 4);
}
static size_t oscar_kmeta(int64_t page, int Hkv, int D, int h, int which) { /* which 0: s, 1: z */
  return (((size_t)page * Hkv + h) * 2 + which) * (size_t)D;
}
static size_t oscar_tmeta(int64_t page, int Hkv, int h, int which) { /* 0: K norm, 1: V s, 2: V z */
  return (((size_t)page * Hkv + h) * 3 + which) * ORACLE_PAGE;
}

/* Codes of values u for a given (s, z): round-half-even(fp32(u - z) * fp32(1/s))
 * clamped to [0, top], the same decision rule as the INT4 path. */
static uint8_t oscar_code(float u, uint16_t s, uint16_t z, int top) {
  float sf = (float)oracle_half_to_double(s);
  float zf = (float)oracle_half_to_double(z);
  float inv = (sf > 0.0f) ? 1.0f / sf : 0.0f;
  double r = nearbyint((double)(u - zf) * (double)inv);
  if (r < 0) r = 0;
  if (r > top) r = top;
  return (uint8_t)r;
}

/* Codes (one per byte, unpacked) of n values for a given (s, z), by the rule
 * of oscar_code; used to compare another implementation's codes under that
 * implementation's own (s, z). */
void oracle_oscar_codes_given(const float* u, int n, uint16_t s, uint16_t z, uint8_t* codes) {
  for (int i = 0; i < n; ++i) codes[i] = oscar_code(u[i], s, z, OSCAR_TOP);
}

/* The Omni-Token factor of a rotated row: n = ||y||_2 rounded to the nearest
 * fp16 (saturating at the largest finite one) is stored; the row is scaled
 * by S = fp32(1/n) (0 when n = 0): u = fp32(y * S). 1/n in fp64 rounded to
 * fp32 is the correctly rounded fp32 quotient, and the product of two fp32
 * values is exact in fp64, so each step rounds once. */
uint16_t oracle_oscar_token_norm(const float* y, int D, float* u) {
  double ss = 0.0;
  for (int c = 0; c < D; ++c) ss += (double)y[c] * (double)y[c];
  uint16_t n = oracle_half_round_nearest(sqrt(ss));
  if ((n & 0x7FFF) >= 0x7C00) n = 0x7BFF;
  double nd = oracle_half_to_double(n);
  float S = (nd > 0.0) ? (float)(1.0 / nd) : 0.0f;
  for (int c = 0; c < D; ++c) u[c] = (float)((double)y[c] * (double)S);
  return n;
}

/* Per-channel INT2 quantization of 16 normalized rows u[16][D]: (s_c, z_c)
 * from the channel's min and max over the 16 rows, codes packed four per byte. */
void oracle_oscar_quant_channels(const float* u, int D, uint8_t* kcodes, uint16_t* ks, uint16_t* kz) {
  uint8_t codes[256];
  for (int c = 0; c < D; ++c) {
    float mn = u[c], mx = u[c];
    for (int t = 1; t < ORACLE_PAGE; ++t) {
      if (u[t * D + c] < mn) mn = u[t * D + c];
      if (u[t * D + c] > mx) mx = u[t * D + c];
    }
    oracle_scale_zero_levels(mn, mx, OSCAR_TOP, &ks[c], &kz[c]);
  }
  for (int t = 0; t < ORACLE_PAGE; ++t) {
    for (int c = 0; c < D; ++c) codes[c] = oscar_code(u[t * D + c], ks[c], kz[c], OSCAR_TOP);
    for (int j = 0; j < D / 4; ++j)
      kcodes[(size_t)t * (D / 4) + j] = (uint8_t)(codes[4 * j] | codes[4 * j + 1] << 2 |
                                                  codes[4 * j + 2] << 4 | codes[4 * j + 3] << 6);
  }
}

/* One page of one kv head: K rows k[16][D], V rows v[16][D] (bf16) -> codes,
 * per-channel (s, z) of K, token norms of K, per-token (s, z) of V. */
int oracle_oscar_quant_page(const uint16_t* k, const uint16_t* v, int D, int b, uint8_t* kcodes,
                            uint8_t* vcodes, uint16_t* ks, uint16_t* kz, uint16_t* kn, uint16_t* vs,
                            uint16_t* vz) {
  float y[ORACLE_PAGE][256], u[ORACLE_PAGE][256];
  uint8_t codes[256];
  if (D > 256 || !valid_block(D, b)) return -1;
  float uf[ORACLE_PAGE * 256];
  for (int t = 0; t < ORACLE_PAGE; ++t) {
    oracle_rotate_row(k + (size_t)t * D, D, b, y[t]);
    kn[t] = oracle_oscar_token_norm(y[t], D, u[t]);
    for (int c = 0; c < D; ++c) uf[t * D + c] = u[t][c];
  }
  oracle_oscar_quant_channels(uf, D, kcodes, ks, kz);
  for (int t = 0; t < ORACLE_PAGE; ++t) {
    float yv[256];
    oracle_rotate_row(v + (size_t)t * D, D, b, yv);
    float mn = yv[0], mx = yv[0];
    for (int c = 1; c < D; ++c) {
      if (yv[c] < mn) mn = yv[c];
      if (yv[c] > mx) mx = yv[c];
    }
    oracle_scale_zero_levels(mn, mx, OSCAR_TOP, &vs[t], &vz[t]);
    for (int c = 0; c < D; ++c) codes[c] = oscar_code(yv[c], vs[t], vz[t], OSCAR_TOP);
    for (int j = 0; j < D / 4; ++j)
      vcodes[(size_t)t * (D / 4) + j] = (uint8_t)(codes[4 * j] | codes[4 * j + 1] << 2 |
                                                  codes[4 * j + 2] << 4 | codes[4 * j + 3] << 6);
  }
  return 0;
}

/* The write: token group g (rows 16 g .. 16 g + 15 of k and v, [T][Hkv][D]
 * bf16) fills page page_ids[g] whole, for every kv head. A page id outside
 * [0, num_pages) is skipped and makes the return -2. */
int oracle_oscar_write(const uint16_t* k, const uint16_t* v, const int32_t* page_ids, int P, int Hkv,
                       int D, int b, int64_t num_pages, uint8_t* cache, uint16_t* kmeta, uint16_t* tmeta) {
  if ((D != 64 && D != 128) || !valid_block(D, b)) return -1;
  int rc = 0;
#pragma omp parallel for schedule(static) collapse(2)
  for (int g = 0; g < P; ++g)
    for (int h = 0; h < Hkv; ++h) {
      int64_t page = page_ids[g];
      if (page < 0 || page >= num_pages) {
#pragma omp critical
        rc = -2;
        continue;
      }
      uint16_t kr[ORACLE_PAGE * 256], vr[ORACLE_PAGE * 256];
      for (int t = 0; t < ORACLE_PAGE; ++t)
        for (int c = 0; c < D; ++c) {
          size_t src = (((size_t)g * ORACLE_PAGE + t) * Hkv + h) * D + c;
          kr[t * D + c] = k[src];
          vr[t * D + c] = v[src];
        }
      oracle_oscar_quant_page(kr, vr, D, b, cache + oscar_code_row(page, Hkv, D, h, 0, 0),
                              cache + oscar_code_row(page, Hkv, D, h, 1, 0),
                              kmeta + oscar_kmeta(page, Hkv, D, h, 0), kmeta + oscar_kmeta(page, Hkv, D, h, 1),
                              tmeta + oscar_tmeta(page, Hkv, h, 0), tmeta + oscar_tmeta(page, Hkv, h, 1),
                              tmeta + oscar_tmeta(page, Hkv, h, 2));
    }
  return rc;
}

/* Dequantized rotated rows of one page-head: K^ = n (code s_c + z_c),
 * V^ = code s + z, [16][D] each, fp64. */
void oracle_oscar_dequant_page(const uint8_t* cache, const uint16_t* kmeta, const uint16_t* tmeta,
                               int64_t page, int Hkv, int D, int h, double* K, double* V) {
  const uint8_t* kc = cache + oscar_code_row(page, Hkv, D, h, 0, 0);
  const uint8_t* vc = cache + oscar_code_row(page, Hkv, D, h, 1, 0);
  const uint16_t* ks = kmeta + oscar_kmeta(page, Hkv, D, h, 0);
  const uint16_t* kz = kmeta + oscar_kmeta(page, Hkv, D, h, 1);
  const uint16_t* kn = tmeta + oscar_tmeta(page, Hkv, h, 0);
  const uint16_t* vs = tmeta + oscar_tmeta(page, Hkv, h, 1);
  const uint16_t* vz = tmeta + oscar_tmeta(page, Hkv, h, 2);
  for (int t = 0; t < ORACLE_PAGE; ++t) {
    const double n = oracle_half_to_double(kn[t]);
    for (int c = 0; c < D; ++c) {
      const int ck = (kc[(size_t)t * (D / 4) + c / 4] >> (2 * (c % 4))) & 3;
      const int cv = (vc[(size_t)t * (D / 4) + c / 4] >> (2 * (c % 4))) & 3;
      K[(size_t)t * D + c] = n * (ck * oracle_half_to_double(ks[c]) + oracle_half_to_double(kz[c]));
      V[(size_t)t * D + c] = cv * oracle_half_to_double(vs[t]) + oracle_half_to_double(vz[t]);
    }
  }
}

/* One (sequence, query head) of the OScaR decode: the context's first
 * 16 * (ctx / 16) tokens from the INT2 pages of page_table[n], the last
 * ctx % 16 from the bf16 rows of the unfinished page, k_tail / v_tail
 * [B][Hkv][16][D]; brute-force fp64 softmax attention as for INT4. */
int oracle_oscar_decode_one(const uint16_t* q_bf16, const uint8_t* cache, const uint16_t* kmeta,
                            const uint16_t* tmeta, const int32_t* page_table, const int32_t* context_lens,
                            const uint16_t* k_tail, const uint16_t* v_tail, int n, int hq, int Hq, int Hkv,
                            int D, int b, int max_pages, int64_t num_pages, double softmax_scale,
                            double* out) {
  if (Hkv <= 0 || Hq % Hkv != 0) return -1;
  const int G = Hq / Hkv, h = hq / G;
  const int ctx = context_lens[n];
  const int full = ctx / ORACLE_PAGE, tail = ctx % ORACLE_PAGE;
  if (ctx < 0 || full > max_pages) return -2;
  const double scale = (softmax_scale == 0.0) ? 1.0 / sqrt((double)D) : softmax_scale;
  double q[256];
  for (int c = 0; c < D; ++c) q[c] = oracle_bf16_to_double(q_bf16[((size_t)n * Hq + hq) * D + c]);
  const size_t rows = (size_t)(ctx > 0 ? ctx : 1);
  double* K = (double*)malloc(sizeof(double) * rows * D);
  double* V = (double*)malloc(sizeof(double) * rows * D);
  int rc = 0;
  for (int p = 0; p < full && rc == 0; ++p) {
    const int64_t page = page_table[(size_t)n * max_pages + p];
    if (page < 0 || page >= num_pages) { rc = -2; break; }
    oracle_oscar_dequant_page(cache, kmeta, tmeta, page, Hkv, D, h, K + (size_t)p * ORACLE_PAGE * D,
                              V + (size_t)p * ORACLE_PAGE * D);
  }
  for (int t = 0; t < tail && rc == 0; ++t) {
    double x[256];
    const size_t src = (((size_t)n * Hkv + h) * ORACLE_PAGE + t) * D;
    const size_t dst = ((size_t)full * ORACLE_PAGE + t) * D;
    for (int c = 0; c < D; ++c) x[c] = oracle_bf16_to_double(k_tail[src + c]);
    oracle_rotate_f64(x, D, b, K + dst);
    for (int c = 0; c < D; ++c) x[c] = oracle_bf16_to_double(v_tail[src + c]);
    oracle_rotate_f64(x, D, b, V + dst);
  }
  if (rc == 0) rc = oracle_attn_rows(q, K, V, ctx, D, b, NULL, scale, out);
  free(K);
  free(V);
  return rc;
}

int oracle_oscar_decode_attn(const uint16_t* q_bf16, const uint8_t* cache, const uint16_t* kmeta,
                             const uint16_t* tmeta, const int32_t* page_table, const int32_t* context_lens,
                             const uint16_t* k_tail, const uint16_t* v_tail, int B, int Hq, int Hkv, int D,
                             int b, int max_pages, int64_t num_pages, double softmax_scale, double* out) {
  if ((D != 64 && D != 128) || !valid_block(D, b) || Hkv <= 0 || Hq % Hkv != 0) return -1;
  int rc = 0;
#pragma omp parallel for schedule(dynamic) collapse(2)
  for (int n = 0; n < B; ++n)
    for (int hq = 0; hq < Hq; ++hq) {
      int r = oracle_oscar_decode_one(q_bf16, cache, kmeta, tmeta, page_table, context_lens, k_tail, v_tail,
                                      n, hq, Hq, Hkv, D, b, max_pages, num_pages, softmax_scale,
                                      out + ((size_t)n * Hq + hq) * D);
      if (r != 0) {
#pragma omp critical
        rc = r;
      }
    }
  return rc;
}
