/*
 * kvq.h - C ABI of the rotated-INT4 paged KV cache (the data-parallel hot
 * path of SAW-INT4: token-wise INT4 quantization with a block-diagonal
 * Hadamard rotation, written into a paged KV cache and read back by a fused
 * decode-attention kernel).
 *
 * Sources (web pages, cited by title and section):
 *  [SAW]   "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World
 *          LLM Serving", Abstract (arXiv 2604.19157 mirror): token-wise INT4
 *          after a Hadamard rotation applied block by block; one kernel
 *          rotates, quantizes and stores into the paged cache; attention
 *          is computed on the quantized cache in the kernel that reads it.
 *  [OSCAR] "OScaR: Occam's Razor for Extreme KV Cache Quantization in LLMs"
 *          (forum summary), section "The OScaR Framework": V^ = Quant(S.(R.V)),
 *          rotate first, then scale, then quantize.
 * The pages fix no layout, rounding rule or API; every such choice below is a
 * reading of this library and is stated where it is made.
 *
 * Conventions shared by every entry point
 *  - All pointers named "device" are CUDA device pointers; the caller owns
 *    every buffer, and no entry point allocates device memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous on that stream.
 *  - Argument errors are reported synchronously, before anything is launched.
 *  - Range errors found on the device (a slot or page id outside the pool, a
 *    context longer than the page table) skip the offending row or page and
 *    record a status in a per-device error word; a bounded wait that ran out
 *    records KVQ_ERR_TIMEOUT there. kvq_get_device_error() reads and clears it.
 *
 * Data layout (this library's reading; the pages only say "paged"):
 *  - page size P = 16 tokens (KVQ_PAGE_SIZE).
 *  - cache : uint8  [num_pages][Hkv][2][P][D/2]  (index 2: 0 = K, 1 = V)
 *            one row = D 4-bit codes of one (token, kv head, K|V);
 *            byte j of a row = code[2j] | (code[2j+1] << 4)  (low nibble = even
 *            channel).
 *  - scales: fp16   [num_pages][Hkv][2][P]   the per-row step s
 *  - zeros : fp16   [num_pages][Hkv][2][P]   the per-row offset z
 *            dequantized value = code * s + z.
 *  - slot  : page * 16 + offset within the page.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_PAGE_SIZE 16
#define KVQ_ABI_VERSION 6

typedef enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned buffer */
  KVQ_ERR_UNSUPPORTED = 2,  /* head_dim, block size or GQA group not built */
  KVQ_ERR_OUT_OF_RANGE = 3, /* device-side: slot/page id/context outside the pool */
  KVQ_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required */
  KVQ_ERR_TIMEOUT = 5,      /* device-side: a bounded wait ran out */
  KVQ_ERR_CUDA = 6          /* a CUDA runtime call or launch failed */
} kvq_status;

/* Shapes of one kv_quant_write call. */
typedef struct kvq_write_desc {
  int32_t num_tokens;   /* T >= 0 new tokens */
  int32_t num_kv_heads; /* Hkv >= 1 */
  int32_t head_dim;     /* D: 64 or 128 */
  int32_t page_size;    /* must be KVQ_PAGE_SIZE */
  int32_t num_pages;    /* pages in the pool; valid slots are [0, num_pages*16) */
  /* Randomized Hadamard: bit c of hadamard_signs[c / 32] set negates channel
   * c before the transform, R = H_b diag(sigma) / sqrt(b) (orthogonal for any
   * signs). All zero: the plain rotation. Must be zero when hadamard_block is
   * 0 and above bit D - 1; a decode of the cache must use the same mask. */
  uint32_t hadamard_signs[4];
} kvq_write_desc;

/* Shapes of one paged_decode_attn_int4 call. */
typedef struct kvq_attn_desc {
  int32_t batch;             /* B sequences, one query token each */
  int32_t num_q_heads;       /* Hq; query head i reads kv head i / (Hq/Hkv) */
  int32_t num_kv_heads;      /* Hkv; Hq/Hkv must be 1, 2, 4 or 8 */
  int32_t head_dim;          /* D: 64 or 128 */
  int32_t page_size;         /* must be KVQ_PAGE_SIZE */
  int32_t num_pages;         /* pages in the pool */
  int32_t max_pages_per_seq; /* columns of page_table */
  int32_t hadamard_block;    /* the block b the cache was written with (0 = none) */
  float softmax_scale;       /* 0 means 1/sqrt(head_dim) */
  int32_t out_dtype;         /* 0 = fp32 output, 1 = bf16 output */
  int32_t flags;             /* 0 or KVQ_ATTN_INPUTS_READY */
  /* Optional host copy of context_lens (B values), or NULL. When given, the
   * work is split per sequence in proportion to its length (longer sequences
   * get more CTAs, the longest start first) instead of evenly; the kernel
   * still reads the lengths from the device array, so a host copy that is
   * out of date costs balance, never correctness. Read during the call only. */
  const int32_t* context_lens_host;
  /* The sign mask the cache was written with (see kvq_write_desc): q is
   * rotated by R and the output by R^T = diag(sigma) H_b / sqrt(b). */
  uint32_t hadamard_signs[4];
} kvq_attn_desc;

/*
 * Every kernel of this library is launched as a programmatic dependent
 * launch: its CTAs may start while the previous kernel on the stream is
 * finishing, and wait for that kernel to complete before touching memory it
 * may have written. KVQ_ATTN_INPUTS_READY tells paged_decode_attn_int4 that
 * q, page_table and context_lens were not written by the kernel launched
 * just before it on the stream (they may be written by anything earlier:
 * every kernel of this library waits for its predecessor before letting its
 * own successor start), so it may read them and rotate q while that kernel
 * is still running. kv_quant_write followed by paged_decode_attn_int4 on
 * the same stream qualifies when q, the page table and the context lengths
 * came from before the write.
 */
#define KVQ_ATTN_INPUTS_READY 1

/*
 * kv_quant_write - fused rotate + token-wise INT4 quantize + paged store
 * ([SAW] Abstract: one kernel rotates, quantizes and stores into the paged
 * cache; [OSCAR] "The OScaR Framework": rotate first, then quantize).
 *
 * For every new token t, kv head h and tensor X in {K, V}, with row x = X[t,h,:]:
 *   1. y = R x, R = diag(H_b/sqrt(b), ...) over contiguous b-channel blocks,
 *      H_b the Sylvester Hadamard matrix in natural order
 *      (H[i][j] = (-1)^popcount(i & j)); b = 0 means R = I (plain INT4).
 *      y is fp32.
 *   2. z = the largest fp16 <= min(y); s = the smallest fp16 >= 0 with
 *      15*s + z >= max(y) (so every element lies in [z, z + 15 s]).
 *   3. code = round-half-even( fp32(y - z) * fp32(1/s) ), in [0, 15]; s = 0
 *      gives code 0.
 *   4. the packed row, s and z go to slot slot_mapping[t]; slot -1 skips t.
 *
 * k, v         : device, bf16 [T][Hkv][D], contiguous, 16-byte aligned.
 * slot_mapping : device, int64 [T]; -1 = skip; any other value outside
 *                [0, num_pages*16) skips the token and records
 *                KVQ_ERR_OUT_OF_RANGE in the device error word.
 * page_table   : accepted for signature compatibility with the decode call and
 *                not read; placement is decided by slot_mapping alone. May be NULL.
 * cache, scales, zeros : device, layouts above, 16-byte aligned.
 * hadamard_block : 0, 32, 64 or 128, and at most D (with desc->hadamard_signs,
 *                the randomized rotation H_b diag(sigma) / sqrt(b)).
 * desc         : host pointer to the shapes.
 * Inputs must be finite and their rotated values must lie within the fp16
 * range (|y| <= 65504); rows outside it get infinite or NaN s/z.
 * num_tokens = 0 launches nothing and returns KVQ_OK (pointers may then be NULL).
 * Returns KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED or KVQ_ERR_CUDA.
 */
kvq_status kv_quant_write(const void* k, const void* v, const int64_t* slot_mapping,
                          const int32_t* page_table, uint8_t* cache, void* scales,
                          void* zeros, int32_t hadamard_block,
                          const kvq_write_desc* desc, void* stream);

/*
 * kvq_attn_workspace_size - bytes of device workspace paged_decode_attn_int4
 * needs for these shapes (0 when the call needs none) on this library's
 * current device (see kvq_set_device). The value depends on the shapes and on
 * how many decode CTAs that device holds at once (the split count fills them
 * in one wave). Returns SIZE_MAX when the shapes are invalid or no device can
 * be queried.
 *
 * The workspace holds the per-split partial results (fp32, each word stored
 * bit-inverted so that a zero word means "not written yet", plus one state
 * word per row used to hand a merge over to another split); it must be
 * zero-filled before its first use, and every call leaves it zero-filled
 * again - except after a call whose bounded waits ran out (kvq_get_device_error
 * returns KVQ_ERR_TIMEOUT): words that arrived after the wait gave up may
 * remain, so clear the workspace before using it again.
 *
 * The split merge needs no co-residency of the launch's CTAs: a merger that
 * waits long (about 0.2 ms) for a split that has not written hands its rows
 * over to that split and exits, so a decode also completes when other
 * streams' kernels hold most SMs.
 */
size_t kvq_attn_workspace_size(const kvq_attn_desc* desc);

/*
 * paged_decode_attn_int4 - one decode step of attention over the INT4 cache
 * ([SAW] Abstract: attention computed on the quantized cache in the kernel
 * that reads it; the rotation is orthogonal,
 * so q.k = (Rq).(Rk) and the output is R^T sum_t p_t (R v_t), with R^T = R
 * because H_b/sqrt(b) is symmetric and its own inverse).
 *
 * For sequence n and query head i (kv head h = i / (Hq/Hkv)), over the
 * context_lens[n] cached tokens t with page = page_table[n][t/16]:
 *   k^_t = code*s + z (per row), likewise v^_t, both in rotated space;
 *   logit_t = softmax_scale * (R q) . k^_t;  p = softmax(logit);
 *   out[n][i] = R (sum_t p_t v^_t).      context_lens[n] = 0 gives out = 0.
 *
 * q            : device, bf16 [B][Hq][D], contiguous, 16-byte aligned.
 * cache, scales, zeros : device, as written by kv_quant_write with the same
 *                hadamard_block.
 * page_table   : device, int32 [B][max_pages_per_seq]; entries past the
 *                context are not read. An id outside [0, num_pages) makes the
 *                page count as empty and records KVQ_ERR_OUT_OF_RANGE.
 * context_lens : device, int32 [B]; a value above max_pages_per_seq*16 is
 *                clamped and records KVQ_ERR_OUT_OF_RANGE.
 * out          : device, [B][Hq][D], fp32 or bf16 (desc->out_dtype).
 * workspace    : device, at least kvq_attn_workspace_size(desc) bytes, 16-byte
 *                aligned, zero-filled before its first use (each call leaves
 *                it zero-filled; after KVQ_ERR_TIMEOUT clear it again); may be
 *                NULL when that size is 0. Calls that overlap on the GPU must
 *                use different workspaces.
 * batch = 0 launches nothing and returns KVQ_OK (pointers may then be NULL).
 * Returns KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_WORKSPACE
 * or KVQ_ERR_CUDA.
 */
kvq_status paged_decode_attn_int4(const void* q, const uint8_t* cache,
                                  const void* scales, const void* zeros,
                                  const int32_t* page_table,
                                  const int32_t* context_lens, void* out,
                                  void* workspace, size_t workspace_bytes,
                                  const kvq_attn_desc* desc, void* stream);

/*
 * paged_decode_append_attn_int4 - one decode step that also appends the
 * step's new token: kv_quant_write of k_new/v_new at slot_mapping followed by
 * paged_decode_attn_int4 over the contexts that include it, in one launch
 * ([SAW] Abstract: the rotate-quantize-store step and the attention over
 * the paged cache, here in a single kernel).
 *
 * For sequence n the new token is position context_lens[n] - 1: its slot
 * (page * 16 + offset) must be page_table[n][(ctx - 1) / 16] * 16 +
 * (ctx - 1) % 16, or -1 for "no new token" (the sequence is then decoded as
 * paged_decode_attn_int4 would). Its K and V rows are rotated, quantized
 * and stored exactly as kv_quant_write defines them (codes may differ from
 * a kv_quant_write call only where both are within the rounding of a code
 * boundary: this path rotates with fp32 butterflies), and the attention uses
 * the stored values.
 *
 * k_new, v_new : device, bf16 [B][Hkv][D], contiguous, 16-byte aligned.
 * slot_mapping : device, int64 [B], 8-byte aligned.
 * cache, scales, zeros : device, written at the new slots, read as in
 *                paged_decode_attn_int4.
 * Every other argument as for paged_decode_attn_int4 (the same workspace
 * size applies). A slot that does not match its sequence's last position,
 * or a new token with context length 0, is not stored and records
 * KVQ_ERR_OUT_OF_RANGE. Returns as paged_decode_attn_int4.
 */
kvq_status paged_decode_append_attn_int4(const void* q, const void* k_new,
                                         const void* v_new,
                                         const int64_t* slot_mapping,
                                         uint8_t* cache, void* scales, void* zeros,
                                         const int32_t* page_table,
                                         const int32_t* context_lens, void* out,
                                         void* workspace, size_t workspace_bytes,
                                         const kvq_attn_desc* desc, void* stream);

/*
 * paged_prefill_attn_int4 - chunked-prefill attention over the INT4 cache
 * ([SAW] Abstract: attention on the quantized paged cache, aimed at serving
 * many requests at once): many queries per sequence, so
 * QK^T and PV run as dense tcgen05 MMAs.
 *
 * Sequence n's chunk is its last L_n = q_start[n+1] - q_start[n] context
 * tokens, already stored by kv_quant_write; query token i of the chunk (row
 * q_start[n] + i of q) is position context_lens[n] - L_n + i and attends to
 * positions 0 .. that position (causal):
 *   out[row][head] = R^T sum_t p_t v^_t, p = softmax over those positions of
 *   softmax_scale * (R q[row][head]) . k^_t      (k^, v^ as in paged_decode_attn_int4).
 *
 * q            : device, bf16 [Tq][Hq][D], D = 64 or 128 (as for the decode),
 *                16-byte aligned.
 * cache, scales, zeros, page_table, desc : as for paged_decode_attn_int4
 *                (desc->context_lens_host and desc->flags are not used).
 * context_lens : device, int32 [B], each >= its chunk length.
 * q_start      : device, int32 [B + 1], non-decreasing, q_start[0] = 0.
 * max_q_len    : host, the largest chunk length (sizes the grid).
 * out          : device, [Tq][Hq][D], fp32 or bf16 (desc->out_dtype).
 * A context shorter than its chunk or longer than max_pages_per_seq * 16, or a
 * chunk longer than max_q_len, records KVQ_ERR_OUT_OF_RANGE and leaves that
 * sequence's rows unwritten.
 * Returns KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED or KVQ_ERR_CUDA.
 */
kvq_status paged_prefill_attn_int4(const void* q, const uint8_t* cache,
                                   const void* scales, const void* zeros,
                                   const int32_t* page_table,
                                   const int32_t* context_lens,
                                   const int32_t* q_start, int32_t max_q_len,
                                   void* out, const kvq_attn_desc* desc, void* stream);

/*
 * paged_decode_attn_int4_static_ws - the same decode step as
 * paged_decode_attn_int4, for callers that are not allowed to allocate device
 * memory. Examples: a plug-in hosted by a serving runtime that owns all GPU
 * memory through its own pool and forbids raw cudaMalloc, or a latency-bound
 * path where an allocation (which may synchronize the device) is unacceptable.
 * The paper has no counterpart; this is a deployment convenience.
 *
 * Instead of a caller-provided workspace, the split-K scratch lives in a
 * fixed device array of KVQ_STATIC_WORKSPACE_BYTES inside this library (every
 * GPU that loads the library holds it until the process exits). The caller
 * still passes all inputs and outputs, exactly as for paged_decode_attn_int4.
 *  - The first call on a device (and the first after that device's context
 *    changed, e.g. after cudaDeviceReset) looks up that array's device
 *    address; make that first call before any stream capture.
 *  - The array starts zeroed and every call leaves it zeroed (each merge
 *    clears the words it read). After a call whose bounded waits ran out,
 *    kvq_get_device_error (which reports KVQ_ERR_TIMEOUT) clears the array on
 *    that device with an asynchronous memset on its stream - nothing else
 *    can, since callers cannot reach the array.
 *  - All calls share the one array per device: calls that overlap on the GPU
 *    (other streams, other host threads) race and give wrong results.
 *  - The uniform split plan needs up to resident CTAs x (query rows per CTA)
 *    x (D + 4) x 4 bytes; shapes whose plan needs more than the array holds
 *    are rejected with KVQ_ERR_WORKSPACE before anything is launched (on a
 *    148-SM B200: up to 2.5 MB when 4 kv heads of GQA 4 share a CTA, so such
 *    shapes are rejected; the benchmark's shapes need at most 0.6 MB). With
 *    desc->context_lens_host, the per-sequence plan runs when its partials
 *    fit, else the uniform plan.
 * No allocation of any kind is made. Returns the same statuses as
 * paged_decode_attn_int4.
 */
#define KVQ_STATIC_WORKSPACE_BYTES (2u * 1024u * 1024u)
kvq_status paged_decode_attn_int4_static_ws(const void* q, const uint8_t* cache,
                                            const void* scales, const void* zeros,
                                            const int32_t* page_table,
                                            const int32_t* context_lens, void* out,
                                            const kvq_attn_desc* desc, void* stream);

/* ------------------------------------------------------------------------ */
/* OScaR variant: INT2 codes, K quantized per channel after a per-token scale */
/* ------------------------------------------------------------------------ */

/* Shapes of one kv_quant_write_oscar call. */
typedef struct kvq_oscar_write_desc {
  int32_t num_groups;   /* P >= 0 token groups of 16, each filling one whole page */
  int32_t num_kv_heads; /* Hkv >= 1 */
  int32_t head_dim;     /* D: 128 */
  int32_t num_pages;    /* pages in the pool */
} kvq_oscar_write_desc;

/*
 * kv_quant_write_oscar - the OScaR write (OScaR forum summary, "The OScaR
 * Framework": V^ = Quant(S (R V)); OScaR abstract: per-channel quantization
 * of K, Token Norm Imbalance, INT2): for every token group g and kv head h,
 * rows 16 g .. 16 g + 15 of k and v become page page_ids[g]:
 *   K: y_t = R k_t; n_t = fp16(||y_t||_2) (saturating); S_t = fp32(1/n_t)
 *      (0 when n_t = 0), u_t = fp32(y_t * S_t); per channel c over the
 *      page's 16 tokens z_c = RD16(min_t u_tc), s_c = the smallest fp16 with
 *      3 s_c + z_c >= max_t u_tc; code = rint(fp32(u - z_c) * fp32(1/s_c))
 *      in 0..3;
 *      dequantized K^_tc = n_t (code s_c + z_c).
 *   V: y_t = R v_t, per token z = RD16(min), s = the smallest fp16 with
 *      3 s + z >= max, codes as for K; V^ = code s + z.
 * A sequence's unfinished last page is not written here: the caller keeps
 * its rows in bf16 and passes them to paged_decode_attn_oscar.
 *
 * k, v         : device, bf16 [16 P][Hkv][D], contiguous, 16-byte aligned.
 * page_ids     : device, int32 [P]; an id outside [0, num_pages) skips that
 *                group and records KVQ_ERR_OUT_OF_RANGE.
 * cache        : device, uint8 [num_pages][Hkv][2][16][D/4]: K codes, then V
 *                codes, four per byte, the lowest channel in the lowest bits.
 * kmeta        : device, fp16 [num_pages][Hkv][2][D]: K per-channel s, then z.
 * tmeta        : device, fp16 [num_pages][Hkv][3][16]: K token norms, V s, V z.
 * hadamard_block : 0, 32, 64 or 128.
 * Returns KVQ_OK, KVQ_ERR_INVALID_ARG (null or misaligned pointers, bad
 * shapes), KVQ_ERR_UNSUPPORTED (D != 128, bad block) or KVQ_ERR_CUDA.
 */
kvq_status kv_quant_write_oscar(const void* k, const void* v, const int32_t* page_ids, uint8_t* cache,
                                void* kmeta, void* tmeta, int32_t hadamard_block,
                                const kvq_oscar_write_desc* desc, void* stream);

/* Shapes of one paged_decode_attn_oscar call (fields as in kvq_attn_desc). */
typedef struct kvq_oscar_attn_desc {
  int32_t batch;
  int32_t num_q_heads;       /* Hq / Hkv must be 1, 2 or 4 */
  int32_t num_kv_heads;
  int32_t head_dim;          /* 128 */
  int32_t num_pages;
  int32_t max_pages_per_seq; /* columns of page_table: full pages only */
  int32_t hadamard_block;
  float softmax_scale;       /* 0 means 1/sqrt(head_dim) */
  int32_t out_dtype;         /* 0 = fp32, 1 = bf16 */
} kvq_oscar_attn_desc;

/*
 * kvq_oscar_workspace_size - bytes of device workspace paged_decode_attn_oscar
 * needs on this library's current device (the splits' partial results; no
 * zero-filling needed). SIZE_MAX for invalid shapes.
 */
size_t kvq_oscar_workspace_size(const kvq_oscar_attn_desc* desc);

/*
 * paged_decode_attn_oscar - one decode step over the OScaR cache. For
 * sequence n with ctx = context_lens[n]: tokens 0 .. 16 (ctx / 16) - 1 are
 * the INT2 pages page_table[n][0 .. ctx / 16 - 1]; the last ctx % 16 tokens
 * are rows 0 .. ctx % 16 - 1 of k_tail[n][h] / v_tail[n][h] (bf16, exact).
 *   logit_t = softmax_scale * q . k_t, p = softmax(logit),
 *   out[n][i] = sum_t p_t v_t, with k_t, v_t the dequantized rows rotated
 *   back (R^T K^, R^T V^) or the bf16 rows of the unfinished page.
 * q            : device, bf16 [B][Hq][D], 16-byte aligned.
 * cache, kmeta, tmeta : as written by kv_quant_write_oscar with the same block.
 * page_table   : device, int32 [B][max_pages_per_seq]; only the first
 *                ctx / 16 entries of row n are read. An id outside
 *                [0, num_pages) skips that page (its tokens get no weight)
 *                and records KVQ_ERR_OUT_OF_RANGE.
 * context_lens : device, int32 [B]; above max_pages_per_seq * 16 + 15 it is
 *                clamped and records KVQ_ERR_OUT_OF_RANGE.
 * k_tail, v_tail : device, bf16 [B][Hkv][16][D].
 * out          : device, [B][Hq][D] fp32 or bf16.
 * workspace    : device, >= kvq_oscar_workspace_size(desc) bytes, 16-byte
 *                aligned (contents need not be zero).
 * Two launches (the split decode, then a merge kernel). Returns KVQ_OK,
 * KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_WORKSPACE or KVQ_ERR_CUDA.
 */
kvq_status paged_decode_attn_oscar(const void* q, const uint8_t* cache, const void* kmeta, const void* tmeta,
                                   const int32_t* page_table, const int32_t* context_lens, const void* k_tail,
                                   const void* v_tail, void* out, void* workspace, size_t workspace_bytes,
                                   const kvq_oscar_attn_desc* desc, void* stream);

/*
 * kvq_get_device_error - synchronizes `stream`, then returns and clears the
 * current device's error word (KVQ_OK when no kernel recorded an error).
 * When the word is KVQ_ERR_TIMEOUT it also clears the static split-K array
 * of paged_decode_attn_int4_static_ws on that device (a memset on `stream`,
 * waited for), since late words may remain there.
 * Returns KVQ_ERR_CUDA if the synchronization itself fails.
 */
kvq_status kvq_get_device_error(void* stream);

/*
 * kvq_static_workspace_nonzero - a test hook with no counterpart in the
 * pages: the number of non-zero bytes in the static split-K array of
 * paged_decode_attn_int4_static_ws on the current device (copied to the host,
 * synchronously), or SIZE_MAX when it cannot be read.
 */
size_t kvq_static_workspace_nonzero(void);

/*
 * kvq_set_device - make `device` this library's current CUDA device (the
 * device kvq_attn_workspace_size plans for). The other calls select the
 * device that owns their cache buffer by themselves. Returns KVQ_OK,
 * KVQ_ERR_INVALID_ARG for a negative ordinal, or KVQ_ERR_CUDA.
 */
kvq_status kvq_set_device(int32_t device);

/*
 * kvq_selftest_bounded_wait - the failure path of the library's bounded
 * waits, for tests: on the current device, one warp runs a wait on a
 * condition that nothing completes, which = 0: an mbarrier wait as in the
 * write and prefill pipelines (gives up after ~4096 rounds of at most ~1 ms);
 * which = 1: the decode's split-merge poll of a word that stays zero (gives
 * up after 2^20 polls 64 ns apart). The wait runs out, records
 * KVQ_ERR_TIMEOUT in the device error word and the kernel returns; nothing
 * faults and the context stays usable. Not part of the hot path. Returns
 * KVQ_OK once launched, KVQ_ERR_INVALID_ARG for another `which`, or
 * KVQ_ERR_CUDA.
 */
kvq_status kvq_selftest_bounded_wait(int32_t which, void* stream);

/*
 * kvq_selftest_occupy - a test hook with no counterpart in the pages: launch
 * `ctas` CTAs (1..65535) on `stream`, each holding most of an SM's shared
 * memory, that wait on the global timer for `microseconds` (0..1000000) and
 * then end on their own. Tests use it to keep SMs busy while a decode runs on
 * another stream. No hot-path call uses it.
 * Returns KVQ_ERR_INVALID_ARG on out-of-range arguments, KVQ_ERR_CUDA when
 * the launch fails.
 */
kvq_status kvq_selftest_occupy(int32_t ctas, int32_t microseconds, void* stream);

/* Static, human-readable name of a status value (never NULL). */
const char* kvq_status_string(int32_t status);

/* KVQ_ABI_VERSION of the built library. */
int32_t kvq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
