/*
 * qjl.h - C ABI of the QJL KV-cache library for NVIDIA B200 (sm_100a).
 *
 * QJL ("QJL: 1-Bit Quantized JL Transform for KV Cache Quantization with Zero
 * Overhead", atlas.scime.ai summary, sections Approach / Surprising findings /
 * Limitations) stores each cached key as the sign bits of a random Gaussian JL
 * projection S k plus the key norm, projects the query with the same S but
 * WITHOUT quantising it, and scores a cached token with the unbiased
 * asymmetric estimator
 *
 *     score(q, k) = sqrt(pi/2)/m * |k_in| * <S q_in, sign(S k_in)>
 *                 + sqrt(pi/2)/m_out * |k_out| * <S_out q_out, sign(S_out k_out)>
 *
 * where k_in / q_in zero the few outlier channels of the head and k_out / q_out
 * keep only them (the outlier channels get a quantiser copy of their own).
 * Values use token-wise asymmetric min-max quantisation (Limitations: standard
 * token-wise quantisation; the min-max grid of "2 numbers out of 128 destroy
 * the entire KV cache", section "The Obvious Fix").
 *
 * Conventions shared by every entry point
 *   - All tensors are caller-owned device memory (except where "host" is said).
 *     The library never allocates per call; only qjl_init allocates (the two
 *     sketch matrices) and qjl_free releases them.
 *   - Every call is asynchronous on the caller's CUDA stream, passed as
 *     `void* stream` (a cudaStream_t; NULL = the legacy default stream), and
 *     returns once the work is enqueued. Only qjl_init, qjl_free and
 *     qjl_ctx_sketch synchronise.
 *   - 16-bit floats cross the ABI as uint16_t bit patterns (fp16 = IEEE
 *     binary16, bf16 = bfloat16).
 *   - Errors: no exception or abort crosses the ABI. A call returns a
 *     qjl_status; on failure nothing was enqueued (argument errors) or the CUDA
 *     error is reported (QJL_ERR_CUDA), and qjl_last_error() returns a message
 *     for the calling thread.
 *   - Head dimension d = 128 (QJL_ERR_UNSUPPORTED otherwise). m and m_out are
 *     multiples of 32 with m in [32, 512] and m_out in [0, 256]; n_outlier is
 *     in [0, 32] and needs m_out > 0 when positive. With n_outlier == 0 the
 *     outlier norm is 0 and the outlier term vanishes (plain QJL).
 *
 * Cache layout (struct qjl_cache). Every (sequence b, kv head h) owns a slab of
 * `cap` token slots (cap a multiple of 64), stored as cap/64 consecutive tiles
 * of 64 tokens; slab (b, h) starts at tile (b * Hkv + h) * (cap / 64). A tile
 * holds, for its 64 tokens j = 0..63 and in this order:
 *   kbits     [64][m/32]      uint32: bit i of word w = [ (S k_in)_{32w+i} >= 0 ]
 *   kbits_out [64][m_out/32]  uint32: the same for S_out k_out
 *   knorm     [64][2]         fp16: (|k_in|, |k_out|)
 *   vcode     [64][d/2]       uint8: code of dim 2i in the low nibble, 2i+1 in the high nibble;
 *                             the 16 bytes of group g (dims 32g..32g+31) of token j sit at
 *                             16-byte chunk g ^ ((j >> 1) & 3) of the token's row
 *   vsz       [64][d/32][2]   fp16: (scale, zero) per group of 32 dims
 * so a tile is 64 * (m/8 + m_out/8 + 4 + d/2 + d/8) bytes (7936 at m = 256,
 * m_out = 64, d = 128) and decode reads several tiles with one contiguous copy.
 * With 2-bit value codes (qjl_init_ex) vcode is instead [d/4 lines][68]
 * uint8: line 8g + r holds, for dims 32g + 4r .. 32g + 4r + 3, the byte of
 * each token j at offset j (the lowest dim in the lowest two bits), then 4
 * bytes of padding (2176 bytes; 6016-byte tiles at m = 256, m_out = 64).
 * qjl_cache_tile_bytes() returns the tile size. outlier_idx is a separate
 * int32 array [B, Hkv, n_outlier] of ascending channel indices.
 * Both pointers must be 16-byte aligned. Decode copies whole tiles; slots past
 * a sequence's length take no part in its result, whatever they hold.
 */
#ifndef QJL_H
#define QJL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct qjl_ctx qjl_ctx; /* opaque: owns the device copies of S and S_out */

typedef enum {
  QJL_OK = 0,
  QJL_ERR_ARG = 1,         /* invalid argument (shape, pointer, alignment, size) */
  QJL_ERR_CUDA = 2,        /* a CUDA runtime call or kernel launch failed */
  QJL_ERR_UNSUPPORTED = 3, /* valid in principle, not implemented (e.g. d != 128) */
  QJL_ERR_OOM = 4,         /* qjl_init could not allocate the sketch matrices */
  QJL_ERR_WORKSPACE = 5,   /* workspace missing or smaller than the *_workspace_bytes query */
  QJL_ERR_TIMEOUT = 6      /* a wait inside a decode kernel ran out (reported by qjl_decode_workspace_status) */
} qjl_status;

typedef enum { QJL_BF16 = 0, QJL_FP32 = 1 } qjl_dtype;

typedef enum {
  QJL_PREFILL = 0, /* select the outlier channels from the given keys, write outlier_idx, then sketch */
  QJL_APPEND = 1   /* use the outlier_idx already in the cache (chosen at prefill) */
} qjl_mode;

typedef struct {
  int32_t* outlier_idx; /* [B, Hkv, n_outlier] */
  void* tiles;          /* [B, Hkv, cap / 64] tiles of qjl_cache_tile_bytes() bytes */
  int B;                /* sequences */
  int Hkv;              /* key/value heads */
  int cap;              /* token capacity of each (sequence, kv head) slab, a multiple of 64 */
} qjl_cache;

/*
 * qjl_init - create a context: draw S (m x d) and S_out (m_out x d) and copy
 * them to the current device.
 *   Definition (QJL summary, Approach: a random Gaussian JL matrix): entries
 *   i.i.d. N(0,1). Generator: SplitMix64 stream `seed` (Steele, Lea & Flood
 *   2014); element e of S (row-major) uses outputs 2e+1, 2e+2 and element e of
 *   S_out uses outputs 2^62+2e+1, 2^62+2e+2, each mapped to (0,1) as
 *   ((x >> 12) + 1/2) * 2^-52; Box-Muller cosine branch
 *   sqrt(-2 ln u1) cos(2 pi u2); rounded to the nearest bf16 (ties to even).
 *   One (S, S_out) pair serves all sequences and heads.
 *   Arguments: d = 128; m, m_out, n_outlier as in the file comment.
 *   Ownership: *out receives a context that the caller releases with qjl_free.
 *   Errors: QJL_ERR_ARG, QJL_ERR_UNSUPPORTED, QJL_ERR_OOM, QJL_ERR_CUDA; *out is
 *   set to NULL on failure. Synchronises the device.
 */
qjl_status qjl_init(uint64_t seed, int d, int m, int m_out, int n_outlier, qjl_ctx** out);

/*
 * qjl_init_ex - qjl_init with a choice of value code width: value_bits = 4
 * (what qjl_init sets) or 2 (levels zero + c * scale, c = 0..3, scale =
 * fp16((max - min) / 3): the 2-bit grid of "2 numbers out of 128 destroy the
 * entire KV cache", section "The Obvious Fix"). Every call with this context
 * uses that width: the cache tile layout (2-bit vcode section in the file
 * comment), qjl_quantize_values, and the decode entry points.
 * Errors: as qjl_init; QJL_ERR_ARG for another value_bits.
 */
qjl_status qjl_init_ex(uint64_t seed, int d, int m, int m_out, int n_outlier, int value_bits, qjl_ctx** out);

/* qjl_free - release a context (NULL is a no-op). Synchronises the device. */
void qjl_free(qjl_ctx* ctx);

/* qjl_last_error - message of the last failed call on this thread ("" if none). */
const char* qjl_last_error(void);

/*
 * qjl_sketch_host - the same S and S_out that qjl_init would draw, written to
 * HOST buffers as bf16 bit patterns (S: m*d, S_out: m_out*d entries; S_out may
 * be NULL when m_out == 0). Needs no GPU.
 */
qjl_status qjl_sketch_host(uint64_t seed, int d, int m, int m_out, uint16_t* S, uint16_t* S_out);

/* qjl_ctx_sketch - copy the context's device S / S_out to HOST buffers (bf16 bits). Synchronises. */
qjl_status qjl_ctx_sketch(const qjl_ctx* ctx, uint16_t* S, uint16_t* S_out);

/* qjl_ctx_guard - the relative guard band used by the key sketch (see qjl_quantize_keys). */
float qjl_ctx_guard(const qjl_ctx* ctx);

/*
 * qjl_cache_tile_bytes - bytes of one 64-token cache tile (layout in the file
 * comment) for head dimension d and sketch sizes m, m_out; 0 when the sizes are
 * not ones qjl_init accepts. Host-only, needs no GPU.
 */
size_t qjl_cache_tile_bytes(int d, int m, int m_out);
/* The same for value_bits (4 or 2) codes; 0 for an invalid shape. */
size_t qjl_cache_tile_bytes_ex(int d, int m, int m_out, int value_bits);

/*
 * qjl_quantize_keys_workspace_bytes - device workspace that qjl_quantize_keys
 * needs for B sequences x Hkv heads in QJL_PREFILL mode (0 for QJL_APPEND).
 */
size_t qjl_quantize_keys_workspace_bytes(const qjl_ctx* ctx, int B, int Hkv, qjl_mode mode);

/*
 * qjl_quantize_keys - QJL key quantisation of T new tokens per (sequence, kv head).
 *   Computes (QJL summary, Approach): in QJL_PREFILL mode first the outlier
 *   channels of each (b, h) - the n_outlier channels with the largest sum over
 *   the T given tokens of k_c^2, exact ties to the lower index, written to
 *   cache->outlier_idx in ascending order; then for every token
 *     kbits     = sign bits of S k_in   (k_in: k with the outlier channels zeroed)
 *     kbits_out = sign bits of S_out k_out (k_out: only the outlier channels)
 *     knorm     = fp16(|k_in|), fp16(|k_out|) (norms computed in fp64)
 *   (all written into the token's tile slot). A sign bit is 1 when the
 *   projection is >= 0. Projections are computed in
 *   fp32; any projection whose magnitude is below guard * |k_part| (guard from
 *   qjl_ctx_guard, above the fp32 rounding bound) is recomputed in fp64, so the
 *   bits equal those of the exact projection except where |S k| is within about
 *   1e-13 |k| of zero.
 *   K: device, dtype `dtype`, element (b, h, t, c) at
 *      K[b*stride_b + h*stride_h + t*stride_t + c] (element strides; c contiguous).
 *   t_start: device int32 [B] or NULL (= 0): token t of sequence b is written at
 *      cache position t_start[b] + t. Positions >= cap are skipped (not written).
 *   workspace: device, at least qjl_quantize_keys_workspace_bytes bytes (PREFILL).
 *   Errors: QJL_ERR_ARG (shapes, NULL or misaligned pointers, T < 0),
 *   QJL_ERR_WORKSPACE, QJL_ERR_CUDA. T == 0 enqueues nothing.
 */
qjl_status qjl_quantize_keys(qjl_ctx* ctx, const qjl_cache* cache, const void* K, qjl_dtype dtype, int T,
                             int64_t stride_b, int64_t stride_h, int64_t stride_t, const int32_t* t_start,
                             qjl_mode mode, void* workspace, size_t workspace_bytes, void* stream);

/*
 * qjl_quantize_values - token-wise asymmetric quantisation of T new value
 * vectors per (sequence, kv head), groups of 32 dims, with the context's
 * value_bits b (4, or 2 from qjl_init_ex).
 *   Computes (QJL summary, Limitations; min-max grid of "2 numbers out of 128",
 *   "The Obvious Fix"): per group, zero = fp16(min), scale =
 *   fp16((max-min)/(2^b - 1)), code = clamp(rint((v - zero)/scale), 0, 2^b - 1),
 *   each step an IEEE fp32 operation rounded to nearest even; code = 0 when
 *   scale == 0.
 *   V, strides, t_start: as K in qjl_quantize_keys.
 *   Errors: QJL_ERR_ARG, QJL_ERR_CUDA. T == 0 enqueues nothing.
 */
qjl_status qjl_quantize_values(qjl_ctx* ctx, const qjl_cache* cache, const void* V, qjl_dtype dtype, int T,
                               int64_t stride_b, int64_t stride_h, int64_t stride_t, const int32_t* t_start,
                               void* stream);

/*
 * qjl_decode_workspace_bytes - device workspace that qjl_decode_attention and
 * qjl_decode_step need for B sequences, Hq query heads, Hkv kv heads and up to
 * T cached tokens: a 256-byte header, one merge counter per (sequence, kv head),
 * a slot per (sequence, kv head) for a prepared query sketch and the partial
 * results of the (sequence, kv head) pairs whose tokens are split between
 * thread blocks.
 * 0 for an invalid shape.
 */
size_t qjl_decode_workspace_bytes(const qjl_ctx* ctx, int B, int Hq, int Hkv, int T);

/*
 * qjl_decode_attention - one decode step of attention over the QJL cache.
 *   Computes for every sequence b and query head h (kv head h / (Hq/Hkv)):
 *     score_t = the QJL estimate of <q, k_t> (formula in the file comment,
 *               QJL summary, Approach), for the cached tokens t < len_b
 *     p       = softmax(sm_scale * score)   (online, split over tokens)
 *     O[b,h]  = sum_t p_t * (zero + code * scale) of token t's values.
 *   Q: device [B, Hq, d], dtype `dtype`, contiguous.
 *   T: tokens in every sequence, or the maximum when seqlens is given;
 *      seqlens: device int32 [B] or NULL; len_b = min(seqlens[b], T) (clamped
 *      at 0). An empty sequence gives O[b,h] = 0.
 *   sm_scale: logit scale; <= 0 selects 1/sqrt(d).
 *   O: device fp32 [B, Hq, d], written.
 *   scores: device fp32 [B, Hq, T] or NULL; when given, score_t (before
 *      sm_scale) is written for t < len_b.
 *   workspace: device, qjl_decode_workspace_bytes bytes, 16-byte aligned,
 *      zero-filled once before its first use. Every call leaves its header
 *      and counters at zero again, so consecutive calls reuse one workspace
 *      without clearing it; after a wait ran out, qjl_decode_workspace_status
 *      clears them. Calls that share one workspace must not overlap on the GPU.
 *   Launch: one persistent kernel, at most one block per SM; the blocks split
 *      the cache tiles of all (sequence, kv head) pairs into equal contiguous
 *      shares, build the projected query sketches of the pairs in their share
 *      and stream it; they never wait for one another. Every wait inside is bounded
 *      (qjl_set_wait_limit); when one runs out, the outputs the block owns
 *      become NaN and qjl_decode_workspace_status reports QJL_ERR_TIMEOUT.
 *   Errors: QJL_ERR_ARG, QJL_ERR_WORKSPACE, QJL_ERR_CUDA.
 */
qjl_status qjl_decode_attention(qjl_ctx* ctx, const qjl_cache* cache, const void* Q, qjl_dtype dtype, int Hq,
                                int T, const int32_t* seqlens, float sm_scale, float* O, float* scores,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * qjl_decode_step - a whole decode step in one launch: append each sequence's
 * new token to the cache, then attend over the cache including it.
 *   Computes (QJL summary, Approach: keys are sketched as they are generated,
 *   with the outlier channels chosen at prefill; the query is projected
 *   without quantisation): for every sequence b and kv head h the new key
 *   K_new[b, h] is sketched exactly as qjl_quantize_keys(QJL_APPEND) would
 *   (sign bits of S k_in and S_out k_out, fp16 norms from fp64) and the new
 *   value V_new[b, h] quantised exactly as qjl_quantize_values would, into
 *   cache slot len_b; then O is what qjl_decode_attention computes over the
 *   len_b + 1 tokens.
 *   K_new, V_new: device, dtype `dtype` (the same as Q), element (b, h, c) at
 *      K_new[b * k_stride_b + h * k_stride_h + c] (element strides, c
 *      contiguous, 16-byte aligned rows), likewise V_new.
 *   T, seqlens: the lengths BEFORE the step, as in qjl_decode_attention; T
 *      must be at most cap - 1 and seqlens[b] <= T.
 *   scores: device fp32 [B, Hq, T + 1] or NULL (t < len_b + 1 written).
 *   Other arguments, workspace and errors: as qjl_decode_attention.
 */
qjl_status qjl_decode_step(qjl_ctx* ctx, const qjl_cache* cache, const void* Q, const void* K_new, int64_t k_stride_b,
                           int64_t k_stride_h, const void* V_new, int64_t v_stride_b, int64_t v_stride_h,
                           qjl_dtype dtype, int Hq, int T, const int32_t* seqlens, float sm_scale, float* O,
                           float* scores, void* workspace, size_t workspace_bytes, void* stream);

/*
 * qjl_decode_attention_partial - this rank's part of a context-parallel decode:
 * qjl_decode_attention over the shard of the context that `cache` holds,
 * reported before normalisation so that the shards of several ranks combine.
 *   Computes ("2 numbers out of 128 destroy the entire KV cache", "The Memory
 *   Math": a long context outgrows one device, so its tokens are split over
 *   ranks; softmax is exp(x - M) / sum exp(x - M) for any M >= max x, "Your
 *   Brain Already Runs on 1-Bit Keys", "Why Truncation Kills"): with logits
 *   x_t = sm_scale * score_t * log2(e) over the shard's tokens,
 *     ML_part[b,h] = (M, L), M = max_t x_t, L = sum_t 2^(x_t - M)
 *     O_part[b,h]  = sum_t 2^(x_t - M) * (zero + code * scale) of token t.
 *   An empty shard gives (-inf, 0) and a zero O_part.
 *   O_part: device fp32 [B, Hq, d], 16-byte aligned; ML_part: device fp32
 *   [B, Hq, 2], 8-byte aligned. Other arguments, launch and errors: as
 *   qjl_decode_attention (scores, when given, are the shard's own).
 */
qjl_status qjl_decode_attention_partial(qjl_ctx* ctx, const qjl_cache* cache, const void* Q, qjl_dtype dtype, int Hq,
                                        int T, const int32_t* seqlens, float sm_scale, float* O_part, float* ML_part,
                                        float* scores, void* workspace, size_t workspace_bytes, void* stream);

/*
 * qjl_merge_partials - the attention output from R ranks' parts (the exchange
 * step of a context-parallel decode happens before: every rank gathers all
 * parts, e.g. with an all-gather).
 *   Computes, per row (sequence, query head), with M = max_r M_r:
 *     O = sum_r 2^(M_r - M) O_parts[r] / sum_r 2^(M_r - M) L_r
 *   (zero when every part is empty; NaN when any part holds NaN).
 *   O_parts: device fp32; rank r's parts [rows, d] start at
 *   O_parts + r * o_stride (floats; 16-byte aligned, o_stride a multiple of
 *   4 and >= rows * d). ML_parts: device fp32; rank r's [rows, 2] at
 *   ML_parts + r * ml_stride (8-byte aligned, ml_stride even and >= 2 rows).
 *   Two arrays [R, rows, d] and [R, rows, 2] (o_stride = rows * d,
 *   ml_stride = 2 rows) and one packed buffer per rank both fit. These are
 *   what qjl_decode_attention_partial writes, with rows = B * Hq.
 *   O: device fp32 [rows, d], written.
 *   Errors: QJL_ERR_ARG (R < 1, rows < 0, NULL, misaligned or overlapping
 *   strides), QJL_ERR_CUDA. rows == 0 enqueues nothing.
 */
qjl_status qjl_merge_partials(const float* O_parts, int64_t o_stride, const float* ML_parts, int64_t ml_stride, int R,
                              int64_t rows, float* O, void* stream);

/*
 * qjl_set_wait_limit - the time limit (ns, > 0) of every wait inside the decode
 * kernels launched with this context from now on (default 2 s).
 */
qjl_status qjl_set_wait_limit(qjl_ctx* ctx, uint64_t ns);

/*
 * qjl_decode_workspace_status - synchronise `stream` and report whether a wait
 * inside a decode kernel that used this workspace (shape B, Hq, Hkv) ran out:
 * QJL_OK, or QJL_ERR_TIMEOUT, in which case the outputs of that call hold NaN
 * and the workspace header and counters are cleared so that the next call
 * starts clean. QJL_ERR_CUDA if the read fails.
 */
qjl_status qjl_decode_workspace_status(const qjl_ctx* ctx, void* workspace, int B, int Hq, int Hkv, void* stream);

/*
 * ---------------------------------------------------------------------------
 * Comparison kernels: decode over an unquantised bf16 cache and over an FP8
 * cache, on the same shapes as the QJL path ("2 numbers out of 128 destroy
 * the entire KV cache" (Towards AI), "The Memory Math"; TurboQuant slides,
 * section 05: FP8 halves the cache with hardware-native support).
 * ---------------------------------------------------------------------------
 */
typedef enum { QJL_KV_BF16 = 0, QJL_KV_FP8_E4M3 = 1, QJL_KV_MINMAX2 = 2, QJL_KV_MINMAX4 = 3 } qjl_kv_format;

/*
 * qjl_minmax_quantize - the token-wise min-max quantiser of "2 numbers out of
 * 128 destroy the entire KV cache", section "The Obvious Fix", for keys or
 * values of a comparison cache: per group of 32 dims, zero = fp16(min),
 * scale = fp16((max - min) / (2^bits - 1)), code = clamp(rint((x - zero) /
 * scale), 0, 2^bits - 1), every step one IEEE fp32 operation (as the QJL
 * value codes; scale == 0 gives code 0).
 *   X: device [n_rows, d] (d = 128), dtype QJL_BF16 or QJL_FP32, contiguous,
 *   16-byte aligned. bits: 2 or 4. out: device [n_rows][d*bits/8 + 16] bytes,
 *   16-byte aligned: a row's codes (the lowest dim in the lowest bits of each
 *   byte), then its four (scale, zero) fp16 pairs.
 *   Errors: QJL_ERR_ARG, QJL_ERR_CUDA. n_rows == 0 enqueues nothing.
 */
qjl_status qjl_minmax_quantize(const void* X, qjl_dtype dtype, int64_t n_rows, int bits, uint8_t* out, void* stream);

/*
 * qjl_fp8_quantize - FP8 E4M3 codes of n values: code = the E4M3 value
 * nearest to fp32(x / scale) (IEEE fp32 division; ties to even; magnitudes
 * beyond 448 saturate to +-448). E4M3 is the OCP "FN" variant: bias 7, 3
 * mantissa bits, no infinities.
 *   X: device, dtype QJL_BF16 or QJL_FP32, n elements, 16-byte aligned;
 *   n: a multiple of 8; scale > 0; out: device, n bytes, 8-byte aligned.
 *   Errors: QJL_ERR_ARG, QJL_ERR_CUDA. n == 0 enqueues nothing.
 */
qjl_status qjl_fp8_quantize(const void* X, qjl_dtype dtype, int64_t n, float scale, uint8_t* out, void* stream);

/*
 * qjl_exact_decode_workspace_bytes - device workspace of qjl_exact_decode for
 * B sequences, Hq query heads and up to T tokens (per-chunk partial outputs).
 */
size_t qjl_exact_decode_workspace_bytes(int B, int Hq, int T);

/*
 * qjl_exact_decode - decode attention over a plain KV cache.
 *   Computes for every sequence b and query head h (kv head h / (Hq/Hkv)):
 *     O[b,h] = softmax(sm_scale * K_hat[b,kv] q) V_hat[b,kv] over the first
 *     len_b tokens, with K_hat = K (QJL_KV_BF16) or K_hat = code * k_scale,
 *     V_hat = code * v_scale (QJL_KV_FP8_E4M3, codes from qjl_fp8_quantize),
 *     or K_hat, V_hat = zero + code * scale (QJL_KV_MINMAX2 / 4, rows from
 *     qjl_minmax_quantize).
 *   K, V: device [B, Hkv, cap] rows of the format (bf16 [d], E4M3 bytes [d],
 *      or min-max rows of d*bits/8 + 16 bytes), contiguous, 16-byte aligned.
 *      k_scale, v_scale: FP8 only (ignored otherwise).
 *   Q: device [B, Hq, d], dtype `q_dtype` (QJL_BF16 or QJL_FP32), contiguous.
 *   T <= cap: tokens per sequence, or the maximum when seqlens (device int32
 *   [B], clamped to [0, T]) is given. sm_scale <= 0 selects 1/sqrt(d).
 *   O: device fp32 [B, Hq, d], written (zero for an empty sequence).
 *   workspace: device, qjl_exact_decode_workspace_bytes(B, Hq, T) bytes,
 *   16-byte aligned, no initial contents needed.
 *   Launch: blocks of 256 tokens of one (sequence, kv head) pair, then the
 *   merge of qjl_merge_partials over the blocks.
 *   Errors: QJL_ERR_ARG, QJL_ERR_UNSUPPORTED (Hq / Hkv not 1, 2, 4 or 8),
 *   QJL_ERR_WORKSPACE, QJL_ERR_CUDA.
 */
qjl_status qjl_exact_decode(qjl_kv_format format, const void* K, const void* V, float k_scale, float v_scale, int B,
                            int Hq, int Hkv, int cap, int T, const void* Q, qjl_dtype q_dtype,
                            const int32_t* seqlens, float sm_scale, float* O, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * qjl_decode_attention_static - qjl_decode_attention without a caller workspace
 * and without any allocation. The pages have no counterpart: this entry point
 * exists for callers that cannot allocate device memory, such as a plugin
 * inside a host runtime that owns all of the device's memory and forbids its
 * plugins to allocate, or a latency-critical caller that cannot accept the
 * implicit synchronisation of cudaMalloc/cudaFree.
 *   Computes exactly what qjl_decode_attention computes, with the same
 *   arguments except the workspace, and the same results.
 *   Scratch: a fixed array of QJL_STATIC_SCRATCH_BYTES inside the library,
 *   held by every GPU that loads the library until the process exits. A call
 *   whose qjl_decode_workspace_bytes exceeds it is rejected with
 *   QJL_ERR_WORKSPACE (use qjl_decode_attention with a caller workspace).
 *   Each call clears the header and counters at the start of the array
 *   (cudaMemsetAsync on the caller's stream) before the decode kernel; the
 *   rest is fully written before it is read. The context's device must be
 *   the current device (else QJL_ERR_ARG).
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture begins.
 *   Sharing: every call uses the same array, so calls whose GPU work overlaps
 *   (other streams, other host threads) race and corrupt each other's results;
 *   the caller must serialise them.
 *   Errors: as qjl_decode_attention, plus QJL_ERR_WORKSPACE for the size limit
 *   and QJL_ERR_CUDA if the set-up or the clear fails. Allocates nothing.
 */
#define QJL_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)
qjl_status qjl_decode_attention_static(qjl_ctx* ctx, const qjl_cache* cache, const void* Q, qjl_dtype dtype,
                                       int Hq, int T, const int32_t* seqlens, float sm_scale, float* O,
                                       float* scores, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QJL_H */
