/*
 * nsn.h -- C ABI of the NSNQuant KV-cache hot path on B200 (sm_100a).
 *
 * The method (sources named by page title and section):
 *   [TS] "NSNQuant: A Double Normalization Approach for Calibration-Free Low-Bit
 *        Vector Quantization of KV Cache", technical summary (gist.science):
 *        Metodologia 1 (Normalize-Shift-Normalize), 2 (Hadamard transform),
 *        3 (vector quantization, codebook from k-means on randn, adaptive scale),
 *        4 (KIVI-style residual window; attention scores that fold in s1, s2, o;
 *        custom CUDA kernels for Hadamard, VQ and dequantization).
 *   [GH] "NSNQuant" repository README: Overview; Codebook tuning (--abs 2-bit
 *        codebook over absolute values, 1-bit codebook).
 *
 * Every token vector x (head_dim 128) of K or V is rotated, y = H x (orthonormal
 * Sylvester Hadamard, natural order), then NSN is applied per block of 128
 * tokens of one (batch, kv-head):
 *   s1 = ||y||/sqrt(d), n1 = y/s1;  o = mean over the block of n1;  z = n1 - o;
 *   s2 = ||z||/sqrt(d), u = z/s2.
 * u is split into 16 sub-vectors of 8; each gets the nearest codeword (squared
 * Euclidean, ties to the lowest index) of one 256 x 8 codebook:
 *   1-bit mode: code over the signed codebook C;
 *   2-bit mode: 8 sign bits (bit i set iff u_i < 0) + code over |u| against an
 *               absolute-value codebook A (entries >= 0).
 * Adaptive scale (flag): alpha = ||u||^2 / (u . u_hat) (1 if u . u_hat <= 0) is
 * folded into the stored s2.  The token is reconstructed as
 *   x_hat = H^T ((u_hat * s2 + o) * s1).
 *
 * Conventions for every entry point:
 *   - All tensors are caller-owned.  The library never allocates or frees memory.
 *   - Device pointers must be 16-byte aligned; row strides are in ELEMENTS and
 *     must keep every 128-element row 16-byte aligned.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t passed as
 *     void*; NULL = legacy default stream).  No call synchronizes.
 *   - Arguments are validated on the host before any launch; an invalid call
 *     returns an error code and launches nothing (the cache is untouched).
 *     A failed launch returns NSN_ERR_CUDA.
 *   - fp16 values are stored as IEEE binary16 bit patterns (uint16_t).
 */
#ifndef NSN_H_
#define NSN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NSN_HEAD_DIM 128 /* d */
#define NSN_SUB_DIM 8    /* sub-vector length */
#define NSN_N_SUB 16     /* sub-vectors per token */
#define NSN_N_CODES 256  /* codebook entries (8-bit code) */
#define NSN_BLOCK 128    /* tokens per NSN block (channel-mean scope) */
#define NSN_MAX_GQA 8    /* query heads per kv-head supported by decode */

typedef enum {
  NSN_OK = 0,
  NSN_ERR_INVALID_ARG = 1, /* null pointer, bad size, stride or alignment */
  NSN_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. window not in {0,128}) */
  NSN_ERR_WORKSPACE = 3,   /* decode workspace too small */
  NSN_ERR_CUDA = 4,        /* a CUDA launch failed; see nsn_last_cuda_error() */
  NSN_ERR_STATE = 5        /* the cache is in a state the call cannot use */
} nsn_status;

typedef enum { NSN_MODE_1BIT = 1, NSN_MODE_2BIT = 2 } nsn_mode;

typedef enum { NSN_DTYPE_F32 = 0, NSN_DTYPE_BF16 = 1, NSN_DTYPE_F16 = 2 } nsn_dtype;

/*
 * Compressed cache of one tensor (K or V) of one layer.  All pointers are
 * device pointers owned by the caller.  Layout (row-major, per (b, h) contiguous):
 *   codes    uint8  [batch][n_kv_heads][capacity][16]   the codes of the even sub-vectors, then
 *                                                       of the odd ones: byte i < 8 holds the
 *                                                       code of sub-vector 2i, byte 8+i that
 *                                                       of sub-vector 2i+1
 *   signs    uint8  [batch][n_kv_heads][capacity][16]   2-bit mode only (NULL in 1-bit): the
 *                                                       128 sign bits of a token as eight
 *                                                       little-endian 16-bit fields; field i
 *                                                       (bytes 2i, 2i+1) bit 15-s is set iff
 *                                                       u[8s+i] < 0 (s = sub-vector 0..15)
 *   norms    fp16   [batch][n_kv_heads][capacity][2]    (s1, alpha*s2) per token
 *   means    fp16   [batch][n_kv_heads][capacity/128][128]   o of each block (rotated domain)
 *   window   fp16   [batch][n_kv_heads][window][128]    residual tokens, original domain
 *   n_quant  int32  [batch][n_kv_heads]                 quantized tokens (multiple of 128
 *                                                       when window > 0)
 *   n_window int32  [batch][n_kv_heads]                 tokens in the residual window
 *   status   int32  [1] or NULL                         device error bits, OR-ed by kernels:
 *                                                       1 = capacity overflow on flush,
 *                                                       2 = decode copy timeout,
 *                                                       4 = ragged prefill length out of range,
 *                                                       8 = chunked-prefill query not in the window
 * capacity must be a positive multiple of 128.  window must be 0 (quantize every
 * token, no append) or 128 (KIVI-style residual of one block).
 *
 * Double quantization (double_quant = 1; [TS] Metodologia 3: the NSN byproducts s1
 * and o are stored in 4 bits).  s1 and o are stored as 4-bit levels of 16 uniform
 * steps between the fp16-rounded min and max of their group (the tokens of a
 * 128-token block for s1, the 128 channels of a block for o); level =
 * round-half-even((x - lo) / step) clamped to 0..15, step = (hi - lo) / 15, and the
 * value read back is lo + level * step.  The NSN itself uses the exact values.  The
 * buffers then change to:
 *   norms     fp16   [batch][n_kv_heads][capacity]          alpha*s2 per token
 *   means     uint8  [batch][n_kv_heads][capacity/128][64]   o levels, channel 2c in the
 *                                                           low nibble of byte c
 *   s1_levels uint8  [batch][n_kv_heads][capacity/2]         s1 levels, token 2t in the
 *                                                           low nibble of byte t
 *   dq_params fp16   [batch][n_kv_heads][capacity/128][8]    (s1 lo, s1 hi, o lo, o hi, 0, 0,
 *                                                           0, 0) of each block
 * With double_quant = 0, s1_levels and dq_params are unused (may be NULL).  The K and
 * V caches given to one append or decode call must both use it or both not.
 *
 * Cosine assignment (assign = 1; [TS] Metodologia 3: the codebook is fine-tuned for
 * the cosine distance between a vector and its quantized version, [GH] Codebook
 * tuning "--method learned"): every sub-vector a (u, or |u| in 2-bit mode) takes the
 * codeword of largest cosine similarity, code = argmax_k a . c_k / ||c_k|| (ties to
 * the lowest index; a zero codeword scores 0), instead of the nearest one.  The
 * stored scalars, the adaptive scale and the decode are unchanged (they use the
 * codebook as given).  assign applies to every quantization of the cache (prefill
 * and flushes); the K and V caches may differ in it.
 */
typedef struct {
  int32_t batch;
  int32_t n_kv_heads;
  int32_t capacity;
  int32_t window;
  int32_t mode;         /* nsn_mode */
  int32_t scale_adjust; /* 1: fold the adaptive scale into the stored s2 */
  uint8_t* codes;
  uint8_t* signs;
  uint16_t* norms;
  uint16_t* means;
  uint16_t* window_buf;
  int32_t* n_quant;
  int32_t* n_window;
  int32_t* status;
  int32_t double_quant; /* 1: s1 and o stored in 4 bits (layout above) */
  uint8_t* s1_levels;
  uint16_t* dq_params;
  int32_t assign;       /* codeword choice of the quantizer: 0 = nearest (squared Euclidean),
                           1 = largest cosine similarity a.c/||c|| (see below) */
} nsn_cache;

/* Byte sizes of the buffers of an nsn_cache with the given shape. */
typedef struct {
  size_t codes, signs, norms, means, window_buf, n_quant, n_window, s1_levels, dq_params;
} nsn_cache_sizes;

/* Library version (major*10000 + minor*100 + patch). */
int nsn_version(void);

/* Human-readable name of a status code (static string). */
const char* nsn_status_string(int status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* nsn_last_cuda_error(void);

/*
 * Fills *out with the byte size of each cache buffer.  signs is 0 in 1-bit mode,
 * window_buf is 0 when window == 0, s1_levels and dq_params are 0 unless
 * double_quant.  Returns NSN_ERR_INVALID_ARG on a bad shape.
 */
nsn_status nsn_cache_buffer_sizes(int batch, int n_kv_heads, int capacity, int window, int mode,
                                  int double_quant, nsn_cache_sizes* out);

/*
 * Builds the codebook on the HOST (no GPU use).  [TS] Metodologia 3: k-means on
 * synthetic standard-normal samples; [GH] Codebook tuning: --abs builds it over
 * absolute values.
 *   seed       stream seed.  Samples are standard normals from Philox4x64-10 (Salmon
 *              et al., SC'11) with key (seed, 0x4E534E51) and counter (j,0,0,0) for
 *              block j; each 64-bit word w -> u = ((w >> 12) + 0.5) * 2^-52; the pairs
 *              (u0,u1), (u2,u3) -> Box-Muller normals (r cos 2 pi u_b, r sin 2 pi u_b),
 *              r = sqrt(-2 ln u_a).  Normal i*dim + c is component c of sample i.
 *   n_samples  >= n_codes.   n_codes, dim > 0.   abs_mode: 1 = use |samples|.
 *   iters      Lloyd iterations (>= 0) from the first n_codes samples as initial
 *              centroids; ties go to the lowest centroid; empty clusters keep theirs.
 *   out        host float[n_codes * dim], row-major; every value is rounded to the
 *              nearest fp16-representable number (so the fp32 quantizer and the fp16
 *              decode read identical codewords).
 */
nsn_status nsn_build_codebook_host(uint64_t seed, int n_samples, int n_codes, int dim,
                                   int abs_mode, int iters, float* out);

/*
 * Cosine-tuned codebook ([TS] Metodologia 3: the k-means codebook is fine-tuned to
 * minimise the cosine distance between vectors and their quantized versions; [GH]
 * Codebook tuning, "--method learned").  The pages give no procedure; this one
 * alternates, cosine_iters times:
 *   1. assign every sample to its nearest codeword (squared Euclidean, lowest index
 *      on ties), as the quantizer assigns;
 *   2. turn codeword c to the normalised sum of its members' unit vectors (the
 *      direction that maximises their summed cosine) and give it the mean projection
 *      of its members on that direction (the least-squares length).  A codeword with
 *      no members, a zero direction sum or a non-positive mean projection is kept.
 * Samples, k-means start (kmeans_iters Lloyd iterations) and the fp16 rounding of
 * the result are those of nsn_build_codebook_host; cosine_iters = 0 gives its result.
 */
nsn_status nsn_build_codebook_cosine_host(uint64_t seed, int n_samples, int n_codes, int dim,
                                          int abs_mode, int kmeans_iters, int cosine_iters,
                                          float* out);

/*
 * Prefill: quantizes n_tokens tokens of every (b, h) of x into a FRESH cache
 * (counters are overwritten).  [TS] Metodologia 1-3 (+ 4 for the residual split).
 *   x          device, dtype element type, token (b, t, h) row at
 *              x + b*stride_b + t*stride_t + h*stride_h (elements), 128 contiguous values.
 *              May be NULL when n_tokens == 0 (only the counters are reset then).
 *   n_tokens   L >= 0, same for every batch row.  With window 128 the first
 *              Q = 128*floor((L-1)/128) tokens are quantized in blocks of 128 and the
 *              remaining L-Q (1..128) are copied (as fp16) to the window; with
 *              window 0 all L are quantized (the last block may be partial).
 *              Requires Q <= capacity.
 *   codebook   device float[256*8] (signed codebook in 1-bit, absolute in 2-bit).
 * Stored values: codes/signs bit-exact to the definition: the nearest codeword of
 * the fp32 sub-vector (scores on the tensor cores, the winner located by the best
 * group and column maxima of the scores, and every near tie within the error bounds
 * re-decided exactly in fp64; ties to the lowest index), s1, alpha*s2 and o rounded
 * to fp16.  Any fp32
 * codebook works; one of fp16-representable values keeps the decision bound tightest.
 */
nsn_status nsn_quantize_kv(nsn_cache* cache, const void* x, int dtype, int64_t stride_b,
                           int64_t stride_t, int64_t stride_h, int n_tokens,
                           const float* codebook, void* stream);

/*
 * Ragged prefill: nsn_quantize_kv with one prompt length per batch row.  Sequence
 * b takes lengths[b] tokens and is split by the same rule as a common length L
 * ([TS] Metodologia 1-4 per sequence; the pages' runs use one sequence at a time).
 *   lengths     device int32[batch], read by the kernels (no host synchronisation).
 *               An entry outside [0, max_tokens] is treated as 0 and sets status
 *               bit 4 (that sequence is left empty).
 *   max_tokens  host bound on the lengths; it must satisfy the capacity rule that
 *               n_tokens satisfies in nsn_quantize_kv.  Rows t >= lengths[b] of
 *               sequence b are never read, so x may be padded or shorter per row.
 * Everything else (x layout, codebook, stored values) is as in nsn_quantize_kv; with
 * every length equal to L the cache bytes equal those of nsn_quantize_kv(..., L, ...).
 */
nsn_status nsn_quantize_kv_ragged(nsn_cache* cache, const void* x, int dtype, int64_t stride_b,
                                  int64_t stride_t, int64_t stride_h, const int32_t* lengths,
                                  int max_tokens, const float* codebook, void* stream);

/*
 * Decode-time append of one new token per (b, h) to K and V ([TS] Metodologia 4,
 * residual: when the window is full it is flushed -- quantized as one block and
 * appended -- and emptied).  For every (b, h) of each cache: if n_window == 128 the
 * window is quantized into block n_quant/128 (n_quant += 128, n_window = 0; if that
 * block does not fit in capacity the token is not appended and status bit 1 is set);
 * then the new token is stored (as fp16) at window[n_window] and n_window += 1.
 *   k_new, v_new  device [b][h][128] rows at base + b*stride_b + h*stride_h (elements).
 *   cb_k, cb_v    device float[256*8] codebooks of the K and V caches.
 * Both caches must have window == 128 and the same batch / n_kv_heads.
 */
nsn_status nsn_append_residual(nsn_cache* k_cache, nsn_cache* v_cache, const void* k_new,
                               const void* v_new, int dtype, int64_t stride_b, int64_t stride_h,
                               const float* cb_k, const float* cb_v, void* stream);

/*
 * Workspace bytes that nsn_decode_attention needs for these caches and n_q_heads.
 * The workspace starts with 2 * batch * n_kv_heads 32-bit merge counters (padded
 * to 256 bytes); the decode partials follow.
 */
size_t nsn_decode_workspace_bytes(const nsn_cache* k_cache, int n_q_heads);

/*
 * Decode attention of one query token per (b, q-head) over the compressed cache
 * followed by the residual window ([TS] Metodologia 4: scores with s1, s2, o folded
 * in).  q-head j uses kv-head j / (n_q_heads / n_kv_heads).
 *   q              device dtype [b][n_q_heads][128], row at q + b*q_stride_b + j*q_stride_h.
 *   n_q_heads      multiple of n_kv_heads, n_q_heads / n_kv_heads <= 8.
 *   softmax_scale  score = softmax_scale * q . k (1/sqrt(128) for standard attention).
 *   cb_k, cb_v     device float[256*8] codebooks; decode reads them rounded to fp16.
 *   out            device float [b][n_q_heads][128].  A (b, h) with no tokens at all
 *                  yields zeros.
 *   workspace      device, >= nsn_decode_workspace_bytes() bytes, 256-byte aligned,
 *                  caller-owned.  It must be zero-filled before its first use with
 *                  caches of a given batch x n_kv_heads (its leading counters must be
 *                  zero); every completed call leaves those counters zero again, so
 *                  later calls need no clearing.  Calls sharing one workspace must not
 *                  overlap on the GPU.
 * One kernel launch: the quantized blocks of each (b, kv-head) are dealt out to
 * splits, the last split also attends the window, and the thread block of the
 * split that completes a (b, kv-head, head group) last merges the partials into
 * `out`.  Status bit 2 of
 * k_cache->status is set if a copy into shared memory did not complete in time
 * (the affected outputs are then not meaningful).
 */
nsn_status nsn_decode_attention(const nsn_cache* k_cache, const nsn_cache* v_cache,
                                const void* q, int dtype, int n_q_heads, int64_t q_stride_b,
                                int64_t q_stride_h, float softmax_scale, const float* cb_k,
                                const float* cb_v, float* out, void* workspace, size_t ws_bytes,
                                void* stream);

/*
 * Chunked-prefill ("extend") attention over the compressed cache ([TS] Metodologia 4:
 * the quantized part and the full-precision residual window; [GH] Note on the split
 * between them at prefill).  After a chunk of n_queries tokens has been added to the
 * cache (they are the last n_queries tokens of every sequence and all sit in the
 * residual window), query i of the chunk (position P - n_queries + i, P = n_quant +
 * n_window) attends every quantized token and the window tokens up to its own:
 *   out[b][i][h] = softmax_scale-softmax attention of q[b][i][h] over
 *                  { k_hat_t : t < n_quant } U { window slots 0 .. n_window - n_queries + i }
 * with the decode's arithmetic (nsn_decode_attention) for each query.
 *   q          device, dtype, query (b, i, h) at q + b*q_stride_b + i*q_stride_t +
 *              h*q_stride_h (elements), 128 contiguous values; all strides multiples of
 *              16 bytes.
 *   n_queries  1 .. window (the caches' window must be 128).
 *   out        device float [batch][n_queries][n_q_heads][128].
 *   workspace  as nsn_decode_attention (nsn_decode_workspace_bytes; zero-filled before
 *              its first use), reused by every query of the chunk.
 * Runs as n_queries passes of the decode kernel (one per query, stream-ordered), each
 * with the window shortened by the tokens that follow its query.  A sequence whose
 * window holds fewer than n_queries tokens sets status bit 8 (its queries then see
 * fewer window tokens).  Errors as nsn_decode_attention; NSN_ERR_UNSUPPORTED for a
 * cache without a window.
 */
nsn_status nsn_extend_attention(const nsn_cache* k_cache, const nsn_cache* v_cache, const void* q, int dtype,
                                int n_q_heads, int n_queries, int64_t q_stride_b, int64_t q_stride_t,
                                int64_t q_stride_h, float softmax_scale, const float* cb_k, const float* cb_v,
                                float* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * Pre-RoPE keys ([TS] Metodologia 4: NSN is applied to the keys BEFORE the rotary
 * position embedding).  The K cache then holds pre-RoPE keys -- both the quantized
 * part and the fp16 window, filled by the same nsn_quantize_kv* / append calls --
 * and the decode rotates every key at its position before the score:
 *   score(q_h, key t) = softmax_scale * q_h . R_pos(t) k_hat_t,
 *   pos(t) = t for quantized token t, n_quant + w for window slot w,
 *   R_pos rotates each pair of dims (i, i + 64), i < 64 ("rotate-half" pairing), by
 *   the angle pos * inv_freq[i]:  (x_i, x_{i+64}) -> (x_i c - x_{i+64} s, x_{i+64} c + x_i s).
 * q is the already-rotated query (the caller applies RoPE to it at its own position).
 * Values are not rotated.  Arguments as nsn_decode_attention, plus
 *   inv_freq       device float[64], 16-byte aligned: theta_i (e.g. base^(-2i/128);
 *                  any table, so scaled-RoPE variants work).  Angles are formed as
 *                  pos * theta_i in fp64 and reduced to [-pi, pi] before sin/cos.
 *   workspace      >= nsn_decode_rope_workspace_bytes() bytes, same zero-fill rule as
 *                  nsn_decode_attention (its leading part is that workspace; the K
 *                  logits follow: batch * n_q_heads * (capacity + window) fp32).
 * Two kernel launches: the K logits of every key (the rotated key is formed in
 * registers from the compressed cache: H u_hat on the tensor cores, the NSN terms and
 * the rotation in fp32), then the decode over those logits and the V cache.
 * Errors as nsn_decode_attention (NSN_ERR_WORKSPACE if ws_bytes is too small).
 */
size_t nsn_decode_rope_workspace_bytes(const nsn_cache* k_cache, int n_q_heads);
nsn_status nsn_decode_attention_rope(const nsn_cache* k_cache, const nsn_cache* v_cache,
                                     const void* q, int dtype, int n_q_heads, int64_t q_stride_b,
                                     int64_t q_stride_h, float softmax_scale, const float* inv_freq,
                                     const float* cb_k, const float* cb_v, float* out,
                                     void* workspace, size_t ws_bytes, void* stream);

/*
 * Allocation-free variant of nsn_decode_attention.  The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory when they
 * decode -- code running inside an allocator or memory-pool callback, frameworks
 * that reserve all device memory up front, hosts that forbid cudaMalloc after
 * start-up.  It takes the same arguments as nsn_decode_attention minus the
 * workspace and computes the same result; its decode partials go to a fixed
 * file-scope device array of NSN_DECODE_SCRATCH_BYTES bytes instead, and its merge
 * counters to a second one of NSN_DECODE_STATIC_COUNTERS 32-bit words (both
 * zero-filled at load); every GPU that loads the library holds them until the
 * process exits.
 *   - Nothing is allocated or freed (no cudaMalloc / cudaFree / allocating library).
 *   - Returns NSN_ERR_WORKSPACE if this shape's partials need more than
 *     NSN_DECODE_SCRATCH_BYTES or 2 * batch * n_kv_heads > NSN_DECODE_STATIC_COUNTERS.
 *   - The first call on a device (in a given CUDA context) resolves the arrays' device
 *     addresses (with that device current) and caches them; make that first call before
 *     any stream capture.  With lazy module loading (the CUDA default) that first call
 *     can also be the moment the module holding the arrays is loaded, which is when
 *     their NSN_DECODE_SCRATCH_BYTES + 4 * NSN_DECODE_STATIC_COUNTERS bytes of device
 *     memory are taken: a caller that reserves all device memory, or that must not
 *     allocate at all later on, makes one warm-up call (or sets CUDA_MODULE_LOADING=EAGER)
 *     before it does so.  Later calls allocate nothing.
 *   - All calls share the one array: two calls whose work overlaps on the GPU (e.g. on
 *     different streams without ordering between them) race on it and must not be
 *     issued.  Every partial the kernel reads is written earlier in the same call and
 *     each completed call leaves the counters it used at zero, so nothing needs
 *     clearing between calls.
 */
#define NSN_DECODE_SCRATCH_BYTES (8u << 20)
#define NSN_DECODE_STATIC_COUNTERS 16384u
nsn_status nsn_decode_attention_static(const nsn_cache* k_cache, const nsn_cache* v_cache, const void* q,
                                       int dtype, int n_q_heads, int64_t q_stride_b, int64_t q_stride_h,
                                       float softmax_scale, const float* cb_k, const float* cb_v, float* out,
                                       void* stream);

/*
 * Double quantization of a codebook's entries ([TS] Metodologia 3: the codebook
 * entries are stored in 4 bits too).  In place on a HOST float array of n_values:
 * 16 uniform levels between the fp16-rounded min and max of all entries, level =
 * round-half-even((x - lo) / step) clamped to 0..15, step = (hi - lo) / 15; every
 * entry becomes the fp16 rounding of lo + level * step.  The result is an ordinary
 * codebook input for the quantizer and the decode.
 */
nsn_status nsn_codebook_4bit_host(float* codebook, int n_values);

/*
 * Diagnostic of the decode's error path for a copy that never lands (the pages
 * have no counterpart).  Launches one warp that announces 16 bytes on an mbarrier,
 * issues no copy, and waits with the decode's bounded wait capped at max_attempts
 * suspended attempts (1..4096, each at most about a millisecond).  The wait gives
 * up, sets bit 2 of *status (device int32) and returns; the context stays usable.
 */
nsn_status nsn_selftest_bounded_wait(int32_t* status, int max_attempts, void* stream);

/*
 * Diagnostic of the quantizer's tensor-core scores ([TS] Metodologia 3: nearest
 * codeword of one global codebook; the pages have no counterpart for the check).
 * For n_rows (1..128) fp32 rows of 8 values (`rows`, DEVICE [n_rows][8]) and a
 * codebook (DEVICE fp32 [256][8]) it stages the codebook, builds the A operand and
 * runs the two tcgen05 MMAs exactly as the prefill search does, and writes the raw
 * fp32 accumulators to `scores` (DEVICE [n_rows][256]):
 *   assign 0: score_k = a . c_k - ||c_k||^2 / 2     (fp16 hi + lo a, fp16 c, fp16 hi + lo bias)
 *   assign 1: score_k = a . c_hat_k                  (c_hat = c / ||c||, fp16 hi + lo on both sides)
 * so the caller can compare them with exact arithmetic.  All pointers 16-byte
 * aligned (status 4-byte); bit 2 of *status (device int32) is set if the MMA
 * completion wait gave up.  Invalid arguments return NSN_ERR_INVALID_ARG before
 * any launch.
 */
nsn_status nsn_selftest_tensor_scores(const float* rows, int n_rows, const float* codebook, int assign,
                                      float* scores, int32_t* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NSN_H_ */
