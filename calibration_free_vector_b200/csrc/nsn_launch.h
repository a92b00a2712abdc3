// Internal interface between the C ABI (nsn_api.cpp) and the kernels.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace nsn {

// Device view of one nsn_cache (same buffers, typed pointers).
struct CacheView {
  int batch, n_kv_heads, capacity, window_len, mode, scale_adjust;
  uint8_t* codes;
  uint8_t* signs;
  __half2* norms;
  __half* means;
  __half* window;
  int32_t* n_quant;
  int32_t* n_window;
  int32_t* status;
  int dq;               // 1: s1 and o stored as 4-bit levels (then `norms` holds fp16 alpha*s2,
  uint8_t* s1_levels;   //    `means` the o levels, s1_levels / dq_params the rest)
  __half* dq_params;
  int assign;           // 0: nearest codeword, 1: largest cosine similarity
};

// Decode split geometry: the quantized blocks of every (b, kv-head) are dealt
// out to nsplit_q warps in contiguous ranges; one more partial slot holds the
// residual window.
struct DecodeGeom {
  int chunk;         // unused (kept 0)
  int nsplit_q;      // splits per sequence over the quantized part (blocks are dealt out evenly)
  int g;             // query heads per kv-head
};

DecodeGeom decode_geometry(int batch, int capacity, int n_q_heads, int n_kv_heads);
// Workspace = merge counters (zero at rest) followed by the partials.
size_t decode_workspace_bytes(int batch, int n_kv_heads, const DecodeGeom& geom);
size_t decode_partial_bytes(int batch, int n_kv_heads, const DecodeGeom& geom);
// Whether a shape fits the allocation-free decode's fixed arrays.
bool decode_static_fits(int batch, int n_kv_heads, const DecodeGeom& geom);

size_t quant_smem_bytes();

// `lengths` (device int32[batch]) is NULL for a common length; otherwise n_tokens is
// the bound of the lengths and q_tokens the quantized prefix of that bound.
cudaError_t launch_quantize_prefill(const void* x, int dtype, int64_t sb, int64_t st, int64_t sh, int q_tokens,
                                    int n_tokens, const int32_t* lengths, const CacheView& cv, const float* cb,
                                    cudaStream_t s);

cudaError_t launch_append(const CacheView& kc, const CacheView& vc, const void* kn, const void* vn, int dtype,
                          int64_t sb, int64_t sh, const float* cbk, const float* cbv, cudaStream_t s);

cudaError_t launch_decode(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                          int64_t qsb, int64_t qsh, float softmax_scale, const float* cbk, const float* cbv,
                          float* out, void* ws, const DecodeGeom& geom, cudaStream_t s);

// Chunked-prefill attention of the last n_queries window tokens (causal inside the window).
cudaError_t launch_extend(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                          int n_queries, int64_t qsb, int64_t qst, int64_t qsh, float softmax_scale, const float* cbk,
                          const float* cbv, float* out, void* ws, const DecodeGeom& geom, cudaStream_t s);

// Pre-RoPE keys: the K logits (keys rotated at their positions by inv_freq) into
// the workspace after the decode partials, then the decode over them.
size_t decode_rope_workspace_bytes(int batch, int n_kv_heads, int capacity, int window_len, const DecodeGeom& geom);
cudaError_t launch_decode_rope(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                               int64_t qsb, int64_t qsh, float softmax_scale, const float* inv_freq, const float* cbk,
                               const float* cbv, float* out, void* ws, const DecodeGeom& geom, cudaStream_t s);

// Same as launch_decode with the file-scope arrays as the workspace.
cudaError_t launch_decode_static(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                                 int64_t qsb, int64_t qsh, float softmax_scale, const float* cbk, const float* cbv,
                                 float* out, const DecodeGeom& geom, cudaStream_t s);

// Bounded-wait diagnostic (see nsn_selftest_bounded_wait).
cudaError_t launch_bounded_wait_selftest(int32_t* status, uint32_t limit, cudaStream_t s);
// Tensor-core score diagnostic (see nsn_selftest_tensor_scores).
cudaError_t launch_tensor_scores_selftest(const float* rows, int n, const float* codebook, int cosine, float* scores,
                                          int32_t* status, cudaStream_t s);

}  // namespace nsn
