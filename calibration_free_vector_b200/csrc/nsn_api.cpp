// C ABI entry points (include/nsn.h): host-side validation, then kernel launches.
// No entry point allocates, frees or synchronizes.

#include <cuda_runtime.h>

#include <cstring>
#include <string>

#include "nsn.h"
#include "nsn_launch.h"

namespace {

thread_local std::string g_last_cuda_error;

nsn_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return NSN_OK;
  g_last_cuda_error = cudaGetErrorString(e);
  return NSN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(int dt) { return dt == NSN_DTYPE_F32 || dt == NSN_DTYPE_BF16 || dt == NSN_DTYPE_F16; }

// Elements per 16 bytes: row offsets must be multiples of this.
int64_t elems16(int dt) { return dt == NSN_DTYPE_F32 ? 4 : 8; }

nsn_status check_cache(const nsn_cache* c) {
  if (!c) return NSN_ERR_INVALID_ARG;
  if (c->batch <= 0 || c->n_kv_heads <= 0) return NSN_ERR_INVALID_ARG;
  if (c->capacity <= 0 || c->capacity % NSN_BLOCK != 0) return NSN_ERR_INVALID_ARG;
  if (c->mode != NSN_MODE_1BIT && c->mode != NSN_MODE_2BIT) return NSN_ERR_INVALID_ARG;
  if (c->window != 0 && c->window != NSN_BLOCK) return NSN_ERR_UNSUPPORTED;
  if (!c->codes || !c->norms || !c->means || !c->n_quant || !c->n_window) return NSN_ERR_INVALID_ARG;
  if (c->mode == NSN_MODE_2BIT && !c->signs) return NSN_ERR_INVALID_ARG;
  if (c->window > 0 && !c->window_buf) return NSN_ERR_INVALID_ARG;
  if (!aligned16(c->codes) || !aligned16(c->norms) || !aligned16(c->means)) return NSN_ERR_INVALID_ARG;
  if (c->signs && !aligned16(c->signs)) return NSN_ERR_INVALID_ARG;
  if (c->window_buf && !aligned16(c->window_buf)) return NSN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(c->n_quant) & 3u) || (reinterpret_cast<uintptr_t>(c->n_window) & 3u))
    return NSN_ERR_INVALID_ARG;
  if (c->double_quant != 0 && c->double_quant != 1) return NSN_ERR_INVALID_ARG;
  if (c->assign != 0 && c->assign != 1) return NSN_ERR_INVALID_ARG;
  if (c->double_quant && (!c->s1_levels || !c->dq_params || !aligned16(c->s1_levels) || !aligned16(c->dq_params)))
    return NSN_ERR_INVALID_ARG;
  return NSN_OK;
}

nsn::CacheView view(const nsn_cache* c) {
  nsn::CacheView v;
  v.batch = c->batch;
  v.n_kv_heads = c->n_kv_heads;
  v.capacity = c->capacity;
  v.window_len = c->window;
  v.mode = c->mode;
  v.scale_adjust = c->scale_adjust ? 1 : 0;
  v.codes = c->codes;
  v.signs = c->mode == NSN_MODE_2BIT ? c->signs : nullptr;
  v.norms = reinterpret_cast<__half2*>(c->norms);
  v.means = reinterpret_cast<__half*>(c->means);
  v.window = reinterpret_cast<__half*>(c->window_buf);
  v.n_quant = c->n_quant;
  v.n_window = c->n_window;
  v.status = c->status;
  v.dq = c->double_quant ? 1 : 0;
  v.assign = c->assign;
  v.s1_levels = c->double_quant ? c->s1_levels : nullptr;
  v.dq_params = c->double_quant ? reinterpret_cast<__half*>(c->dq_params) : nullptr;
  return v;
}

// K and V caches used together must agree in shape and in double quantization.
bool same_shape(const nsn_cache* a, const nsn_cache* b) {
  return a->batch == b->batch && a->n_kv_heads == b->n_kv_heads && a->capacity == b->capacity &&
         a->window == b->window && a->double_quant == b->double_quant;
}

}  // namespace

extern "C" {

int nsn_version(void) { return 100; }

const char* nsn_status_string(int status) {
  switch (status) {
    case NSN_OK: return "ok";
    case NSN_ERR_INVALID_ARG: return "invalid argument";
    case NSN_ERR_UNSUPPORTED: return "unsupported";
    case NSN_ERR_WORKSPACE: return "workspace too small";
    case NSN_ERR_CUDA: return "cuda error";
    case NSN_ERR_STATE: return "bad cache state";
    default: return "unknown status";
  }
}

const char* nsn_last_cuda_error(void) { return g_last_cuda_error.c_str(); }

nsn_status nsn_cache_buffer_sizes(int batch, int n_kv_heads, int capacity, int window, int mode,
                                  int double_quant, nsn_cache_sizes* out) {
  if (!out || batch <= 0 || n_kv_heads <= 0 || capacity <= 0 || capacity % NSN_BLOCK != 0)
    return NSN_ERR_INVALID_ARG;
  if (mode != NSN_MODE_1BIT && mode != NSN_MODE_2BIT) return NSN_ERR_INVALID_ARG;
  if (window != 0 && window != NSN_BLOCK) return NSN_ERR_UNSUPPORTED;
  const size_t seqs = (size_t)batch * n_kv_heads;
  out->codes = seqs * capacity * NSN_N_SUB;
  out->signs = mode == NSN_MODE_2BIT ? out->codes : 0;
  const size_t blocks = seqs * (capacity / NSN_BLOCK);
  if (double_quant) {
    out->norms = seqs * capacity * sizeof(uint16_t);
    out->means = blocks * (NSN_HEAD_DIM / 2);
    out->s1_levels = seqs * capacity / 2;
    out->dq_params = blocks * 8 * sizeof(uint16_t);
  } else {
    out->norms = seqs * capacity * 2 * sizeof(uint16_t);
    out->means = blocks * NSN_HEAD_DIM * sizeof(uint16_t);
    out->s1_levels = 0;
    out->dq_params = 0;
  }
  out->window_buf = seqs * (size_t)window * NSN_HEAD_DIM * sizeof(uint16_t);
  out->n_quant = seqs * sizeof(int32_t);
  out->n_window = seqs * sizeof(int32_t);
  return NSN_OK;
}

// Validation shared by the common-length and ragged prefills; sets q, the
// quantized prefix of n_tokens.
static nsn_status check_prefill(const nsn_cache* cache, const void* x, int dtype, int64_t stride_b, int64_t stride_t,
                                int64_t stride_h, int n_tokens, const float* codebook, int* q_out) {
  nsn_status st = check_cache(cache);
  if (st != NSN_OK) return st;
  if (!codebook || !valid_dtype(dtype) || n_tokens < 0) return NSN_ERR_INVALID_ARG;
  if (n_tokens > 0 && !x) return NSN_ERR_INVALID_ARG;   // x is not read when n_tokens == 0
  if (!aligned16(x) || !aligned16(codebook)) return NSN_ERR_INVALID_ARG;
  const int64_t e16 = elems16(dtype);
  if (stride_b < 0 || stride_t < 0 || stride_h < 0) return NSN_ERR_INVALID_ARG;
  if (stride_b % e16 || stride_t % e16 || stride_h % e16) return NSN_ERR_INVALID_ARG;
  int q;
  if (n_tokens == 0) q = 0;
  else if (cache->window == 0) q = n_tokens;
  else q = NSN_BLOCK * ((n_tokens - 1) / NSN_BLOCK);
  if (q > cache->capacity) return NSN_ERR_INVALID_ARG;
  if (n_tokens - q > cache->window) return NSN_ERR_INVALID_ARG;
  *q_out = q;
  return NSN_OK;
}

nsn_status nsn_quantize_kv_ragged(nsn_cache* cache, const void* x, int dtype, int64_t stride_b, int64_t stride_t,
                                  int64_t stride_h, const int32_t* lengths, int max_tokens, const float* codebook,
                                  void* stream) {
  if (!lengths || (reinterpret_cast<uintptr_t>(lengths) & 3u)) return NSN_ERR_INVALID_ARG;
  int q = 0;
  const nsn_status st = check_prefill(cache, x, dtype, stride_b, stride_t, stride_h, max_tokens, codebook, &q);
  if (st != NSN_OK) return st;
  return cuda_status(nsn::launch_quantize_prefill(x, dtype, stride_b, stride_t, stride_h, q, max_tokens, lengths,
                                                  view(cache), codebook, static_cast<cudaStream_t>(stream)));
}

nsn_status nsn_quantize_kv(nsn_cache* cache, const void* x, int dtype, int64_t stride_b, int64_t stride_t,
                           int64_t stride_h, int n_tokens, const float* codebook, void* stream) {
  int q = 0;
  const nsn_status st = check_prefill(cache, x, dtype, stride_b, stride_t, stride_h, n_tokens, codebook, &q);
  if (st != NSN_OK) return st;
  return cuda_status(nsn::launch_quantize_prefill(x, dtype, stride_b, stride_t, stride_h, q, n_tokens, nullptr,
                                                  view(cache), codebook, static_cast<cudaStream_t>(stream)));
}

nsn_status nsn_append_residual(nsn_cache* k_cache, nsn_cache* v_cache, const void* k_new, const void* v_new,
                               int dtype, int64_t stride_b, int64_t stride_h, const float* cb_k, const float* cb_v,
                               void* stream) {
  nsn_status st = check_cache(k_cache);
  if (st != NSN_OK) return st;
  st = check_cache(v_cache);
  if (st != NSN_OK) return st;
  if (!same_shape(k_cache, v_cache)) return NSN_ERR_INVALID_ARG;
  if (k_cache->window != NSN_BLOCK) return NSN_ERR_UNSUPPORTED;
  if (!k_new || !v_new || !cb_k || !cb_v || !valid_dtype(dtype)) return NSN_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(cb_k) || !aligned16(cb_v)) return NSN_ERR_INVALID_ARG;
  const int64_t e16 = elems16(dtype);
  if (stride_b < 0 || stride_h < 0 || stride_b % e16 || stride_h % e16) return NSN_ERR_INVALID_ARG;
  return cuda_status(nsn::launch_append(view(k_cache), view(v_cache), k_new, v_new, dtype, stride_b, stride_h, cb_k,
                                        cb_v, static_cast<cudaStream_t>(stream)));
}

size_t nsn_decode_workspace_bytes(const nsn_cache* k_cache, int n_q_heads) {
  if (check_cache(k_cache) != NSN_OK || n_q_heads <= 0 || n_q_heads % k_cache->n_kv_heads) return 0;
  const nsn::DecodeGeom g = nsn::decode_geometry(k_cache->batch, k_cache->capacity, n_q_heads, k_cache->n_kv_heads);
  return nsn::decode_workspace_bytes(k_cache->batch, k_cache->n_kv_heads, g);
}

nsn_status nsn_decode_attention(const nsn_cache* k_cache, const nsn_cache* v_cache, const void* q, int dtype,
                                int n_q_heads, int64_t q_stride_b, int64_t q_stride_h, float softmax_scale,
                                const float* cb_k, const float* cb_v, float* out, void* workspace, size_t ws_bytes,
                                void* stream) {
  nsn_status st = check_cache(k_cache);
  if (st != NSN_OK) return st;
  st = check_cache(v_cache);
  if (st != NSN_OK) return st;
  if (!same_shape(k_cache, v_cache)) return NSN_ERR_INVALID_ARG;
  if (!q || !cb_k || !cb_v || !out || !workspace || !valid_dtype(dtype)) return NSN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(cb_k) || !aligned16(cb_v) || !aligned16(out) || !aligned16(workspace))
    return NSN_ERR_INVALID_ARG;
  if (n_q_heads <= 0 || n_q_heads % k_cache->n_kv_heads) return NSN_ERR_INVALID_ARG;
  const int g = n_q_heads / k_cache->n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return NSN_ERR_UNSUPPORTED;
  const int64_t e16 = elems16(dtype);
  if (q_stride_b < 0 || q_stride_h < 0 || q_stride_b % e16 || q_stride_h % e16) return NSN_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return NSN_ERR_INVALID_ARG;
  const nsn::DecodeGeom geom = nsn::decode_geometry(k_cache->batch, k_cache->capacity, n_q_heads, k_cache->n_kv_heads);
  if (ws_bytes < nsn::decode_workspace_bytes(k_cache->batch, k_cache->n_kv_heads, geom)) return NSN_ERR_WORKSPACE;
  return cuda_status(nsn::launch_decode(view(k_cache), view(v_cache), q, dtype, n_q_heads, q_stride_b, q_stride_h,
                                        softmax_scale, cb_k, cb_v, out, workspace, geom,
                                        static_cast<cudaStream_t>(stream)));
}

nsn_status nsn_extend_attention(const nsn_cache* k_cache, const nsn_cache* v_cache, const void* q, int dtype,
                                int n_q_heads, int n_queries, int64_t q_stride_b, int64_t q_stride_t,
                                int64_t q_stride_h, float softmax_scale, const float* cb_k, const float* cb_v,
                                float* out, void* workspace, size_t ws_bytes, void* stream) {
  nsn_status st = check_cache(k_cache);
  if (st != NSN_OK) return st;
  st = check_cache(v_cache);
  if (st != NSN_OK) return st;
  if (!same_shape(k_cache, v_cache)) return NSN_ERR_INVALID_ARG;
  if (k_cache->window == 0) return NSN_ERR_UNSUPPORTED;
  if (n_queries < 1 || n_queries > k_cache->window) return NSN_ERR_INVALID_ARG;
  if (!q || !cb_k || !cb_v || !out || !workspace || !valid_dtype(dtype)) return NSN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(cb_k) || !aligned16(cb_v) || !aligned16(out) || !aligned16(workspace))
    return NSN_ERR_INVALID_ARG;
  if (n_q_heads <= 0 || n_q_heads % k_cache->n_kv_heads) return NSN_ERR_INVALID_ARG;
  const int g = n_q_heads / k_cache->n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return NSN_ERR_UNSUPPORTED;
  const int64_t e16 = elems16(dtype);
  if (q_stride_b < 0 || q_stride_t < 0 || q_stride_h < 0 || q_stride_b % e16 || q_stride_t % e16 ||
      q_stride_h % e16)
    return NSN_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return NSN_ERR_INVALID_ARG;
  const nsn::DecodeGeom geom = nsn::decode_geometry(k_cache->batch, k_cache->capacity, n_q_heads, k_cache->n_kv_heads);
  if (ws_bytes < nsn::decode_workspace_bytes(k_cache->batch, k_cache->n_kv_heads, geom)) return NSN_ERR_WORKSPACE;
  return cuda_status(nsn::launch_extend(view(k_cache), view(v_cache), q, dtype, n_q_heads, n_queries, q_stride_b,
                                        q_stride_t, q_stride_h, softmax_scale, cb_k, cb_v, out, workspace, geom,
                                        static_cast<cudaStream_t>(stream)));
}

size_t nsn_decode_rope_workspace_bytes(const nsn_cache* k_cache, int n_q_heads) {
  if (check_cache(k_cache) != NSN_OK || n_q_heads <= 0 || n_q_heads % k_cache->n_kv_heads) return 0;
  const nsn::DecodeGeom g = nsn::decode_geometry(k_cache->batch, k_cache->capacity, n_q_heads, k_cache->n_kv_heads);
  return nsn::decode_rope_workspace_bytes(k_cache->batch, k_cache->n_kv_heads, k_cache->capacity, k_cache->window,
                                          g);
}

nsn_status nsn_decode_attention_rope(const nsn_cache* k_cache, const nsn_cache* v_cache, const void* q, int dtype,
                                     int n_q_heads, int64_t q_stride_b, int64_t q_stride_h, float softmax_scale,
                                     const float* inv_freq, const float* cb_k, const float* cb_v, float* out,
                                     void* workspace, size_t ws_bytes, void* stream) {
  nsn_status st = check_cache(k_cache);
  if (st != NSN_OK) return st;
  st = check_cache(v_cache);
  if (st != NSN_OK) return st;
  if (!same_shape(k_cache, v_cache)) return NSN_ERR_INVALID_ARG;
  if (!q || !inv_freq || !cb_k || !cb_v || !out || !workspace || !valid_dtype(dtype)) return NSN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(inv_freq) || !aligned16(cb_k) || !aligned16(cb_v) || !aligned16(out) ||
      !aligned16(workspace))
    return NSN_ERR_INVALID_ARG;
  if (n_q_heads <= 0 || n_q_heads % k_cache->n_kv_heads) return NSN_ERR_INVALID_ARG;
  const int g = n_q_heads / k_cache->n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return NSN_ERR_UNSUPPORTED;
  const int64_t e16 = elems16(dtype);
  if (q_stride_b < 0 || q_stride_h < 0 || q_stride_b % e16 || q_stride_h % e16) return NSN_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return NSN_ERR_INVALID_ARG;
  const nsn::DecodeGeom geom = nsn::decode_geometry(k_cache->batch, k_cache->capacity, n_q_heads, k_cache->n_kv_heads);
  if (ws_bytes < nsn::decode_rope_workspace_bytes(k_cache->batch, k_cache->n_kv_heads, k_cache->capacity,
                                                  k_cache->window, geom))
    return NSN_ERR_WORKSPACE;
  return cuda_status(nsn::launch_decode_rope(view(k_cache), view(v_cache), q, dtype, n_q_heads, q_stride_b,
                                             q_stride_h, softmax_scale, inv_freq, cb_k, cb_v, out, workspace, geom,
                                             static_cast<cudaStream_t>(stream)));
}

nsn_status nsn_decode_attention_static(const nsn_cache* k_cache, const nsn_cache* v_cache, const void* q, int dtype,
                                       int n_q_heads, int64_t q_stride_b, int64_t q_stride_h, float softmax_scale,
                                       const float* cb_k, const float* cb_v, float* out, void* stream) {
  nsn_status st = check_cache(k_cache);
  if (st != NSN_OK) return st;
  st = check_cache(v_cache);
  if (st != NSN_OK) return st;
  if (!same_shape(k_cache, v_cache)) return NSN_ERR_INVALID_ARG;
  if (!q || !cb_k || !cb_v || !out || !valid_dtype(dtype)) return NSN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(cb_k) || !aligned16(cb_v) || !aligned16(out)) return NSN_ERR_INVALID_ARG;
  if (n_q_heads <= 0 || n_q_heads % k_cache->n_kv_heads) return NSN_ERR_INVALID_ARG;
  const int g = n_q_heads / k_cache->n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return NSN_ERR_UNSUPPORTED;
  const int64_t e16 = elems16(dtype);
  if (q_stride_b < 0 || q_stride_h < 0 || q_stride_b % e16 || q_stride_h % e16) return NSN_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return NSN_ERR_INVALID_ARG;
  const nsn::DecodeGeom geom = nsn::decode_geometry(k_cache->batch, k_cache->capacity, n_q_heads, k_cache->n_kv_heads);
  // the partials and counters of this shape must fit in the fixed arrays
  if (!nsn::decode_static_fits(k_cache->batch, k_cache->n_kv_heads, geom)) return NSN_ERR_WORKSPACE;
  return cuda_status(nsn::launch_decode_static(view(k_cache), view(v_cache), q, dtype, n_q_heads, q_stride_b,
                                               q_stride_h, softmax_scale, cb_k, cb_v, out, geom,
                                               static_cast<cudaStream_t>(stream)));
}

nsn_status nsn_selftest_bounded_wait(int32_t* status, int max_attempts, void* stream) {
  if (!status || (reinterpret_cast<uintptr_t>(status) & 3u) || max_attempts <= 0 || max_attempts > 4096)
    return NSN_ERR_INVALID_ARG;
  return cuda_status(nsn::launch_bounded_wait_selftest(status, (uint32_t)max_attempts,
                                                       static_cast<cudaStream_t>(stream)));
}

nsn_status nsn_selftest_tensor_scores(const float* rows, int n_rows, const float* codebook, int assign,
                                      float* scores, int32_t* status, void* stream) {
  if (!rows || !codebook || !scores || !status || n_rows <= 0 || n_rows > 128 || (assign != 0 && assign != 1))
    return NSN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(rows) | reinterpret_cast<uintptr_t>(codebook) |
       reinterpret_cast<uintptr_t>(scores)) & 15u || (reinterpret_cast<uintptr_t>(status) & 3u))
    return NSN_ERR_INVALID_ARG;
  return cuda_status(nsn::launch_tensor_scores_selftest(rows, n_rows, codebook, assign, scores, status,
                                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
