// NSNQuant decode attention over the compressed KV cache (sm_100a).
//
// Method: "NSNQuant: A Double Normalization Approach for Calibration-Free Low-Bit
// Vector Quantization of KV Cache", technical summary, Metodologia 4: attention
// scores fold the NSN byproducts s1, s2, o in directly, and a full-precision
// residual window holds the most recent tokens.
//
// For a quantized token t of block b:  k_hat = H^T((u_hat s2 + o_b) s1), so
//   q . k_hat = s1 (s2 (Hq) . u_hat + (Hq) . o_b)
// and the value sum stays in the rotated domain until the very end:
//   sum_t p_t v_hat_t = H [ sum_t (p_t s1 s2) u_hat_t + sum_b (sum_{t in b} p_t s1) o_b ].
// Residual-window tokens are attended in the original domain.
//
// Kernels:
//   decode_split_kernel     one CTA per (split of the quantized range, kv-head, batch):
//                           rotated query, scores from the codes, online softmax,
//                           value accumulation from the codewords -> partial (m, l, acc)
//   decode_window_kernel    one CTA per (kv-head, batch): the residual window -> partial
//   decode_combine_kernel   one warp per (q-head, batch): log-sum-exp merge of the
//                           partials, H applied to the rotated sum, normalisation.
// Scores are carried in log2 units (the query is pre-scaled by softmax_scale*log2 e).

#include "nsn_common.cuh"
#include "nsn_launch.h"

namespace nsn {

constexpr float LOG2E = 1.4426950408889634f;
constexpr float INV_SQRT_D = 0.08838834764831845f;  // 1/sqrt(128)

__device__ __forceinline__ void load8_rt(const void* base, int64_t off, int dtype, float* out) {
  if (dtype == NSN_DTYPE_F32) load8<NSN_DTYPE_F32>(base, off, out);
  else if (dtype == NSN_DTYPE_BF16) load8<NSN_DTYPE_BF16>(base, off, out);
  else load8<NSN_DTYPE_F16>(base, off, out);
}

__device__ __forceinline__ float f16r(float x) { return __half2float(__float2half_rn(x)); }

// Block-wide reduction of N values per thread (128 threads): op = sum or max.
template <int N, bool IS_MAX>
__device__ __forceinline__ void block_reduce(float* vals, float (*red)[16]) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    float x = vals[i];
    x = IS_MAX ? warp_max(x) : warp_sum(x);
    if (lane == 0) red[w][i] = x;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < N; ++i) {
    float a = red[0][i], b = red[1][i], c = red[2][i], d = red[3][i];
    vals[i] = IS_MAX ? fmaxf(fmaxf(a, b), fmaxf(c, d)) : (a + b) + (c + d);
  }
  __syncthreads();
}

// Loads the g query rows of kv-head hk, rotates them (H q = FWHT(q)/sqrt(128))
// when `rotate`, scales by `scale` and stores [g][128] fp32 to qt.
template <int G>
__device__ void load_queries(float* qt, const void* q, int dtype, int64_t qsb, int64_t qsh, int b, int hk,
                             float scale, bool rotate) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  for (int h = w; h < G; h += 4) {
    const int64_t off = (int64_t)b * qsb + (int64_t)(hk * G + h) * qsh + 4 * lane;
    float v[4];
    if (dtype == NSN_DTYPE_F32) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(q) + off));
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else if (dtype == NSN_DTYPE_BF16) {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(q) + off));
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
      v[0] = a.x; v[1] = a.y; v[2] = c.x; v[3] = c.y;
    } else {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(static_cast<const __half*>(q) + off));
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&r.x));
      const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&r.y));
      v[0] = a.x; v[1] = a.y; v[2] = c.x; v[3] = c.y;
    }
    float sc = scale;
    if (rotate) {
      fwht128_warp(v, lane);
      sc *= INV_SQRT_D;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) qt[h * D + 4 * lane + i] = v[i] * sc;
  }
}

// Workspace layout: [P][G][2] (m, l) floats, then -- from a 16-byte aligned
// offset -- [P][G][128] accumulators; P = batch * kv-heads * (nsplit_q + 1).
__device__ __host__ __forceinline__ int64_t acc_offset(int64_t P, int G) { return ((P * G * 2 + 3) / 4) * 4; }
__device__ __forceinline__ float* partial_ml(float* ws, int64_t p, int G, int h) { return ws + (p * G + h) * 2; }

// ---------------------------------------------------------------------------
// Tensor-core building blocks (mma.sync m16n8k16, fp16 in / fp32 accumulate;
// ldmatrix gathers of whole 8-dim codewords).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

// d += A(16x16, rows a0/a1/a2/a3) * B(16x8, b0/b1); rows 8-15 of A are zero here.
__device__ __forceinline__ void mma_rows0_7(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_full(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2^x with the hardware approximation (ex2.approx.ftz: ~2 ulp); 2^(-1e30) = 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Applies stored sign bits to a half2 fragment: `w` holds the two signs at bits
// 15 - s and 31 - s; after the shift by s they sit on the fp16 sign bits.
__device__ __forceinline__ uint32_t apply_signs(uint32_t x, uint32_t w, int s) {
  return x ^ ((w << s) & 0x80008000u);
}

__device__ __forceinline__ uint32_t u4_word(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// ---------------------------------------------------------------------------
// Quantized part.  One CTA of 16 warps per SM; every warp owns one split: a
// contiguous range of 128-token blocks of one (batch, kv-head) sequence, and
// writes its own partial (m, l, O).  The CTA shares only the two replicated
// fp16 codebooks (staged once).  Compressed tokens stream through a per-warp
// double-buffered ring of 64-token stages filled by cp.async, so one stage is
// always in flight while the previous one is consumed.
//
// Per 16-token tile a warp computes, on the tensor cores,
//   S^T[h][t]  = sum_k q~[h][k] u_hat[t][k]   (M = heads, N = 8 tokens, K = 16 dims)
//   O^T[d][h] += sum_t u_hat_v[t][d] w[t][h]   (M = 16 dims, N = heads, K = 16 tokens)
// with u_hat fragments gathered by ldmatrix from an 8-fold replicated fp16
// codebook (replica r of code c at byte 128c + 16r: the 8 rows of each 8x8
// matrix always hit 8 different bank groups), stored sign bits XOR-ed onto the
// fp16 sign bits (2-bit mode), and w = p * s1 * s2 of the value tokens.  The S^T
// accumulator fragment (head g, tokens 2p, 2p+1) is exactly the B fragment of
// the value product, so no transpose is needed.  A rows g + 8 carry the fp16
// rounding residual of q~ (the score adds both accumulator rows).
// ---------------------------------------------------------------------------
constexpr int DEC_WARPS = 16;
constexpr int STAGE_TOK = 64;
// stage layout (bytes): K codes | K signs | K norms | V codes | V signs | V norms | K mean | V mean
constexpr int ST_KC = 0, ST_KS = 1024, ST_KN = 2048, ST_VC = 2304, ST_VS = 3328, ST_VN = 4352, ST_KM = 4608,
              ST_VM = 4864, STAGE_BYTES = 5120;

struct DecSmem {
  alignas(128) uint4 cbk[NCODES][8];  // replicated fp16 codebooks (32 KB each)
  alignas(128) uint4 cbv[NCODES][8];
  alignas(128) unsigned char stage[DEC_WARPS][2][STAGE_BYTES];
};

__device__ __forceinline__ uint4 cb_row_f16(const float* __restrict__ cb, int c) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(cb + c * SUB));
  const float4 b = __ldg(reinterpret_cast<const float4*>(cb + c * SUB) + 1);
  return make_uint4(pack_half2(a.x, a.y), pack_half2(a.z, a.w), pack_half2(b.x, b.y), pack_half2(b.z, b.w));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Copies `bytes` (multiple of 16) from global src to shared dst, lanes striding 16 B.
__device__ __forceinline__ void warp_copy(uint32_t dst, const unsigned char* src, int bytes, int lane) {
  for (int o = lane * 16; o < bytes; o += 32 * 16) cp_async16(dst + o, src + o);
}

template <int MK, int MV>
__device__ __forceinline__ void issue_stage(uint32_t dst, const CacheView& kc, const CacheView& vc, int64_t seq,
                                           int t0, int lane) {
  const int64_t cap = kc.capacity;
  const int64_t tok = seq * cap + t0;
  const int64_t mrow = (seq * (cap / BLK) + t0 / BLK) * D;
  warp_copy(dst + ST_KC, kc.codes + tok * NSUB, STAGE_TOK * 16, lane);
  if constexpr (MK == NSN_MODE_2BIT) warp_copy(dst + ST_KS, kc.signs + tok * NSUB, STAGE_TOK * 16, lane);
  warp_copy(dst + ST_KN, reinterpret_cast<const unsigned char*>(kc.norms + tok), STAGE_TOK * 4, lane);
  warp_copy(dst + ST_VC, vc.codes + tok * NSUB, STAGE_TOK * 16, lane);
  if constexpr (MV == NSN_MODE_2BIT) warp_copy(dst + ST_VS, vc.signs + tok * NSUB, STAGE_TOK * 16, lane);
  warp_copy(dst + ST_VN, reinterpret_cast<const unsigned char*>(vc.norms + tok), STAGE_TOK * 4, lane);
  warp_copy(dst + ST_KM, reinterpret_cast<const unsigned char*>(kc.means + mrow), D * 2, lane);
  warp_copy(dst + ST_VM, reinterpret_cast<const unsigned char*>(vc.means + mrow), D * 2, lane);
  cp_async_commit();
}

template <int G, int MK, int MV>
__global__ void __launch_bounds__(32 * DEC_WARPS, 1)
decode_split_kernel(CacheView kc, CacheView vc, const void* __restrict__ q, int dtype, int64_t qsb, int64_t qsh,
                    float qscale, const float* __restrict__ cbk_g, const float* __restrict__ cbv_g,
                    float* __restrict__ ws, DecodeGeom geom) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, p = lane & 3;

  // ---- stage the replicated fp16 codebooks (whole CTA, once) ----
  for (int e = tid; e < NCODES * 8; e += blockDim.x) {
    const int c = e >> 3, r = e & 7;
    sm.cbk[c][r] = cb_row_f16(cbk_g, c);
    sm.cbv[c][r] = cb_row_f16(cbv_g, c);
  }
  __syncthreads();

  const int nseq = kc.batch * kc.n_kv_heads;
  const int gw = blockIdx.x * DEC_WARPS + warp;  // global split id
  if (gw >= nseq * geom.nsplit_q) return;
  const int64_t seq = gw / geom.nsplit_q;
  const int split = gw % geom.nsplit_q;
  const int b = (int)(seq / kc.n_kv_heads), hk = (int)(seq % kc.n_kv_heads);
  const int64_t pidx = seq * (geom.nsplit_q + 1) + split;
  const int64_t P = (int64_t)nseq * (geom.nsplit_q + 1);
  float* ws_acc = ws + acc_offset(P, G);

  const int nq = min(min(kc.n_quant[seq], vc.n_quant[seq]), kc.capacity);
  const int nblk = (nq + BLK - 1) / BLK;
  const int bps = (nblk + geom.nsplit_q - 1) / geom.nsplit_q;  // blocks per split
  const int tok_begin = split * bps * BLK;
  const int tok_end = min(nq, (split + 1) * bps * BLK);
  if (tok_begin >= tok_end) {
    for (int i = lane; i < G * D; i += 32) ws_acc[pidx * G * D + i] = 0.f;
    if (lane < G) {
      partial_ml(ws, pidx, G, lane)[0] = NEG_BIG;
      partial_ml(ws, pidx, G, lane)[1] = 0.f;
    }
    return;
  }
  const int nstages = (tok_end - tok_begin + STAGE_TOK - 1) / STAGE_TOK;
  const uint32_t st_base = smem_addr(&sm.stage[warp][0][0]);

  // prologue: two stages in flight
  issue_stage<MK, MV>(st_base, kc, vc, seq, tok_begin, lane);
  if (nstages > 1) issue_stage<MK, MV>(st_base + STAGE_BYTES, kc, vc, seq, tok_begin + STAGE_TOK, lane);
  else cp_async_commit();

  // ---- rotated query fragments (built in registers while the copies fly) ----
  // A row g = fp16(q~_g), row g + 8 = fp16(q~_g - fp16(q~_g)).
  uint32_t qa[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) qa[j][0] = qa[j][1] = qa[j][2] = qa[j][3] = 0u;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const int64_t off = (int64_t)b * qsb + (int64_t)(hk * G + h) * qsh + 4 * lane;
    float v[4];
    if (dtype == NSN_DTYPE_F32) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(q) + off));
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(q) + off));
      float2 a, c;
      if (dtype == NSN_DTYPE_BF16) {
        a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
        c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
      } else {
        a = __half22float2(*reinterpret_cast<const __half2*>(&r.x));
        c = __half22float2(*reinterpret_cast<const __half2*>(&r.y));
      }
      v[0] = a.x; v[1] = a.y; v[2] = c.x; v[3] = c.y;
    }
    fwht128_warp(v, lane);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] *= qscale * INV_SQRT_D;
    // element c lives in lane c/4, slot c%4; lane (g, p) needs c = 16j + 8hf + 2p, +1
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int src = 4 * j + 2 * hf + (p >> 1);
        const float e0 = __shfl_sync(0xffffffffu, v[0], src), e2 = __shfl_sync(0xffffffffu, v[2], src);
        const float e1 = __shfl_sync(0xffffffffu, v[1], src), e3 = __shfl_sync(0xffffffffu, v[3], src);
        const float x0 = (p & 1) ? e2 : e0, x1 = (p & 1) ? e3 : e1;
        if (g == h) {
          const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
          qa[j][2 * hf] = pack_half2(__half2float(h0), __half2float(h1));
          qa[j][2 * hf + 1] = pack_half2(x0 - __half2float(h0), x1 - __half2float(h1));
        }
      }
    }
  }

  const uint32_t lane_row = (uint32_t)(lane & 7) * 16u;
  const uint32_t cbk_base = smem_addr(&sm.cbk[0][0]) + lane_row;
  const uint32_t cbv_base = smem_addr(&sm.cbv[0][0]) + lane_row;
  const uint32_t sel_k = 0x4440u | (uint32_t)(lane >> 3);
  const uint32_t sel_v0 = 0x4440u | (uint32_t)((lane >> 3) & 1);
  const uint32_t sel_v1 = 0x4440u | (uint32_t)(2 + ((lane >> 3) & 1));

  float m = NEG_BIG, l = 0.f;
  float O[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) O[i][0] = O[i][1] = O[i][2] = O[i][3] = 0.f;

  for (int st = 0; st < nstages; ++st) {
    cp_async_wait<1>();
    __syncwarp();
    const int t_stage = tok_begin + st * STAGE_TOK;
    const unsigned char* sb = &sm.stage[warp][st & 1][0];
    const uint32_t sba = st_base + (uint32_t)((st & 1) * STAGE_BYTES);

    // (H q) . o_K of this stage's block, for head g (the mean row as all 8 "tokens")
    float qo;
    {
      float d4[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t mrow = sba + ST_KM + (uint32_t)(lane >> 3) * 16u;
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        uint32_t bb[4];
        ldsm_x4(mrow + 64u * qq, bb);
        mma_full(d4, qa[2 * qq], bb[0], bb[1]);
        mma_full(d4, qa[2 * qq + 1], bb[2], bb[3]);
      }
      qo = d4[0] + d4[2];
    }
    float cmean = 0.f;
    const int ntile = min(STAGE_TOK, tok_end - t_stage + 15) >> 4;
    const bool full = t_stage + STAGE_TOK <= tok_end;  // every token of the stage is valid
    for (int tile = 0; tile < ntile; ++tile) {
      const int tt = 16 * tile;  // token offset inside the stage
      const uint4 kc0 = *reinterpret_cast<const uint4*>(sb + ST_KC + (tt + (lane & 7)) * 16);
      const uint4 kc1 = *reinterpret_cast<const uint4*>(sb + ST_KC + (tt + 8 + (lane & 7)) * 16);
      uint32_t ks0 = 0u, ks1 = 0u;
      if constexpr (MK == NSN_MODE_2BIT) {
        ks0 = *reinterpret_cast<const uint32_t*>(sb + ST_KS + (tt + g) * 16 + 4 * p);
        ks1 = *reinterpret_cast<const uint32_t*>(sb + ST_KS + (tt + 8 + g) * 16 + 4 * p);
      }
      const uint2 kn0 = *reinterpret_cast<const uint2*>(sb + ST_KN + (tt + 2 * p) * 4);
      const uint2 kn1 = *reinterpret_cast<const uint2*>(sb + ST_KN + (tt + 8 + 2 * p) * 4);
      const uint4 vcw = *reinterpret_cast<const uint4*>(sb + ST_VC + (tt + (lane & 7) + 8 * (lane >> 4)) * 16);
      uint32_t W0 = 0u, W1 = 0u;
      if constexpr (MV == NSN_MODE_2BIT) {
        const uint16_t* vs = reinterpret_cast<const uint16_t*>(sb + ST_VS);
        W0 = (uint32_t)vs[(tt + 2 * p) * 8 + g] | ((uint32_t)vs[(tt + 2 * p + 1) * 8 + g] << 16);
        W1 = (uint32_t)vs[(tt + 8 + 2 * p) * 8 + g] | ((uint32_t)vs[(tt + 9 + 2 * p) * 8 + g] << 16);
      }
      const uint2 vn0 = *reinterpret_cast<const uint2*>(sb + ST_VN + (tt + 2 * p) * 4);
      const uint2 vn1 = *reinterpret_cast<const uint2*>(sb + ST_VN + (tt + 8 + 2 * p) * 4);

      // ---- scores S^T = q~ u_hat^T for the two 8-token groups ----
      float S[2][2];
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        const uint4 kcw = grp ? kc1 : kc0;
        const uint32_t ksw = grp ? ks1 : ks0;
        float Sa[4] = {0.f, 0.f, 0.f, 0.f}, Sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const uint32_t code = __byte_perm(u4_word(kcw, qq), 0u, sel_k);
          uint32_t bb[4];
          ldsm_x4(cbk_base + code * 128u, bb);
          if constexpr (MK == NSN_MODE_2BIT) {
#pragma unroll
            for (int i = 0; i < 4; ++i) bb[i] = apply_signs(bb[i], ksw, 4 * qq + i);
          }
          mma_full(Sa, qa[2 * qq], bb[0], bb[1]);
          mma_full(Sb, qa[2 * qq + 1], bb[2], bb[3]);
        }
        S[grp][0] = (Sa[0] + Sa[2]) + (Sb[0] + Sb[2]);  // rows g and g + 8
        S[grp][1] = (Sa[1] + Sa[3]) + (Sb[1] + Sb[3]);
      }

      // ---- scores with the NSN byproducts, online softmax (head g) ----
      const __half2* kh0 = reinterpret_cast<const __half2*>(&kn0);
      const __half2* kh1 = reinterpret_cast<const __half2*>(&kn1);
      const __half2* vh0 = reinterpret_cast<const __half2*>(&vn0);
      const __half2* vh1 = reinterpret_cast<const __half2*>(&vn1);
      const float2 kn[4] = {__half22float2(kh0[0]), __half22float2(kh0[1]), __half22float2(kh1[0]),
                            __half22float2(kh1[1])};
      const float2 vn[4] = {__half22float2(vh0[0]), __half22float2(vh0[1]), __half22float2(vh1[0]),
                            __half22float2(vh1[1])};
      const float dk[4] = {S[0][0], S[0][1], S[1][0], S[1][1]};  // tokens 2p, 2p+1, 8+2p, 9+2p
      const int tk[4] = {tt + 2 * p, tt + 2 * p + 1, tt + 8 + 2 * p, tt + 9 + 2 * p};
      float sc[4];
      float tmax = NEG_BIG;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool ok = (g < G) && (full || t_stage + tk[i] < tok_end);
        sc[i] = ok ? kn[i].x * fmaf(kn[i].y, dk[i], qo) : NEG_BIG;
        tmax = fmaxf(tmax, sc[i]);
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
      const float mnew = fmaxf(m, tmax);
      if (__any_sync(0xffffffffu, mnew > m)) {
        const float corr = fast_exp2(m - mnew);
        const float ca = __shfl_sync(0xffffffffu, corr, 8 * p);
        const float cb = __shfl_sync(0xffffffffu, corr, 8 * p + 4);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          O[i][0] *= ca; O[i][1] *= cb; O[i][2] *= ca; O[i][3] *= cb;
        }
        l *= corr;
        cmean *= corr;
        m = mnew;
      }
      float w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float pr = (g < G) ? fast_exp2(sc[i] - m) : 0.f;
        l += pr;
        cmean = fmaf(pr, vn[i].x, cmean);
        w[i] = pr * vn[i].x * vn[i].y;
      }
      const uint32_t pb0 = pack_half2(w[0], w[1]);
      const uint32_t pb1 = pack_half2(w[2], w[3]);

      // ---- values: O^T += u_hat_v^T w ----
#pragma unroll
      for (int mm = 0; mm < 8; ++mm) {
        const uint32_t code = __byte_perm(u4_word(vcw, mm >> 1), 0u, (mm & 1) ? sel_v1 : sel_v0);
        uint32_t aa[4];
        ldsm_x4_t(cbv_base + code * 128u, aa);
        if constexpr (MV == NSN_MODE_2BIT) {
          aa[0] = apply_signs(aa[0], W0, 2 * mm);
          aa[1] = apply_signs(aa[1], W0, 2 * mm + 1);
          aa[2] = apply_signs(aa[2], W1, 2 * mm);
          aa[3] = apply_signs(aa[3], W1, 2 * mm + 1);
        }
        mma_full(O[mm], aa, pb0, pb1);
      }
    }

    // ---- block mean of V for this stage's tokens: O^T[d][h] += o_V[d] * sum_t p_t s1_t ----
    cmean += __shfl_xor_sync(0xffffffffu, cmean, 1);
    cmean += __shfl_xor_sync(0xffffffffu, cmean, 2);
    {
      const float ca = __shfl_sync(0xffffffffu, cmean, 8 * p);
      const float cb = __shfl_sync(0xffffffffu, cmean, 8 * p + 4);
      const __half* ov = reinterpret_cast<const __half*>(sb + ST_VM);
#pragma unroll
      for (int mm = 0; mm < 8; ++mm) {
        const float oa = __half2float(ov[16 * mm + g]);
        const float ob = __half2float(ov[16 * mm + 8 + g]);
        O[mm][0] = fmaf(oa, ca, O[mm][0]);
        O[mm][1] = fmaf(oa, cb, O[mm][1]);
        O[mm][2] = fmaf(ob, ca, O[mm][2]);
        O[mm][3] = fmaf(ob, cb, O[mm][3]);
      }
    }
    __syncwarp();  // every lane is done with this stage buffer
    if (st + 2 < nstages) issue_stage<MK, MV>(sba, kc, vc, seq, t_stage + 2 * STAGE_TOK, lane);
    else cp_async_commit();  // keep the group count uniform for wait_group
  }
  cp_async_wait<0>();
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);

  // ---- this warp's partial ----
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int h = 2 * p + hh;
    if (h < G) {
      float* dst = ws_acc + (pidx * G + h) * D;
#pragma unroll
      for (int mm = 0; mm < 8; ++mm) {
        dst[16 * mm + g] = O[mm][hh];
        dst[16 * mm + 8 + g] = O[mm][2 + hh];
      }
    }
  }
  if (p == 0 && g < G) {
    partial_ml(ws, pidx, G, g)[0] = m;
    partial_ml(ws, pidx, G, g)[1] = l;
  }
}

// ---------------------------------------------------------------------------
// Residual window: grid (kv-heads, batch), 128 threads; thread t owns window
// token t for the scores and dim t for the value sum.  Original domain.
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(128)
decode_window_kernel(CacheView kc, CacheView vc, const void* __restrict__ q, int dtype, int64_t qsb, int64_t qsh,
                     float qscale, float* __restrict__ ws, DecodeGeom geom) {
  __shared__ float qp[G][D];
  __shared__ float pw[BLK][G];
  __shared__ float red[4][16];
  const int hk = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const int64_t seq = (int64_t)b * kc.n_kv_heads + hk;
  const int64_t pidx = seq * (geom.nsplit_q + 1) + geom.nsplit_q;
  const int64_t P = (int64_t)kc.batch * kc.n_kv_heads * (geom.nsplit_q + 1);
  float* ws_acc = ws + acc_offset(P, G);
  const int nw = (kc.window_len > 0) ? min(min(kc.n_window[seq], vc.n_window[seq]), kc.window_len) : 0;
  if (nw <= 0) {
    for (int i = t; i < G * D; i += blockDim.x) ws_acc[pidx * G * D + i] = 0.f;
    if (t < G) {
      partial_ml(ws, pidx, G, t)[0] = NEG_BIG;
      partial_ml(ws, pidx, G, t)[1] = 0.f;
    }
    return;
  }
  load_queries<G>(&qp[0][0], q, dtype, qsb, qsh, b, hk, qscale, false);
  __syncthreads();
  const bool valid = t < nw;
  float sc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) sc[h] = 0.f;
  if (valid) {
    const __half* krow = kc.window + (seq * kc.window_len + t) * D;
#pragma unroll 4
    for (int c = 0; c < D; c += 8) {
      float kv[8];
      load8<NSN_DTYPE_F16>(krow, c, kv);
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) sc[h] = fmaf(qp[h][c + i], kv[i], sc[h]);
    }
  }
  float tmax[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    sc[h] = valid ? sc[h] : NEG_BIG;
    tmax[h] = sc[h];
  }
  block_reduce<G, true>(tmax, red);
  float sums[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float p = valid ? exp2f(sc[h] - tmax[h]) : 0.f;
    pw[t][h] = p;
    sums[h] = p;
  }
  block_reduce<G, false>(sums, red);
  float acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = 0.f;
  const __half* vbase = vc.window + seq * vc.window_len * D;
  for (int j = 0; j < nw; ++j) {
    const float vv = __half2float(vbase[(int64_t)j * D + t]);
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = fmaf(pw[j][h], vv, acc[h]);
  }
#pragma unroll
  for (int h = 0; h < G; ++h) ws_acc[(pidx * G + h) * D + t] = acc[h];
  if (t < G) {
    partial_ml(ws, pidx, G, t)[0] = tmax[t];
    partial_ml(ws, pidx, G, t)[1] = sums[t];
  }
}

// ---------------------------------------------------------------------------
// Combine: grid (q-heads, batch), 32 threads.  Lane l owns dims 4l..4l+3.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32)
decode_combine_kernel(const float* __restrict__ ws, float* __restrict__ out, int n_q_heads, int n_kv_heads,
                      int batch, DecodeGeom geom) {
  const int hq = blockIdx.x, b = blockIdx.y, lane = threadIdx.x;
  const int G = geom.g;
  const int hk = hq / G, h = hq % G;
  const int nslots = geom.nsplit_q + 1;
  const int64_t P = (int64_t)batch * n_kv_heads * nslots;
  const float* ws_acc = ws + acc_offset(P, G);
  const int64_t p0 = ((int64_t)b * n_kv_heads + hk) * nslots;

  float mrot = NEG_BIG;
  for (int s = 0; s < geom.nsplit_q; ++s) mrot = fmaxf(mrot, ws[((p0 + s) * G + h) * 2]);
  float lrot = 0.f, a[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < geom.nsplit_q; ++s) {
    const float* ml = ws + ((p0 + s) * G + h) * 2;
    const float l = ml[1];
    if (l == 0.f) continue;
    const float f = exp2f(ml[0] - mrot);
    lrot = fmaf(l, f, lrot);
    const float4 v = *reinterpret_cast<const float4*>(ws_acc + ((p0 + s) * G + h) * D + 4 * lane);
    a[0] = fmaf(v.x, f, a[0]); a[1] = fmaf(v.y, f, a[1]); a[2] = fmaf(v.z, f, a[2]); a[3] = fmaf(v.w, f, a[3]);
  }
  fwht128_warp(a, lane);
  const int64_t pr = p0 + geom.nsplit_q;
  const float mres = ws[(pr * G + h) * 2], lres = ws[(pr * G + h) * 2 + 1];
  const float4 r = *reinterpret_cast<const float4*>(ws_acc + (pr * G + h) * D + 4 * lane);
  const float mt = fmaxf(mrot, mres);
  const float fa = lrot > 0.f ? exp2f(mrot - mt) : 0.f;
  const float fr = lres > 0.f ? exp2f(mres - mt) : 0.f;
  const float den = lrot * fa + lres * fr;
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float4 o;
  o.x = (a[0] * INV_SQRT_D * fa + r.x * fr) * inv;
  o.y = (a[1] * INV_SQRT_D * fa + r.y * fr) * inv;
  o.z = (a[2] * INV_SQRT_D * fa + r.z * fr) * inv;
  o.w = (a[3] * INV_SQRT_D * fa + r.w * fr) * inv;
  *reinterpret_cast<float4*>(out + ((int64_t)b * n_q_heads + hq) * D + 4 * lane) = o;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static int sm_count() {
  static int cached = 0;
  if (cached == 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      cached = n;
    else
      cached = 148;
  }
  return cached;
}

DecodeGeom decode_geometry(int batch, int capacity, int n_q_heads, int n_kv_heads) {
  DecodeGeom g;
  g.g = n_q_heads / n_kv_heads;
  g.chunk = 0;
  // splits per sequence: fill one 16-warp CTA per SM, at most one split per block
  const int nseq = batch * n_kv_heads;
  const int warps = sm_count() * DEC_WARPS;
  int sp = warps / (nseq > 0 ? nseq : 1);
  const int maxsp = capacity / BLK;
  if (sp > maxsp) sp = maxsp;
  if (sp < 1) sp = 1;
  g.nsplit_q = sp;
  return g;
}

size_t decode_workspace_bytes(int batch, int n_kv_heads, const DecodeGeom& geom) {
  const int64_t P = (int64_t)batch * n_kv_heads * (geom.nsplit_q + 1);
  return (size_t)(acc_offset(P, geom.g) + P * geom.g * D) * sizeof(float);
}

template <int G, int MK, int MV>
static cudaError_t launch_split_t(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int64_t qsb,
                                  int64_t qsh, float qscale, const float* cbk, const float* cbv, float* ws,
                                  const DecodeGeom& geom, cudaStream_t s) {
  const size_t smem = sizeof(DecSmem);
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<G, MK, MV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nwarps = kc.batch * kc.n_kv_heads * geom.nsplit_q;
  dim3 grid((nwarps + DEC_WARPS - 1) / DEC_WARPS);
  decode_split_kernel<G, MK, MV><<<grid, 32 * DEC_WARPS, smem, s>>>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, ws, geom);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(kc.n_kv_heads, kc.batch);
  decode_window_kernel<G><<<g2, 128, 0, s>>>(kc, vc, q, dtype, qsb, qsh, qscale, ws, geom);
  return cudaGetLastError();
}

template <int G>
static cudaError_t launch_modes(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int64_t qsb,
                                int64_t qsh, float qscale, const float* cbk, const float* cbv, float* ws,
                                const DecodeGeom& geom, cudaStream_t s) {
  if (kc.mode == NSN_MODE_1BIT && vc.mode == NSN_MODE_1BIT)
    return launch_split_t<G, 1, 1>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, ws, geom, s);
  if (kc.mode == NSN_MODE_1BIT && vc.mode == NSN_MODE_2BIT)
    return launch_split_t<G, 1, 2>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, ws, geom, s);
  if (kc.mode == NSN_MODE_2BIT && vc.mode == NSN_MODE_1BIT)
    return launch_split_t<G, 2, 1>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, ws, geom, s);
  return launch_split_t<G, 2, 2>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, ws, geom, s);
}

cudaError_t launch_decode(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                          int64_t qsb, int64_t qsh, float softmax_scale, const float* cbk, const float* cbv,
                          float* out, void* ws, const DecodeGeom& geom, cudaStream_t s) {
  const float qscale = softmax_scale * LOG2E;
  float* w = static_cast<float*>(ws);
  cudaError_t e;
  switch (geom.g) {
    case 1: e = launch_modes<1>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, w, geom, s); break;
    case 2: e = launch_modes<2>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, w, geom, s); break;
    case 4: e = launch_modes<4>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, w, geom, s); break;
    default: e = launch_modes<8>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, w, geom, s); break;
  }
  if (e != cudaSuccess) return e;
  dim3 g3(n_q_heads, kc.batch);
  decode_combine_kernel<<<g3, 32, 0, s>>>(w, out, n_q_heads, kc.n_kv_heads, kc.batch, geom);
  return cudaGetLastError();
}

}  // namespace nsn
