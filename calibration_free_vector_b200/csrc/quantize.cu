// NSNQuant KV quantizer kernels (sm_100a).
//
// Method: "NSNQuant: A Double Normalization Approach for Calibration-Free Low-Bit
// Vector Quantization of KV Cache", technical summary, Metodologia 1 (NSN),
// 2 (Hadamard), 3 (VQ with one global codebook, adaptive scale) and 4 (KIVI-style
// residual that is flushed into the quantized part when full).
//
// One CTA of 256 threads quantizes one block of <= 128 tokens of one (batch,
// kv-head); the adjacent lanes 2t, 2t+1 own token t (64 dims, 8 sub-vectors
// each).  Per block:
//   r      = column mean of the raw tokens (fp64 sum, stored as fp32)
//   d_t    = FWHT(x_t - r)                 fp32, in registers (exact algebra:
//   w_t    = d_t + FWHT(r)                 FWHT is linear; FWHT(r) in fp64)
//   s1     = ||x_t|| / sqrt(128)  (= ||H x_t|| / sqrt(128), H orthonormal)
//   n1_t   = w_t rr_t, rr_t = 1/||x_t||;  o = FWHT(r) mean(rr) + mean_t(d_t rr_t)
//   z_t    = d_t rr_t + FWHT(r)(rr_t - mean rr) - mean_t(d_t rr_t)       (fp64 -> fp32)
//   s2     = ||z_t|| / sqrt(128),  u_t = z_t / s2                          (u: fp32)
// Subtracting r before the fp32 transform keeps the large token-constant channel
// offsets (outliers) out of the fp32 rounding, so u carries fp32 precision
// relative to the token-varying part that survives the shift step.
//
// Nearest codeword: exhaustive scores score_k = u.c_k - ||c_k||^2/2 of all 256
// codewords on the tensor cores (a token's 16 sub-vectors are the rows of one
// m16n8k16 tile, K = the fp16 hi and lo parts of u against the fp16 codebook
// twice, the bias as the accumulator's start), the best group of 8 codewords per
// sub-vector, then the 8 codewords of that group rescanned in sequential fp32.
// Whenever a rival lies within the error bounds of the best (the fp32 bound inside
// the group, that plus a wide tensor-accumulation bound outside it), the
// sub-vector is re-decided exactly in fp64 by a whole warp over all codewords
// inside the bound (ties to the lowest index).  The stored code is therefore the
// exact nearest codeword of the fp32 u.

#include "nsn_common.cuh"
#include "nsn_launch.h"

namespace nsn {

// Shared-memory fp64 load that the compiler may not merge with other loads of the
// same address (keeps 128-entry fp64 tables from being cached in registers).
__device__ __forceinline__ double lds_f64(const double* p) {
  double r;
  asm volatile("ld.shared.f64 %0, [%1];" : "=d"(r) : "r"((unsigned)__cvta_generic_to_shared(p)));
  return r;
}

// ldmatrix / mma.sync / three-input max for the tensor-core codeword scores.
__device__ __forceinline__ uint32_t q_smem(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void q_ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// d += A (16 x 16) * B (16 x 8) with both K halves of B equal to `b`
__device__ __forceinline__ void q_mma_bb(float (&d)[4], const uint32_t (&a)[4], uint32_t b) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %8}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b));
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }

constexpr int QTHREADS = 2 * BLK;  // two threads per token
constexpr int HD = D / 2;           // dims per thread
constexpr int HSUB = NSUB / 2;      // sub-vectors per thread

struct QuantSmem {
  // codebook (fp32), rows padded to 48 bytes: lanes gathering random rows (the
  // group rescan, the adaptive scale) spread over all eight 16-byte bank groups
  alignas(16) float cb[NCODES][SUB + 4];
  alignas(16) float bias[NCODES];      // -||c_k||^2 / 2
  alignas(16) float biasq[NCODES];     // the same, per (group G of 32 codes, quad lane p): codes 32G + 8i + 2p + e at 32G + 8p + 2i + e
  alignas(16) float cnorm[4];          // [0] = max ||c||, [1] = max ||c||^2, [2] = max ||c - fp16(c)|| (rounded up)
  alignas(16) __half cbh[NCODES][SUB]; // codebook rounded to fp16, dims in the order 0 4 1 5 2 6 3 7 (tensor-core operand)
  alignas(16) double rr[BLK];          // 1 / ||x_t|| (0 for a zero token)
  alignas(16) double s1[BLK];          // per-token s1 and s2 (fp64) until the final store
  alignas(16) double s2[BLK];
  alignas(16) double big_r[D];         // FWHT(r) in fp64
  alignas(16) double o[D];             // D_c = mean_t(d_t,c rr_t) (the token-varying part of o)
  alignas(16) double part[2][D];       // per-half column partial sums
  alignas(16) double dev_part[2];      // per-half sums of rr_t - rr_0
  alignas(16) float r[D];              // column mean of raw tokens (fp32)
  alignas(16) float tile[BLK][D + 4];  // raw tokens, then d_t rows, then u rows; padded by 16 B
  alignas(16) float thr[BLK][NSUB + 1];  // per (token, sub-vector) threshold of the exact re-decision
  alignas(16) uint8_t code[BLK][NSUB]; // chosen codes
  alignas(16) uint8_t grp[BLK][NSUB];  // winning (group of 8 codes, lane) of the tensor-core scores
  alignas(16) uint16_t flag[BLK * NSUB];  // (token, sub-vector) pairs for the exact re-decision
  int nflag;
  alignas(16) uint32_t sgn[BLK][4];    // packed sign bits (2-bit mode)
  // double quantization
  alignas(16) double ofull[D];         // o of the block (fp64) until its levels are formed
  alignas(16) double red[2][QTHREADS / 32][2];  // per-warp (min, max) of s1 and of o
  alignas(16) double dq[2][3];         // (lo, hi, step) of s1 and of o
  alignas(16) uint8_t lev[2][BLK];     // 4-bit levels of s1 (per token) and of o (per channel)
};

// Destination of the stored scalars of one block: either fp16 (s1, alpha*s2) pairs
// and fp16 o, or (double quantization) fp16 alpha*s2, 4-bit s1 and o levels and the
// block's (lo, hi) pairs.
struct BlockOut {
  __half2* norms;        // [n] (s1, alpha*s2)            -- plain
  __half* means;         // [128] o                        -- plain
  __half* s2;            // [n] alpha*s2                   -- double quantization
  uint8_t* s1_levels;    // [64]  two levels per byte       -- double quantization
  uint8_t* o_levels;     // [64]                            -- double quantization
  __half* params;        // [8] (s1 lo, s1 hi, o lo, o hi, 0, 0, 0, 0) -- double quantization
  bool dq;
};

__device__ __forceinline__ BlockOut block_out(const CacheView& c, int64_t seq, int64_t tok0, int blk) {
  BlockOut o;
  const int64_t bi = seq * (c.capacity / BLK) + blk;
  o.dq = c.dq != 0;
  o.norms = c.norms + tok0;
  o.means = c.means + bi * D;
  o.s2 = reinterpret_cast<__half*>(c.norms) + tok0;
  o.s1_levels = c.s1_levels ? c.s1_levels + tok0 / 2 : nullptr;
  o.o_levels = reinterpret_cast<uint8_t*>(c.means) + bi * (D / 2);
  o.params = c.dq_params ? c.dq_params + bi * 8 : nullptr;
  return o;
}

// Stages the codebook, its biases and norm bounds.  All QTHREADS threads.
__device__ void stage_codebook(QuantSmem& sm, const float* __restrict__ codebook) {
  const int t = threadIdx.x;
  for (int i = t; i < NCODES * SUB / 4; i += blockDim.x)
    *reinterpret_cast<float4*>(&sm.cb[i >> 1][4 * (i & 1)]) = __ldg(reinterpret_cast<const float4*>(codebook) + i);
  __syncthreads();
  float my_max = 0.f, my_dev = 0.f;
  for (int k = t; k < NCODES; k += blockDim.x) {
    float s = 0.f, e = 0.f;
#pragma unroll
    for (int i = 0; i < SUB; ++i) {
      s = fmaf(sm.cb[k][i], sm.cb[k][i], s);
      const __half c16 = __float2half_rn(sm.cb[k][i]);
      sm.cbh[k][i < 4 ? 2 * i : 2 * (i - 4) + 1] = c16;  // K order of the MMA: dims p, p + 4 at slots 2p, 2p + 1
      const float d = sm.cb[k][i] - __half2float(c16);
      e = fmaf(d, d, e);
    }
    sm.bias[k] = -0.5f * s;
    sm.biasq[(k & ~31) + 8 * ((k >> 1) & 3) + 2 * ((k >> 3) & 3) + (k & 1)] = -0.5f * s;
    my_max = fmaxf(my_max, s);
    my_dev = fmaxf(my_dev, e);
  }
  my_max = warp_max(my_max);
  my_dev = warp_max(my_dev);
  __shared__ float red[QTHREADS / 32][2];
  if ((t & 31) == 0) {
    red[t >> 5][0] = my_max;
    red[t >> 5][1] = my_dev;
  }
  __syncthreads();
  if (t == 0) {
    float m = 0.f, e = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      m = fmaxf(m, red[w][0]);
      e = fmaxf(e, red[w][1]);
    }
    m *= 1.0001f;  // upper bound on max ||c||^2 despite the fp32 rounding above
    sm.cnorm[1] = m;
    sm.cnorm[0] = sqrtf(m) * 1.0001f;
    sm.cnorm[2] = e > 0.f ? sqrtf(e) * 1.001f : 0.f;  // 0 for a codebook of fp16 values
  }
  __syncthreads();
}

__device__ __forceinline__ double shfl_pair_sum(double x) { return x + __shfl_xor_sync(0xffffffffu, x, 1); }

__device__ __forceinline__ double warp_min_d(double x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x = fmin(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}
__device__ __forceinline__ double warp_max_d(double x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x = fmax(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

// Double quantization of a block's stored scalars ([TS] Metodologia 3): s1 over
// the n tokens and o over the 128 channels, each as 4-bit levels of 16 uniform
// steps between the fp16-rounded min and max of the group:
//   lo = fp16(min), hi = fp16(max), step = (hi - lo) / 15 (fp64),
//   level = round-half-even((x - lo) / step) clamped to 0..15 (step = 0: level 0).
// Threads 0..127 handle s1 (token t), threads 128..255 o (channel t - 128).
// sm.s1 and sm.ofull hold the exact fp64 values.  All QTHREADS threads.
__device__ void store_double_quant(QuantSmem& sm, int n, const BlockOut& bo) {
  __syncthreads();  // sm.s1 of every token is final
  const int t = threadIdx.x, grp = t >> 7, i = t & (BLK - 1), warp = t >> 5, lane = t & 31;
  const bool have = grp == 1 || i < n;
  const double x = grp == 0 ? (i < n ? sm.s1[i] : 0.0) : sm.ofull[i];
  const double mn = warp_min_d(have ? x : INFINITY), mx = warp_max_d(have ? x : -INFINITY);
  if (lane == 0) {
    sm.red[grp][warp & 3][0] = mn;
    sm.red[grp][warp & 3][1] = mx;
  }
  __syncthreads();
  if (t < 2) {
    double a = INFINITY, b = -INFINITY;
    for (int w = 0; w < 4; ++w) {
      a = fmin(a, sm.red[t][w][0]);
      b = fmax(b, sm.red[t][w][1]);
    }
    const double lo = (double)__half2float(__double2half(a));
    const double hi = (double)__half2float(__double2half(b));
    sm.dq[t][0] = lo;
    sm.dq[t][1] = hi;
    sm.dq[t][2] = (hi - lo) / 15.0;
  }
  __syncthreads();
  {
    const double lo = sm.dq[grp][0], step = sm.dq[grp][2];
    int level = 0;
    if (have && step > 0.0) level = (int)fmin(15.0, fmax(0.0, rint((x - lo) / step)));
    sm.lev[grp][i] = (uint8_t)level;
  }
  __syncthreads();
  if (t < 64) bo.s1_levels[t] = (uint8_t)(sm.lev[0][2 * t] | (sm.lev[0][2 * t + 1] << 4));
  else if (t < 128) bo.o_levels[t - 64] = (uint8_t)(sm.lev[1][2 * (t - 64)] | (sm.lev[1][2 * (t - 64) + 1] << 4));
  else if (t < 136) {
    const int k = t - 128;
    const double v = k == 0 ? sm.dq[0][0] : k == 1 ? sm.dq[0][1] : k == 2 ? sm.dq[1][0] : k == 3 ? sm.dq[1][1] : 0.0;
    bo.params[k] = __double2half(v);
  }
}

// Quantizes one block of n (1..128) tokens with QTHREADS threads: thread
// t = 2 tk + h works on token tk, dims 64h .. 64h+63 (sub-vectors 8h .. 8h+7).
// Rows are at src + row0 + tk*row_stride (elements).  Output pointers are
// already offset to the block's first token (codes, signs, norms) and to its
// mean row (means).
template <int DT, int MODE>
__device__ void quantize_block_dev(QuantSmem& sm, const void* __restrict__ src, int64_t row0,
                                   int64_t row_stride, int n, uint8_t* __restrict__ codes,
                                   uint8_t* __restrict__ signs, const CacheView& cv, int64_t seq,
                                   int64_t tok0, int blk, int scale_adjust) {
  const int t = threadIdx.x, tk = t >> 1, h = t & 1;
  const int col = t & (D - 1), rhalf = t >> 7;  // column-sum roles: column, half of the rows
  const bool valid = tk < n;
  if (t == 0) sm.nflag = 0;  // read only after the barriers below
  constexpr int ESZ = (DT == NSN_DTYPE_F32) ? 4 : 2;
  constexpr int CHUNKS = D * ESZ / 16;  // 16-byte chunks per row

  // ---- cooperative, coalesced load of the raw tile into shared memory --------
  {
    char* tile_bytes = reinterpret_cast<char*>(&sm.tile[0][0]);
    constexpr int ROWB = (D + 4) * 4;  // padded row stride in bytes (fits both dtypes)
    for (int q = t; q < BLK * CHUNKS; q += QTHREADS) {
      const int row = q / CHUNKS, ch = q % CHUNKS;
      if (row < n) {
        const char* g = static_cast<const char*>(src) + (row0 + (int64_t)row * row_stride) * ESZ + ch * 16;
        *reinterpret_cast<uint4*>(tile_bytes + row * ROWB + ch * 16) = __ldg(reinterpret_cast<const uint4*>(g));
      }
    }
  }
  __syncthreads();

  auto raw_at = [&](int row, int c) -> float {
    const char* tb = reinterpret_cast<const char*>(&sm.tile[0][0]) + row * (D + 4) * 4;
    if constexpr (DT == NSN_DTYPE_F32) return reinterpret_cast<const float*>(tb)[c];
    else if constexpr (DT == NSN_DTYPE_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(tb)[c]);
    else return __half2float(reinterpret_cast<const __half*>(tb)[c]);
  };

  // ---- reference r = column mean of the raw tokens ---------------------------
  // Column `col`, rows split in two halves (two accumulators each), combined in
  // a fixed order.
  {
    const int lo = rhalf * (BLK / 2), hi = min(n, lo + BLK / 2);
    double s0 = 0.0, s1 = 0.0;
    int row = lo;
    for (; row + 1 < hi; row += 2) {
      s0 += (double)raw_at(row, col);
      s1 += (double)raw_at(row + 1, col);
    }
    if (row < hi) s0 += (double)raw_at(row, col);
    sm.part[rhalf][col] = s0 + s1;
  }
  __syncthreads();
  if (t < D) sm.r[t] = (float)((sm.part[0][t] + sm.part[1][t]) / n);
  __syncthreads();
  // FWHT(r) in fp64 by warp 0 (lane l holds elements 4l..4l+3).
  if (t < 32) {
    double v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = (double)sm.r[4 * t + i];
    double a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    v[0] = a0 + a2; v[2] = a0 - a2; v[1] = a1 + a3; v[3] = a1 - a3;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const bool upper = (t & m) != 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        double other = __shfl_xor_sync(0xffffffffu, v[i], m);
        v[i] = upper ? (other - v[i]) : (v[i] + other);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) sm.big_r[4 * t + i] = v[i];
  }

  // ---- d_t = FWHT(x_t - r) over the lane pair; ||x_t||^2 from the raw values --
  float v[HD];
  double ssx0 = 0.0, ssx1 = 0.0;
  if (valid) {
    const char* tb = reinterpret_cast<const char*>(&sm.tile[tk][0]) + HD * ESZ * h;
    constexpr int HCHUNKS = CHUNKS / 2;
    constexpr int PER = (DT == NSN_DTYPE_F32) ? 4 : 8;
#pragma unroll
    for (int ch = 0; ch < HCHUNKS; ++ch) {
      const uint4 raw = *reinterpret_cast<const uint4*>(tb + ch * 16);
      float xs[8];
      if constexpr (DT == NSN_DTYPE_F32) {
        const float* f = reinterpret_cast<const float*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) xs[i] = f[i];
      } else if constexpr (DT == NSN_DTYPE_BF16) {
        const __nv_bfloat162* f = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 p = __bfloat1622float2(f[i]);
          xs[2 * i] = p.x;
          xs[2 * i + 1] = p.y;
        }
      } else {
        const __half2* f = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 p = __half22float2(f[i]);
          xs[2 * i] = p.x;
          xs[2 * i + 1] = p.y;
        }
      }
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        v[PER * ch + i] = xs[i] - sm.r[HD * h + PER * ch + i];
        if (i & 1) ssx1 = fma((double)xs[i], (double)xs[i], ssx1);
        else ssx0 = fma((double)xs[i], (double)xs[i], ssx0);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < HD; ++c) v[c] = 0.f;
  }
  fwht128_pair(v, h);
  const double ssx = shfl_pair_sum(ssx0 + ssx1);
  __syncthreads();  // raw tile fully consumed; big_r ready

  // ---- first normalization: s1 = ||H x|| / sqrt(128) = ||x|| / sqrt(128) -----
  // (H is orthonormal.)  n1_t = w_t * rr_t with w_t = FWHT(x_t) = d_t + FWHT(r)
  // and rr_t = 1/||x_t|| (||w_t|| = sqrt(128) ||x_t||); a zero token gets rr = 0.
  {
    const double norm_x = sqrt(ssx);
    const double rr = (ssx > 0.0) ? 1.0 / norm_x : 0.0;
    if (valid) {
#pragma unroll
      for (int c = 0; c < HD; c += 4)
        *reinterpret_cast<float4*>(&sm.tile[tk][HD * h + c]) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
      if (h == 0) {
        sm.rr[tk] = rr;
        sm.s1[tk] = norm_x / 11.313708498984761;
      }
    }
  }
  __syncthreads();

  // ---- shift: o = mean_t n1_t = FWHT(r) * mean(rr) + mean_t(d_t rr_t) --------
  // mean(rr) is accumulated as deviations from rr_0 so that equal rr give it
  // exactly (identical tokens then give z = 0 exactly, as the definition does).
  // Column `col`, rows split in two halves, combined in a fixed order.
  {
    const double rr0 = sm.rr[0];
    const int lo = rhalf * (BLK / 2), hi = min(n, lo + BLK / 2);
    double dev = 0.0, sd0 = 0.0, sd1 = 0.0;
    int row = lo;
    for (; row + 1 < hi; row += 2) {
      const double ra = sm.rr[row], rb = sm.rr[row + 1];
      dev += (ra - rr0) + (rb - rr0);
      sd0 = fma((double)sm.tile[row][col], ra, sd0);
      sd1 = fma((double)sm.tile[row + 1][col], rb, sd1);
    }
    if (row < hi) {
      const double ra = sm.rr[row];
      dev += ra - rr0;
      sd0 = fma((double)sm.tile[row][col], ra, sd0);
    }
    sm.part[rhalf][col] = sd0 + sd1;
    if (col == 0) sm.dev_part[rhalf] = dev;
  }
  __syncthreads();
  const double rr_mean = sm.rr[0] + (sm.dev_part[0] + sm.dev_part[1]) / n;
  if (t < D) {
    const double dc = (sm.part[0][t] + sm.part[1][t]) / n;
    sm.o[t] = dc;  // D_c = mean_t(d_t,c rr_t)
    const double o_t = fma(sm.big_r[t], rr_mean, dc);
    if (cv.dq) sm.ofull[t] = o_t;
    else cv.means[(seq * (cv.capacity / BLK) + blk) * D + t] = __double2half(o_t);
  }
  __syncthreads();

  // ---- second normalization --------------------------------------------------
  // z_t = n1_t - o = d_t rr_t + FWHT(r) (rr_t - mean rr) - D.  The last two terms
  // are formed in fp64 and rounded once (they are at the scale of z), then one
  // fp32 fma per channel.
  const double rr_t = valid ? sm.rr[tk] : 0.0;
  const double delta = rr_t - rr_mean;
  const float rrf = (float)rr_t;
  double zz0 = 0.0, zz1 = 0.0;
#pragma unroll
  for (int c = 0; c < HD; c += 2) {
    const int cg = HD * h + c;
    const float c0 = (float)fma(lds_f64(&sm.big_r[cg]), delta, -lds_f64(&sm.o[cg]));
    const float c1 = (float)fma(lds_f64(&sm.big_r[cg + 1]), delta, -lds_f64(&sm.o[cg + 1]));
    const float z0 = fmaf(v[c], rrf, c0);
    const float z1 = fmaf(v[c + 1], rrf, c1);
    v[c] = z0;
    v[c + 1] = z1;
    zz0 = fma((double)z0, (double)z0, zz0);
    zz1 = fma((double)z1, (double)z1, zz1);
  }
  const double zz = shfl_pair_sum(zz0 + zz1);
  if (valid && h == 0) sm.s2[tk] = sqrt(zz) / 11.313708498984761;
  const float inv2 = (zz > 0.0) ? (float)(11.313708498984761 / sqrt(zz)) : 0.f;
#pragma unroll
  for (int c = 0; c < HD; ++c) v[c] *= inv2;
  // v now holds u (fp32) for dims 64h .. 64h+63.

  // ---- sign bits (2-bit) and search operand a = |u| or u ---------------------
  // In 2-bit mode v is replaced by |u| after the sign bits are taken; every later
  // use only needs |u| (u_c * u_hat_c = |u_c| * A_code,c because the signs match).
  // Sign-bit layout (see include/nsn.h): 16-bit field i (i = dim within the
  // sub-vector) holds the sign of u[8s + i] at bit 15 - s; fields 2j, 2j+1 form
  // 32-bit word j (bit 15 - s and bit 31 - s).
  uint32_t sgn[4] = {0u, 0u, 0u, 0u};
  if constexpr (MODE == NSN_MODE_2BIT) {
#pragma unroll
    for (int c = 0; c < HD; ++c) {
      const int s = HSUB * h + (c >> 3), i = c & 7;
      sgn[i >> 1] |= (v[c] < 0.f ? 1u : 0u) << (16 * (i & 1) + 15 - s);
      v[c] = fabsf(v[c]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) sgn[k] |= __shfl_xor_sync(0xffffffffu, sgn[k], 1);
    if (h == 0) *reinterpret_cast<uint4*>(&sm.sgn[tk][0]) = make_uint4(sgn[0], sgn[1], sgn[2], sgn[3]);
  }

  // ---- nearest codeword: tensor-core scores, exact decision ------------------
  // score_k = a.c_k - ||c_k||^2 / 2 (maximised) for every sub-vector a.
  // (1) The 16 sub-vectors of a token are the 16 rows of one m16n8k16 tile with
  //     K = [a_hi | a_lo] (the fp32 a split into two fp16 parts, exact to 2^-22)
  //     against B = [c | c] (the codebook in fp16) and the bias as the
  //     accumulator's start: 32 MMAs give the 256 scores of 16 sub-vectors.
  // (2) Lane p of a quad sees codes 8n + 2p, 8n + 2p + 1 of every n-tile n: a
  //     running max per group of 4 n-tiles (8 codes), then the best and
  //     second-best group maxima and the best group, merged over the quad.
  // (3) The owner lane rescans the 8 codes of the winning group in sequential
  //     fp32 (the arithmetic of the exact path below) for the code (lowest index
  //     on ties) and the in-group runner-up.
  // (4) When the runner-up -- another group's tensor score or an fp32 score
  //     inside the group -- comes within the error bounds of the best, a whole
  //     warp re-decides the sub-vector exactly in fp64.
  // Error bounds: the sequential fp32 score is within gamma_9 (max||c||^2 +
  // ||a|| max||c||) of the exact one.  The tensor score's error is bounded by
  // TC_REL (sum |a_i c_i| + |bias|) for the accumulation inside the MMA (its
  // order and rounding are the hardware's, so the bound is taken wide: 2^-16
  // against 17 terms of at most 2^-24 relative each), plus ||a|| ||c - fp16(c)||
  // for a codebook that is not fp16-representable.
  const float cmax = sm.cnorm[0], cmax2 = sm.cnorm[1], cdel = sm.cnorm[2];
  constexpr float GAMMA9 = 9.0f * 5.9604645e-8f * 1.0001f;  // 9u/(1-9u), u = 2^-24
  constexpr float TC_REL = 1.52587890625e-05f;               // 2^-16
  const int warp = t >> 5, lane = t & 31, qg = lane >> 2, qp = lane & 3;
  // (1) this warp's 16 tokens x 16 sub-vectors as rows of 8 fp32 (the exact
  // search operand a), in the warp's own 16 tile rows (free since the column
  // sums).  Row r of token m sits at R = 16 m + (r ^ (m & 3)) and its two 16-byte
  // halves (dims 0-3, 4-7) swap when bit 2 xor bit 3 of R is set: the 8 rows of
  // an ldmatrix fetch and the 8 rows of a store phase (4 tokens x 2 halves of the
  // sub-vectors) both land in 8 different 16-byte bank groups.  The rows stay
  // there for the rescan, the exact path and the adaptive scale.
  auto a_phys = [](int m, int r) { return 16 * m + (r ^ (m & 3)); };
  auto a_flip = [](int R) { return ((R >> 2) ^ (R >> 3)) & 1; };
  auto urow = [&](int tok, int j, int half) -> const float4* {
    const unsigned char* base = reinterpret_cast<const unsigned char*>(&sm.tile[16 * (tok >> 4)][0]);
    const int R = a_phys(tok & 15, j);
    return reinterpret_cast<const float4*>(base + R * 32 + 16 * (half ^ a_flip(R)));
  };
  unsigned char* arow = reinterpret_cast<unsigned char*>(&sm.tile[16 * warp][0]);
  {
    const int m_own = lane >> 1;
#pragma unroll
    for (int jj = 0; jj < HSUB; ++jj) {
      const int R = a_phys(m_own, HSUB * h + jj), sw = a_flip(R);
      const float4 lo4 = valid ? make_float4(v[8 * jj], v[8 * jj + 1], v[8 * jj + 2], v[8 * jj + 3])
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 hi4 = valid ? make_float4(v[8 * jj + 4], v[8 * jj + 5], v[8 * jj + 6], v[8 * jj + 7])
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(arow + R * 32 + 16 * sw) = lo4;
      *reinterpret_cast<float4*>(arow + R * 32 + 16 * (sw ^ 1)) = hi4;
    }
  }
  __syncwarp();
  // (2) scores and group maxima, two tokens (m-tiles) at a time sharing the
  // codebook fragments.  ldmatrix of the fp32 rows gives lane (g, p) dims p and
  // p + 4 of rows g and g + 8; their fp16 hi and lo parts are the A fragment in
  // the K order of the permuted fp16 codebook.
  {
    const uint32_t abase = q_smem(arow);
    const uint32_t cb_lane = q_smem(&sm.cbh[0][0]) + 16u * (uint32_t)lane;  // x4: n-tiles 4G .. 4G + 3
    const int arow_l = (lane & 7) + 8 * ((lane >> 3) & 1), ahalf = lane >> 4;
#pragma unroll 1
    for (int mp = 0; mp < 8; ++mp) {
      uint32_t A[2][4];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int R = a_phys(2 * mp + q, arow_l);
        uint32_t w[4];
        q_ldsm_x4(abase + (uint32_t)(R * 32 + 16 * (ahalf ^ a_flip(R))), w);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {  // row g (words 0, 2) and row g + 8 (words 1, 3)
          const float x0 = __uint_as_float(w[rr]), x1 = __uint_as_float(w[rr + 2]);
          const __half2 hh = __floats2half2_rn(x0, x1);
          const float2 hf = __half22float2(hh);
          A[q][rr] = h2_bits(hh);
          A[q][2 + rr] = h2_bits(__floats2half2_rn(x0 - hf.x, x1 - hf.y));
        }
      }
      float b1[2][2], b2[2][2];
      int bg[2][2];
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          b1[q][r] = -INFINITY;
          b2[q][r] = -INFINITY;
          bg[q][r] = 0;
        }
#pragma unroll
      for (int G = 0; G < NCODES / 32; ++G) {
        uint32_t B4[4];
        q_ldsm_x4(cb_lane + 512u * (uint32_t)G, B4);
        const float4 bz01 = *reinterpret_cast<const float4*>(&sm.biasq[32 * G + 8 * qp]);
        const float4 bz23 = *reinterpret_cast<const float4*>(&sm.biasq[32 * G + 8 * qp + 4]);
        const float bzv[8] = {bz01.x, bz01.y, bz01.z, bz01.w, bz23.x, bz23.y, bz23.z, bz23.w};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float d[4][4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            d[i][0] = bzv[2 * i]; d[i][1] = bzv[2 * i + 1]; d[i][2] = bzv[2 * i]; d[i][3] = bzv[2 * i + 1];
            q_mma_bb(d[i], A[q], B4[i]);
          }
          // group maxima of rows g (0, 1) and g + 8 (2, 3) as shallow trees
          const float gm[2] = {max3f(max3f(d[0][0], d[0][1], d[1][0]), max3f(d[1][1], d[2][0], d[2][1]),
                                     fmaxf(d[3][0], d[3][1])),
                               max3f(max3f(d[0][2], d[0][3], d[1][2]), max3f(d[1][3], d[2][2], d[2][3]),
                                     fmaxf(d[3][2], d[3][3]))};
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float lo = fminf(b1[q][r], gm[r]);
            bg[q][r] = (gm[r] > b1[q][r]) ? G : bg[q][r];
            b1[q][r] = fmaxf(b1[q][r], gm[r]);
            b2[q][r] = fmaxf(b2[q][r], lo);
          }
        }
      }
      // merge over the quad: best group maximum, its (group, lane), and the
      // largest maximum of every other group
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float x1 = b1[q][r], x2 = b2[q][r];
          int id = 4 * bg[q][r] + qp;
#pragma unroll
          for (int m = 1; m <= 2; m <<= 1) {
            const float y1 = __shfl_xor_sync(0xffffffffu, x1, m), y2 = __shfl_xor_sync(0xffffffffu, x2, m);
            const int yid = __shfl_xor_sync(0xffffffffu, id, m);
            x2 = fmaxf(fmaxf(x2, y2), fminf(x1, y1));
            id = (y1 > x1 || (y1 == x1 && yid < id)) ? yid : id;
            x1 = fmaxf(x1, y1);
          }
          if (qp == 0) {
            const int tok = 16 * warp + 2 * mp + q, j = qg + 8 * r;
            sm.grp[tok][j] = (uint8_t)id;
            sm.thr[tok][j] = x2;  // other groups' best tensor score, until (3) overwrites it
          }
        }
    }
  }
  __syncwarp();
  // (3) exact-arithmetic rescan of the winning group by the owner lane
  uint32_t need = 0u;
#pragma unroll 2
  for (int jj = 0; jj < HSUB; ++jj) {
    const int j = HSUB * h + jj;
    const int id = sm.grp[tk][j];
    const float other = sm.thr[tk][j];
    const float4 u0 = *urow(tk, j, 0), u1 = *urow(tk, j, 1);
    const float a[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    const int kbase = 32 * (id >> 2) + 2 * (id & 3);
    float best = -INFINITY, second = -INFINITY;
    int idx = kbase;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = kbase + 8 * i + e;
        const float4 c0 = *reinterpret_cast<const float4*>(&sm.cb[k][0]);
        const float4 c1 = *reinterpret_cast<const float4*>(&sm.cb[k][4]);
        float sc = sm.bias[k];
        sc = fmaf(a[0], c0.x, sc);
        sc = fmaf(a[1], c0.y, sc);
        sc = fmaf(a[2], c0.z, sc);
        sc = fmaf(a[3], c0.w, sc);
        sc = fmaf(a[4], c1.x, sc);
        sc = fmaf(a[5], c1.y, sc);
        sc = fmaf(a[6], c1.z, sc);
        sc = fmaf(a[7], c1.w, sc);
        const float lo = fminf(best, sc);
        idx = (sc > best) ? k : idx;
        best = fmaxf(best, sc);
        second = fmaxf(second, lo);
      }
    float na = 0.f;
#pragma unroll
    for (int i = 0; i < SUB; ++i) na = fmaf(a[i], a[i], na);
    na = sqrtf(na) * 1.0001f;
    // a rival within twice the fp32 bound of the best may be the true best; so may
    // another group whose tensor score is within the fp32 and tensor bounds
    const float margin = 2.0f * GAMMA9 * (cmax2 + na * cmax) * 1.01f;
    const float m_tc = (TC_REL * (1.001f * na * cmax + 0.5f * cmax2) + na * cdel) * 1.01f;
    sm.thr[tk][j] = best - margin;
    sm.code[tk][j] = (uint8_t)idx;
    need |= ((second >= best - margin || other >= best - 0.5f * margin - m_tc) ? 1u : 0u) << jj;
  }

  if (valid) {
#pragma unroll 1
    for (int jj = 0; jj < HSUB; ++jj)
      if ((need >> jj) & 1u) sm.flag[atomicAdd(&sm.nflag, 1)] = (uint16_t)(tk * NSUB + HSUB * h + jj);
  }
  __syncthreads();

  // ---- (4) exact fp64 re-decision of the flagged sub-vectors, a warp each ----
  // Candidates: codewords whose sequential fp32 score reaches the threshold
  // (best - twice the fp32 bound); the winner by fp64 squared distance, ties to
  // the lowest index.
  {
    const int nflag = sm.nflag;
#pragma unroll 1
    for (int f = warp; f < nflag; f += QTHREADS / 32) {
      const int ftk = sm.flag[f] / NSUB, fj = sm.flag[f] % NSUB;
      const float4 fa0 = *urow(ftk, fj, 0), fa1 = *urow(ftk, fj, 1);
      const float a[8] = {fa0.x, fa0.y, fa0.z, fa0.w, fa1.x, fa1.y, fa1.z, fa1.w};
      const float thr = sm.thr[ftk][fj];
      double bestd = INFINITY;
      int bi = NCODES;
#pragma unroll 1
      for (int k = lane; k < NCODES; k += 32) {
        float sc = sm.bias[k];
#pragma unroll
        for (int i = 0; i < SUB; ++i) sc = fmaf(a[i], sm.cb[k][i], sc);
        if (sc >= thr) {
          double dd = 0.0;
#pragma unroll
          for (int i = 0; i < SUB; ++i) {
            const double e = (double)a[i] - (double)sm.cb[k][i];
            dd = fma(e, e, dd);
          }
          if (dd < bestd) { bestd = dd; bi = k; }
        }
      }
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) {
        const double od = __shfl_xor_sync(0xffffffffu, bestd, m);
        const int ob = __shfl_xor_sync(0xffffffffu, bi, m);
        if (od < bestd || (od == bestd && ob < bi)) { bestd = od; bi = ob; }
      }
      if (lane == 0 && bi < NCODES) sm.code[ftk][fj] = (uint8_t)bi;
    }
  }
  __syncthreads();

  // ---- adaptive scale: alpha = ||u||^2 / (u . u_hat) --------------------------
  double dot = 0.0, uu = 0.0;
#pragma unroll 4
  for (int jj = 0; jj < HSUB; ++jj) {
    const int j = HSUB * h + jj;
    const int cj = sm.code[tk][j];
    const float4 q0 = *reinterpret_cast<const float4*>(&sm.cb[cj][0]);
    const float4 q1 = *reinterpret_cast<const float4*>(&sm.cb[cj][4]);
    const float4 u0 = *urow(tk, j, 0), u1 = *urow(tk, j, 1);
    const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    float dj = 0.f, uj = 0.f;
#pragma unroll
    for (int i = 0; i < SUB; ++i) {
      dj = fmaf(uv[i], qv[i], dj);
      uj = fmaf(uv[i], uv[i], uj);
    }
    dot += (double)dj;
    uu += (double)uj;
  }
  // halves combined in a fixed order (low half first) so both lanes agree bit for bit
  const double dot_o = __shfl_xor_sync(0xffffffffu, dot, 1), uu_o = __shfl_xor_sync(0xffffffffu, uu, 1);
  dot = h ? dot_o + dot : dot + dot_o;
  uu = h ? uu_o + uu : uu + uu_o;
  double alpha = (dot > 0.0) ? uu / dot : 1.0;
  if (!scale_adjust) alpha = 1.0;

  // ---- packed stores ---------------------------------------------------------
  if (valid) {
    *reinterpret_cast<uint2*>(codes + (int64_t)tk * NSUB + HSUB * h) =
        *reinterpret_cast<const uint2*>(&sm.code[tk][HSUB * h]);
    if (h == 0) {
      if constexpr (MODE == NSN_MODE_2BIT)
        *reinterpret_cast<uint4*>(signs + (int64_t)tk * NSUB) = *reinterpret_cast<const uint4*>(&sm.sgn[tk][0]);
      const BlockOut bo = block_out(cv, seq, tok0, blk);
      if (bo.dq) bo.s2[tk] = __double2half(alpha * sm.s2[tk]);
      else bo.norms[tk] = __halves2half2(__double2half(sm.s1[tk]), __double2half(alpha * sm.s2[tk]));
    }
  }
  if (cv.dq) store_double_quant(sm, n, block_out(cv, seq, tok0, blk));
  __syncthreads();  // shared memory is reused by the caller's next block
}

// ---------------------------------------------------------------------------
// Prefill: grid (blocks, kv-heads, batch).
// ---------------------------------------------------------------------------
// Tokens of sequence b and its quantized prefix.  Without `lengths` every
// sequence has the common n_tokens / q_tokens; with it, sequence b has
// lengths[b] tokens (an entry outside [0, max_tokens] counts as 0 and is
// flagged) and the same split rule: window 0 quantizes all of them, window 128
// quantizes 128 floor((L - 1) / 128) and keeps the rest (1..128) in the window.
struct PrefillSplit {
  int n, q;
  bool bad;
};

__device__ __forceinline__ PrefillSplit prefill_split(const int32_t* __restrict__ lengths, int b, int n_tokens,
                                                      int q_tokens, int window_len) {
  if (!lengths) return {n_tokens, q_tokens, false};
  int L = lengths[b];
  const bool bad = L < 0 || L > n_tokens;
  if (bad) L = 0;
  const int q = L == 0 ? 0 : (window_len == 0 ? L : BLK * ((L - 1) / BLK));
  return {L, q, bad};
}

template <int DT, int MODE>
__global__ void __launch_bounds__(QTHREADS, 2)
quantize_prefill_kernel(const void* __restrict__ x, int64_t sb, int64_t st, int64_t sh, int q_tokens, int n_tokens,
                        const int32_t* __restrict__ lengths, CacheView cv, const float* __restrict__ codebook) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  QuantSmem& sm = *reinterpret_cast<QuantSmem*>(smem_raw);
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const PrefillSplit ps = prefill_split(lengths, b, n_tokens, q_tokens, cv.window_len);
  const int n = min(BLK, ps.q - blk * BLK);
  if (n <= 0) return;
  stage_codebook(sm, codebook);
  const int64_t seq = (int64_t)b * cv.n_kv_heads + h;
  const int64_t tok0 = seq * cv.capacity + (int64_t)blk * BLK;
  quantize_block_dev<DT, MODE>(sm, x, (int64_t)b * sb + (int64_t)blk * BLK * st + (int64_t)h * sh, st, n,
                               cv.codes + tok0 * NSUB, MODE == NSN_MODE_2BIT ? cv.signs + tok0 * NSUB : nullptr,
                               cv, seq, tok0, blk, cv.scale_adjust);
}

// Prefill tail: copies tokens [q, L) of each sequence to the residual window
// (fp16) and sets the counters; a rejected ragged length sets status bit 4.
// grid (kv-heads, batch), 128 threads.
template <int DT>
__global__ void window_fill_kernel(const void* __restrict__ x, int64_t sb, int64_t st, int64_t sh, int q_tokens,
                                   int n_tokens, const int32_t* __restrict__ lengths, CacheView cv) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int64_t seq = (int64_t)b * cv.n_kv_heads + h;
  const PrefillSplit ps = prefill_split(lengths, b, n_tokens, q_tokens, cv.window_len);
  const int nw = ps.n - ps.q;
  for (int q = threadIdx.x; q < nw * (D / 8); q += blockDim.x) {
    const int row = q / (D / 8), ch = q % (D / 8);
    float vals[8];
    load8<DT>(x, (int64_t)b * sb + (int64_t)(ps.q + row) * st + (int64_t)h * sh + ch * 8, vals);
    *reinterpret_cast<uint4*>(cv.window + (seq * cv.window_len + row) * D + ch * 8) = pack8_f16(vals);
  }
  if (threadIdx.x == 0) {
    cv.n_quant[seq] = ps.q;
    cv.n_window[seq] = nw;
    if (ps.bad && h == 0 && cv.status) atomicOr(cv.status, 4);
  }
}

// ---------------------------------------------------------------------------
// Append one token per (b, h) to K (blockIdx.z == 0) and V (blockIdx.z == 1),
// flushing a full window into the quantized part first.  grid (kv-heads, batch, 2).
// ---------------------------------------------------------------------------
template <int DTN>
__global__ void __launch_bounds__(QTHREADS, 2)
append_kernel(CacheView kc, CacheView vc, const void* __restrict__ k_new, const void* __restrict__ v_new,
              int64_t sb, int64_t sh, const float* __restrict__ cbk, const float* __restrict__ cbv) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  QuantSmem& sm = *reinterpret_cast<QuantSmem*>(smem_raw);
  __shared__ int state[2];
  const bool is_v = blockIdx.z == 1;
  const CacheView c = is_v ? vc : kc;
  const void* src_new = is_v ? v_new : k_new;
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const int64_t seq = (int64_t)b * c.n_kv_heads + h;
  if (t == 0) { state[0] = c.n_quant[seq]; state[1] = c.n_window[seq]; }
  __syncthreads();
  int nq = state[0], nw = state[1];
  bool ok = true;
  if (nw >= c.window_len) {
    if (nq + BLK > c.capacity || (nq % BLK) != 0) {
      ok = false;
      if (t == 0 && c.status) atomicOr(c.status, 1);
    } else {
      stage_codebook(sm, is_v ? cbv : cbk);
      const int64_t tok0 = seq * c.capacity + nq;
      const int blk = nq / BLK;
      uint8_t* sg = c.mode == NSN_MODE_2BIT ? c.signs + tok0 * NSUB : nullptr;
      if (c.mode == NSN_MODE_2BIT)
        quantize_block_dev<NSN_DTYPE_F16, NSN_MODE_2BIT>(sm, c.window, seq * c.window_len * D, D, BLK,
                                                         c.codes + tok0 * NSUB, sg, c, seq, tok0, blk, c.scale_adjust);
      else
        quantize_block_dev<NSN_DTYPE_F16, NSN_MODE_1BIT>(sm, c.window, seq * c.window_len * D, D, BLK,
                                                         c.codes + tok0 * NSUB, sg, c, seq, tok0, blk, c.scale_adjust);
      nq += BLK;
      nw = 0;
    }
  }
  __syncthreads();  // the flushed window rows are consumed before row 0 is overwritten
  if (!ok) return;
  if (t < D / 8) {
    float vals[8];
    load8<DTN>(src_new, (int64_t)b * sb + (int64_t)h * sh + t * 8, vals);
    *reinterpret_cast<uint4*>(c.window + (seq * c.window_len + nw) * D + t * 8) = pack8_f16(vals);
  }
  if (t == 0) {
    c.n_quant[seq] = nq;
    c.n_window[seq] = nw + 1;
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
size_t quant_smem_bytes() { return sizeof(QuantSmem); }

template <int DT, int MODE>
static cudaError_t launch_prefill_t(const void* x, int64_t sb, int64_t st, int64_t sh, int q_tokens, int n_tokens,
                                    const int32_t* lengths, const CacheView& cv, const float* cb, cudaStream_t s) {
  const size_t smem = sizeof(QuantSmem);
  cudaError_t e = cudaFuncSetAttribute(quantize_prefill_kernel<DT, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nblk = (q_tokens + BLK - 1) / BLK;
  if (nblk > 0) {
    dim3 grid(nblk, cv.n_kv_heads, cv.batch);
    quantize_prefill_kernel<DT, MODE><<<grid, QTHREADS, smem, s>>>(x, sb, st, sh, q_tokens, n_tokens, lengths, cv, cb);
  }
  return cudaGetLastError();
}

template <int MODE>
static cudaError_t launch_prefill_m(const void* x, int dtype, int64_t sb, int64_t st, int64_t sh, int q_tokens,
                                    int n_tokens, const int32_t* lengths, const CacheView& cv, const float* cb,
                                    cudaStream_t s) {
  if (dtype == NSN_DTYPE_F32)
    return launch_prefill_t<NSN_DTYPE_F32, MODE>(x, sb, st, sh, q_tokens, n_tokens, lengths, cv, cb, s);
  if (dtype == NSN_DTYPE_BF16)
    return launch_prefill_t<NSN_DTYPE_BF16, MODE>(x, sb, st, sh, q_tokens, n_tokens, lengths, cv, cb, s);
  return launch_prefill_t<NSN_DTYPE_F16, MODE>(x, sb, st, sh, q_tokens, n_tokens, lengths, cv, cb, s);
}

cudaError_t launch_quantize_prefill(const void* x, int dtype, int64_t sb, int64_t st, int64_t sh, int q_tokens,
                                    int n_tokens, const int32_t* lengths, const CacheView& cv, const float* cb,
                                    cudaStream_t s) {
  if (q_tokens > 0) {
    const cudaError_t e =
        cv.mode == NSN_MODE_1BIT
            ? launch_prefill_m<NSN_MODE_1BIT>(x, dtype, sb, st, sh, q_tokens, n_tokens, lengths, cv, cb, s)
            : launch_prefill_m<NSN_MODE_2BIT>(x, dtype, sb, st, sh, q_tokens, n_tokens, lengths, cv, cb, s);
    if (e != cudaSuccess) return e;
  }
  dim3 g2(cv.n_kv_heads, cv.batch);
  if (dtype == NSN_DTYPE_F32)
    window_fill_kernel<NSN_DTYPE_F32><<<g2, 128, 0, s>>>(x, sb, st, sh, q_tokens, n_tokens, lengths, cv);
  else if (dtype == NSN_DTYPE_BF16)
    window_fill_kernel<NSN_DTYPE_BF16><<<g2, 128, 0, s>>>(x, sb, st, sh, q_tokens, n_tokens, lengths, cv);
  else
    window_fill_kernel<NSN_DTYPE_F16><<<g2, 128, 0, s>>>(x, sb, st, sh, q_tokens, n_tokens, lengths, cv);
  return cudaGetLastError();
}

template <int DTN>
static cudaError_t launch_append_t(const CacheView& kc, const CacheView& vc, const void* kn, const void* vn,
                                   int64_t sb, int64_t sh, const float* cbk, const float* cbv, cudaStream_t s) {
  const size_t smem = sizeof(QuantSmem);
  cudaError_t e = cudaFuncSetAttribute(append_kernel<DTN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(kc.n_kv_heads, kc.batch, 2);
  append_kernel<DTN><<<grid, QTHREADS, smem, s>>>(kc, vc, kn, vn, sb, sh, cbk, cbv);
  return cudaGetLastError();
}

cudaError_t launch_append(const CacheView& kc, const CacheView& vc, const void* kn, const void* vn, int dtype,
                          int64_t sb, int64_t sh, const float* cbk, const float* cbv, cudaStream_t s) {
  if (dtype == NSN_DTYPE_F32) return launch_append_t<NSN_DTYPE_F32>(kc, vc, kn, vn, sb, sh, cbk, cbv, s);
  if (dtype == NSN_DTYPE_BF16) return launch_append_t<NSN_DTYPE_BF16>(kc, vc, kn, vn, sb, sh, cbk, cbv, s);
  return launch_append_t<NSN_DTYPE_F16>(kc, vc, kn, vn, sb, sh, cbk, cbv, s);
}

}  // namespace nsn
