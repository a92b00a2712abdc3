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
// Quantized part: grid (nsplit_q, kv-heads, batch), 128 threads.
// ---------------------------------------------------------------------------
// Every member is 16-byte aligned (vector loads); unused tables shrink to 4 floats.
template <int G, int MK, int MV>
struct SplitSmem {
  alignas(16) float qt[G][D];
  alignas(16) float lut[MK == NSN_MODE_1BIT ? NSUB * NCODES * G : 4];  // [s][k][h]
  alignas(16) float cbk[MK == NSN_MODE_2BIT ? NCODES * SUB : 4];
  alignas(16) float cbv[NCODES * SUB];
  alignas(16) float w[BLK][G];
  alignas(16) uint4 vcode[BLK];
  alignas(16) uint4 vsign[BLK];
  alignas(16) float red[4][16];
  alignas(16) float racc[8][G][D];  // final reduction over the 8 token groups
};

template <int G, int MK, int MV>
__global__ void __launch_bounds__(128)
decode_split_kernel(CacheView kc, CacheView vc, const void* __restrict__ q, int dtype, int64_t qsb, int64_t qsh,
                    float qscale, const float* __restrict__ cbk, const float* __restrict__ cbv,
                    float* __restrict__ ws, DecodeGeom geom) {
  static_assert(2 * G <= 16, "reduction scratch holds 16 values");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  using Smem = SplitSmem<G, MK, MV>;
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
  const int64_t seq = (int64_t)b * kc.n_kv_heads + hk;
  const int64_t pidx = seq * (geom.nsplit_q + 1) + split;
  const int64_t P = (int64_t)kc.batch * kc.n_kv_heads * (geom.nsplit_q + 1);
  float* ws_acc = ws + acc_offset(P, G);

  const int nq = min(min(kc.n_quant[seq], vc.n_quant[seq]), kc.capacity);
  const int start = split * geom.chunk;
  const int end = min(start + geom.chunk, nq);
  if (start >= end) {
    for (int i = t; i < G * D; i += blockDim.x) ws_acc[pidx * G * D + i] = 0.f;
    if (t < G) {
      partial_ml(ws, pidx, G, t)[0] = NEG_BIG;
      partial_ml(ws, pidx, G, t)[1] = 0.f;
    }
    return;
  }

  load_queries<G>(&sm.qt[0][0], q, dtype, qsb, qsh, b, hk, qscale, true);
  for (int i = t; i < NCODES * SUB; i += blockDim.x) {
    sm.cbv[i] = f16r(__ldg(cbv + i));
    if constexpr (MK == NSN_MODE_2BIT) sm.cbk[i] = f16r(__ldg(cbk + i));
  }
  __syncthreads();
  if constexpr (MK == NSN_MODE_1BIT) {
    for (int e = t; e < NSUB * NCODES; e += blockDim.x) {
      const int s = e / NCODES, k = e % NCODES;
      float c[SUB];
#pragma unroll
      for (int i = 0; i < SUB; ++i) c[i] = f16r(__ldg(cbk + k * SUB + i));
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < SUB; ++i) acc = fmaf(sm.qt[h][SUB * s + i], c[i], acc);
        sm.lut[e * G + h] = acc;
      }
    }
    __syncthreads();
  }

  const int64_t cap = kc.capacity;
  const int64_t nblk_cap = cap / BLK;
  const uint4* kcodes = reinterpret_cast<const uint4*>(kc.codes) + seq * cap;
  const uint4* ksigns = MK == NSN_MODE_2BIT ? reinterpret_cast<const uint4*>(kc.signs) + seq * cap : nullptr;
  const __half2* knorm = kc.norms + seq * cap;
  const __half* kmean = kc.means + seq * nblk_cap * D;
  const uint4* vcodes = reinterpret_cast<const uint4*>(vc.codes) + seq * cap;
  const uint4* vsigns = MV == NSN_MODE_2BIT ? reinterpret_cast<const uint4*>(vc.signs) + seq * cap : nullptr;
  const __half2* vnorm = vc.norms + seq * cap;
  const __half* vmean = vc.means + seq * nblk_cap * D;

  float m_run[G], l_run[G], accm[G], acc[G][SUB];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_run[h] = NEG_BIG;
    l_run[h] = 0.f;
    accm[h] = 0.f;
#pragma unroll
    for (int i = 0; i < SUB; ++i) acc[h][i] = 0.f;
  }
  const int my_s = t % NSUB, my_tg = t / NSUB;

  for (int tile0 = start; tile0 < end; tile0 += BLK) {
    const int tok = tile0 + t;
    const bool valid = tok < end;
    const int blk = tile0 / BLK;
    const float oK = __half2float(kmean[(int64_t)blk * D + t]);
    const float oV = __half2float(vmean[(int64_t)blk * D + t]);

    uint4 kcw = make_uint4(0, 0, 0, 0), ksw = make_uint4(0, 0, 0, 0), vcw = make_uint4(0, 0, 0, 0),
          vsw = make_uint4(0, 0, 0, 0);
    float2 kn = make_float2(0.f, 0.f), vn = make_float2(0.f, 0.f);
    if (valid) {
      kcw = kcodes[tok];
      if constexpr (MK == NSN_MODE_2BIT) ksw = ksigns[tok];
      kn = __half22float2(knorm[tok]);
      vcw = vcodes[tok];
      if constexpr (MV == NSN_MODE_2BIT) vsw = vsigns[tok];
      vn = __half22float2(vnorm[tok]);
    }
    sm.vcode[t] = vcw;
    sm.vsign[t] = vsw;

    // (Hq) . o_b for the K block of this tile
    float qo[G];
#pragma unroll
    for (int h = 0; h < G; ++h) qo[h] = sm.qt[h][t] * oK;
    block_reduce<G, false>(qo, sm.red);

    // q~ . u_hat from the codes
    float dot[G];
#pragma unroll
    for (int h = 0; h < G; ++h) dot[h] = 0.f;
    const uint32_t kcs[4] = {kcw.x, kcw.y, kcw.z, kcw.w};
    const uint32_t kss[4] = {ksw.x, ksw.y, ksw.z, ksw.w};
#pragma unroll
    for (int s = 0; s < NSUB; ++s) {
      const int code = (kcs[s >> 2] >> (8 * (s & 3))) & 0xff;
      if constexpr (MK == NSN_MODE_1BIT) {
        const float* e = &sm.lut[(s * NCODES + code) * G];
#pragma unroll
        for (int h = 0; h < G; ++h) dot[h] += e[h];
      } else {
        const uint32_t sb = (kss[s >> 2] >> (8 * (s & 3))) & 0xff;
        const float4 c0 = *reinterpret_cast<const float4*>(&sm.cbk[code * SUB]);
        const float4 c1 = *reinterpret_cast<const float4*>(&sm.cbk[code * SUB + 4]);
        float cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int i = 0; i < SUB; ++i) cw[i] = ((sb >> i) & 1) ? -cw[i] : cw[i];
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
          for (int i = 0; i < SUB; ++i) dot[h] = fmaf(sm.qt[h][SUB * s + i], cw[i], dot[h]);
        }
      }
    }
    float sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) sc[h] = valid ? kn.x * fmaf(kn.y, dot[h], qo[h]) : NEG_BIG;

    // online softmax
    float tmax[G];
#pragma unroll
    for (int h = 0; h < G; ++h) tmax[h] = sc[h];
    block_reduce<G, true>(tmax, sm.red);
    float corr[G], sums[2 * G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mn = fmaxf(m_run[h], tmax[h]);
      corr[h] = exp2f(m_run[h] - mn);
      m_run[h] = mn;
      const float p = valid ? exp2f(sc[h] - mn) : 0.f;
      sm.w[t][h] = p * vn.x * vn.y;
      sums[h] = p;
      sums[G + h] = p * vn.x;
    }
    block_reduce<2 * G, false>(sums, sm.red);  // also publishes sm.w / vcode / vsign
#pragma unroll
    for (int h = 0; h < G; ++h) {
      l_run[h] = fmaf(l_run[h], corr[h], sums[h]);
      accm[h] = fmaf(accm[h], corr[h], sums[G + h] * oV);
#pragma unroll
      for (int i = 0; i < SUB; ++i) acc[h][i] *= corr[h];
    }

    // value accumulation in the rotated domain: thread (s, tg) takes tokens tg, tg+8, ...
    const int nvalid = min(BLK, end - tile0);
    for (int tt = my_tg; tt < nvalid; tt += 8) {
      const uint4 cw4 = sm.vcode[tt];
      const uint32_t cws[4] = {cw4.x, cw4.y, cw4.z, cw4.w};
      const int code = (cws[my_s >> 2] >> (8 * (my_s & 3))) & 0xff;
      const float4 c0 = *reinterpret_cast<const float4*>(&sm.cbv[code * SUB]);
      const float4 c1 = *reinterpret_cast<const float4*>(&sm.cbv[code * SUB + 4]);
      float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      if constexpr (MV == NSN_MODE_2BIT) {
        const uint4 sw4 = sm.vsign[tt];
        const uint32_t sws[4] = {sw4.x, sw4.y, sw4.z, sw4.w};
        const uint32_t sb = (sws[my_s >> 2] >> (8 * (my_s & 3))) & 0xff;
#pragma unroll
        for (int i = 0; i < SUB; ++i) cv[i] = ((sb >> i) & 1) ? -cv[i] : cv[i];
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float wt = sm.w[tt][h];
#pragma unroll
        for (int i = 0; i < SUB; ++i) acc[h][i] = fmaf(wt, cv[i], acc[h][i]);
      }
    }
    __syncthreads();  // w / vcode / vsign are rewritten by the next tile
  }

  // reduce the 8 token groups; thread t owns rotated dim t
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int i = 0; i < SUB; ++i) sm.racc[my_tg][h][my_s * SUB + i] = acc[h][i];
  __syncthreads();
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float s = accm[h];
#pragma unroll
    for (int g2 = 0; g2 < 8; ++g2) s += sm.racc[g2][h][t];
    ws_acc[(pidx * G + h) * D + t] = s;
  }
  if (t < G) {
    partial_ml(ws, pidx, G, t)[0] = m_run[t];
    partial_ml(ws, pidx, G, t)[1] = l_run[t];
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
DecodeGeom decode_geometry(int capacity, int n_q_heads, int n_kv_heads) {
  DecodeGeom g;
  g.g = n_q_heads / n_kv_heads;
  g.chunk = capacity < 1024 ? capacity : 1024;
  g.nsplit_q = (capacity + g.chunk - 1) / g.chunk;
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
  const size_t smem = sizeof(SplitSmem<G, MK, MV>);
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<G, MK, MV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(geom.nsplit_q, kc.n_kv_heads, kc.batch);
  decode_split_kernel<G, MK, MV><<<grid, 128, smem, s>>>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, ws, geom);
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
