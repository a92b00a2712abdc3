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
// One kernel (decode_kernel) does the whole call:
//   - one warp per split (a contiguous range of 64-token stages of one (batch,
//     kv-head) and a group of up to 4 query heads): rotated query, scores from the
//     codes, online softmax, value accumulation from the codewords -> partial
//     (m, l, acc) in the rotated domain;
//   - the last split of a sequence also attends the residual window (original
//     domain) -> a second partial;
//   - the thread block of the warp that finishes a (sequence, head group) last
//     (a self-resetting counter decides) merges the partials by log-sum-exp,
//     applies H to the rotated value sum and writes the output rows.
// Scores are carried in log2 units (the query is pre-scaled by softmax_scale*log2 e).

#include <mutex>

#include "nsn_common.cuh"
#include "nsn_launch.h"

namespace nsn {

constexpr float LOG2E = 1.4426950408889634f;
constexpr float INV_SQRT_D = 0.08838834764831845f;  // 1/sqrt(128)

// Partials layout: [P][G][2] (m, l) floats, then -- from a 16-byte aligned
// offset -- [P][G][128] accumulators; P = batch * kv-heads * (nsplit_q + 1)
// (slot nsplit_q of each sequence is its residual window).
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

// Two 8x8 matrices (row addresses from lanes 0-15): for A operands whose rows
// 8-15 repeat rows 0-7, half the shared-memory reads of an x4.
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
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

// Code of k-step j (0..7) from the 8 code bytes a lane reads: the cache stores a
// token's codes as the even sub-vectors' (bytes 0-7) then the odd ones' (bytes
// 8-15), and a lane whose ldmatrix row is sub-vector 2j + par reads half par.
__device__ __forceinline__ uint32_t code_byte(const uint2& w, int j) {
  return __byte_perm(j < 4 ? w.x : w.y, 0u, 0x4440u | (uint32_t)(j & 3));
}

// ---------------------------------------------------------------------------
// Quantized part.  One CTA of 16 warps per SM; every warp owns one split: a
// contiguous range of 64-token stages of one (batch, kv-head) sequence, and
// writes its own partial (m, l, O).  The CTA shares the two replicated fp16
// codebooks (staged once) and, at the end, the merge.  Compressed tokens stream
// through a per-warp double-buffered ring of 64-token stages filled by 1-D bulk
// copies, so one stage is always in flight while the previous one is consumed.
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
// stage layout (bytes): K codes | K signs | K norms | V codes | V signs | V norms
constexpr int ST_KC = 0, ST_KS = 1024, ST_KN = 2048, ST_VC = 2304, ST_VS = 3328, ST_VN = 4352, STAGE_BYTES = 4608;
constexpr int MEAN_BYTES = 512;  // K mean row | V mean row of one block (fp16)
// The running max is re-based only when a score exceeds it by more than this
// (log2 units): weights stay below 2^8 and exact in fp32, and most tiles skip the
// max reduction.
constexpr float LAZY_MAX_SLACK = 8.0f;
// Upper bound on suspended mbarrier wait attempts before a wait gives up (error
// flag, no hang): a few seconds in total.
constexpr uint32_t WAIT_LIMIT = 4096u;

struct DecSmem {
  alignas(128) uint4 cbk[NCODES][8];  // replicated fp16 codebooks (32 KB each)
  alignas(128) uint4 cbv[NCODES][8];
  alignas(128) unsigned char stage[DEC_WARPS][2][STAGE_BYTES];
  alignas(128) unsigned char means[DEC_WARPS][2][MEAN_BYTES];
  alignas(8) uint64_t bar[DEC_WARPS][2];
  int merge_n;                    // (sequence, head group)s whose last ticket a warp of this CTA took
  int merge_seq[DEC_WARPS];
  int merge_hg[DEC_WARPS];
};

__device__ __forceinline__ uint4 cb_row_f16(const float* __restrict__ cb, int c) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(cb + c * SUB));
  const float4 b = __ldg(reinterpret_cast<const float4*>(cb + c * SUB) + 1);
  return make_uint4(pack_half2(a.x, a.y), pack_half2(a.z, a.w), pack_half2(b.x, b.y), pack_half2(b.z, b.w));
}

// ---- mbarrier + 1-D bulk copy (TMA) helpers ----
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// One wait attempt: the thread may sleep in hardware for up to SUSPEND_NS while the
// phase is incomplete (no polling instructions are issued meanwhile).
constexpr uint32_t SUSPEND_NS = 1000000u;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity), "r"(SUSPEND_NS)
      : "memory");
  return done != 0;
}
// Bounded wait (at most `limit` suspended attempts); false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t limit = WAIT_LIMIT) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Lane 0 issues the bulk copies of one 64-token stage (+ the block's mean rows
// when `with_means`) and arms the stage's barrier with the byte count.
// With double quantization (DQ) the norms region receives alpha*s2 (fp16, 128 B)
// followed by the 4-bit s1 levels (32 B), and the mean slot receives, from byte
// 256 on, the K and V o levels (64 B each) and their (lo, hi) parameters (16 B
// each); the fp16 mean rows are formed from them in shared memory.
constexpr int DQ_LEV = 2 * D;           // o levels of K at +256, of V at +320
constexpr int DQ_PAR = 2 * D + D;       // parameters of K at +384, of V at +400
// With RGH > 0 (pre-RoPE keys) the K logits of the stage were computed by
// rope_scores_kernel: the stage's 64 x RGH fp32 logits (from `rsrc`, this warp's
// (sequence, head group) row of them) take the place of the K codes, and the K
// signs and norms are not copied.
template <int MK, int MV, bool DQ, int RGH = 0>
__device__ __forceinline__ void issue_stage(uint32_t dst, uint32_t mdst, uint32_t bar, const CacheView& kc,
                                           const CacheView& vc, int64_t seq, int t0, bool with_means,
                                           const float* rsrc = nullptr) {
  const int64_t cap = kc.capacity;
  const int64_t tok = seq * cap + t0;
  constexpr uint32_t CB = STAGE_TOK * 16;
  constexpr uint32_t NB = DQ ? STAGE_TOK * 2 + STAGE_TOK / 2 : STAGE_TOK * 4;
  constexpr uint32_t MB = DQ ? 2 * (D / 2) + 2 * 16 : MEAN_BYTES;
  constexpr uint32_t RB = STAGE_TOK * RGH * 4;
  static_assert(RB <= ST_KS - ST_KC, "the stage's logits fit the K code area");
  constexpr uint32_t KB = RGH > 0 ? RB : CB + NB + (MK == NSN_MODE_2BIT ? CB : 0);
  const uint32_t bytes = KB + CB + NB + (MV == NSN_MODE_2BIT ? CB : 0) + (with_means ? MB : 0);
  mbar_expect_tx(bar, bytes);
  if constexpr (RGH > 0) {
    bulk_g2s(dst + ST_KC, rsrc + (int64_t)t0 * RGH, RB, bar);
  } else {
    bulk_g2s(dst + ST_KC, kc.codes + tok * NSUB, CB, bar);
    if constexpr (MK == NSN_MODE_2BIT) bulk_g2s(dst + ST_KS, kc.signs + tok * NSUB, CB, bar);
  }
  bulk_g2s(dst + ST_VC, vc.codes + tok * NSUB, CB, bar);
  if constexpr (MV == NSN_MODE_2BIT) bulk_g2s(dst + ST_VS, vc.signs + tok * NSUB, CB, bar);
  const int64_t blk = seq * (cap / BLK) + t0 / BLK;
  if constexpr (DQ) {
    if constexpr (RGH == 0) {
      bulk_g2s(dst + ST_KN, reinterpret_cast<const __half*>(kc.norms) + tok, STAGE_TOK * 2, bar);
      bulk_g2s(dst + ST_KN + STAGE_TOK * 2, kc.s1_levels + tok / 2, STAGE_TOK / 2, bar);
    }
    bulk_g2s(dst + ST_VN, reinterpret_cast<const __half*>(vc.norms) + tok, STAGE_TOK * 2, bar);
    bulk_g2s(dst + ST_VN + STAGE_TOK * 2, vc.s1_levels + tok / 2, STAGE_TOK / 2, bar);
    if (with_means) {
      bulk_g2s(mdst + DQ_LEV, reinterpret_cast<const uint8_t*>(kc.means) + blk * (D / 2), D / 2, bar);
      bulk_g2s(mdst + DQ_LEV + D / 2, reinterpret_cast<const uint8_t*>(vc.means) + blk * (D / 2), D / 2, bar);
      bulk_g2s(mdst + DQ_PAR, kc.dq_params + blk * 8, 16, bar);
      bulk_g2s(mdst + DQ_PAR + 16, vc.dq_params + blk * 8, 16, bar);
    }
  } else {
    if constexpr (RGH == 0) bulk_g2s(dst + ST_KN, kc.norms + tok, NB, bar);
    bulk_g2s(dst + ST_VN, vc.norms + tok, NB, bar);
    if (with_means) {
      bulk_g2s(mdst, kc.means + blk * D, D * 2, bar);
      bulk_g2s(mdst + D * 2, vc.means + blk * D, D * 2, bar);
    }
  }
}

// A 4-bit level (the low nibble of `bits`) as a float without an int-to-float
// conversion: 2^23 + level is exact in fp32, and subtracting 2^23 leaves the level.
__device__ __forceinline__ float nibble_f(uint32_t bits) {
  return __uint_as_float((bits & 15u) | 0x4B000000u) - 8388608.0f;
}

// (lo, step) of a 4-bit group from its fp16 (lo, hi) pair.
__device__ __forceinline__ float2 dq_lo_step(const unsigned char* par) {
  const float2 lh = __half22float2(*reinterpret_cast<const __half2*>(par));
  return make_float2(lh.x, (lh.y - lh.x) * (1.0f / 15.0f));
}

// Writes the fp16 mean row of one block (128 channels, lane l: channels 4l..4l+3)
// from its 4-bit levels into `row`.
__device__ __forceinline__ void dq_mean_row(unsigned char* row, const unsigned char* levels, const unsigned char* par,
                                            int lane) {
  const float2 ls = dq_lo_step(par);
  const uint32_t two = *reinterpret_cast<const uint16_t*>(levels + 2 * lane);
  const float c0 = fmaf(nibble_f(two), ls.y, ls.x), c1 = fmaf(nibble_f(two >> 4), ls.y, ls.x);
  const float c2 = fmaf(nibble_f(two >> 8), ls.y, ls.x), c3 = fmaf(nibble_f(two >> 12), ls.y, ls.x);
  *reinterpret_cast<uint2*>(row + 8 * lane) = make_uint2(pack_half2(c0, c1), pack_half2(c2, c3));
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// ---- residual-window chunks: 8 fp16 rows of K and of V per stage buffer ----
// Rows are copied one by one (one lane per row) into 272-byte slots so that the
// 8 rows of an ldmatrix fetch start in 8 different bank groups.
constexpr int WCHUNK = 8;
constexpr int WROWB = (D + 8) * 2;    // 272
constexpr int WC_V = WCHUNK * WROWB;  // V rows follow the K rows
static_assert(2 * WC_V <= STAGE_BYTES, "a window chunk fits one stage buffer");
// The residual window counts as this many 64-token stages when the quantized
// stages of a sequence are dealt out to its splits (the last split takes it).
constexpr int WINDOW_COST_STAGES = 4;

__device__ __forceinline__ void issue_window_chunk(uint32_t dst, uint32_t bar, const __half* krow, const __half* vrow,
                                                   int rows, int lane) {
  if (lane == 0) mbar_expect_tx(bar, (uint32_t)rows * 2u * (uint32_t)(D * 2));
  __syncwarp();
  if (lane < 2 * rows) {
    const int r = lane >> 1;
    const bool isv = (lane & 1) != 0;
    bulk_g2s(dst + (isv ? WC_V : 0) + (uint32_t)(r * WROWB), (isv ? vrow : krow) + r * D, D * 2, bar);
  }
}

// Query rows of the GH heads of a group: lane l receives elements 4l..4l+3.
template <int GH>
__device__ __forceinline__ void load_q_rows(float (&v)[GH][4], const void* __restrict__ q, int dtype, int64_t off0,
                                            int64_t qsh, int lane) {
#pragma unroll
  for (int h = 0; h < GH; ++h) {
    const int64_t off = off0 + (int64_t)h * qsh + 4 * lane;
    if (dtype == NSN_DTYPE_F32) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(q) + off));
      v[h][0] = f.x; v[h][1] = f.y; v[h][2] = f.z; v[h][3] = f.w;
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
      v[h][0] = a.x; v[h][1] = a.y; v[h][2] = c.x; v[h][3] = c.y;
    }
  }
}

// B operand of the score product for GH query heads: lane (g, p) holds column g
// (head g for g < 4, the fp16 rounding residual of head g - 4 for g >= 4), k rows
// 2p, 2p+1 (qb[j][0]) and 8+2p, 9+2p (qb[j][1]) of k-step j.  With `rotate` the
// query is taken to the Hadamard domain first (orthonormal H).  Each lane
// converts its own 4 values per head once and stores them as rows of an 8 x 128
// fp16 matrix (rows 0-3: fp16 of the heads, 4-7: rounding residuals; 272-byte
// rows) in `qs`, a free 2176-byte stretch of this warp's shared memory; four
// ldmatrix.x4 then deliver the fragments.
constexpr int QS_ROW = (D + 8) * 2;
template <int GH>
__device__ __forceinline__ void build_q_operand(uint32_t (&qb)[8][2], const float (&rows)[GH][4], float scale,
                                                bool rotate, int lane, unsigned char* qs) {
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    uint2 hi = make_uint2(0u, 0u), lo = make_uint2(0u, 0u);
    if (h < GH) {
      float v[4] = {rows[h < GH ? h : 0][0], rows[h < GH ? h : 0][1], rows[h < GH ? h : 0][2],
                    rows[h < GH ? h : 0][3]};
      if (rotate) fwht128_warp(v, lane);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] *= scale;
      split_half2(v[0], v[1], hi.x, lo.x);
      split_half2(v[2], v[3], hi.y, lo.y);
    }
    *reinterpret_cast<uint2*>(qs + h * QS_ROW + 8 * lane) = hi;
    *reinterpret_cast<uint2*>(qs + (h + 4) * QS_ROW + 8 * lane) = lo;
  }
  __syncwarp();
  const uint32_t base = smem_addr(qs) + (uint32_t)((lane & 7) * QS_ROW + 16 * (lane >> 3));
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    uint32_t r4[4];
    ldsm_x4(base + 64u * jj, r4);
    qb[2 * jj][0] = r4[0];
    qb[2 * jj][1] = r4[1];
    qb[2 * jj + 1][0] = r4[2];
    qb[2 * jj + 1][1] = r4[3];
  }
  __syncwarp();  // every lane has read the stretch ...
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // ... before a bulk copy may overwrite it
}

// Online-softmax state of one warp for its head pair (h0, h0 + 1): running max in
// log2 units, denominator and the O^T accumulator fragment (rows = dims, columns =
// heads).  `lazy_update` re-bases the running max only when a score exceeds it by
// more than LAZY_MAX_SLACK, so most tiles skip the max reduction.
struct SoftmaxState {
  float m0, m1, l0, l1;
  float O[8][4];
};

__device__ __forceinline__ void lazy_update(SoftmaxState& st, float sc0, float sc1, float& cm0, float& cm1) {
  if (__any_sync(0xffffffffu, fmaxf(sc0 - st.m0, sc1 - st.m1) > LAZY_MAX_SLACK)) {
    float t0 = sc0, t1 = sc1;
#pragma unroll
    for (int x = 2; x < 32; x <<= 1) {  // lanes sharing the head pair: xor 2, 4, 8, 16
      t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, x));
      t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, x));
    }
    const float n0 = fmaxf(st.m0, t0), n1 = fmaxf(st.m1, t1);
    const float c0 = fast_exp2(st.m0 - n0), c1 = fast_exp2(st.m1 - n1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      st.O[i][0] *= c0; st.O[i][1] *= c1; st.O[i][2] *= c0; st.O[i][3] *= c1;
    }
    st.l0 *= c0; st.l1 *= c1; cm0 *= c0; cm1 *= c1;
    st.m0 = n0; st.m1 = n1;
  }
}

// Writes a warp's partial (m, l, O^T) for the GH heads of its group: lanes p < 2
// own heads 2p, 2p + 1.  Reduces l across the lanes first.
template <int GH>
__device__ __forceinline__ void store_partial(SoftmaxState& st, float* __restrict__ ws, float* __restrict__ ws_acc,
                                              int64_t slot, int G, int hbase, int lane) {
  const int g = lane >> 2, p = lane & 3, h0 = 2 * (p & 1);
#pragma unroll
  for (int x = 2; x < 32; x <<= 1) {
    st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, x);
    st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, x);
  }
  if (p < 2) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int h = 2 * p + hh;
      if (h < GH) {
        float* dst = ws_acc + (slot * G + hbase + h) * D;
#pragma unroll
        for (int mm = 0; mm < 8; ++mm) {
          dst[16 * mm + g] = st.O[mm][hh];
          dst[16 * mm + 8 + g] = st.O[mm][2 + hh];
        }
      }
    }
    if (g == 0) {
      if (h0 < GH) {
        partial_ml(ws, slot, G, hbase + h0)[0] = st.m0;
        partial_ml(ws, slot, G, hbase + h0)[1] = st.l0;
      }
      if (h0 + 1 < GH) {
        partial_ml(ws, slot, G, hbase + h0 + 1)[0] = st.m1;
        partial_ml(ws, slot, G, hbase + h0 + 1)[1] = st.l1;
      }
    }
  }
}

// Log-sum-exp merge of the partials of one (sequence, head group), done by all
// threads of the CTA whose warp finished the group last.  Slots 0 .. nsplit-1
// hold the quantized part (rotated domain), slot nsplit the residual window
// (original domain).  The rotated value sum is taken back with H (H^T = H)
// before both parts are normalised together.  Partials written by other SMs are
// read through L2.  `scratch` is shared memory no longer in use (the stage
// buffers): (nsplit + 1) * GH float2 weights, then GH * 128 floats.
template <int GH>
__device__ __noinline__ void cta_merge(const float* ws, const float* ws_acc, int64_t p0, int nsplit, int G, int hbase,
                                       float* __restrict__ out_rows, float* scratch) {
  constexpr int CH = 32;  // slots whose accumulators a thread holds in registers at once
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nslot = nsplit + 1;
  float2* wt = reinterpret_cast<float2*>(scratch);          // [slot][h]: (m, l), then (weight, l)
  float* rot = scratch + 2 * ((nslot * GH + 1) & ~1);       // [h][128] rotated sums, [h][128] window sums, [h] max
  float* win = rot + GH * D;
  const bool own = tid < GH * D;                            // thread (h, d) owns one output element
  const int h = own ? tid / D : 0, d = tid % D;
  const float* acc_hd = ws_acc + (p0 * G + hbase + h) * D + d;   // slot s at + s * G * D
  // The accumulators of the first CH slots and the window element are requested
  // together with the (m, l) pairs, so all of them share one L2 round trip.
  float vals[CH];
#pragma unroll
  for (int k = 0; k < CH; ++k) vals[k] = (own && k < nsplit) ? __ldcg(acc_hd + (int64_t)k * G * D) : 0.f;
  const float wv = own ? __ldcg(acc_hd + (int64_t)nsplit * G * D) : 0.f;
  for (int i = tid; i < nslot * GH; i += blockDim.x) {
    const int slot = i / GH, hh = i % GH;
    wt[i] = __ldcg(reinterpret_cast<const float2*>(ws + ((p0 + slot) * G + hbase + hh) * 2));
  }
  __syncthreads();
  if (warp < GH) {  // warp hh: running max of the quantized slots, then their weights
    const int hh = warp;
    float mx = NEG_BIG;
    for (int s = lane; s < nsplit; s += 32) {
      const float2 ml = wt[s * GH + hh];
      if (ml.y > 0.f) mx = fmaxf(mx, ml.x);
    }
    mx = warp_max(mx);
    for (int s = lane; s < nsplit; s += 32) {
      const float2 ml = wt[s * GH + hh];
      wt[s * GH + hh] = make_float2(ml.y > 0.f ? fast_exp2(ml.x - mx) : 0.f, ml.y);
    }
    if (lane == 0) win[GH * D + hh] = mx;
  }
  __syncthreads();
  if (own) {  // thread (h, d): weighted sum over the quantized slots
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < CH; ++k)
      if (k < nsplit) acc = fmaf(vals[k], wt[k * GH + h].x, acc);
    for (int s = CH; s < nsplit; ++s) acc = fmaf(__ldcg(acc_hd + (int64_t)s * G * D), wt[s * GH + h].x, acc);
    rot[h * D + d] = acc;
    win[h * D + d] = wv;
  }
  __syncthreads();
  if (warp < GH) {  // warp hh: H applied to the rotated sum, window part, normalisation
    const int hh = warp;
    float lr = 0.f;
    for (int s = lane; s < nsplit; s += 32) {
      const float2 wl = wt[s * GH + hh];
      lr = fmaf(wl.y, wl.x, lr);
    }
    lr = warp_sum(lr);
    const float mrot = win[GH * D + hh];
    float a[4], aw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[i] = rot[hh * D + 4 * lane + i];
      aw[i] = win[hh * D + 4 * lane + i];
    }
    fwht128_warp(a, lane);
    const float2 mlw = wt[nsplit * GH + hh];
    const float mw = mlw.y > 0.f ? mlw.x : NEG_BIG, lw = mlw.y;
    const float mt = fmaxf(mrot, mw);
    const float fa = lr > 0.f ? fast_exp2(mrot - mt) : 0.f;
    const float fr = lw > 0.f ? fast_exp2(mw - mt) : 0.f;
    const float den = lr * fa + lw * fr;
    const float inv = den > 0.f ? 1.f / den : 0.f;
    float4 o;
    o.x = (a[0] * INV_SQRT_D * fa + aw[0] * fr) * inv;
    o.y = (a[1] * INV_SQRT_D * fa + aw[1] * fr) * inv;
    o.z = (a[2] * INV_SQRT_D * fa + aw[2] * fr) * inv;
    o.w = (a[3] * INV_SQRT_D * fa + aw[3] * fr) * inv;
    *reinterpret_cast<float4*>(out_rows + (int64_t)hh * D + 4 * lane) = o;
  }
  __syncthreads();  // the scratch may be reused by the next merge of this CTA
}

// One warp = one split of one (sequence, head group); GH <= 4 query heads per
// warp (a group of 8 runs as two head groups).  A split is a contiguous range of
// 64-token stages (it may start or end inside a 128-token block); the last split
// of a sequence also attends the residual window.  The CTA of the warp that
// completes a (sequence, head group) last merges its partials into the output,
// so one launch does the whole decode.
//
// Scores:  S[t][c] = sum_k u_hat[t][k] Qc[k][c]   M = 16 tokens, N = 8 columns, K = 16
//          (columns 0-3: fp16(q~) of the GH heads, 4-7: their fp16 rounding residual),
//          accumulated in two independent chains (even and odd k-steps).
//          A lane swap (xor 2) adds the two halves so that lane (g, p) holds the
//          scores of token g + 8 (p >> 1) for heads 2 (p & 1), 2 (p & 1) + 1.
// Values:  O^T[d][h] += sum_t u_hat_v[t][d] w[t][h]  M = 16 dims, N = 8 heads, K = 16 tokens;
//          the B operand is the weight matrix moved into place with movmatrix.trans.
// RP (pre-RoPE keys): the K logits of every quantized and window token come
// precomputed from rope_scores_kernel (`rscores`, rs_cap tokens per (sequence,
// head group)); the kernel then reads neither the query nor the K cache.
template <int GH, int MK, int MV, bool DQ, bool RP = false>
__global__ void __launch_bounds__(32 * DEC_WARPS, 1)
decode_kernel(CacheView kc, CacheView vc, const void* __restrict__ q, int dtype, int64_t qsb, int64_t qsh,
              float qscale, const float* __restrict__ cbk_g, const float* __restrict__ cbv_g,
              unsigned int* __restrict__ counters, float* __restrict__ ws, float* __restrict__ out, int n_q_heads,
              DecodeGeom geom, const float* __restrict__ rscores, int rs_cap, int nw_cut, int64_t out_sb) {
  static_assert(GH == 1 || GH == 2 || GH == 4, "1, 2 or 4 heads per warp");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, p = lane & 3;
  const int G = geom.g;           // query heads per kv-head
  const int ngroups = G / GH;     // head groups per kv-head
  const int nsplit = geom.nsplit_q;
  const int nseq = kc.batch * kc.n_kv_heads;
  const int gw = blockIdx.x * DEC_WARPS + warp;  // global warp job id
  const bool active = gw < nseq * nsplit * ngroups;
  const int hg = gw % ngroups;
  const int64_t seq = active ? (gw / ngroups) / nsplit : 0;
  const int split = (gw / ngroups) % nsplit;
  const int b = (int)(seq / kc.n_kv_heads), hk = (int)(seq % kc.n_kv_heads);
  const int hbase = hg * GH;                      // first head of the group within the kv-head
  const int64_t p0 = seq * (nsplit + 1);          // first partial slot of the sequence
  const int64_t P = (int64_t)nseq * (nsplit + 1);
  float* ws_acc = ws + acc_offset(P, G);
  const int64_t q_off = (int64_t)b * qsb + (int64_t)(hk * G + hbase) * qsh;
  const float* rsrc = RP ? rscores + ((int64_t)(seq * ngroups + hg) * rs_cap) * GH : nullptr;
  constexpr int RGH = RP ? GH : 0;

  // The query rows are requested first, before the codebook staging and the bulk
  // copies, so that they do not queue behind the copies of every warp.
  // Prologue order: the query rows, the cache counters and this thread's codeword
  // are requested first; each warp then arms its own barriers and issues its
  // first bulk copy (no CTA barrier needed), builds its query operand while that
  // copy flies, issues its second copy, and only then does the CTA store the
  // codebooks and meet at the one barrier.
  float qrows[GH][4];
  if (!RP && active) load_q_rows<GH>(qrows, q, dtype, q_off, qsh, lane);
  static_assert(32 * DEC_WARPS == 2 * NCODES, "one codeword per thread");
  const int cb_c = tid & (NCODES - 1);
  const bool cb_isv = tid >= NCODES;
  const uint4 cb_row = cb_row_f16(cb_isv ? cbv_g : cbk_g, cb_c);

  const int nq = active ? min(min(kc.n_quant[seq], vc.n_quant[seq]), kc.capacity) : 0;
  // nw_cut > 0 (chunked-prefill queries): the last nw_cut window tokens lie after
  // this query and are not attended; status bit 8 if the query's own token is not
  // in the window.
  const int nw_all = (kc.window_len > 0) ? max(0, min(min(kc.n_window[seq], vc.n_window[seq]), kc.window_len)) : 0;
  const int nw = max(0, nw_all - nw_cut);
  if (nw_cut > 0 && active && split == 0 && hg == 0 && lane == 0 && nw_all <= nw_cut && kc.status)
    atomicOr(kc.status, 8);
  // Splits are dealt whole 64-token stages, so a split may start or end inside
  // a 128-token block (the block's mean terms are then split between them too).
  const int nst_all = (nq + STAGE_TOK - 1) / STAGE_TOK;
  const int sps = max(1, (nst_all + (nw > 0 ? WINDOW_COST_STAGES : 0) + nsplit - 1) / nsplit);  // stages per split
  const int tok_begin = min(nq, split * sps * STAGE_TOK);
  const int tok_end = min(nq, (split + 1) * sps * STAGE_TOK);
  const bool has_window = active && split == nsplit - 1;
  const uint32_t st_base = smem_addr(&sm.stage[warp][0][0]);
  const uint32_t mb_base = smem_addr(&sm.means[warp][0][0]);
  const uint32_t bar0 = smem_addr(&sm.bar[warp][0]);
  const int nstages = (tok_end - tok_begin + STAGE_TOK - 1) / STAGE_TOK;

  if (lane == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8u, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    if (nstages > 0)
      issue_stage<MK, MV, DQ, RGH>(st_base, mb_base + (uint32_t)(((tok_begin / BLK) & 1) * MEAN_BYTES), bar0, kc, vc,
                                   seq, tok_begin, true, rsrc);
  }
  __syncwarp();

  // ---- query operand (B of the score product), built while stage 0 flies, in
  // the second stage buffer, which is filled only afterwards ----
  uint32_t qb[8][2];
  if (!RP && active) build_q_operand<GH>(qb, qrows, qscale * INV_SQRT_D, true, lane, &sm.stage[warp][1][0]);
  if (lane == 0 && nstages > 1) {
    const int t1 = tok_begin + STAGE_TOK;
    issue_stage<MK, MV, DQ, RGH>(st_base + STAGE_BYTES, mb_base + (uint32_t)(((t1 / BLK) & 1) * MEAN_BYTES), bar0 + 8,
                                 kc, vc, seq, t1, (t1 % BLK) == 0, rsrc);
  }

  // ---- stage the replicated fp16 codebooks (whole CTA, once) ----
  // One codeword per thread, stored as 8 replicas in a rotated order so that the
  // 8 lanes of a quarter-warp hit 8 bank groups.
  {
    uint4* dst = cb_isv ? &sm.cbv[cb_c][0] : &sm.cbk[cb_c][0];
#pragma unroll
    for (int r = 0; r < 8; ++r) dst[(r + cb_c) & 7] = cb_row;
  }
  if (tid == 0) sm.merge_n = 0;
  __syncthreads();

  const uint32_t lane_row = (uint32_t)(lane & 7) * 16u;
  const uint32_t cbk_base = smem_addr(&sm.cbk[0][0]) + lane_row;
  const uint32_t cbv_base = smem_addr(&sm.cbv[0][0]) + lane_row;
  // The K and V ldmatrix rows use one lane map: lane l reads token (l & 7) + 8 (l >> 4),
  // sub-vector parity (l >> 3) & 1, so the 8-byte code loads of a half-warp cover
  // 128 contiguous bytes (no bank conflict).  For K this puts the matrices of rows
  // 8-15 and of k 8-15 in the other order: the gather swaps registers 1 and 2.
  const int tok_a = (lane & 7) + 8 * (lane >> 4);         // token of this lane's K ldmatrix row
  const int tok_v = (lane & 7) + 8 * (lane >> 4);         // token of this lane's V ldmatrix row
  const int kpar = (lane >> 3) & 1, vpar = kpar;       // sub-vector parity of the K / V ldmatrix row
  const bool lo_lane = p < 2;                      // keeps token g (else g + 8) after the swap
  const int t_l = g + (lo_lane ? 0 : 8);           // token of this lane's two scores
  const int h0 = 2 * (p & 1);                      // its two heads: h0, h0 + 1 (within the group)
  // Padding heads get a running max of +1e30: their weights are exactly 0 and they
  // never trigger a re-base.
  const float m_init0 = h0 < GH ? NEG_BIG : -NEG_BIG, m_init1 = h0 + 1 < GH ? NEG_BIG : -NEG_BIG;
  SoftmaxState sx;
  sx.m0 = m_init0; sx.m1 = m_init1; sx.l0 = sx.l1 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) sx.O[i][0] = sx.O[i][1] = sx.O[i][2] = sx.O[i][3] = 0.f;
  float cm0 = 0.f, cm1 = 0.f, qo0 = 0.f, qo1 = 0.f;
  uint32_t phase = 0u;
  bool failed = false;
  int pending = 0;  // buffers whose copy may still be in flight when a wait gives up (bit per buffer)

  for (int st = 0; st < nstages; ++st) {
    const int buf = st & 1;
    const bool arrived = mbar_wait(bar0 + 8u * buf, (phase >> buf) & 1u);
    if (!__all_sync(0xffffffffu, arrived)) {
      failed = true;
      pending = (1 << buf) | (st + 1 < nstages ? (1 << (buf ^ 1)) : 0);
      break;
    }
    phase ^= 1u << buf;
    const int t_stage = tok_begin + st * STAGE_TOK;
    const bool block_start = (t_stage % BLK) == 0 || st == 0;  // (q~ . o_b needed from the split's first stage)
    const bool block_end = ((t_stage + STAGE_TOK) % BLK) == 0 || st == nstages - 1;
    const int mbuf = (t_stage / BLK) & 1;
    const unsigned char* sb = &sm.stage[warp][buf][0];
    unsigned char* mb = &sm.means[warp][mbuf][0];
    float2 k_s1 = make_float2(0.f, 0.f), v_s1 = make_float2(0.f, 0.f);  // (lo, step) of the s1 levels
    if constexpr (DQ) {
      k_s1 = dq_lo_step(mb + DQ_PAR);
      v_s1 = dq_lo_step(mb + DQ_PAR + 16);
    }

    if (!RP && block_start) {
      if constexpr (DQ) {  // the fp16 o_K row, from its levels
        dq_mean_row(mb, mb + DQ_LEV, mb + DQ_PAR + 4, lane);
        __syncwarp();
      }
      // (H q) . o_K of this block: the mean row as all 16 "tokens" of one score tile
      // (rows 8-15 repeat rows 0-7, so an x2 load gives all four A registers)
      float d4[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t mrow = mb_base + (uint32_t)(mbuf * MEAN_BYTES) + (uint32_t)((lane >> 3) & 1) * 16u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t aa[4];
        ldsm_x2(mrow + 32u * j, aa[0], aa[2]);
        aa[1] = aa[0];
        aa[3] = aa[2];
        mma_full(d4, aa, qb[j][0], qb[j][1]);
      }
      const float r0 = __shfl_xor_sync(0xffffffffu, lo_lane ? d4[2] : d4[0], 2);
      const float r1 = __shfl_xor_sync(0xffffffffu, lo_lane ? d4[3] : d4[1], 2);
      qo0 = (lo_lane ? d4[0] : d4[2]) + r0;
      qo1 = (lo_lane ? d4[1] : d4[3]) + r1;
    }
    const int ntile = min(STAGE_TOK, tok_end - t_stage + 15) >> 4;
    const bool full = t_stage + STAGE_TOK <= tok_end;  // every token of the stage is valid
    for (int tile = 0; tile < ntile; ++tile) {
      const int tt = 16 * tile;  // token offset inside the stage
      uint2 kcw = make_uint2(0u, 0u);
      if constexpr (!RP) kcw = *reinterpret_cast<const uint2*>(sb + ST_KC + (tt + tok_a) * 16 + 8 * kpar);
      uint32_t ks0 = 0u, ks1 = 0u;
      if constexpr (!RP && MK == NSN_MODE_2BIT) {
        ks0 = *reinterpret_cast<const uint32_t*>(sb + ST_KS + (tt + g) * 16 + 4 * p);
        ks1 = *reinterpret_cast<const uint32_t*>(sb + ST_KS + (tt + 8 + g) * 16 + 4 * p);
      }
      uint32_t knw = 0u, vnw = 0u;
      if constexpr (!DQ && !RP) knw = *reinterpret_cast<const uint32_t*>(sb + ST_KN + (tt + t_l) * 4);
      const uint2 vcw = *reinterpret_cast<const uint2*>(sb + ST_VC + (tt + tok_v) * 16 + 8 * vpar);
      uint32_t W0 = 0u, W1 = 0u;
      if constexpr (MV == NSN_MODE_2BIT) {
        const uint16_t* vs = reinterpret_cast<const uint16_t*>(sb + ST_VS);
        W0 = __byte_perm((uint32_t)vs[(tt + 2 * p) * 8 + g], (uint32_t)vs[(tt + 2 * p + 1) * 8 + g], 0x5410u);
        W1 = __byte_perm((uint32_t)vs[(tt + 8 + 2 * p) * 8 + g], (uint32_t)vs[(tt + 9 + 2 * p) * 8 + g], 0x5410u);
      }
      if constexpr (!DQ) vnw = *reinterpret_cast<const uint32_t*>(sb + ST_VN + (tt + t_l) * 4);

      // ---- scores: 8 k-steps of 16 dims in two independent accumulation chains ----
      float S[4] = {0.f, 0.f, 0.f, 0.f}, S2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < (RP ? 0 : 8); ++j) {
        const uint32_t code = code_byte(kcw, j);
        uint32_t aa[4];
        ldsm_x4(cbk_base + code * 128u, aa);
        {  // matrices 1 and 2 hold tokens 0-7 of k 8-15 and tokens 8-15 of k 0-7
          const uint32_t t = aa[1];
          aa[1] = aa[2];
          aa[2] = t;
        }
        if constexpr (MK == NSN_MODE_2BIT) {
          aa[0] = apply_signs(aa[0], ks0, 2 * j);
          aa[1] = apply_signs(aa[1], ks1, 2 * j);
          aa[2] = apply_signs(aa[2], ks0, 2 * j + 1);
          aa[3] = apply_signs(aa[3], ks1, 2 * j + 1);
        }
        if (j & 1) mma_full(S2, aa, qb[j][0], qb[j][1]);
        else mma_full(S, aa, qb[j][0], qb[j][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) S[i] += S2[i];
      // hi + lo columns -> (token t_l, heads h0, h0 + 1)
      const float r0 = __shfl_xor_sync(0xffffffffu, lo_lane ? S[2] : S[0], 2);
      const float r1 = __shfl_xor_sync(0xffffffffu, lo_lane ? S[3] : S[1], 2);
      const float d0 = (lo_lane ? S[0] : S[2]) + r0;
      const float d1 = (lo_lane ? S[1] : S[3]) + r1;

      // ---- scores with the NSN byproducts; online softmax (lazy re-basing) ----
      float2 kn = make_float2(0.f, 0.f), vn;  // (s1, s2) of token t_l
      if constexpr (DQ) {
        const int tk = tt + t_l;
        const uint32_t sh = 4u * (uint32_t)(tk & 1);
        if constexpr (!RP) {
          const float kl = nibble_f((uint32_t)sb[ST_KN + STAGE_TOK * 2 + (tk >> 1)] >> sh);
          kn = make_float2(fmaf(kl, k_s1.y, k_s1.x), __half2float(reinterpret_cast<const __half*>(sb + ST_KN)[tk]));
        }
        const float vl = nibble_f((uint32_t)sb[ST_VN + STAGE_TOK * 2 + (tk >> 1)] >> sh);
        vn = make_float2(fmaf(vl, v_s1.y, v_s1.x), __half2float(reinterpret_cast<const __half*>(sb + ST_VN)[tk]));
      } else {
        kn = __half22float2(*reinterpret_cast<const __half2*>(&knw));
        vn = __half22float2(*reinterpret_cast<const __half2*>(&vnw));
      }
      float sc0, sc1;
      if constexpr (RP) {  // padding heads (h >= GH) carry a running max of +1e30: any finite value will do
        const float* lg = reinterpret_cast<const float*>(sb + ST_KC) + (tt + t_l) * GH;
        sc0 = h0 < GH ? lg[h0] : 0.f;
        sc1 = h0 + 1 < GH ? lg[h0 + 1] : 0.f;
      } else {
        sc0 = kn.x * fmaf(kn.y, d0, qo0);
        sc1 = kn.x * fmaf(kn.y, d1, qo1);
      }
      if (!full && t_stage + tt + t_l >= tok_end) {  // past the end: no weight, and no stale norms
        sc0 = sc1 = NEG_BIG;
        vn = make_float2(0.f, 0.f);
      }
      lazy_update(sx, sc0, sc1, cm0, cm1);
      const float pr0 = fast_exp2(sc0 - sx.m0), pr1 = fast_exp2(sc1 - sx.m1);
      sx.l0 += pr0;
      sx.l1 += pr1;
      cm0 = fmaf(pr0, vn.x, cm0);
      cm1 = fmaf(pr1, vn.x, cm1);
      const float s12 = vn.x * vn.y;
      const uint32_t wpk = pack_half2(pr0 * s12, pr1 * s12);
      const uint32_t wother = __shfl_xor_sync(0xffffffffu, wpk, 2);
      const uint32_t pb0 = movmatrix_t(lo_lane ? wpk : 0u);     // tokens 0-7
      const uint32_t pb1 = movmatrix_t(lo_lane ? wother : 0u);  // tokens 8-15

      // ---- values: O^T += u_hat_v^T w ----
#pragma unroll
      for (int mm = 0; mm < 8; ++mm) {
        const uint32_t code = code_byte(vcw, mm);
        uint32_t aa[4];
        ldsm_x4_t(cbv_base + code * 128u, aa);
        if constexpr (MV == NSN_MODE_2BIT) {
          aa[0] = apply_signs(aa[0], W0, 2 * mm);
          aa[1] = apply_signs(aa[1], W0, 2 * mm + 1);
          aa[2] = apply_signs(aa[2], W1, 2 * mm);
          aa[3] = apply_signs(aa[3], W1, 2 * mm + 1);
        }
        mma_full(sx.O[mm], aa, pb0, pb1);
      }
    }

    if (block_end) {
      // ---- block mean of V: O^T[d][h] += o_V[d] * sum_{t in block} p_t s1_t ----
      float c0 = cm0, c1 = cm1;
#pragma unroll
      for (int x = 2; x < 32; x <<= 1) {
        c0 += __shfl_xor_sync(0xffffffffu, c0, x);
        c1 += __shfl_xor_sync(0xffffffffu, c1, x);
      }
      if constexpr (DQ) {  // the fp16 o_V row, from its levels (the o_K row is no longer needed)
        dq_mean_row(mb, mb + DQ_LEV + D / 2, mb + DQ_PAR + 16 + 4, lane);
        __syncwarp();
      }
      const __half* ov = reinterpret_cast<const __half*>(mb + (DQ ? 0 : D * 2));
#pragma unroll
      for (int mm = 0; mm < 8; ++mm) {
        const float oa = __half2float(ov[16 * mm + g]);
        const float ob = __half2float(ov[16 * mm + 8 + g]);
        sx.O[mm][0] = fmaf(oa, c0, sx.O[mm][0]);
        sx.O[mm][1] = fmaf(oa, c1, sx.O[mm][1]);
        sx.O[mm][2] = fmaf(ob, c0, sx.O[mm][2]);
        sx.O[mm][3] = fmaf(ob, c1, sx.O[mm][3]);
      }
      cm0 = cm1 = 0.f;
    }
    __syncwarp();  // every lane is done with this stage buffer (and, at a block end, its means)
    if (lane == 0 && st + 2 < nstages) {
      const int tn = t_stage + 2 * STAGE_TOK;
      issue_stage<MK, MV, DQ, RGH>(st_base + (uint32_t)(buf * STAGE_BYTES),
                                   mb_base + (uint32_t)(((tn / BLK) & 1) * MEAN_BYTES), bar0 + 8u * buf, kc, vc, seq, tn,
                                   (tn % BLK) == 0, rsrc);
    }
  }
  if (active) store_partial<GH>(sx, ws, ws_acc, p0 + split, G, hbase, lane);

  // ---- residual window (original domain), last split only ----
  if (has_window) {
    sx.m0 = m_init0; sx.m1 = m_init1; sx.l0 = sx.l1 = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) sx.O[i][0] = sx.O[i][1] = sx.O[i][2] = sx.O[i][3] = 0.f;
    const int nch = failed ? 0 : (nw + WCHUNK - 1) / WCHUNK;
    if (nch > 0) {
      const __half* kw0 = kc.window + seq * kc.window_len * D;
      const __half* vw0 = vc.window + seq * vc.window_len * D;
      issue_window_chunk(st_base, bar0, kw0, vw0, min(WCHUNK, nw), lane);
      if constexpr (!RP) {
        float wrows[GH][4];  // reloaded: keeping the first rows alive would cost registers in the main loop
        load_q_rows<GH>(wrows, q, dtype, q_off, qsh, lane);
        build_q_operand<GH>(qb, wrows, qscale, false, lane, &sm.stage[warp][1][0]);
      }
      if (nch > 1) issue_window_chunk(st_base + STAGE_BYTES, bar0 + 8u, kw0 + WCHUNK * D, vw0 + WCHUNK * D,
                                      min(WCHUNK, nw - WCHUNK), lane);
      const int wr = lane & 7;  // ldmatrix row (token) of this lane; rows 8-15 repeat rows 0-7
      for (int c = 0; c < nch; ++c) {
        const int buf = c & 1;
        const bool arrived = mbar_wait(bar0 + 8u * buf, (phase >> buf) & 1u);
        if (!__all_sync(0xffffffffu, arrived)) {
          failed = true;
          pending = (1 << buf) | (c + 1 < nch ? (1 << (buf ^ 1)) : 0);
          break;
        }
        phase ^= 1u << buf;
        const int rows = min(WCHUNK, nw - c * WCHUNK);
        const uint32_t kbuf = st_base + (uint32_t)(buf * STAGE_BYTES);
        const uint32_t vbuf = kbuf + (uint32_t)WC_V;
        const uint32_t rowoff = (uint32_t)(min(wr, rows - 1) * WROWB);
        float sc0, sc1;
        if constexpr (RP) {  // logits of window slot w at position n_quant + w
          const float* lg = rsrc + (int64_t)(nq + c * WCHUNK + min(t_l, rows - 1)) * GH;
          sc0 = h0 < GH ? lg[h0] : 0.f;
          sc1 = h0 + 1 < GH ? lg[h0 + 1] : 0.f;
        } else {
          float S[4] = {0.f, 0.f, 0.f, 0.f}, S2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t aa[4];  // rows 8-15 repeat rows 0-7
            ldsm_x2(kbuf + rowoff + (uint32_t)(32 * j + 16 * ((lane >> 3) & 1)), aa[0], aa[2]);
            aa[1] = aa[0];
            aa[3] = aa[2];
            if (j & 1) mma_full(S2, aa, qb[j][0], qb[j][1]);
            else mma_full(S, aa, qb[j][0], qb[j][1]);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) S[i] += S2[i];
          const float r0 = __shfl_xor_sync(0xffffffffu, lo_lane ? S[2] : S[0], 2);
          const float r1 = __shfl_xor_sync(0xffffffffu, lo_lane ? S[3] : S[1], 2);
          sc0 = (lo_lane ? S[0] : S[2]) + r0;
          sc1 = (lo_lane ? S[1] : S[3]) + r1;
        }
        if (t_l >= rows) sc0 = sc1 = NEG_BIG;  // tokens 8-15 of the tile and rows past the window
        float unused0 = 0.f, unused1 = 0.f;
        lazy_update(sx, sc0, sc1, unused0, unused1);
        const float pr0 = fast_exp2(sc0 - sx.m0), pr1 = fast_exp2(sc1 - sx.m1);
        sx.l0 += pr0;
        sx.l1 += pr1;
        const uint32_t wpk = pack_half2(pr0, pr1);
        const uint32_t pb0 = movmatrix_t(lo_lane ? wpk : 0u);  // tokens 0-7; tokens 8-15 weigh 0
#pragma unroll
        for (int mm = 0; mm < 8; ++mm) {
          uint32_t aa[4];  // tokens 8-15 repeat tokens 0-7 (and weigh 0)
          ldsm_x2_t(vbuf + rowoff + (uint32_t)(32 * mm + 16 * ((lane >> 3) & 1)), aa[0], aa[1]);
          aa[2] = aa[0];
          aa[3] = aa[1];
          mma_full(sx.O[mm], aa, pb0, 0u);
        }
        __syncwarp();
        if (c + 2 < nch) {
          const int t2 = (c + 2) * WCHUNK;
          issue_window_chunk(kbuf, bar0 + 8u * buf, kw0 + t2 * D, vw0 + t2 * D, min(WCHUNK, nw - t2), lane);
        }
      }
    }
    store_partial<GH>(sx, ws, ws_acc, p0 + nsplit, G, hbase, lane);
  }

  if (failed) {
    if (lane == 0 && kc.status) atomicOr(kc.status, 2);
    // let copies that may still be in flight land before the CTA can exit
    if (pending & 1) mbar_wait(bar0, phase & 1u);
    if (pending & 2) mbar_wait(bar0 + 8u, (phase >> 1) & 1u);
  }

  // ---- the last warp of this (sequence, head group) hands it to its CTA ----
  __threadfence();  // this warp's partial stores are visible device-wide ...
  __syncwarp();     // ... for every lane before lane 0 takes the ticket
  if (active && lane == 0) {
    const unsigned int ticket = atomicInc(&counters[seq * ngroups + hg], (unsigned int)(nsplit - 1));
    if (ticket == (unsigned int)(nsplit - 1)) {
      __threadfence();
      const int k = atomicAdd(&sm.merge_n, 1);
      sm.merge_seq[k] = (int)seq;
      sm.merge_hg[k] = hg;
    }
  }

  // ---- the whole CTA merges the groups whose last ticket it took ----
  __syncthreads();  // every warp is done with its stage buffers, the merge list is complete
  const int n_merge = sm.merge_n;
  if (n_merge == 0) return;
  __threadfence();
  float* scratch = reinterpret_cast<float*>(&sm.stage[0][0][0]);
  for (int m = 0; m < n_merge; ++m) {
    const int mseq = sm.merge_seq[m], mhg = sm.merge_hg[m];
    const int mb = mseq / kc.n_kv_heads, mhk = mseq % kc.n_kv_heads;
    cta_merge<GH>(ws, ws + acc_offset(P, G), (int64_t)mseq * (nsplit + 1), nsplit, G, mhg * GH,
                  out + (int64_t)mb * out_sb + (int64_t)(mhk * G + mhg * GH) * D, scratch);
  }
}

// ---------------------------------------------------------------------------
// Pre-RoPE keys: the K logits ([TS] Metodologia 4 -- NSN is applied to the keys
// before the rotary position embedding, so the cache holds pre-RoPE keys and each
// is rotated at its own position when it is attended).  For key t of a (batch,
// kv-head) at position pos (its index in the sequence: quantized tokens first,
// then the window) and query head h of one head group:
//   quantized:  logit = qscale * s1_t * q_h . R_pos(s2_t H u_hat_t + H o_b)
//   window:     logit = qscale * q_h . R_pos(k_t)        (k_t the stored fp16 row)
// with H the orthonormal Hadamard matrix and R_pos the rotate-half rotation of
// dims (i, i + 64) by pos * theta_i.  The logits (log2 units) go to a workspace
// array that decode_kernel<..., RP = true> reads in place of its K path.
//
// Per 16-token tile a warp forms H u_hat on the tensor cores.  With dim
// k = 16a + b, H_128 = H_8 (x) H_16, so output k-step a' accumulates k-step a of
// u_hat times H_8[a'][a] H_16: the B operand is always +H_16 or -H_16 (4 constant
// registers each) and the sum is exact up to fp32 accumulation.  On the
// accumulator fragments the lane holds dims i and i + 64 of the same tokens in the
// same register slot, so the NSN affine terms and the rotation run in fp32 in
// registers; the rotated key is split into fp16 hi + lo and multiplied by the
// fp16 hi + lo query (the accumulator layout is the A layout, no shuffle).
// Rotations compose, q . R_(pos0 + r) k = (R_(-pos0) q) . (R_r k): the query is
// rotated back by the 64-token stage start pos0 once per stage (angles reduced in
// fp64), and each key by its offset r < 64 from a CTA table of (cos, sin)(r theta_i).
// ---------------------------------------------------------------------------
constexpr int RS_WARPS = 8;
constexpr int RS_WK_HOB = 8 * QS_ROW;             // per-warp area: query staging (8 fp16 rows) ...
constexpr int RS_WK_BASE = RS_WK_HOB + D * 4;     // ... H o_b (128 fp32) ...
constexpr int RS_WK_BYTES = RS_WK_BASE + (D / 2) * 8;  // ... (cos, sin)(pos0 theta_i), 64 pairs
constexpr int RS_OFF_ROW = STAGE_TOK + 8;  // float2 per table row: 64 + padding, so 8 lanes of a
                                           // 16-byte fetch on two rows hit different banks
struct RsSmem {
  alignas(128) uint4 cbk[NCODES][8];                    // replicated fp16 K codebook (as in decode_kernel)
  alignas(16) float2 off[STAGE_TOK][RS_OFF_ROW];        // (cos, sin)(r theta_i), r < 64, i < 64
  alignas(128) unsigned char wk[RS_WARPS][RS_WK_BYTES];  // per warp: query staging | H o_b | stage angles
};

// (cos a, sin a) with a reduced to [-pi, pi] in fp64 first.
__device__ __forceinline__ float2 rope_cs(double a) {
  const double two_pi = 6.283185307179586;
  const double r = a - two_pi * rint(a * (1.0 / two_pi));
  float sn, cs;
  sincosf((float)r, &sn, &cs);
  return make_float2(cs, sn);
}

__device__ __forceinline__ void mma_zero(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %10, %10, %10};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// Compressed inputs of one 16-token K tile, loaded one tile ahead.
struct RsTileIn {
  uint4 codes;      // code record of this lane's ldmatrix token (the lane uses half lane >> 4)
  uint32_t ks0, ks1;  // sign words (2-bit) of tokens g, g + 8
  uint32_t n[2];    // tokens g, g + 8: (s1, s2) fp16 pair, or (alpha*s2 fp16 | s1 level << 16) with DQ
};

template <int MK, bool DQ>
__device__ __forceinline__ void rs_load_tile(RsTileIn& in, const CacheView& kc, int64_t tq, int tok_a, int g, int p) {
  in.codes = __ldg(reinterpret_cast<const uint4*>(kc.codes + (tq + tok_a) * NSUB));
  in.ks0 = in.ks1 = 0u;
  if constexpr (MK == NSN_MODE_2BIT) {
    in.ks0 = __ldg(reinterpret_cast<const uint32_t*>(kc.signs + (tq + g) * NSUB) + p);
    in.ks1 = __ldg(reinterpret_cast<const uint32_t*>(kc.signs + (tq + 8 + g) * NSUB) + p);
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int64_t tk = tq + g + 8 * rr;
    if constexpr (DQ) {
      const uint32_t s2b = __ldg(reinterpret_cast<const unsigned short*>(kc.norms) + tk);
      const uint32_t lv = ((uint32_t)__ldg(kc.s1_levels + tk / 2) >> (4 * (uint32_t)(tk & 1))) & 15u;
      in.n[rr] = s2b | (lv << 16);
    } else {
      in.n[rr] = __ldg(reinterpret_cast<const uint32_t*>(kc.norms) + tk);
    }
  }
}

template <int GH, int MK, bool DQ>
__global__ void __launch_bounds__(32 * RS_WARPS, 2)
rope_scores_kernel(CacheView kc, const int32_t* __restrict__ v_nquant, const int32_t* __restrict__ v_nwindow,
                   const void* __restrict__ q, int dtype, int64_t qsb, int64_t qsh, float qscale,
                   const float* __restrict__ inv_freq, const float* __restrict__ cbk_g, float* __restrict__ rscores,
                   int rs_cap, int G, int nchunk) {
  static_assert(GH == 1 || GH == 2 || GH == 4, "1, 2 or 4 heads per warp");
  static_assert(32 * RS_WARPS == NCODES, "one codeword per thread");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  RsSmem& sm = *reinterpret_cast<RsSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, p = lane & 3;
  {
    const uint4 row = cb_row_f16(cbk_g, tid);
#pragma unroll
    for (int r = 0; r < 8; ++r) sm.cbk[tid][(r + tid) & 7] = row;
    for (int e = tid; e < STAGE_TOK * (D / 2); e += 32 * RS_WARPS) {
      const int r = e / (D / 2), i = e % (D / 2);
      sm.off[r][i] = rope_cs((double)r * (double)__ldg(inv_freq + i));
    }
  }
  __syncthreads();  // the only CTA barrier

  const int ngroups = G / GH;
  const int nseq = kc.batch * kc.n_kv_heads;
  const int gw = blockIdx.x * RS_WARPS + warp;
  if (gw >= nseq * ngroups * nchunk) return;
  const int chunk = gw % nchunk;
  const int hg = (gw / nchunk) % ngroups;
  const int64_t seq = (gw / nchunk) / ngroups;
  const int b = (int)(seq / kc.n_kv_heads), hk = (int)(seq % kc.n_kv_heads);
  // the same token counts as decode_kernel
  const int nq = min(min(kc.n_quant[seq], v_nquant[seq]), kc.capacity);
  const int nw = (kc.window_len > 0) ? max(0, min(min(kc.n_window[seq], v_nwindow[seq]), kc.window_len)) : 0;
  const int nst_q = (nq + STAGE_TOK - 1) / STAGE_TOK;
  const int nst = nst_q + (nw + STAGE_TOK - 1) / STAGE_TOK;
  const int spc = (nst + nchunk - 1) / nchunk;
  const int st_first = chunk * spc, st_last = min(nst, st_first + spc);
  if (st_first >= st_last) return;
  float* rdst = rscores + ((int64_t)(seq * ngroups + hg) * rs_cap) * GH;

  // query operand (original domain, fp16 hi rows 0-3, residual rows 4-7), rebuilt
  // per stage rotated back by the stage start
  unsigned char* wk = &sm.wk[warp][0];
  const int64_t q_off = (int64_t)b * qsb + (int64_t)(hk * G + hg * GH) * qsh;
  uint32_t qb[8][2];
  float* hob = reinterpret_cast<float*>(wk + RS_WK_HOB);      // H o_b of the current block (128 fp32)
  float2* base = reinterpret_cast<float2*>(wk + RS_WK_BASE);  // (cos, sin)(pos0 theta_i), 64

  // H_16 as the B operand: column n = g + 8 nt, rows 2p, 2p+1 | 2p+8, 2p+9
  uint32_t Hb[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int n = g + 8 * nt;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int k0 = 2 * p + 8 * r;
      const uint32_t e0 = (__popc(k0 & n) & 1) ? 0xBC00u : 0x3C00u;
      const uint32_t e1 = (__popc((k0 + 1) & n) & 1) ? 0xBC00u : 0x3C00u;
      Hb[nt][r] = e0 | (e1 << 16);
    }
  }
  const uint32_t cbk_base = smem_addr(&sm.cbk[0][0]) + (uint32_t)(lane & 7) * 16u;
  const int tok_a = (lane & 7) + 8 * ((lane >> 3) & 1);
  const int kpar = lane >> 4;
  const bool lo_lane = p < 2;
  const int t_l = g + (lo_lane ? 0 : 8);
  const int h0 = 2 * (p & 1);
  const int64_t cap = kc.capacity;
  const int q_end = min(nq, st_last * STAGE_TOK);  // this job's quantized positions end here
  int cur_blk = -1;
  RsTileIn nxt;
  if (st_first < nst_q) rs_load_tile<MK, DQ>(nxt, kc, seq * cap + st_first * STAGE_TOK, tok_a, g, p);

  for (int st = st_first; st < st_last; ++st) {
    const bool win = st >= nst_q;
    const int pos0 = win ? nq + (st - nst_q) * STAGE_TOK : st * STAGE_TOK;
    const int pend = win ? nq + nw : nq;  // positions below this are keys
    __syncwarp();  // the previous stage is done with `base` and `hob`
    {
      const float2 th = __ldg(reinterpret_cast<const float2*>(inv_freq) + lane);
      base[2 * lane] = rope_cs((double)pos0 * (double)th.x);
      base[2 * lane + 1] = rope_cs((double)pos0 * (double)th.y);
    }
    float2 s1ls = make_float2(0.f, 0.f);  // (lo, step) of the block's s1 levels
    if (!win) {
      const int64_t blk = seq * (cap / BLK) + pos0 / BLK;
      if constexpr (DQ) s1ls = dq_lo_step(reinterpret_cast<const unsigned char*>(kc.dq_params + blk * 8));
      if (pos0 / BLK != cur_blk) {
        cur_blk = pos0 / BLK;
        float v[4];
        if constexpr (DQ) {
          const float2 ls = dq_lo_step(reinterpret_cast<const unsigned char*>(kc.dq_params + blk * 8 + 2));
          const uint32_t two = reinterpret_cast<const uint16_t*>(kc.means)[blk * (D / 4) + lane];
#pragma unroll
          for (int i = 0; i < 4; ++i)  // o is stored as the fp16 rounding of its level's value
            v[i] = __half2float(__float2half_rn(fmaf(nibble_f(two >> (4 * i)), ls.y, ls.x)));
        } else {
          const uint2 r = __ldg(reinterpret_cast<const uint2*>(kc.means + blk * D) + lane);
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&r.x));
          const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&r.y));
          v[0] = a.x; v[1] = a.y; v[2] = c.x; v[3] = c.y;
        }
        fwht128_warp(v, lane);
        *reinterpret_cast<float4*>(hob + 4 * lane) =
            make_float4(v[0] * INV_SQRT_D, v[1] * INV_SQRT_D, v[2] * INV_SQRT_D, v[3] * INV_SQRT_D);
      }
    } else if (cur_blk != -2) {  // window keys: no mean term
      cur_blk = -2;
      *reinterpret_cast<float4*>(hob + 4 * lane) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncwarp();
    // the query rotated back by the stage start: q . R_(pos0 + r) k = (R_(-pos0) q) . (R_r k)
    {
      float qrows[GH][4];
      load_q_rows<GH>(qrows, q, dtype, q_off, qsh, lane);
      const int i0 = (4 * lane) & (D / 2 - 1);  // dims 4l .. 4l+3; their pair partners sit in lane l ^ 16
      const float4 cs01 = *reinterpret_cast<const float4*>(base + i0);
      const float4 cs23 = *reinterpret_cast<const float4*>(base + i0 + 2);
      const float cc[4] = {cs01.x, cs01.z, cs23.x, cs23.z}, ss[4] = {cs01.y, cs01.w, cs23.y, cs23.w};
      const bool upper = lane >= 16;  // dims i + 64
#pragma unroll
      for (int hh = 0; hh < GH; ++hh)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float mine = qrows[hh][e], other = __shfl_xor_sync(0xffffffffu, mine, 16);
          qrows[hh][e] = fmaf(mine, cc[e], (upper ? -other : other) * ss[e]);
        }
      build_q_operand<GH>(qb, qrows, qscale, false, lane, wk);
    }

    for (int m = 0; m < STAGE_TOK / 16; ++m) {
      const int tt = pos0 + 16 * m;  // position of the tile's first token
      if (tt >= pend) break;
      // E[a'][nt][r]: dim 16 a' + 8 nt + 2p + (r & 1) of token row g + 8 (r >> 1), before the NSN terms
      float E[8][2][4];
      float xs[2] = {1.f, 1.f}, s1r[2] = {1.f, 1.f};  // per row: scale of E, and s1
      if (!win) {
        const RsTileIn cur = nxt;
        if (tt + 16 < q_end) rs_load_tile<MK, DQ>(nxt, kc, seq * cap + tt + 16, tok_a, g, p);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          if constexpr (DQ) {
            xs[rr] = __half2float(__ushort_as_half((unsigned short)(cur.n[rr] & 0xFFFFu))) * INV_SQRT_D;
            s1r[rr] = fmaf(nibble_f(cur.n[rr] >> 16), s1ls.y, s1ls.x);
          } else {
            const float2 n2 = __half22float2(*reinterpret_cast<const __half2*>(&cur.n[rr]));
            s1r[rr] = n2.x;
            xs[rr] = n2.y * INV_SQRT_D;
          }
        }
        // u_hat k-steps a and a + 4 times +-H_16: their sum and difference are the
        // H_8 stage across bit 2 of the k-step, accumulated on the tensor cores;
        // the stages across bits 0 and 1 follow in fp32
        auto gather = [&](int a, uint32_t (&A)[4]) {
          // (the whole 16-byte record is loaded: an 8-byte load here costs this kernel spills)
          const uint32_t code = code_byte(kpar ? make_uint2(cur.codes.z, cur.codes.w) : make_uint2(cur.codes.x, cur.codes.y), a);
          ldsm_x4(cbk_base + code * 128u, A);
          if constexpr (MK == NSN_MODE_2BIT) {
            A[0] = apply_signs(A[0], cur.ks0, 2 * a);
            A[1] = apply_signs(A[1], cur.ks1, 2 * a);
            A[2] = apply_signs(A[2], cur.ks0, 2 * a + 1);
            A[3] = apply_signs(A[3], cur.ks1, 2 * a + 1);
          }
        };
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          uint32_t A0[4], A1[4];
          gather(a, A0);
          gather(a + 4, A1);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            mma_zero(E[a][nt], A0, Hb[nt][0], Hb[nt][1]);
            mma_full(E[a][nt], A1, Hb[nt][0], Hb[nt][1]);
            mma_zero(E[a + 4][nt], A0, Hb[nt][0], Hb[nt][1]);
            mma_full(E[a + 4][nt], A1, Hb[nt][0] ^ 0x80008000u, Hb[nt][1] ^ 0x80008000u);
          }
        }
#pragma unroll
        for (int sstep = 1; sstep < 4; sstep <<= 1)
#pragma unroll
          for (int a = 0; a < 8; ++a)
            if (!(a & sstep))
#pragma unroll
              for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                  const float u = E[a][nt][r], w = E[a + sstep][nt][r];
                  E[a][nt][r] = u + w;
                  E[a + sstep][nt][r] = u - w;
                }
      } else {
        const __half* wrow = kc.window + seq * (int64_t)kc.window_len * D;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int w = min(tt - nq + g + 8 * rr, nw - 1);
#pragma unroll
          for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              const float2 kv = __half22float2(
                  *reinterpret_cast<const __half2*>(wrow + (int64_t)w * D + 16 * a + 8 * nt + 2 * p));
              E[a][nt][2 * rr] = kv.x;
              E[a][nt][2 * rr + 1] = kv.y;
            }
        }
      }
      // NSN terms, rotation of dims (i, i + 64), fp16 hi + lo, and the query product
      // (one k16 MMA per 16 dims for the hi part and one for the lo part)
      const int r_off = 16 * m + g;  // offset-table rows of this lane's tokens: r_off, r_off + 8
      float S[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ap = 0; ap < 4; ++ap) {
        uint32_t ahi[2][4], alo[2][4];  // [h][A fragment register]: rows g, g + 8 of k-halves nt = 0, 1
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int i0 = 16 * ap + 8 * nt + 2 * p;
          const float2 olo = *reinterpret_cast<const float2*>(hob + i0);
          const float2 ohi = *reinterpret_cast<const float2*>(hob + i0 + 64);
          float y0[4], y1[4];
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const float4 oo = *reinterpret_cast<const float4*>(&sm.off[r_off + 8 * rr][i0]);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int r = 2 * rr + e;
              const float lo = fmaf(xs[rr], E[ap][nt][r], e ? olo.y : olo.x);
              const float hi = fmaf(xs[rr], E[ap + 4][nt][r], e ? ohi.y : ohi.x);
              const float c = e ? oo.z : oo.x, sn = e ? oo.w : oo.y;  // (cos, sin)(r theta_i)
              y0[r] = fmaf(lo, c, -hi * sn);
              y1[r] = fmaf(hi, c, lo * sn);
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float* y = h ? y1 : y0;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) split_half2(y[2 * rr], y[2 * rr + 1], ahi[h][2 * nt + rr], alo[h][2 * nt + rr]);
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          mma_full(S[h], ahi[h], qb[ap + 4 * h][0], qb[ap + 4 * h][1]);
          mma_full(S[h], alo[h], qb[ap + 4 * h][0], qb[ap + 4 * h][1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) S[0][i] += S[1][i];
      // hi + lo query columns -> (token t_l, heads h0, h0 + 1)
      const float r0 = __shfl_xor_sync(0xffffffffu, lo_lane ? S[0][2] : S[0][0], 2);
      const float r1 = __shfl_xor_sync(0xffffffffu, lo_lane ? S[0][3] : S[0][1], 2);
      const float s1 = lo_lane ? s1r[0] : s1r[1];
      const float sc0 = s1 * ((lo_lane ? S[0][0] : S[0][2]) + r0);
      const float sc1 = s1 * ((lo_lane ? S[0][1] : S[0][3]) + r1);
      const int pos = tt + t_l;
      if (pos < pend) {
        float* dst = rdst + (int64_t)pos * GH;
        if constexpr (GH == 1) {
          if (h0 == 0) dst[0] = sc0;
        } else {
          if (h0 + 1 < GH) *reinterpret_cast<float2*>(dst + h0) = make_float2(sc0, sc1);
        }
      }
    }
  }
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
  const int groups = g.g > 4 ? g.g / 4 : 1;
  const int warps = sm_count() * DEC_WARPS;
  int sp = warps / (nseq * groups > 0 ? nseq * groups : 1);
  const int maxsp = capacity / BLK;
  if (sp > maxsp) sp = maxsp;
  if (sp < 1) sp = 1;
  g.nsplit_q = sp;
  return g;
}

// Merge counters: two 32-bit words per (batch, kv-head) (one per head group),
// padded to 256 bytes.
static int64_t counter_words(int64_t nseq) { return ((2 * nseq + 63) / 64) * 64; }

size_t decode_partial_bytes(int batch, int n_kv_heads, const DecodeGeom& geom) {
  const int64_t P = (int64_t)batch * n_kv_heads * (geom.nsplit_q + 1);
  return (size_t)(acc_offset(P, geom.g) + P * geom.g * D) * sizeof(float);
}

size_t decode_workspace_bytes(int batch, int n_kv_heads, const DecodeGeom& geom) {
  return (size_t)counter_words((int64_t)batch * n_kv_heads) * 4u + decode_partial_bytes(batch, n_kv_heads, geom);
}

template <int G, int MK, int MV, bool DQ>
static cudaError_t launch_t(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                            int64_t qsb, int64_t qsh, float qscale, const float* cbk, const float* cbv, float* out,
                            unsigned int* counters, float* partials, const DecodeGeom& geom, cudaStream_t s,
                            int nw_cut, int64_t out_sb) {
  constexpr int GH = G < 4 ? G : 4;  // heads per warp job
  const size_t smem = sizeof(DecSmem);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<GH, MK, MV, DQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int nwarps = kc.batch * kc.n_kv_heads * geom.nsplit_q * (G / GH);
  dim3 grid((nwarps + DEC_WARPS - 1) / DEC_WARPS);
  decode_kernel<GH, MK, MV, DQ><<<grid, 32 * DEC_WARPS, smem, s>>>(kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv,
                                                               counters, partials, out, n_q_heads, geom, nullptr, 0,
                                                               nw_cut, out_sb);
  return cudaGetLastError();
}

template <int G>
static cudaError_t launch_g(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                            int64_t qsb, int64_t qsh, float qscale, const float* cbk, const float* cbv, float* out,
                            unsigned int* counters, float* partials, const DecodeGeom& geom, cudaStream_t s,
                            int nw_cut, int64_t out_sb) {
#define NSN_LAUNCH(MK_, MV_)                                                                                    \
  return kc.dq ? launch_t<G, MK_, MV_, true>(kc, vc, q, dtype, n_q_heads, qsb, qsh, qscale, cbk, cbv, out, counters,  \
                                             partials, geom, s, nw_cut, out_sb)                                       \
               : launch_t<G, MK_, MV_, false>(kc, vc, q, dtype, n_q_heads, qsb, qsh, qscale, cbk, cbv, out, counters, \
                                              partials, geom, s, nw_cut, out_sb)
  if (kc.mode == NSN_MODE_1BIT && vc.mode == NSN_MODE_1BIT) NSN_LAUNCH(1, 1);
  if (kc.mode == NSN_MODE_1BIT && vc.mode == NSN_MODE_2BIT) NSN_LAUNCH(1, 2);
  if (kc.mode == NSN_MODE_2BIT && vc.mode == NSN_MODE_1BIT) NSN_LAUNCH(2, 1);
  NSN_LAUNCH(2, 2);
#undef NSN_LAUNCH
}

static cudaError_t launch_any(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                              int64_t qsb, int64_t qsh, float softmax_scale, const float* cbk, const float* cbv,
                              float* out, unsigned int* counters, float* partials, const DecodeGeom& geom,
                              cudaStream_t s, int nw_cut = 0, int64_t out_sb = -1) {
  const float qscale = softmax_scale * LOG2E;
  if (out_sb < 0) out_sb = (int64_t)n_q_heads * D;
#define NSN_G(G_) \
  return launch_g<G_>(kc, vc, q, dtype, n_q_heads, qsb, qsh, qscale, cbk, cbv, out, counters, partials, geom, s, \
                      nw_cut, out_sb)
  switch (geom.g) {
    case 1: NSN_G(1);
    case 2: NSN_G(2);
    case 4: NSN_G(4);
    default: NSN_G(8);
  }
#undef NSN_G
}

cudaError_t launch_decode(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                          int64_t qsb, int64_t qsh, float softmax_scale, const float* cbk, const float* cbv,
                          float* out, void* ws, const DecodeGeom& geom, cudaStream_t s) {
  unsigned int* counters = static_cast<unsigned int*>(ws);
  float* partials = static_cast<float*>(ws) + counter_words((int64_t)kc.batch * kc.n_kv_heads);
  return launch_any(kc, vc, q, dtype, n_q_heads, qsb, qsh, softmax_scale, cbk, cbv, out, counters, partials, geom, s);
}

// Chunked-prefill ("extend") attention: the last n_queries tokens of every
// sequence sit in the residual window; query i attends the quantized part and the
// window up to its own slot.  One decode pass per query, each with the window
// shortened by the n_queries - 1 - i tokens that follow it, all sharing the
// workspace (stream-ordered; the merge counters return to zero after each pass).
cudaError_t launch_extend(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                          int n_queries, int64_t qsb, int64_t qst, int64_t qsh, float softmax_scale, const float* cbk,
                          const float* cbv, float* out, void* ws, const DecodeGeom& geom, cudaStream_t s) {
  unsigned int* counters = static_cast<unsigned int*>(ws);
  float* partials = static_cast<float*>(ws) + counter_words((int64_t)kc.batch * kc.n_kv_heads);
  const int64_t esz = dtype == NSN_DTYPE_F32 ? 4 : 2;
  const int64_t out_sb = (int64_t)n_queries * n_q_heads * D;
  for (int i = 0; i < n_queries; ++i) {
    const cudaError_t e = launch_any(kc, vc, static_cast<const char*>(q) + (int64_t)i * qst * esz, dtype, n_q_heads,
                                     qsb, qsh, softmax_scale, cbk, cbv, out + (int64_t)i * n_q_heads * D, counters,
                                     partials, geom, s, n_queries - 1 - i, out_sb);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ---- pre-RoPE keys: logits kernel, then decode_kernel<..., RP = true> ----
// Workspace: the decode workspace, then (256-byte aligned) the logits, rs_cap
// tokens per (sequence, head group) of GH fp32 each.
static int rope_rs_cap(int capacity, int window_len) {
  return ((capacity + window_len + STAGE_TOK - 1) / STAGE_TOK) * STAGE_TOK;
}
static size_t rope_scores_offset(int batch, int n_kv_heads, const DecodeGeom& geom) {
  return (decode_workspace_bytes(batch, n_kv_heads, geom) + 255u) / 256u * 256u;
}
size_t decode_rope_workspace_bytes(int batch, int n_kv_heads, int capacity, int window_len, const DecodeGeom& geom) {
  return rope_scores_offset(batch, n_kv_heads, geom) +
         (size_t)batch * n_kv_heads * geom.g * (size_t)rope_rs_cap(capacity, window_len) * sizeof(float);
}

template <int G, int MK, int MV, bool DQ>
static cudaError_t launch_rope_t(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                                 int64_t qsb, int64_t qsh, float qscale, const float* inv_freq, const float* cbk,
                                 const float* cbv, float* out, void* ws, const DecodeGeom& geom, cudaStream_t s) {
  constexpr int GH = G < 4 ? G : 4;
  const int nseq = kc.batch * kc.n_kv_heads;
  const int rs_cap = rope_rs_cap(kc.capacity, kc.window_len);
  float* rscores = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) +
                                            rope_scores_offset(kc.batch, kc.n_kv_heads, geom));
  // logits: jobs of contiguous 64-token stages per (sequence, head group), about
  // two resident 8-warp CTAs per SM, twice over
  const int jobs_per_chunk = nseq * (G / GH);
  const int max_chunks = rs_cap / STAGE_TOK;
  int nchunk = (sm_count() * 2 * RS_WARPS * 2 + jobs_per_chunk - 1) / jobs_per_chunk;
  if (nchunk > max_chunks) nchunk = max_chunks;
  if (nchunk < 1) nchunk = 1;
  const size_t smem_a = sizeof(RsSmem);
  cudaError_t e = cudaFuncSetAttribute(rope_scores_kernel<GH, MK, DQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_a);
  if (e != cudaSuccess) return e;
  const int64_t nw_a = (int64_t)jobs_per_chunk * nchunk;
  rope_scores_kernel<GH, MK, DQ><<<(unsigned)((nw_a + RS_WARPS - 1) / RS_WARPS), 32 * RS_WARPS, smem_a, s>>>(
      kc, vc.n_quant, vc.n_window, q, dtype, qsb, qsh, qscale, inv_freq, cbk, rscores, rs_cap, G, nchunk);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // decode over the logits (the K cache is not read: one instantiation for both K modes)
  const size_t smem = sizeof(DecSmem);
  e = cudaFuncSetAttribute(decode_kernel<GH, NSN_MODE_2BIT, MV, DQ, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  unsigned int* counters = static_cast<unsigned int*>(ws);
  float* partials = static_cast<float*>(ws) + counter_words((int64_t)nseq);
  const int nwarps = nseq * geom.nsplit_q * (G / GH);
  decode_kernel<GH, NSN_MODE_2BIT, MV, DQ, true><<<(nwarps + DEC_WARPS - 1) / DEC_WARPS, 32 * DEC_WARPS, smem, s>>>(
      kc, vc, q, dtype, qsb, qsh, qscale, cbk, cbv, counters, partials, out, n_q_heads, geom, rscores, rs_cap, 0,
      (int64_t)n_q_heads * D);
  return cudaGetLastError();
}

template <int G>
static cudaError_t launch_rope_g(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                                 int64_t qsb, int64_t qsh, float qscale, const float* inv_freq, const float* cbk,
                                 const float* cbv, float* out, void* ws, const DecodeGeom& geom, cudaStream_t s) {
#define NSN_LAUNCH_R(MK_, MV_)                                                                                      \
  return kc.dq ? launch_rope_t<G, MK_, MV_, true>(kc, vc, q, dtype, n_q_heads, qsb, qsh, qscale, inv_freq, cbk, cbv, \
                                                  out, ws, geom, s)                                                  \
               : launch_rope_t<G, MK_, MV_, false>(kc, vc, q, dtype, n_q_heads, qsb, qsh, qscale, inv_freq, cbk, cbv, \
                                                   out, ws, geom, s)
  if (kc.mode == NSN_MODE_1BIT && vc.mode == NSN_MODE_1BIT) NSN_LAUNCH_R(1, 1);
  if (kc.mode == NSN_MODE_1BIT && vc.mode == NSN_MODE_2BIT) NSN_LAUNCH_R(1, 2);
  if (kc.mode == NSN_MODE_2BIT && vc.mode == NSN_MODE_1BIT) NSN_LAUNCH_R(2, 1);
  NSN_LAUNCH_R(2, 2);
#undef NSN_LAUNCH_R
}

cudaError_t launch_decode_rope(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                               int64_t qsb, int64_t qsh, float softmax_scale, const float* inv_freq, const float* cbk,
                               const float* cbv, float* out, void* ws, const DecodeGeom& geom, cudaStream_t s) {
  const float qscale = softmax_scale * LOG2E;
  switch (geom.g) {
    case 1: return launch_rope_g<1>(kc, vc, q, dtype, n_q_heads, qsb, qsh, qscale, inv_freq, cbk, cbv, out, ws, geom, s);
    case 2: return launch_rope_g<2>(kc, vc, q, dtype, n_q_heads, qsb, qsh, qscale, inv_freq, cbk, cbv, out, ws, geom, s);
    case 4: return launch_rope_g<4>(kc, vc, q, dtype, n_q_heads, qsb, qsh, qscale, inv_freq, cbk, cbv, out, ws, geom, s);
    default: return launch_rope_g<8>(kc, vc, q, dtype, n_q_heads, qsb, qsh, qscale, inv_freq, cbk, cbv, out, ws, geom, s);
  }
}

// ---------------------------------------------------------------------------
// Diagnostic of the bounded wait: one warp arms an mbarrier for a copy that is
// never issued and waits on it with the decode's wait helper, capped at `limit`
// attempts.  The wait must give up, set status bit 2 and return, so the error
// path of a copy that never lands can be tested without a fault or a hang.
// ---------------------------------------------------------------------------
__global__ void bounded_wait_selftest_kernel(int32_t* status, uint32_t limit) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    mbar_expect_tx(b, 16u);  // 16 bytes are announced; none will arrive
  }
  __syncwarp();
  const bool arrived = mbar_wait(b, 0u, limit);
  if (!__all_sync(0xffffffffu, arrived) && threadIdx.x == 0 && status) atomicOr(status, 2);
}

cudaError_t launch_bounded_wait_selftest(int32_t* status, uint32_t limit, cudaStream_t s) {
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(status, limit);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free decode.  Some callers cannot allocate device memory at the
// moment they need to attend: code running inside a custom allocator or a
// memory-pool callback, processes whose device memory is fully reserved up
// front by a framework, or embedded hosts that forbid cudaMalloc after start-up.
// For them the decode partials live in this fixed file-scope device array
// instead of a caller-provided workspace, and the merge counters in a second
// one.  Every GPU that loads the library holds both until the process exits.
// All calls share them, so two such calls that overlap on the GPU (different
// streams, no ordering) race on them.  The kernel writes every partial it later
// reads, and each completed call leaves every counter it used at zero (both
// arrays start zero-filled), so nothing needs clearing between calls.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_decode_scratch[NSN_DECODE_SCRATCH_BYTES];
static __device__ __align__(256) unsigned int g_decode_counters[NSN_DECODE_STATIC_COUNTERS];

bool decode_static_fits(int batch, int n_kv_heads, const DecodeGeom& geom) {
  return decode_partial_bytes(batch, n_kv_heads, geom) <= (size_t)NSN_DECODE_SCRATCH_BYTES &&
         2 * (int64_t)batch * n_kv_heads <= (int64_t)NSN_DECODE_STATIC_COUNTERS;
}

// The current CUDA context (driver handle), or null.  cuCtxGetCurrent is looked
// up through the runtime, so the library does not link the driver library.
typedef int (*CtxGetCurrentFn)(void**);
static void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  void* ctx = nullptr;
  if (fn && fn(&ctx) != 0) ctx = nullptr;
  return ctx;
}

// Device addresses of the two arrays for the current device.  Resolved with
// cudaGetSymbolAddress (that device current) at the device's first call and cached
// together with the CUDA context they belong to; a different context on the same
// device (one created after cudaDeviceReset, for instance, which loads the module
// again) resolves them anew, so a stale address is never used.
static cudaError_t decode_static_ptrs(void** scratch, void** counters) {
  static std::mutex mu;
  struct Entry { void* ctx; void* scratch; void* counters; };
  static Entry cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  void* ctx = current_context();
  Entry& en = cache[dev];
  if (!en.scratch || !ctx || en.ctx != ctx) {
    void* p = nullptr;
    void* c = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    e = cudaGetSymbolAddress(&c, g_decode_counters);
    if (e != cudaSuccess) return e;
    en = Entry{current_context(), p, c};
  }
  *scratch = en.scratch;
  *counters = en.counters;
  return cudaSuccess;
}

cudaError_t launch_decode_static(const CacheView& kc, const CacheView& vc, const void* q, int dtype, int n_q_heads,
                                 int64_t qsb, int64_t qsh, float softmax_scale, const float* cbk, const float* cbv,
                                 float* out, const DecodeGeom& geom, cudaStream_t s) {
  void* scratch = nullptr;
  void* counters = nullptr;
  const cudaError_t e = decode_static_ptrs(&scratch, &counters);
  if (e != cudaSuccess) return e;
  return launch_any(kc, vc, q, dtype, n_q_heads, qsb, qsh, softmax_scale, cbk, cbv, out,
                    static_cast<unsigned int*>(counters), static_cast<float*>(scratch), geom, s);
}

}  // namespace nsn
