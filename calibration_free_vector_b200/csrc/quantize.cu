// NSNQuant KV quantizer kernels (sm_100a).
//
// Method: "NSNQuant: A Double Normalization Approach for Calibration-Free Low-Bit
// Vector Quantization of KV Cache", technical summary, Metodologia 1 (NSN),
// 2 (Hadamard), 3 (VQ with one global codebook, adaptive scale) and 4 (KIVI-style
// residual that is flushed into the quantized part when full).
//
// Prefill runs one persistent, warp-specialized CTA per SM (quantize_prefill_ws_kernel):
// 8 normalizer warps run the NSN of one block of <= 128 tokens of a (batch, kv-head)
// while two warpgroups of search warps find the codewords of the previous block.
// Residual-window flushes run one CTA of 256 threads per block (append_kernel).
// In NSN the adjacent lanes 2t, 2t+1 of the normalizers own token t (64 dims, 8
// sub-vectors each).  Per block:
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
// Nearest codeword, on the 5th-generation tensor cores: the 2048 sub-vectors of a
// block form 16 tiles of 128 rows (8 tokens x 16 sub-vectors).  Per tile two
// tcgen05.mma (M = 128, N = 256 codewords, K = 16, fp16 operands from shared
// memory, fp32 accumulators in tensor memory) write every score
//   score_k = a . c_k - ||c_k||^2 / 2        (a = u, or |u| in 2-bit mode)
// The first MMA writes the bias (A = [1, 1, 0...], B = the fp16 hi and lo parts of
// -||c_k||^2/2), the second adds K = [a_hi | a_lo] (the fp32 a split into two fp16
// parts, exact to 2^-22) times [c | c] (the codebook in fp16).  Each TMEM lane
// holds one sub-vector's 256 scores; its thread reads them back with tcgen05.ld and
// keeps, with three-input max trees, the best and second-best maxima of the 32
// groups of 8 codewords (the group number rides in the low mantissa bits).
//   Prefill: the thread also keeps the maxima of the 8 columns (position within a
//   group) over all groups.  The best score lies in the best group G and the best
//   column J, so it is codeword 8 G + J; every other score is below the second-best
//   group or column maximum.  If the best beats both by more than twice the
//   tensor-score bound the code is certain.
//   Window flushes: the 8 codewords of the winning group are rescanned in
//   sequential fp32 from an fp32 copy of the codebook in shared memory, and the
//   in-group decision uses the fp32 bound.
// Whenever a rival lies within the bounds, the sub-vector is re-decided exactly in
// fp64 by a whole warp over all codewords inside the bound (ties to the lowest
// index).  The stored code is therefore the exact nearest codeword of the fp32 u.

#include <algorithm>

#include "nsn_common.cuh"
#include "nsn_launch.h"

namespace nsn {

__device__ __forceinline__ uint32_t q_smem(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor core) helpers
// ---------------------------------------------------------------------------
// Shared-memory operand layout of one [rows][16] fp16 tile, K-major without
// swizzle: 8-row x 16-byte core matrices; the two 8-element K halves of an 8-row
// group are 128 B apart (leading byte offset), consecutive 8-row groups 256 B apart
// (stride byte offset).
__host__ __device__ constexpr uint32_t kmaj_off(int row, int k) {
  return (uint32_t)((row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}
// Matrix descriptor: start address, leading / stride byte offsets (16-byte units),
// descriptor version 1 (sm_100), no swizzle.
__device__ __forceinline__ uint64_t tc_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Instruction descriptor of kind::f16: fp32 accumulator (bit 4), fp16 A and B,
// both K-major, N = 256 (bits 17-22: N >> 3), M = 128 (bits 24-28: M >> 4).
constexpr uint32_t TC_IDESC = (1u << 4) | ((256u >> 3) << 17) | ((128u >> 4) << 24);
constexpr int TC_COLS = 256;  // tensor-memory columns of one CTA: the 256 fp32 scores of 128 rows

__device__ __forceinline__ void tc_mma(uint32_t dtmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile("{.reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;}"
               :: "r"(dtmem), "l"(adesc), "l"(bdesc), "r"(TC_IDESC), "r"(accumulate) : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(mbar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// Bounded wait on an mbarrier phase; false after `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, int limit) {
  for (int it = 0; it < limit; ++it) {
    uint32_t done;
    asm volatile("{.reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p;}"
                 : "=r"(done) : "r"(mbar), "r"(parity) : "memory");
    if (done) return true;
  }
  return false;
}
// 32 consecutive fp32 columns of this warp's 32 TMEM lanes (one lane per thread).
// The registers are valid only after tc_wait_ld(); tc_regs_ready() then keeps the
// compiler from reading them before the wait.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
               "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
                 "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                 "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
               : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_regs_ready(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                 "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

constexpr int QTHREADS = 2 * BLK;  // two threads per token
constexpr int HD = D / 2;           // dims per thread
constexpr int HSUB = NSUB / 2;      // sub-vectors per thread
constexpr int MBAR_POLLS = 1 << 22;  // bounded wait for the MMAs of one tile
// Kind of the staged codebook: fp16-representable (the tensor-core operand is exact),
// any other (the operand is its fp16 rounding), or the unit codewords c_hat of the
// cosine assignment (operand c_hat_hi, second operand c_hat_lo, bias 0).
constexpr int TAB_F16 = 0, TAB_GLOBAL = 1, TAB_COSINE = 2;

// Shared-memory state of the quantizer, in four parts so that a warp-specialized
// CTA can keep two blocks in flight: the staged codebook (per launch), the search's
// operands and barriers, the NSN scratch, and one block's data.
struct QTables {
  // ---- operands of the tensor-core scores ----
  alignas(128) unsigned char bop[NCODES * 32];    // B: codebook fp16 [c | c], K-major canonical layout
  alignas(128) unsigned char bop2[NCODES * 16];   // B of the bias MMA: per codeword [b_hi, b_lo, 0 x 6]; K half 1 aliases K half 0
  alignas(128) unsigned char aop2[256];           // A of the bias MMA: one core matrix of rows [1, 1, 0 ...] + a zero one
  // ---- codebook for the exact arithmetic (fp32: c, or c_hat for the cosine assignment), two
  // replicas: replica p of codeword k at floats 16 k + 8 p .. 16 k + 8 p + 7, so a 16-byte half h of it
  // lies in bank group 4 (k & 1) + 2 p + h.  The bias -||c_k||^2/2 (fp32, sequential; 0 for the cosine
  // assignment) in four replicas, replica r at word 4 k + r.  A lane l reading codeword 8 G + ((i + l) & 7)
  // from replica (l >> 2) & 1, half (l >> 1) & 1 first, with bias replica l >> 3, hits with the 8 lanes of a
  // phase 8 different bank groups, and with the 32 lanes 32 different bias banks, whatever their groups G;
  // the exact re-decision and the adaptive scale read it, and the flush's group rescan. ----
  alignas(16) float cw[NCODES * 16];
  alignas(16) float cbias[NCODES * 4];
  alignas(16) float cnorm[4];                     // [0] max ||c||, [1] max ||c||^2, [2] max ||c - fp16(c)|| (rounded up)
  int tab;                                        // TAB_F16, TAB_GLOBAL or TAB_COSINE
};

struct QSearch {
  alignas(128) unsigned char aop[2][BLK * 32];    // A: [a_hi | a_lo] of the 128 rows of a tile (double-buffered)
  alignas(8) unsigned long long mbar[2];          // MMA completion barriers (one per tensor-memory buffer)
  uint32_t tmem;                                  // tensor-memory base address of this CTA
  int nflag;
  alignas(16) uint16_t flag[BLK * NSUB];          // (token, sub-vector) pairs for the exact re-decision
};

struct QNsn {
  alignas(16) double rr[BLK];          // 1 / ||x_t|| (0 for a zero token)
  alignas(16) float r[D];              // column mean of raw tokens (fp32)
  union {                              // NSN column sums, then the search's warp-pair exchanges
    struct {
      double part[2][D];               // per-half column partial sums
      double dev_part[2];              // per-half sums of rr_t - rr_0
      double big_r[D];                 // FWHT(r) in fp64
      float big_rf[D];                 // FWHT(r) and D_c = mean_t(d_t,c rr_t) rounded to fp32 (the constant terms of z)
      float dcf[D];
    };
    struct {
      float2 xch1[2][BLK];             // group maxima (best key, second) per half
      float4 xch2[BLK];                // rescan (best, second, index) of the upper half
    };
  };
  // double quantization
  alignas(16) double red[2][QTHREADS / 32][2];  // per-warp (min, max) of s1 and of o
  alignas(16) double dq[2][3];         // (lo, hi, step) of s1 and of o
  alignas(16) uint8_t lev[2][BLK];     // 4-bit levels of s1 (per token) and of o (per channel)
};

struct QBlock {
  alignas(16) float tile[BLK][D + 4];  // raw tokens, then d_t rows, then u rows (|u| in 2-bit mode); padded by 16 B
  alignas(16) double s1[BLK];          // per-token s1 and s2 (fp64) until the final store
  alignas(16) double s2[BLK];
  alignas(16) double ofull[D];         // o of the block (fp64) until its levels are formed
  alignas(16) uint8_t code[BLK][NSUB]; // chosen codes
};

// One CTA, one block at a time (2 CTAs per SM): prefill flushes of the residual window.
struct QuantSmem {
  QTables tb;
  QSearch se;
  QNsn ns;
  QBlock bk;
};

// The parts a phase works on (the warp-specialized CTA passes one of its two blocks).
struct QRefs {
  QTables* tb;
  QSearch* se;
  QNsn* ns;
  QBlock* bk;
};

__device__ __forceinline__ QRefs refs(QuantSmem& sm) { return QRefs{&sm.tb, &sm.se, &sm.ns, &sm.bk}; }

// A set of threads that synchronize among themselves: the whole CTA (id 0,
// __syncthreads) or `n` threads on named barrier `id`; t = index within the set.
struct Grp {
  int id, n, t;
  __device__ __forceinline__ void sync() const {
    if (id == 0) __syncthreads();
    else asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(n) : "memory");
  }
};
__device__ __forceinline__ Grp cta_grp() { return Grp{0, (int)blockDim.x, (int)threadIdx.x}; }

// Tensor-memory allocation and the MMA barriers of one CTA.
struct TcState {
  uint32_t tmem;
  uint32_t phase;  // parity bit per barrier
  uint32_t ncols;
};

// Allocates `ncols` tensor-memory columns (warp 0) and initialises `nbar` MMA
// barriers; every thread of the CTA calls it.
__device__ TcState tc_setup(QSearch& se, uint32_t ncols, int nbar) {
  const int t = threadIdx.x;
  if (t < nbar) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(q_smem(&se.mbar[t])));
  if (t == 0) asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  if ((t >> 5) == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(q_smem(&se.tmem)), "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return TcState{se.tmem, 0u, ncols};
}

__device__ void tc_teardown(const TcState& tcs) {
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tcs.tmem), "r"(tcs.ncols));
}

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

// Stages the codebook: the tensor-core operands (fp16 codebook, fp16 hi/lo bias,
// the constant bias rows), the fp16 rows and fp32 biases of the exact arithmetic,
// and the norm bounds.  All QTHREADS threads (one codeword each).
//
// Cosine assignment (cosine = 1): the scores are a . c_hat with c_hat = c / ||c||
// (fp64 division, rounded once to fp32; 0 for a zero codeword).  The score MMA
// takes c_hat's fp16 high part as B, the second MMA (in place of the bias MMA)
// adds the same A rows times its fp16 low part, the exact arithmetic reads the
// fp32 c_hat from the table (bias 0), and the bounds are those of c_hat.
__device__ void stage_codebook(const QRefs& q, const float* __restrict__ codebook, int cosine) {
  const int t = threadIdx.x;
  float my_max = 0.f, my_dev = 0.f;
  for (int k = t; k < NCODES; k += blockDim.x) {
    float c[SUB];
    float4 c0 = __ldg(reinterpret_cast<const float4*>(codebook + k * SUB));
    float4 c1 = __ldg(reinterpret_cast<const float4*>(codebook + k * SUB) + 1);
    c[0] = c0.x; c[1] = c0.y; c[2] = c0.z; c[3] = c0.w; c[4] = c1.x; c[5] = c1.y; c[6] = c1.z; c[7] = c1.w;
    if (cosine) {
      double nn = 0.0;
#pragma unroll
      for (int i = 0; i < SUB; ++i) nn = fma((double)c[i], (double)c[i], nn);
      const double nrm = sqrt(nn);
#pragma unroll
      for (int i = 0; i < SUB; ++i) c[i] = nrm > 0.0 ? (float)((double)c[i] / nrm) : 0.f;
      c0 = make_float4(c[0], c[1], c[2], c[3]);
      c1 = make_float4(c[4], c[5], c[6], c[7]);
    }
    float ss = 0.f, e = 0.f;
    __half ch[SUB];
#pragma unroll
    for (int i = 0; i < SUB; ++i) {
      ss = fmaf(c[i], c[i], ss);
      ch[i] = __float2half_rn(c[i]);
      const float dlt = c[i] - __half2float(ch[i]);
      e = fmaf(dlt, dlt, e);
    }
    const float bias = -0.5f * ss;
    // B operand: K = 0..7 and 8..15 both hold the codeword (multiplied by a_hi and a_lo)
    *reinterpret_cast<uint4*>(q.tb->bop + kmaj_off(k, 0)) = *reinterpret_cast<const uint4*>(ch);
    *reinterpret_cast<uint4*>(q.tb->bop + kmaj_off(k, 8)) = *reinterpret_cast<const uint4*>(ch);
    uint4 brow = make_uint4(0u, 0u, 0u, 0u);
    // fp32 codeword (c_hat) for the exact arithmetic, both replicas, and its bias replicas
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      *reinterpret_cast<float4*>(q.tb->cw + 16 * k + 8 * p) = c0;
      *reinterpret_cast<float4*>(q.tb->cw + 16 * k + 8 * p + 4) = c1;
    }
    const float bstore = cosine ? 0.f : bias;
    *reinterpret_cast<float4*>(q.tb->cbias + 4 * k) = make_float4(bstore, bstore, bstore, bstore);
    if (cosine) {
      // second-MMA operand: fp16(c_hat - fp16(c_hat))
      __half cl[SUB];
#pragma unroll
      for (int i = 0; i < SUB; ++i) cl[i] = __float2half_rn(c[i] - __half2float(ch[i]));
      brow = *reinterpret_cast<const uint4*>(cl);
      e = 0.f;  // hi + lo carries c_hat to 2^-22, inside the tensor bound
    } else {
      // bias operand: (b_hi, b_lo) with b_hi + b_lo = bias to 2^-22 relative
      const __half bh = __float2half_rn(bias);
      const __half bl = __float2half_rn(bias - __half2float(bh));
      brow.x = (uint32_t)__half_as_ushort(bh) | ((uint32_t)__half_as_ushort(bl) << 16);
    }
    *reinterpret_cast<uint4*>(q.tb->bop2 + (k >> 3) * 128 + (k & 7) * 16) = brow;
    my_max = fmaxf(my_max, ss);
    my_dev = fmaxf(my_dev, e);
  }
  if (t < 16) {  // bias A operand: 8 rows [1, 1, 0, ...] (K half 0) and a zero core matrix (K half 1)
    const uint32_t one2 = 0x3C003C00u;  // fp16 (1, 1)
    *reinterpret_cast<uint4*>(q.tb->aop2 + 16 * t) = t < 8 ? make_uint4(one2, 0u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
  }
  my_max = warp_max(my_max);
  my_dev = warp_max(my_dev);
  __shared__ float red[32][2];  // per-warp maxima (up to 32 warps)
  if ((t & 31) == 0) {
    red[t >> 5][0] = my_max;
    red[t >> 5][1] = my_dev;
  }
  fence_async_smem();  // operands written by the generic proxy, read by the tensor cores
  __syncthreads();
  if (t == 0) {
    float m = 0.f, e = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      m = fmaxf(m, red[w][0]);
      e = fmaxf(e, red[w][1]);
    }
    m *= 1.0001f;  // upper bound on max ||c||^2 despite the fp32 rounding above
    q.tb->cnorm[1] = m;
    q.tb->cnorm[0] = sqrtf(m) * 1.0001f;
    q.tb->cnorm[2] = e > 0.f ? sqrtf(e) * 1.001f : 0.f;  // 0 for a codebook of fp16 values
    q.tb->tab = cosine ? TAB_COSINE : (e > 0.f ? TAB_GLOBAL : TAB_F16);
  }
  __syncthreads();
}

// Codeword k as the exact arithmetic uses it (fp32, natural order; c_hat for the cosine
// assignment) from replica p of the table, and its bias.
__device__ __forceinline__ float codeword(const QRefs& q, int k, int p, float (&c)[SUB]) {
  const float4 c0 = *reinterpret_cast<const float4*>(q.tb->cw + 16 * k + 8 * p);
  const float4 c1 = *reinterpret_cast<const float4*>(q.tb->cw + 16 * k + 8 * p + 4);
  c[0] = c0.x; c[1] = c0.y; c[2] = c0.z; c[3] = c0.w; c[4] = c1.x; c[5] = c1.y; c[6] = c1.z; c[7] = c1.w;
  return q.tb->cbias[4 * k + p];
}

// Codeword k as stored in the codebook (the reconstruction's u_hat), fp32.
__device__ __forceinline__ void codeword_given(const QRefs& q, const float* __restrict__ cb_global, int tab,
                                               int k, int p, float (&c)[SUB]) {
  if (tab == TAB_COSINE) {
    const float4 c0 = __ldg(reinterpret_cast<const float4*>(cb_global + k * SUB));
    const float4 c1 = __ldg(reinterpret_cast<const float4*>(cb_global + k * SUB) + 1);
    c[0] = c0.x; c[1] = c0.y; c[2] = c0.z; c[3] = c0.w; c[4] = c1.x; c[5] = c1.y; c[6] = c1.z; c[7] = c1.w;
  } else {
    codeword(q, k, p, c);
  }
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
// q.bk->s1 and q.bk->ofull hold the exact fp64 values.  All QTHREADS threads.
__device__ void store_double_quant(const QRefs& q, const Grp& gr, int n, const BlockOut& bo) {
  gr.sync();  // s1 of every token is final
  const int t = gr.t, grp = t >> 7, i = t & (BLK - 1), warp = t >> 5, lane = t & 31;
  const bool have = grp == 1 || i < n;
  const double x = grp == 0 ? (i < n ? q.bk->s1[i] : 0.0) : q.bk->ofull[i];
  const double mn = warp_min_d(have ? x : INFINITY), mx = warp_max_d(have ? x : -INFINITY);
  if (lane == 0) {
    q.ns->red[grp][warp & 3][0] = mn;
    q.ns->red[grp][warp & 3][1] = mx;
  }
  gr.sync();
  if (t < 2) {
    double a = INFINITY, b = -INFINITY;
    for (int w = 0; w < 4; ++w) {
      a = fmin(a, q.ns->red[t][w][0]);
      b = fmax(b, q.ns->red[t][w][1]);
    }
    const double lo = (double)__half2float(__double2half(a));
    const double hi = (double)__half2float(__double2half(b));
    q.ns->dq[t][0] = lo;
    q.ns->dq[t][1] = hi;
    q.ns->dq[t][2] = (hi - lo) / 15.0;
  }
  gr.sync();
  {
    const double lo = q.ns->dq[grp][0], step = q.ns->dq[grp][2];
    int level = 0;
    if (have && step > 0.0) level = (int)fmin(15.0, fmax(0.0, rint((x - lo) / step)));
    q.ns->lev[grp][i] = (uint8_t)level;
  }
  gr.sync();
  if (t < 64) bo.s1_levels[t] = (uint8_t)(q.ns->lev[0][2 * t] | (q.ns->lev[0][2 * t + 1] << 4));
  else if (t < 128) bo.o_levels[t - 64] = (uint8_t)(q.ns->lev[1][2 * (t - 64)] | (q.ns->lev[1][2 * (t - 64) + 1] << 4));
  else if (t < 136) {
    const int k = t - 128;
    const double v = k == 0 ? q.ns->dq[0][0] : k == 1 ? q.ns->dq[0][1] : k == 2 ? q.ns->dq[1][0] : k == 3 ? q.ns->dq[1][1] : 0.0;
    bo.params[k] = __double2half(v);
  }
}

// Nearest codeword of the sub-vectors of one block (rows of q.bk->tile: a = u, or |u|
// in 2-bit mode; rows of tokens past n are zero), written to q.bk->code.  Sub-vectors
// whose decision lies within the error bounds are appended to q.se->flag for the
// exact re-decision.  All QTHREADS threads.
//
// Tile t = tokens 8t .. 8t+7: row L (TMEM lane L) = token 8t + L/16, sub-vector L%16.
// Warp w reads TMEM lanes 32(w%4) .. 32(w%4)+31 and columns 128(w/4) .. +127, so
// warps w and w+4 form a pair over the same rows.  Per tile:
//   (1) thread 0 issues the bias MMA (D = b_hi + b_lo) and the score MMA
//       (D += [a_hi | a_lo] [c | c]) and commits them to the barrier;
//   (2) meanwhile every thread writes its half of the next tile's A rows;
//   (3) after the barrier, each warp reads its 128 scores per row in chunks of 32
//       and keeps the best and second-best of its 16 group maxima (group = 8
//       consecutive codewords; the group number replaces the 5 low mantissa bits,
//       so the maximum carries its group);
//   (4) the pair merges its halves (both sides get the best group G and the best
//       maximum among the other groups), thread 0 issues the next tile's MMAs,
//       and each side rescans 4 codewords of group G in sequential fp32;
//   (5) the lower warp merges the rescans and applies the decision bounds:
//       the sequential fp32 score is within gamma_9 (max||c||^2 + ||a|| max||c||)
//       of the exact one; the tensor score within tensor_bound() (accumulation
//       order and rounding inside the MMA are the hardware's, so that term is taken
//       wide: 17 terms of at most 2^-24 relative error each need about 2^-19.9);
//       the group number adds at most 32 ulp to a maximum.
//       A rival inside the group within twice the fp32 bound, or another group's
//       maximum within the fp32 plus the tensor bound, flags the sub-vector.
// Bound on |tensor score - exact score| of a row of norm na (rounded up), for a
// codebook with max ||c|| = cmax, max ||c||^2 = cmax2 and max ||c - fp16(c)|| = cdel:
//   2^-16 (na cmax + cmax2 / 2)   accumulation inside the MMA (taken wide: its order
//                                  and rounding are the hardware's);
//   + na cdel                     the fp16 operand of a codebook that is not fp16-representable;
//   + 2^-25 sqrt(8) (cmax + na)   an fp16 lo part below the normal range (of a, and of c_hat in
//                                  the cosine rule) is off by up to half its 2^-24 spacing, so
//                                  hi + lo is exact to 2^-22 only relative to larger elements;
// with 1 % and an absolute 1.2e-7 (the lo part of the bias) on top.  The raw MMA scores are
// compared with this bound by nsn_selftest_tensor_scores.
__device__ __forceinline__ float tensor_bound(float na, float cmax, float cmax2, float cdel) {
  constexpr float TC_REL = 1.52587890625e-05f;        // 2^-16
  constexpr float SUBN = 2.98023223876953125e-08f * 2.8285f;  // 2^-25 sqrt(8), rounded up
  return (TC_REL * (1.001f * na * cmax + 0.5f * cmax2) + na * cdel + SUBN * (cmax + na)) * 1.01f + 1.2e-7f;
}

__device__ void search_block(const QRefs& q, TcState& tcs, const float* __restrict__ cb_global, int n,
                             int32_t* status) {
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int qd = warp & 3, hf = warp >> 2;
  const int L = 32 * qd + lane;
  const float cmax = q.tb->cnorm[0], cmax2 = q.tb->cnorm[1], cdel = q.tb->cnorm[2];
  const int tab = q.tb->tab;
  constexpr float GAMMA9 = 9.0f * 5.9604645e-8f * 1.0001f;  // 9u/(1-9u), u = 2^-24
  const uint32_t taddr = tcs.tmem + ((uint32_t)(32 * qd) << 16) + (uint32_t)(128 * hf);
  const uint64_t db = tc_desc(q_smem(q.tb->bop), 128, 256);
  const uint64_t da2 = tc_desc(q_smem(q.tb->aop2), 128, 0);  // every 8-row group reads the same [1, 1, 0...] rows
  const uint64_t db2 = tc_desc(q_smem(q.tb->bop2), 0, 128);  // K half 1 re-reads K half 0 (times A's zero half)
  const uint32_t mbar = q_smem(&q.se->mbar[0]);
  const int ntiles = (n + 7) >> 3;

  // The A rows of a tile; the row's decision bounds are formed here too, off the
  // critical path of the decision: margin = twice the fp32 bound, mtc = the tensor bound.
  auto build_a = [&](int tile, float (&a)[SUB], float& margin, float& mtc) {
    const int tkk = 8 * tile + (L >> 4), j = L & 15;
    const float4 a0 = *reinterpret_cast<const float4*>(&q.bk->tile[tkk][SUB * j]);
    const float4 a1 = *reinterpret_cast<const float4*>(&q.bk->tile[tkk][SUB * j + 4]);
    a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
    a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
    float na = 0.f;
#pragma unroll
    for (int d = 0; d < SUB; ++d) na = fmaf(a[d], a[d], na);
    na = sqrtf(na) * 1.0001f;
    margin = 2.0f * GAMMA9 * (cmax2 + na * cmax) * 1.01f;
    mtc = tensor_bound(na, cmax, cmax2, cdel);
    uint32_t w[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const __half2 hh = __floats2half2_rn(a[2 * p], a[2 * p + 1]);
      w[p] = h2_bits(hh);
      if (hf != 0)
        w[p] = h2_bits(__floats2half2_rn(sub_f16(a[2 * p], (uint16_t)(w[p] & 0xFFFFu)),
                                         sub_f16(a[2 * p + 1], (uint16_t)(w[p] >> 16))));
    }
    *reinterpret_cast<uint4*>(q.se->aop[tile & 1] + kmaj_off(L, 8 * hf)) = make_uint4(w[0], w[1], w[2], w[3]);
  };
  auto issue = [&](int tile) {
    const uint64_t da = tc_desc(q_smem(q.se->aop[tile & 1]), 128, 256);
    if (tab == TAB_COSINE) {  // D = [a_hi | a_lo] [c_hat_hi | c_hat_hi] + [a_hi | a_lo] [c_hat_lo | c_hat_lo]
      tc_mma(tcs.tmem, da, db, 0u);
      tc_mma(tcs.tmem, da, db2, 1u);
    } else {                  // D = b_hi + b_lo, then D += [a_hi | a_lo] [c | c]
      tc_mma(tcs.tmem, da2, db2, 0u);
      tc_mma(tcs.tmem, da, db, 1u);
    }
    tc_commit(mbar);
  };

  float a[SUB], an[SUB], margin, mtc, margin_n = 0.f, mtc_n = 0.f;
  build_a(0, a, margin, mtc);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (t == 0) issue(0);
#pragma unroll 1
  for (int tile = 0; tile < ntiles; ++tile) {
    if (tile + 1 < ntiles) {
      build_a(tile + 1, an, margin_n, mtc_n);
      fence_async_smem();
    }
    if (!mbar_wait(mbar, tcs.phase, MBAR_POLLS) && lane == 0 && status) atomicOr(status, 2);
    tcs.phase ^= 1u;
    tc_fence_after();

    // (3) best and second-best group maxima of this warp's 128 columns
    float b1 = -INFINITY, b2 = -INFINITY;
    uint32_t r[32];
    tc_ld32(taddr, r);
    tc_wait_ld();
    tc_regs_ready(r);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t rn[32];
      if (c < 3) tc_ld32(taddr + 32 * (c + 1), rn);
      float key[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float m = max3f(max3f(__uint_as_float(r[8 * g]), __uint_as_float(r[8 * g + 1]), __uint_as_float(r[8 * g + 2])),
                              max3f(__uint_as_float(r[8 * g + 3]), __uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5])),
                              fmaxf(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7])));
        key[g] = __uint_as_float((__float_as_uint(m) & ~31u) | (uint32_t)(16 * hf + 4 * c + g));
      }
      const float h01 = fmaxf(key[0], key[1]), l01 = fminf(key[0], key[1]);
      const float h23 = fmaxf(key[2], key[3]), l23 = fminf(key[2], key[3]);
      const float hi = fmaxf(h01, h23);
      const float lo = max3f(l01, l23, fminf(h01, h23));
      b2 = max3f(b2, lo, fminf(b1, hi));
      b1 = fmaxf(b1, hi);
      if (c < 3) {
        tc_wait_ld();
        tc_regs_ready(rn);
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = rn[i];
      }
    }

    // (4) merge the pair's halves; the scores are read, so the next tile may start
    q.ns->xch1[hf][L] = make_float2(b1, b2);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0 && tile + 1 < ntiles) issue(tile + 1);
    const float2 o1 = q.ns->xch1[hf ^ 1][L];
    const float m1 = fmaxf(b1, o1.x);
    const float m2 = max3f(b2, o1.y, fminf(b1, o1.x));
    const int G = (int)(__float_as_uint(m1) & 31u);
    float best = -INFINITY, second = -INFINITY;
    int idx = 8 * G + 4 * hf;
    {
      // this half's 4 codewords, in an order rotated by lane (bank-conflict free);
      // the index keeps the lowest of equal scores explicitly
      const int rep = (lane >> 2) & 1;
      float cw[4][SUB], sc[4];
      int kk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        kk[i] = 8 * G + 4 * hf + ((i + lane) & 3);
        sc[i] = codeword(q, kk[i], rep, cw[i]);
      }
#pragma unroll
      for (int d = 0; d < SUB; ++d)
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[i] = fmaf(a[d], cw[i][d], sc[i]);
      idx = NCODES;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = fminf(best, sc[i]);
        idx = (sc[i] > best || (sc[i] == best && kk[i] < idx)) ? kk[i] : idx;
        best = fmaxf(best, sc[i]);
        second = fmaxf(second, lo);
      }
    }
    if (hf == 1) q.ns->xch2[L] = make_float4(best, second, __int_as_float(idx), 0.f);
    asm volatile("bar.sync %0, 64;" :: "r"(1 + qd) : "memory");  // the two warps of the pair only

    // (5) decision and bounds (lower warp of the pair)
    if (hf == 0) {
      const float4 o2 = q.ns->xch2[L];
      second = max3f(second, o2.y, fminf(best, o2.x));
      idx = (o2.x > best) ? __float_as_int(o2.z) : idx;  // the upper half holds the larger indices
      best = fmaxf(best, o2.x);
      const float other = m2 + fabsf(m2) * 3.82e-6f;  // + 32 ulp: the group number in the low bits
      const int tkk = 8 * tile + (L >> 4), j = L & 15;
      q.bk->code[tkk][j] = (uint8_t)idx;
      const bool need = second >= best - margin || other >= best - 0.5f * margin - mtc;
      if (need && tkk < n) q.se->flag[atomicAdd(&q.se->nflag, 1)] = (uint16_t)(tkk * NSUB + j);
    }
#pragma unroll
    for (int i = 0; i < SUB; ++i) a[i] = an[i];
    margin = margin_n;
    mtc = mtc_n;
  }
  __syncthreads();
}

// NSN of one block of n (1..128) tokens by a set of 256 threads: thread
// t = 2 tk + h works on token tk, dims 64h .. 64h+63 (sub-vectors 8h .. 8h+7).
// Rows are at src + row0 + tk*row_stride (elements).  Leaves the u rows (|u| in
// 2-bit mode; zero rows past n) in q.bk->tile, s1 and s2 (fp64) in q.bk, o in
// q.bk->ofull (double quantization) or stored; sign bits (2-bit) are stored.
template <int DT, int MODE>
__device__ void nsn_phase(const QRefs& q, const Grp& gr, const void* __restrict__ src, int64_t row0,
                          int64_t row_stride, int n, uint8_t* __restrict__ signs, const CacheView& cv, int64_t seq,
                          int blk) {
  const int t = gr.t, tk = t >> 1, h = t & 1;
  const int col = t & (D - 1), rhalf = t >> 7;  // column-sum roles: column, half of the rows
  const bool valid = tk < n;
  constexpr int ESZ = (DT == NSN_DTYPE_F32) ? 4 : 2;
  constexpr int CHUNKS = D * ESZ / 16;  // 16-byte chunks per row

  // ---- cooperative, coalesced load of the raw tile into shared memory --------
  {
    char* tile_bytes = reinterpret_cast<char*>(&q.bk->tile[0][0]);
    constexpr int ROWB = (D + 4) * 4;  // padded row stride in bytes (fits both dtypes)
    for (int qq = t; qq < BLK * CHUNKS; qq += gr.n) {
      const int row = qq / CHUNKS, ch = qq % CHUNKS;
      if (row < n) {
        const char* g = static_cast<const char*>(src) + (row0 + (int64_t)row * row_stride) * ESZ + ch * 16;
        *reinterpret_cast<uint4*>(tile_bytes + row * ROWB + ch * 16) = __ldg(reinterpret_cast<const uint4*>(g));
      }
    }
  }
  gr.sync();

  auto raw_at = [&](int row, int c) -> float {
    const char* tb = reinterpret_cast<const char*>(&q.bk->tile[0][0]) + row * (D + 4) * 4;
    if constexpr (DT == NSN_DTYPE_F32) return reinterpret_cast<const float*>(tb)[c];
    else if constexpr (DT == NSN_DTYPE_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(tb)[c]);
    else return __half2float(reinterpret_cast<const __half*>(tb)[c]);
  };

  // ---- reference r = column mean of the raw tokens ---------------------------
  // r only conditions the fp32 transform (FWHT(x - r) + FWHT(r) = FWHT(x) for any
  // r), so it is formed in fp32: the first token plus the mean deviation from it,
  // which makes r equal the tokens exactly when they are all equal.  Column `col`,
  // rows split in two halves (two accumulators each), combined in a fixed order.
  {
    const int lo = rhalf * (BLK / 2), hi = min(n, lo + BLK / 2);
    const float x0 = raw_at(0, col);
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int row = lo;
    for (; row + 3 < hi; row += 4) {
      s0 += raw_at(row, col) - x0;
      s1 += raw_at(row + 1, col) - x0;
      s2 += raw_at(row + 2, col) - x0;
      s3 += raw_at(row + 3, col) - x0;
    }
    for (; row < hi; ++row) s0 += raw_at(row, col) - x0;
    reinterpret_cast<float*>(&q.ns->part[0][0])[rhalf * D + col] = (s0 + s1) + (s2 + s3);
  }
  gr.sync();
  if (t < D) {
    const float* ps = reinterpret_cast<const float*>(&q.ns->part[0][0]);
    q.ns->r[t] = raw_at(0, t) + (ps[t] + ps[D + t]) / (float)n;
  }
  gr.sync();
  // FWHT(r) in fp64 by warp 0 (lane l holds elements 4l..4l+3).
  if (t < 32) {
    double v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = (double)q.ns->r[4 * t + i];
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
    for (int i = 0; i < 4; ++i) q.ns->big_r[4 * t + i] = v[i];
  }

  // ---- d_t = FWHT(x_t - r) over the lane pair; ||x_t||^2 from the raw values --
  float v[HD];
  double ssx0 = 0.0, ssx1 = 0.0;
  if (valid) {
    const char* tb = reinterpret_cast<const char*>(&q.bk->tile[tk][0]) + HD * ESZ * h;
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
        v[PER * ch + i] = xs[i] - q.ns->r[HD * h + PER * ch + i];
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
  gr.sync();  // raw tile fully consumed; big_r ready

  // ---- first normalization: s1 = ||H x|| / sqrt(128) = ||x|| / sqrt(128) -----
  // (H is orthonormal.)  n1_t = w_t * rr_t with w_t = FWHT(x_t) = d_t + FWHT(r)
  // and rr_t = 1/||x_t|| (||w_t|| = sqrt(128) ||x_t||); a zero token gets rr = 0.
  {
    const double norm_x = sqrt(ssx);
    const double rr = (ssx > 0.0) ? 1.0 / norm_x : 0.0;
    if (valid) {
#pragma unroll
      for (int c = 0; c < HD; c += 4)
        *reinterpret_cast<float4*>(&q.bk->tile[tk][HD * h + c]) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
      if (h == 0) {
        q.ns->rr[tk] = rr;
        q.bk->s1[tk] = norm_x / 11.313708498984761;
      }
    }
  }
  gr.sync();

  // ---- shift: o = mean_t n1_t = FWHT(r) * mean(rr) + mean_t(d_t rr_t) --------
  // mean(rr) is accumulated as deviations from rr_0 so that equal rr give it
  // exactly (identical tokens then give z = 0 exactly, as the definition does).
  // Column `col`, rows split in two halves, combined in a fixed order.
  {
    const double rr0 = q.ns->rr[0];
    const int lo = rhalf * (BLK / 2), hi = min(n, lo + BLK / 2);
    double dev = 0.0, sd0 = 0.0, sd1 = 0.0, sd2 = 0.0, sd3 = 0.0;
    int row = lo;
    for (; row + 3 < hi; row += 4) {
      const double ra = q.ns->rr[row], rb = q.ns->rr[row + 1], rc = q.ns->rr[row + 2], rd = q.ns->rr[row + 3];
      dev += ((ra - rr0) + (rb - rr0)) + ((rc - rr0) + (rd - rr0));
      sd0 = fma((double)q.bk->tile[row][col], ra, sd0);
      sd1 = fma((double)q.bk->tile[row + 1][col], rb, sd1);
      sd2 = fma((double)q.bk->tile[row + 2][col], rc, sd2);
      sd3 = fma((double)q.bk->tile[row + 3][col], rd, sd3);
    }
    for (; row < hi; ++row) {
      const double ra = q.ns->rr[row];
      dev += ra - rr0;
      sd0 = fma((double)q.bk->tile[row][col], ra, sd0);
    }
    q.ns->part[rhalf][col] = (sd0 + sd1) + (sd2 + sd3);
    if (col == 0) q.ns->dev_part[rhalf] = dev;
  }
  gr.sync();
  const double rr_mean = q.ns->rr[0] + (q.ns->dev_part[0] + q.ns->dev_part[1]) / n;
  if (t < D) {
    const double dc = (q.ns->part[0][t] + q.ns->part[1][t]) / n;  // D_c = mean_t(d_t,c rr_t)
    q.ns->big_rf[t] = (float)q.ns->big_r[t];
    q.ns->dcf[t] = (float)dc;
    const double o_t = fma(q.ns->big_r[t], rr_mean, dc);
    if (cv.dq) q.bk->ofull[t] = o_t;
    else cv.means[(seq * (cv.capacity / BLK) + blk) * D + t] = __double2half(o_t);
  }
  gr.sync();

  // ---- second normalization --------------------------------------------------
  // z_t = n1_t - o = d_t rr_t + FWHT(r) (rr_t - mean rr) - D.  The constant part
  // c = FWHT(r) (rr_t - mean rr) - D enters z rounded to fp32; it is formed by one
  // fp32 fma from fp32 copies of FWHT(r), D and rr_t - mean rr (three roundings of
  // the size of the one fp32 rounding of c), then one fp32 fma per channel.
  const double rr_t = valid ? q.ns->rr[tk] : 0.0;
  const float deltaf = (float)(rr_t - rr_mean);
  const float rrf = (float)rr_t;
  double zz0 = 0.0, zz1 = 0.0;
#pragma unroll
  for (int c = 0; c < HD; c += 4) {
    const int cg = HD * h + c;
    const float4 br = *reinterpret_cast<const float4*>(&q.ns->big_rf[cg]);
    const float4 dd = *reinterpret_cast<const float4*>(&q.ns->dcf[cg]);
    const float brv[4] = {br.x, br.y, br.z, br.w}, ddv[4] = {dd.x, dd.y, dd.z, dd.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float z = fmaf(v[c + i], rrf, fmaf(brv[i], deltaf, -ddv[i]));
      v[c + i] = z;
      if (i & 1) zz1 = fma((double)z, (double)z, zz1);
      else zz0 = fma((double)z, (double)z, zz0);
    }
  }
  const double zz = shfl_pair_sum(zz0 + zz1);
  if (valid && h == 0) q.bk->s2[tk] = sqrt(zz) / 11.313708498984761;
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
    if (h == 0 && valid) *reinterpret_cast<uint4*>(signs + (int64_t)tk * NSUB) = make_uint4(sgn[0], sgn[1], sgn[2], sgn[3]);
  }

  // ---- u rows (|u| in 2-bit mode) to shared memory; zeros past the n tokens --
  // The raw tile and the d_t rows are no longer read (the column sums are done).
#pragma unroll
  for (int c = 0; c < HD; c += 4)
    *reinterpret_cast<float4*>(&q.bk->tile[tk][HD * h + c]) =
        valid ? make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
  gr.sync();
}

// Exact fp64 re-decision of the flagged sub-vectors of q.bk (q.se->flag), one
// warp per sub-vector, by the warps of `gr`.
__device__ void exact_phase(const QRefs& q, const Grp& gr, const float* __restrict__ cb_global) {
  // ---- exact fp64 re-decision of the flagged sub-vectors, a warp each --------
  // Each lane scores its 8 codewords in sequential fp32 (bias first, one fma per
  // dim); candidates are the codewords within twice the fp32 bound of the best of
  // these scores; the winner by fp64 squared distance (cosine assignment: largest
  // fp64 inner product with c_hat), ties to the lowest index.
  {
    const int warp = gr.t >> 5, lane = gr.t & 31;
    const float cmax = q.tb->cnorm[0], cmax2 = q.tb->cnorm[1];
    constexpr float GAMMA9 = 9.0f * 5.9604645e-8f * 1.0001f;  // 9u/(1-9u), u = 2^-24
    const int tab = q.tb->tab;
    const int nflag = q.se->nflag;
#pragma unroll 1
    for (int f = warp; f < nflag; f += gr.n / 32) {
      const int ftk = q.se->flag[f] / NSUB, fj = q.se->flag[f] % NSUB;
      const float4 fa0 = *reinterpret_cast<const float4*>(&q.bk->tile[ftk][SUB * fj]);
      const float4 fa1 = *reinterpret_cast<const float4*>(&q.bk->tile[ftk][SUB * fj + 4]);
      const float a[8] = {fa0.x, fa0.y, fa0.z, fa0.w, fa1.x, fa1.y, fa1.z, fa1.w};
      float na = 0.f;
#pragma unroll
      for (int i = 0; i < SUB; ++i) na = fmaf(a[i], a[i], na);
      na = sqrtf(na) * 1.0001f;
      const float margin = 2.0f * GAMMA9 * (cmax2 + na * cmax) * 1.01f;
      float sc[NCODES / 32];
      float best = -INFINITY;
#pragma unroll
      for (int m = 0; m < NCODES / 32; ++m) {
        const int k = lane + 32 * m;
        float c[SUB];
        float x = codeword(q, k, (lane >> 2) & 1, c);
#pragma unroll
        for (int i = 0; i < SUB; ++i) x = fmaf(a[i], c[i], x);
        sc[m] = x;
        best = fmaxf(best, x);
      }
      const float thr = warp_max(best) - margin;
      double bestd = INFINITY;
      int bi = NCODES;
#pragma unroll
      for (int m = 0; m < NCODES / 32; ++m) {
        if (sc[m] >= thr) {
          const int k = lane + 32 * m;
          float c[SUB];
          codeword(q, k, (lane >> 2) & 1, c);
          double dd = 0.0;  // fp64 squared distance, or minus the fp64 inner product with c_hat
          if (tab == TAB_COSINE) {
#pragma unroll
            for (int i = 0; i < SUB; ++i) dd = fma(-(double)a[i], (double)c[i], dd);
          } else {
#pragma unroll
            for (int i = 0; i < SUB; ++i) {
              const double e = (double)a[i] - (double)c[i];
              dd = fma(e, e, dd);
            }
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
      if (lane == 0 && bi < NCODES) q.bk->code[ftk][fj] = (uint8_t)bi;
    }
  }
  gr.sync();
}

// Adaptive scale and stores of one block of n tokens (codes final in q.bk->code)
// by a set of 256 threads (two per token, as in nsn_phase).
__device__ void finish_phase(const QRefs& q, const Grp& gr, const float* __restrict__ cb_global,
                             uint8_t* __restrict__ codes, const CacheView& cv, int64_t seq, int64_t tok0, int blk,
                             int n, int scale_adjust) {
  const int t = gr.t, tk = t >> 1, h = t & 1;
  const bool valid = tk < n;
  // ---- adaptive scale: alpha = ||u||^2 / (u . u_hat) --------------------------
  double dot = 0.0, uu = 0.0;
  {
    const int tab = q.tb->tab;
#pragma unroll 4
    for (int jj = 0; jj < HSUB; ++jj) {
      const int j = HSUB * h + jj;
      float qv[SUB];
      codeword_given(q, cb_global, tab, q.bk->code[tk][j], (t >> 2) & 1, qv);
      const float4 u0 = *reinterpret_cast<const float4*>(&q.bk->tile[tk][SUB * j]);
      const float4 u1 = *reinterpret_cast<const float4*>(&q.bk->tile[tk][SUB * j + 4]);
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
  }
  // halves combined in a fixed order (low half first) so both lanes agree bit for bit
  const double dot_o = __shfl_xor_sync(0xffffffffu, dot, 1), uu_o = __shfl_xor_sync(0xffffffffu, uu, 1);
  dot = h ? dot_o + dot : dot + dot_o;
  uu = h ? uu_o + uu : uu + uu_o;
  double alpha = (dot > 0.0) ? uu / dot : 1.0;
  if (!scale_adjust) alpha = 1.0;

  // ---- packed stores ---------------------------------------------------------
  if (valid) {
    // stored order: the even sub-vectors' codes (h = 0), then the odd ones' (h = 1)
    const uint4 cw = *reinterpret_cast<const uint4*>(&q.bk->code[tk][0]);
    const uint32_t sel = h ? 0x7531u : 0x6420u;
    *reinterpret_cast<uint2*>(codes + (int64_t)tk * NSUB + HSUB * h) =
        make_uint2(__byte_perm(cw.x, cw.y, sel), __byte_perm(cw.z, cw.w, sel));
    if (h == 0) {
      const BlockOut bo = block_out(cv, seq, tok0, blk);
      if (bo.dq) bo.s2[tk] = __double2half(alpha * q.bk->s2[tk]);
      else bo.norms[tk] = __halves2half2(__double2half(q.bk->s1[tk]), __double2half(alpha * q.bk->s2[tk]));
    }
  }
  if (cv.dq) store_double_quant(q, gr, n, block_out(cv, seq, tok0, blk));
  gr.sync();  // shared memory is reused by the caller's next block
}

// Quantizes one block of n (1..128) tokens with the whole CTA of QTHREADS threads
// (NSN, codeword search, exact re-decision, adaptive scale and stores).  Output
// pointers are already offset to the block's first token (codes, signs).
template <int DT, int MODE>
__device__ void quantize_block_dev(QuantSmem& sm, TcState& tcs, const float* __restrict__ cb_global,
                                   const void* __restrict__ src, int64_t row0,
                                   int64_t row_stride, int n, uint8_t* __restrict__ codes,
                                   uint8_t* __restrict__ signs, const CacheView& cv, int64_t seq,
                                   int64_t tok0, int blk, int scale_adjust) {
  const QRefs q = refs(sm);
  const Grp gr = cta_grp();
  if (gr.t == 0) sm.se.nflag = 0;  // read only after the barriers below
  nsn_phase<DT, MODE>(q, gr, src, row0, row_stride, n, signs, cv, seq, blk);
  search_block(q, tcs, cb_global, n, cv.status);
  exact_phase(q, gr, cb_global);
  finish_phase(q, gr, cb_global, codes, cv, seq, tok0, blk, n, scale_adjust);
}

// ---------------------------------------------------------------------------
// Prefill: which tokens of each sequence are quantized.
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


// Row `row` of a tile's A operand, [a_hi | a_lo] (a_hi = fp16(a), a_lo = fp16(a -
// a_hi), so a_hi + a_lo = a to 2^-22), stored in the natural K order; a[0..3] holds
// dims 4h .. 4h + 3 and a[4..7] the other half.
__device__ __forceinline__ void store_a_row(unsigned char* ap, int row, const float (&a)[SUB], int h) {
  uint32_t hi[4], lo[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) split_half2(a[2 * p], a[2 * p + 1], hi[p], lo[p]);
  *reinterpret_cast<uint2*>(ap + kmaj_off(row, 4 * h)) = make_uint2(hi[0], hi[1]);
  *reinterpret_cast<uint2*>(ap + kmaj_off(row, 4 - 4 * h)) = make_uint2(hi[2], hi[3]);
  *reinterpret_cast<uint2*>(ap + kmaj_off(row, 8 + 4 * h)) = make_uint2(lo[0], lo[1]);
  *reinterpret_cast<uint2*>(ap + kmaj_off(row, 12 - 4 * h)) = make_uint2(lo[2], lo[3]);
}

// The two MMAs of one tile's 256 scores per row into the 256 tensor-memory columns
// at `dtmem`, then the commit to `mbar`; issued by one thread.
//   nearest codeword: D = bias + [a_hi | a_lo] [c | c]
//   cosine rule:      D = [a_hi | a_lo] [c_hat_hi | c_hat_hi] + [a_hi | a_lo] [c_hat_lo | c_hat_lo]
__device__ __forceinline__ void issue_scores(const QRefs& q, uint32_t dtmem, const unsigned char* ap, uint32_t mbar) {
  const uint64_t da = tc_desc(q_smem(ap), 128, 256);
  const uint64_t db = tc_desc(q_smem(q.tb->bop), 128, 256);
  const uint64_t da2 = tc_desc(q_smem(q.tb->aop2), 128, 0);  // every 8-row group reads the same [1, 1, 0...] rows
  const uint64_t db2 = tc_desc(q_smem(q.tb->bop2), 0, 128);  // K half 1 re-reads K half 0
  if (q.tb->tab == TAB_COSINE) {
    tc_mma(dtmem, da, db, 0u);
    tc_mma(dtmem, da, db2, 1u);
  } else {
    tc_mma(dtmem, da2, db2, 0u);
    tc_mma(dtmem, da, db, 1u);
  }
  tc_commit(mbar);
}

// ---------------------------------------------------------------------------
// Warp-specialized prefill: one persistent CTA per SM, 16 warps, two blocks in
// flight.  Warps 0-7 (the searchers) form two warpgroups; warpgroup g searches the
// tiles g, g + 2, ... of a block in its own 256-column tensor-memory buffer, so the
// two warpgroups' MMA waits and score reductions overlap.  A searcher thread owns
// one tile row (= tensor-memory lane): it builds the row's A operand, one thread
// per warpgroup issues the MMAs, then each thread reads its row's 256 scores,
// keeps the two best group maxima and the two best column maxima, and decides
// (codeword 8 G + J, certified by the tensor-score bound); after the block the 8
// warps re-decide the flagged sub-vectors.  Warps 8-15 (the normalizers) run the NSN of block j into
// one of two block buffers while the searchers work on block j - 1, and then the
// adaptive scale and stores of block j - 2.  Named barriers hand a block over:
// U (u rows ready, normalizers -> searchers) and D (codes final, searchers ->
// normalizers), one of each per buffer.
// ---------------------------------------------------------------------------
constexpr int WS_SWG = 2;                              // search warpgroups
constexpr int WS_SWARPS = 4 * WS_SWG, WS_NWARPS = 8;
constexpr int WS_THREADS = 32 * (WS_SWARPS + WS_NWARPS);
constexpr int WS_BAR_G = 1;                            // ids 1, 2: one warpgroup of searchers
constexpr int WS_BAR_S = 3, WS_BAR_N = 4;              // all searchers; all normalizers
constexpr int WS_BAR_U = 5, WS_BAR_D = 7;              // ids +0 / +1 by block buffer
constexpr uint32_t WS_TC_COLS = WS_SWG * TC_COLS;

struct QuantSmemWS {
  QTables tb;
  QSearch se;
  QNsn ns;
  QBlock bk[2];
};

__device__ __forceinline__ void bar_arrive(int id, int n) { asm volatile("bar.arrive %0, %1;" :: "r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(n) : "memory"); }

// Search of the tiles wg, wg + 2, ... of one block by search warpgroup wg (thread
// L = tile row = tensor-memory lane).  The tensor-score bound is tensor_bound().
__device__ void search_tiles_ws(const QRefs& q, TcState& tcs, const float* __restrict__ cb_global, int n, int wg,
                                int32_t* status) {
  const int L = threadIdx.x & 127, wq = L >> 5, lane = L & 31;
  const Grp g{WS_BAR_G + wg, 128, L};
  const float cmax = q.tb->cnorm[0], cmax2 = q.tb->cnorm[1], cdel = q.tb->cnorm[2];
  const uint32_t tbuf = tcs.tmem + (uint32_t)(TC_COLS * wg);
  const uint32_t taddr = tbuf + ((uint32_t)(32 * wq) << 16);
  unsigned char* ap = q.se->aop[wg];
  const uint32_t mb = q_smem(&q.se->mbar[wg]);
  const int ntiles = (n + 7) >> 3;
  // this lane reads its row's half hf first: the 8 lanes of a phase then hit 8
  // different bank groups
  const int hf = (lane >> 2) & 1;
  const int j = L & 15;

#pragma unroll 1
  for (int tile = wg; tile < ntiles; tile += WS_SWG) {
    const int tkk = 8 * tile + (L >> 4);
    // ---- the row's A operand (hi and lo halves) and its decision bound ----
    // a[0..3] = dims 4 hf .. 4 hf + 3, a[4..7] = the other half; the A operand
    // keeps the natural order.
    float a[SUB];
    {
      const float4 a0 = *reinterpret_cast<const float4*>(&q.bk->tile[tkk][SUB * j + 4 * hf]);
      const float4 a1 = *reinterpret_cast<const float4*>(&q.bk->tile[tkk][SUB * j + 4 - 4 * hf]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
      a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      store_a_row(ap, L, a, hf);
    }
    // A rows written (generic proxy -> tensor cores) and the previous tile's scores read
    fence_async_smem();
    tc_fence_before();
    g.sync();
    tc_fence_after();
    if (L == 0) issue_scores(q, tbuf, ap, mb);
    float na = 0.f;
#pragma unroll
    for (int d = 0; d < SUB; ++d) na = fmaf(a[d], a[d], na);
    na = sqrtf(na) * 1.0001f;
    const float mtc = tensor_bound(na, cmax, cmax2, cdel);
    if (!mbar_wait(mb, (tcs.phase >> wg) & 1u, MBAR_POLLS) && lane == 0 && status) atomicOr(status, 2);
    tcs.phase ^= 1u << wg;
    tc_fence_after();

    // ---- best and second-best of the 32 group maxima of the row's 256 scores ----
    // (two register buffers in turn: chunk c + 1 loads while chunk c is reduced)
    // and the maxima of the 8 columns (index within a group) over all groups
    float b1 = -INFINITY, b2 = -INFINITY;
    float cm[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) cm[jj] = -INFINITY;
    uint32_t rb[2][32];
    tc_ld32(taddr, rb[0]);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t (&r)[32] = rb[c & 1];
      tc_wait_ld();
      tc_regs_ready(r);
      if (c < 7) tc_ld32(taddr + 32 * (c + 1), rb[(c + 1) & 1]);
      float key[4];
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) {
        const float m = max3f(max3f(__uint_as_float(r[8 * gg]), __uint_as_float(r[8 * gg + 1]), __uint_as_float(r[8 * gg + 2])),
                              max3f(__uint_as_float(r[8 * gg + 3]), __uint_as_float(r[8 * gg + 4]), __uint_as_float(r[8 * gg + 5])),
                              fmaxf(__uint_as_float(r[8 * gg + 6]), __uint_as_float(r[8 * gg + 7])));
        key[gg] = __uint_as_float((__float_as_uint(m) & ~31u) | (uint32_t)(4 * c + gg));
      }
      const float h01 = fmaxf(key[0], key[1]), l01 = fminf(key[0], key[1]);
      const float h23 = fmaxf(key[2], key[3]), l23 = fminf(key[2], key[3]);
      const float hi = fmaxf(h01, h23);
      const float lo = max3f(l01, l23, fminf(h01, h23));
      b2 = max3f(b2, lo, fminf(b1, hi));
      b1 = fmaxf(b1, hi);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        cm[jj] = max3f(cm[jj], __uint_as_float(r[jj]), __uint_as_float(r[8 + jj]));
        cm[jj] = max3f(cm[jj], __uint_as_float(r[16 + jj]), __uint_as_float(r[24 + jj]));
      }
    }
    const int G = (int)(__float_as_uint(b1) & 31u);
    // best and second-best column maximum, the column number in the low 3 bits
    float c1 = -INFINITY, c2 = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const float key = __uint_as_float((__float_as_uint(cm[jj]) & ~7u) | (uint32_t)jj);
      c2 = fmaxf(c2, fminf(c1, key));
      c1 = fmaxf(c1, key);
    }
    const int J = (int)(__float_as_uint(c1) & 7u);

    // ---- the best tensor score lies in group G (best group maximum) and column J
    // (best column maximum), so it is codeword 8 G + J.  Every other score is below
    // the second-best group maximum or the second-best column maximum; if the best
    // beats both by more than twice the tensor bound (after the key bits: 32 ulp for
    // a group number, 8 ulp for a column number), the code is the exact nearest
    // codeword; otherwise the sub-vector is re-decided exactly. ----
    const int idx = 8 * G + J;
    const float top = b1 - fabsf(b1) * 3.82e-6f;
    const float rival = fmaxf(b2 + fabsf(b2) * 3.82e-6f, c2 + fabsf(c2) * 9.6e-7f);
    q.bk->code[tkk][j] = (uint8_t)idx;
    const bool need = rival >= top - 2.0f * mtc;
    if (need && tkk < n) q.se->flag[atomicAdd(&q.se->nflag, 1)] = (uint16_t)(tkk * NSUB + j);
  }
  tc_fence_before();
}

struct WsBlock {
  const void* src;
  int64_t row0, seq, tok0;
  int n, blk;
};

template <int DT, int MODE>
__global__ void __launch_bounds__(WS_THREADS, 1)
quantize_prefill_ws_kernel(const void* __restrict__ x, int64_t sb, int64_t st, int64_t sh, int q_tokens,
                           int n_tokens, const int32_t* __restrict__ lengths, CacheView cv,
                           const float* __restrict__ codebook, int nblk) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  QuantSmemWS& sm = *reinterpret_cast<QuantSmemWS*>(smem_raw);
  TcState tcs = tc_setup(sm.se, WS_TC_COLS, WS_SWG);
  stage_codebook(QRefs{&sm.tb, &sm.se, &sm.ns, &sm.bk[0]}, codebook, cv.assign);
  const int nwork = nblk * cv.n_kv_heads * cv.batch;
  auto block_at = [&](int w) {
    WsBlock bl;
    const int blk = w % nblk, h = (w / nblk) % cv.n_kv_heads, b = w / (nblk * cv.n_kv_heads);
    const PrefillSplit ps = prefill_split(lengths, b, n_tokens, q_tokens, cv.window_len);
    bl.n = min(BLK, ps.q - blk * BLK);
    bl.blk = blk;
    bl.seq = (int64_t)b * cv.n_kv_heads + h;
    bl.tok0 = bl.seq * cv.capacity + (int64_t)blk * BLK;
    bl.row0 = (int64_t)b * sb + (int64_t)blk * BLK * st + (int64_t)h * sh;
    bl.src = x;
    return bl;
  };
  const int warp = threadIdx.x >> 5;
  if (warp < WS_SWARPS) {
    // ---- searchers ----
    const Grp sg{WS_BAR_S, 32 * WS_SWARPS, (int)threadIdx.x};
    const int wg = warp >> 2;
    int j = 0;
#pragma unroll 1
    for (int w = blockIdx.x; w < nwork; w += gridDim.x) {
      const WsBlock bl = block_at(w);
      if (bl.n <= 0) continue;
      const QRefs q{&sm.tb, &sm.se, &sm.ns, &sm.bk[j & 1]};
      bar_sync(WS_BAR_U + (j & 1), WS_THREADS);
      if (sg.t == 0) sm.se.nflag = 0;
      sg.sync();
      search_tiles_ws(q, tcs, codebook, bl.n, wg, cv.status);
      sg.sync();  // every code and flag of the block written
      exact_phase(q, sg, codebook);
      bar_arrive(WS_BAR_D + (j & 1), WS_THREADS);
      ++j;
    }
  } else {
    // ---- normalizers ----
    const Grp ng{WS_BAR_N, 32 * WS_NWARPS, (int)threadIdx.x - 32 * WS_SWARPS};
    WsBlock hist[2];
    int j = 0;
    auto finish = [&](int jj, const WsBlock& bl) {
      bar_sync(WS_BAR_D + (jj & 1), WS_THREADS);
      const QRefs q{&sm.tb, &sm.se, &sm.ns, &sm.bk[jj & 1]};
      finish_phase(q, ng, codebook, cv.codes + bl.tok0 * NSUB, cv, bl.seq, bl.tok0, bl.blk, bl.n, cv.scale_adjust);
    };
#pragma unroll 1
    for (int w = blockIdx.x; w < nwork; w += gridDim.x) {
      const WsBlock bl = block_at(w);
      if (bl.n <= 0) continue;
      if (j >= 2) finish(j - 2, hist[j & 1]);
      const QRefs q{&sm.tb, &sm.se, &sm.ns, &sm.bk[j & 1]};
      nsn_phase<DT, MODE>(q, ng, bl.src, bl.row0, st, bl.n,
                          MODE == NSN_MODE_2BIT ? cv.signs + bl.tok0 * NSUB : nullptr, cv, bl.seq, bl.blk);
      bar_arrive(WS_BAR_U + (j & 1), WS_THREADS);
      hist[j & 1] = bl;
      ++j;
    }
    for (int jj = max(0, j - 2); jj < j; ++jj) finish(jj, hist[jj & 1]);
  }
  tc_teardown(tcs);
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
  extern __shared__ __align__(1024) unsigned char smem_raw[];
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
      const float* cb = is_v ? cbv : cbk;
      TcState tcs = tc_setup(sm.se, TC_COLS, 1);
      stage_codebook(refs(sm), cb, c.assign);
      const int64_t tok0 = seq * c.capacity + nq;
      const int blk = nq / BLK;
      uint8_t* sg = c.mode == NSN_MODE_2BIT ? c.signs + tok0 * NSUB : nullptr;
      if (c.mode == NSN_MODE_2BIT)
        quantize_block_dev<NSN_DTYPE_F16, NSN_MODE_2BIT>(sm, tcs, cb, c.window, seq * c.window_len * D, D, BLK,
                                                         c.codes + tok0 * NSUB, sg, c, seq, tok0, blk, c.scale_adjust);
      else
        quantize_block_dev<NSN_DTYPE_F16, NSN_MODE_1BIT>(sm, tcs, cb, c.window, seq * c.window_len * D, D, BLK,
                                                         c.codes + tok0 * NSUB, sg, c, seq, tok0, blk, c.scale_adjust);
      tc_teardown(tcs);
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
  const size_t smem = sizeof(QuantSmemWS);
  cudaError_t e = cudaFuncSetAttribute(quantize_prefill_ws_kernel<DT, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nblk = (q_tokens + BLK - 1) / BLK;
  if (nblk > 0) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long nwork = (long long)nblk * cv.n_kv_heads * cv.batch;
    const int grid = (int)std::min<long long>(nwork, (long long)sms);  // one persistent CTA per SM
    quantize_prefill_ws_kernel<DT, MODE><<<grid, WS_THREADS, smem, s>>>(x, sb, st, sh, q_tokens, n_tokens, lengths,
                                                                        cv, cb, nblk);
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

// ---------------------------------------------------------------------------
// Diagnostic: the tensor-core scores of up to 128 fp32 rows against a codebook,
// formed exactly as the prefill search forms them (codebook staging, A operand
// rows, the two MMAs into tensor memory) and read back raw, so that their error
// against exact arithmetic can be measured.  One CTA of 128 threads, thread =
// row = tensor-memory lane; rows past n are zero and not written back.
// ---------------------------------------------------------------------------
struct TsSmem {
  QTables tb;
  QSearch se;
};

__global__ void __launch_bounds__(BLK, 1)
tensor_scores_selftest_kernel(const float* __restrict__ rows, int n, const float* __restrict__ codebook, int cosine,
                              float* __restrict__ scores, int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TsSmem& sm = *reinterpret_cast<TsSmem*>(smem_raw);
  TcState tcs = tc_setup(sm.se, TC_COLS, 1);
  const QRefs q{&sm.tb, &sm.se, nullptr, nullptr};
  stage_codebook(q, codebook, cosine);
  const int L = threadIdx.x, lane = L & 31;
  float a[SUB];
#pragma unroll
  for (int d = 0; d < SUB; ++d) a[d] = L < n ? rows[(int64_t)L * SUB + d] : 0.f;
  store_a_row(sm.se.aop[0], L, a, 0);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (L == 0) issue_scores(q, tcs.tmem, sm.se.aop[0], q_smem(&sm.se.mbar[0]));
  if (!mbar_wait(q_smem(&sm.se.mbar[0]), 0u, MBAR_POLLS) && lane == 0 && status) atomicOr(status, 2);
  tc_fence_after();
  const uint32_t taddr = tcs.tmem + ((uint32_t)(32 * (L >> 5)) << 16);
#pragma unroll 1
  for (int c = 0; c < NCODES / 32; ++c) {
    uint32_t r[32];
    tc_ld32(taddr + 32 * c, r);
    tc_wait_ld();
    tc_regs_ready(r);
    if (L < n) {
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(scores + (int64_t)L * NCODES + 32 * c + i) =
            make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                        __uint_as_float(r[i + 3]));
    }
  }
  tc_teardown(tcs);
}

cudaError_t launch_tensor_scores_selftest(const float* rows, int n, const float* codebook, int cosine, float* scores,
                                          int32_t* status, cudaStream_t s) {
  const size_t smem = sizeof(TsSmem);
  cudaError_t e = cudaFuncSetAttribute(tensor_scores_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  tensor_scores_selftest_kernel<<<1, BLK, smem, s>>>(rows, n, codebook, cosine, scores, status);
  return cudaGetLastError();
}

}  // namespace nsn
