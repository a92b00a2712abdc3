// Device helpers shared by the NSNQuant kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nsn.h"

namespace nsn {

constexpr int D = NSN_HEAD_DIM;     // 128
constexpr int SUB = NSN_SUB_DIM;    // 8
constexpr int NSUB = NSN_N_SUB;     // 16
constexpr int NCODES = NSN_N_CODES; // 256
constexpr int BLK = NSN_BLOCK;      // 128 tokens per NSN block

// Sentinel used instead of -inf for "no score yet" so that differences of two
// sentinels stay finite (exp2 of them is 0, never NaN).
constexpr float NEG_BIG = -1.0e30f;

// ---------------------------------------------------------------------------
// Loads of 8 consecutive elements (16 B for 16-bit types, 32 B for fp32) as fp32.
// ---------------------------------------------------------------------------
template <int DT>
__device__ __forceinline__ void load8(const void* base, int64_t elem_off, float* out);

template <>
__device__ __forceinline__ void load8<NSN_DTYPE_F32>(const void* base, int64_t elem_off, float* out) {
  const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem_off);
  float4 a = __ldg(p), b = __ldg(p + 1);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

template <>
__device__ __forceinline__ void load8<NSN_DTYPE_BF16>(const void* base, int64_t elem_off, float* out) {
  uint4 r = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem_off));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}

template <>
__device__ __forceinline__ void load8<NSN_DTYPE_F16>(const void* base, int64_t elem_off, float* out) {
  uint4 r = __ldg(reinterpret_cast<const uint4*>(static_cast<const __half*>(base) + elem_off));
  const __half2* h = reinterpret_cast<const __half2*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}

// y minus an fp16 value h, in fp32, by one mixed-precision fma ((-1) * h + y with
// an fp16 multiplicand, sm_100).  When h = fp16(y) the difference is exact: it is
// a multiple of the fp32 ulp of y and below 2^-11 |y|.
__device__ __forceinline__ float sub_f16(float y, uint16_t h) {
  float d;
  asm("{\n\t.reg .b16 m1;\n\tmov.b16 m1, 0xBC00;\n\tfma.rn.f32.f16 %0, %1, m1, %2;\n\t}" : "=f"(d) : "h"(h), "f"(y));
  return d;
}

// fp16 high and low parts of two fp32 values, each packed as a half2 (first value
// in the low half): hi = fp16(y), lo = fp16(y - hi), so hi + lo = y to 2^-22.
__device__ __forceinline__ void split_half2(float y0, float y1, uint32_t& hi, uint32_t& lo) {
  const __half2 hh = __floats2half2_rn(y0, y1);
  hi = *reinterpret_cast<const uint32_t*>(&hh);
  const __half2 ll = __floats2half2_rn(sub_f16(y0, (uint16_t)(hi & 0xFFFFu)), sub_f16(y1, (uint16_t)(hi >> 16)));
  lo = *reinterpret_cast<const uint32_t*>(&ll);
}

// Converts 8 values to fp16 (round to nearest even) packed in 16 bytes.
__device__ __forceinline__ uint4 pack8_f16(const float* v) {
  uint4 r;
  __half2* h = reinterpret_cast<__half2*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
  return r;
}

// ---------------------------------------------------------------------------
// Unnormalized Walsh-Hadamard transform, w_i = sum_j (-1)^popcount(i & j) v_j
// (Sylvester / natural order), of 128 values held by a pair of adjacent lanes:
// lane 2k + h holds elements 64h .. 64h+63 in v[0..63].  Six butterfly stages in
// registers (compile-time strides, so the array stays in registers), then the
// stride-64 stage across the pair with one shuffle per element.
// ---------------------------------------------------------------------------
template <int H>
__device__ __forceinline__ void fwht64_stage(float* v) {
#pragma unroll
  for (int i = 0; i < D / 2; i += 2 * H) {
#pragma unroll
    for (int j = 0; j < H; ++j) {
      const float a = v[i + j], b = v[i + j + H];
      v[i + j] = a + b;
      v[i + j + H] = a - b;
    }
  }
}

__device__ __forceinline__ void fwht128_pair(float* v, int h) {
  fwht64_stage<1>(v);
  fwht64_stage<2>(v);
  fwht64_stage<4>(v);
  fwht64_stage<8>(v);
  fwht64_stage<16>(v);
  fwht64_stage<32>(v);
#pragma unroll
  for (int i = 0; i < D / 2; ++i) {
    const float o = __shfl_xor_sync(0xffffffffu, v[i], 1);
    v[i] = h ? (o - v[i]) : (v[i] + o);  // (a + b, a - b) with a in the low half
  }
}

// Unnormalized WHT of 128 values spread over a warp, lane l holding elements
// 4l..4l+3 in v[0..3].  Stages 1, 2 in registers, stages 4..64 by shuffles.
__device__ __forceinline__ void fwht128_warp(float* v, int lane) {
  {
    float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    v[0] = a0 + a2; v[2] = a0 - a2; v[1] = a1 + a3; v[3] = a1 - a3;
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float other = __shfl_xor_sync(0xffffffffu, v[r], m);
      v[r] = upper ? (other - v[r]) : (v[r] + other);
    }
  }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

}  // namespace nsn
