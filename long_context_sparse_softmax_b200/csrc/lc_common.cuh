// Device helpers shared by the kernels of the CSA / HCA attention library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lc.h"

namespace lc {

constexpr int kWarp = 32;

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Two floats -> two E4M3 bytes (round to nearest even, saturating at +-448), packed
// little-endian: a in the low byte.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float a, float b) {
  return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t v) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v), __NV_E4M3);
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ void set_status(int32_t* status, int32_t bit) {
  if (status) atomicOr(status, bit);
}

// RoPE frequencies base^(-2i/d_r), i < d_r / 2, computed once per call on the host in
// double precision and passed by value to the kernels.
constexpr int kMaxRopePairs = 64;
struct RopeTable {
  double inv_freq[kMaxRopePairs];
};

// cos / sin of pos * inv_freq.  The angle reaches ~1e6 rad at a 1M-token position, so it
// is formed and reduced to [-pi, pi] in double precision (two-constant additive
// reduction, Cody & Waite 1980) before the single-precision sincosf.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float* c, float* s) {
  const double ang = static_cast<double>(pos) * inv_freq;
  const double kTwoPiHi = 6.283185307179586232;        // nearest double to 2*pi
  const double kTwoPiLo = 2.449293598294706e-16;       // 2*pi - kTwoPiHi
  const double k = rint(ang * 0.15915494309189535);    // ang / (2*pi), nearest integer
  double r = fma(-k, kTwoPiHi, ang);
  r = fma(-k, kTwoPiLo, r);
  sincosf(static_cast<float>(r), s, c);
}

// A group of 8 consecutive dims of a row, held in registers.
struct Vec8 {
  float v[8];
};

// Load 8 dims [d, d+8) of an FP32 or BF16 row (16-byte aligned).
template <bool kF32>
__device__ __forceinline__ Vec8 load8(const void* row, int d) {
  Vec8 r;
  if (kF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(row) + d);
    float4 a = __ldg(p), b = __ldg(p + 1);
    r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
    r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
  } else {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(row) + d));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      r.v[2 * j] = __uint_as_float(w[j] << 16);
      r.v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
  return r;
}

// Streaming (evict-first) variant for data read exactly once.
template <bool kF32>
__device__ __forceinline__ Vec8 load8_stream(const void* row, int d) {
  Vec8 r;
  if (kF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(row) + d);
    float4 a = __ldcs(p), b = __ldcs(p + 1);
    r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
    r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
  } else {
    uint4 u = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(row) + d));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      r.v[2 * j] = __uint_as_float(w[j] << 16);
      r.v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
  return r;
}

// Store 8 dims [d, d+8) of row `r` of `out` in its format.  In LC_FMT_E4M3_BF16 the
// dims below D - d_r go to the E4M3 part, the rest to the BF16 RoPE part.
__device__ __forceinline__ void store8(const lc_rows& out, int64_t r, int D, int d_r, int d, const Vec8& v) {
  if (out.fmt == LC_FMT_F32) {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(out.x) + r * D + d);
    p[0] = make_float4(v.v[0], v.v[1], v.v[2], v.v[3]);
    p[1] = make_float4(v.v[4], v.v[5], v.v[6], v.v[7]);
    return;
  }
  const int d_n = D - d_r;
  if (out.fmt == LC_FMT_BF16 || d >= d_n) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = static_cast<uint32_t>(f32_to_bf16_bits(v.v[2 * j])) |
             (static_cast<uint32_t>(f32_to_bf16_bits(v.v[2 * j + 1])) << 16);
    uint16_t* base = (out.fmt == LC_FMT_BF16) ? static_cast<uint16_t*>(out.x) + r * D + d
                                               : static_cast<uint16_t*>(out.rope) + r * d_r + (d - d_n);
    *reinterpret_cast<uint4*>(base) = make_uint4(w[0], w[1], w[2], w[3]);
    return;
  }
  uint32_t lo = static_cast<uint32_t>(f32x2_to_e4m3x2(v.v[0], v.v[1])) |
                (static_cast<uint32_t>(f32x2_to_e4m3x2(v.v[2], v.v[3])) << 16);
  uint32_t hi = static_cast<uint32_t>(f32x2_to_e4m3x2(v.v[4], v.v[5])) |
                (static_cast<uint32_t>(f32x2_to_e4m3x2(v.v[6], v.v[7])) << 16);
  *reinterpret_cast<uint2*>(static_cast<uint8_t*>(out.x) + r * d_n + d) = make_uint2(lo, hi);
}

// Load 8 logical dims [d, d+8) of row r of a row set in any format, as floats.
__device__ __forceinline__ Vec8 load8_rows(const lc_rows& in, int64_t r, int D, int d_r, int d) {
  if (in.fmt == LC_FMT_F32) return load8<true>(static_cast<const float*>(in.x) + r * D, d);
  if (in.fmt == LC_FMT_BF16) return load8<false>(static_cast<const uint16_t*>(in.x) + r * D, d);
  const int d_n = D - d_r;
  if (d >= d_n) return load8<false>(static_cast<const uint16_t*>(in.rope) + r * d_r, d - d_n);
  uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(in.x) + r * d_n + d));
  Vec8 v;
  const uint32_t w[2] = {u.x, u.y};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float2 a = e4m3x2_to_f32x2(static_cast<uint16_t>(w[j] & 0xffffu));
    float2 b = e4m3x2_to_f32x2(static_cast<uint16_t>(w[j] >> 16));
    v.v[4 * j + 0] = a.x; v.v[4 * j + 1] = a.y; v.v[4 * j + 2] = b.x; v.v[4 * j + 3] = b.y;
  }
  return v;
}

}  // namespace lc
