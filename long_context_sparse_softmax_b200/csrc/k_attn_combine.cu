// Merge of the key splits of a split decode attention (k_attn_tc / k_attn_tc8 with more
// than one key split per query): split s left, for each (query, head) row, its partial
// output o_s = sum_k e^(l_k - m_s) v_k (576 FP32 dims) and (m_s, l_s = sum_k e^(l_k - m_s)),
// exponents in log2 units.  With the sink logit in the same units,
//   M = max(sink, max_s m_s),  Z = e^(sink - M) + sum_s l_s e^(m_s - M),
//   o = sum_s o_s e^(m_s - M) / Z,  lse = (M + log2 Z) ln 2,
// the same softmax over every key of the row as one unsplit pass ("解读 DeepSeek V4",
// 其他架构细节: the sink lets a head give weight to nothing).  The splits are added in
// split order, so the result is deterministic.
#include "lc_internal.h"

namespace lc {

namespace {

constexpr int kAD = 576;             // dims of the split partial rows
constexpr int kCombineThreads = 256;
constexpr int kQuads = kAD / 4;      // float4 groups per row

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  return static_cast<uint32_t>(f32_to_bf16_bits(lo)) | (static_cast<uint32_t>(f32_to_bf16_bits(hi)) << 16);
}

}  // namespace

// S > 0: exactly S splits, every load issued before any arithmetic (one memory round trip);
// S = 0: any split count, one split after another.  Both add the splits in split order.
template <int S>
__global__ void __launch_bounds__(kCombineThreads) k_attn_combine(lc_attn_args a, int n_split,
                                                                  const float* __restrict__ ws_o,
                                                                  const float* __restrict__ ws_ml) {
  const int64_t rows = static_cast<int64_t>(a.n_q) * a.dims.H;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x;
  const int Dv = a.v_nope ? kAD - a.dims.d_r : kAD;  // output dims (the partial rows keep all kAD)
  const int nq = Dv / 4;
  if (t >= rows * nq) return;
  const int64_t row = t / nq;
  const int c4 = static_cast<int>(t % nq);
  const int h = static_cast<int>(row % a.dims.H);
  const float sk = __ldg(a.sink + h) * 1.4426950408889634f;
  const float2* ml = reinterpret_cast<const float2*>(ws_ml) + row * n_split;
  const float4* src = reinterpret_cast<const float4*>(ws_o) + row * kQuads + c4;
  const int64_t split_stride = rows * kQuads;
  float M = sk, Z;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  if constexpr (S > 0) {
    float2 mc[S];
    float4 v[S];
#pragma unroll
    for (int c = 0; c < S; ++c) {
      mc[c] = __ldg(ml + c);
      v[c] = __ldg(src + c * split_stride);
    }
#pragma unroll
    for (int c = 0; c < S; ++c) M = fmaxf(M, mc[c].x);
    Z = exp2f(sk - M);
#pragma unroll
    for (int c = 0; c < S; ++c) {
      const float w = mc[c].x == -INFINITY ? 0.f : exp2f(mc[c].x - M);
      Z = fmaf(mc[c].y, w, Z);
      o.x = fmaf(v[c].x, w, o.x);
      o.y = fmaf(v[c].y, w, o.y);
      o.z = fmaf(v[c].z, w, o.z);
      o.w = fmaf(v[c].w, w, o.w);
    }
  } else {
    for (int c = 0; c < n_split; ++c) M = fmaxf(M, __ldg(ml + c).x);
    Z = exp2f(sk - M);
#pragma unroll 4
    for (int c = 0; c < n_split; ++c) {
      const float2 mc = __ldg(ml + c);
      const float4 v = __ldg(src + c * split_stride);
      const float w = mc.x == -INFINITY ? 0.f : exp2f(mc.x - M);
      Z = fmaf(mc.y, w, Z);
      o.x = fmaf(v.x, w, o.x);
      o.y = fmaf(v.y, w, o.y);
      o.z = fmaf(v.z, w, o.z);
      o.w = fmaf(v.w, w, o.w);
    }
  }
  const float inv = 1.f / Z;
  if (a.out_fmt == LC_FMT_BF16) {
    uint2 pk;
    pk.x = pack_bf16(o.x * inv, o.y * inv);
    pk.y = pack_bf16(o.z * inv, o.w * inv);
    reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + row * Dv)[c4] = pk;
  } else {
    reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * Dv)[c4] =
        make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
  }
  if (a.lse && c4 == 0) a.lse[row] = (M + log2f(Z)) * 0.6931471805599453f;
}

static unsigned combine_blocks(const lc_attn_args& a) {
  const int64_t n = static_cast<int64_t>(a.n_q) * a.dims.H * kQuads;
  return static_cast<unsigned>((n + kCombineThreads - 1) / kCombineThreads);
}

static void combine_launch(const lc_attn_args& a, int n_split, const float* ws_o, const float* ws_ml,
                           cudaStream_t st) {
  const unsigned g = combine_blocks(a);
  switch (n_split) {
    case 2: k_attn_combine<2><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 3: k_attn_combine<3><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 4: k_attn_combine<4><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 5: k_attn_combine<5><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 6: k_attn_combine<6><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 7: k_attn_combine<7><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 8: k_attn_combine<8><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    default: k_attn_combine<0><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
  }
}

cudaError_t launch_attn_combine(const lc_attn_args& a, int n_split, cudaStream_t st) {
  float* ws_o = static_cast<float*>(a.workspace);
  float* ws_ml = ws_o + static_cast<size_t>(a.n_q) * a.dims.H * n_split * kAD;
  combine_launch(a, n_split, ws_o, ws_ml, st);
  return cudaGetLastError();
}

}  // namespace lc
