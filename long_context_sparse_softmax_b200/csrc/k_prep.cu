// Query / window-row preparation and KV compression kernels.
//
// qk_prep: RMSNorm (unit weight) over the D dims of a row, RoPE on its RoPE dims at the
//   token's position, cast to the output format (10100.com analysis §三.1, "辅助优化":
//   RMSNorm on queries and KV entries, partial RoPE).
// compress: each complete block of m tokens becomes one entry: block-softmax gate
//   weights over the m tokens, weighted sum of the raw rows, RMSNorm, RoPE at the
//   block's last position, cast ("解读 DeepSeek V4", CSA m = 4 / HCA m' = 128 sections;
//   "DeepSeek-V4 论文分析" §5.2: learned per-token weights rather than an average).
//
// All of them stream HBM: 16-byte vector loads of 8 dims per lane, one warp per row
// (qk_prep), per entry (CSA compress) or one CTA per entry (HCA compress, 128 tokens).
#include <cmath>

#include "lc_internal.h"

namespace lc {

constexpr int kMaxGroupsPerLane = 4;  // D <= 1024: 128 groups of 8 dims over 32 lanes

// RMSNorm + RoPE + store of one row held by a warp as groups of 8 dims.
__device__ __forceinline__ void norm_rope_store(Vec8 (&v)[kMaxGroupsPerLane], int lane, int D, int d_r,
                                                int rope_off, float eps, int pos, const RopeTable& rt,
                                                const lc_rows& out, int64_t out_row) {
  const int G = D >> 3;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxGroupsPerLane; ++i) {
    const int g = lane + kWarp * i;
    if (g < G) {
#pragma unroll
      for (int j = 0; j < 8; ++j) ss = fmaf(v[i].v[j], v[i].v[j], ss);
    }
  }
  ss = warp_sum(ss);
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(D) + eps);
#pragma unroll
  for (int i = 0; i < kMaxGroupsPerLane; ++i) {
    const int g = lane + kWarp * i;
    if (g >= G) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) v[i].v[j] *= inv;
    const int d = g << 3;
    if (d >= rope_off && d < rope_off + d_r) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float c, s;
        rope_cos_sin(pos, rt.inv_freq[((d - rope_off) >> 1) + j], &c, &s);
        const float a = v[i].v[2 * j], b = v[i].v[2 * j + 1];
        v[i].v[2 * j] = a * c - b * s;
        v[i].v[2 * j + 1] = a * s + b * c;
      }
    }
    store8(out, out_row, D, d_r, d, v[i]);
  }
}

template <bool kF32In>
__global__ void __launch_bounds__(256) k_qk_prep(const void* __restrict__ x, const int32_t* __restrict__ pos,
                                                 const int64_t* __restrict__ out_tok, lc_rows out,
                                                 int64_t n_rows, int H, int D, int d_r, int rope_off,
                                                 float eps, RopeTable rt) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const int G = D >> 3;
  const size_t esz = kF32In ? 4 : 2;
  const void* rp = static_cast<const char*>(x) + static_cast<size_t>(row) * D * esz;
  Vec8 v[kMaxGroupsPerLane];
#pragma unroll
  for (int i = 0; i < kMaxGroupsPerLane; ++i) {
    const int g = lane + kWarp * i;
    if (g < G) v[i] = load8_stream<kF32In>(rp, g << 3);
  }
  const int64_t tok = row / H;
  const int p = __ldg(pos + tok);
  const int64_t orow = out_tok ? __ldg(out_tok + tok) * H + (row - tok * H) : row;
  norm_rope_store(v, lane, D, d_r, rope_off, eps, p, rt, out, orow);
}

// One warp per entry (CSA, m <= 64).
template <bool kF32In>
__global__ void __launch_bounds__(256) k_compress_warp(lc_compress_args a, RopeTable rt) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= __ldg(a.blk_count + b)) return;
  const int m = a.m, D = a.dims.D;
  const int j = __ldg(a.blk_first + b) + i;
  const int pos0 = __ldg(a.tok_pos0 + b);
  const int first = j * m;
  if (first < pos0 || first + m > pos0 + __ldg(a.tok_len + b)) {
    if (lane == 0) set_status(a.status, LC_DEV_BAD_BLOCK);
    return;
  }
  const int64_t row0 = __ldg(a.tok_row0 + b) + (first - pos0);
  // gate softmax over the block: lanes hold tokens lane and lane + 32
  float g0 = lane < m ? __ldg(a.g + row0 + lane) : -INFINITY;
  float g1 = lane + 32 < m ? __ldg(a.g + row0 + lane + 32) : -INFINITY;
  const float gmax = warp_max(fmaxf(g0, g1));
  float e0 = lane < m ? expf(g0 - gmax) : 0.f;
  float e1 = lane + 32 < m ? expf(g1 - gmax) : 0.f;
  const float esum = warp_sum(e0 + e1);
  e0 /= esum;
  e1 /= esum;
  const int G = D >> 3;
  const size_t esz = kF32In ? 4 : 2;
  Vec8 acc[kMaxGroupsPerLane];
#pragma unroll
  for (int q = 0; q < kMaxGroupsPerLane; ++q)
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[q].v[t] = 0.f;
  for (int t = 0; t < m; ++t) {
    const float al = __shfl_sync(0xffffffffu, t < 32 ? e0 : e1, t & 31);
    const void* rp = static_cast<const char*>(a.x) + static_cast<size_t>(row0 + t) * D * esz;
#pragma unroll
    for (int q = 0; q < kMaxGroupsPerLane; ++q) {
      const int g = lane + kWarp * q;
      if (g < G) {
        Vec8 v = load8_stream<kF32In>(rp, g << 3);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[q].v[u] = fmaf(al, v.v[u], acc[q].v[u]);
      }
    }
  }
  norm_rope_store(acc, lane, D, a.dims.d_r, a.dims.rope_off, a.eps, (j + 1) * m - 1, rt, a.out,
                  __ldg(a.ent_start + b) + j);
}

// One CTA (8 warps) per entry (HCA, m >= 64): warp w sums tokens w, w + 8, ...; the
// partial sums meet in shared memory and are added in a fixed order.
template <bool kF32In>
__global__ void __launch_bounds__(256) k_compress_cta(lc_compress_args a, RopeTable rt) {
  extern __shared__ float smem[];  // [8][D] partial sums, then [m] gate weights
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.y;
  const int i = blockIdx.x;
  if (i >= __ldg(a.blk_count + b)) return;
  const int m = a.m, D = a.dims.D;
  const int j = __ldg(a.blk_first + b) + i;
  const int pos0 = __ldg(a.tok_pos0 + b);
  const int first = j * m;
  if (first < pos0 || first + m > pos0 + __ldg(a.tok_len + b)) {
    if (threadIdx.x == 0) set_status(a.status, LC_DEV_BAD_BLOCK);
    return;
  }
  const int64_t row0 = __ldg(a.tok_row0 + b) + (first - pos0);
  float* part = smem;
  float* alpha = smem + 8 * D;
  __shared__ float red[8];
  // gate softmax over the m tokens
  float gm = -INFINITY;
  for (int t = threadIdx.x; t < m; t += blockDim.x) gm = fmaxf(gm, __ldg(a.g + row0 + t));
  gm = warp_max(gm);
  if (lane == 0) red[warp] = gm;
  __syncthreads();
  gm = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) gm = fmaxf(gm, red[w]);
  __syncthreads();
  float es = 0.f;
  for (int t = threadIdx.x; t < m; t += blockDim.x) {
    const float e = expf(__ldg(a.g + row0 + t) - gm);
    alpha[t] = e;
    es += e;
  }
  es = warp_sum(es);
  if (lane == 0) red[warp] = es;
  __syncthreads();
  es = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) es += red[w];
  const float inv_es = 1.0f / es;
  const int G = D >> 3;
  const size_t esz = kF32In ? 4 : 2;
  Vec8 acc[kMaxGroupsPerLane];
#pragma unroll
  for (int q = 0; q < kMaxGroupsPerLane; ++q)
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[q].v[u] = 0.f;
#pragma unroll 4
  for (int t = warp; t < m; t += 8) {
    const float al = alpha[t] * inv_es;
    const void* rp = static_cast<const char*>(a.x) + static_cast<size_t>(row0 + t) * D * esz;
#pragma unroll
    for (int q = 0; q < kMaxGroupsPerLane; ++q) {
      const int g = lane + kWarp * q;
      if (g < G) {
        Vec8 v = load8_stream<kF32In>(rp, g << 3);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[q].v[u] = fmaf(al, v.v[u], acc[q].v[u]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kMaxGroupsPerLane; ++q) {
    const int g = lane + kWarp * q;
    if (g < G)
#pragma unroll
      for (int u = 0; u < 8; ++u) part[warp * D + (g << 3) + u] = acc[q].v[u];
  }
  __syncthreads();
  if (warp != 0) return;
#pragma unroll
  for (int q = 0; q < kMaxGroupsPerLane; ++q) {
    const int g = lane + kWarp * q;
    if (g < G) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float s = part[(g << 3) + u];
#pragma unroll
        for (int w = 1; w < 8; ++w) s += part[w * D + (g << 3) + u];
        acc[q].v[u] = s;
      }
    }
  }
  norm_rope_store(acc, lane, D, a.dims.d_r, a.dims.rope_off, a.eps, (j + 1) * m - 1, rt, a.out,
                  __ldg(a.ent_start + b) + j);
}

RopeTable make_rope_table(int d_r, float base) {
  RopeTable t{};
  for (int i = 0; i < d_r / 2 && i < kMaxRopePairs; ++i)
    t.inv_freq[i] = std::pow(static_cast<double>(base), -2.0 * i / static_cast<double>(d_r));
  return t;
}

cudaError_t launch_qk_prep(const lc_qk_prep_args& a, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(a.n_tok) * a.dims.H;
  if (rows == 0) return cudaSuccess;
  const RopeTable rt = make_rope_table(a.dims.d_r, a.rope_base);
  const int wpb = 8;
  const dim3 grid(static_cast<unsigned>((rows + wpb - 1) / wpb));
  if (a.in_fmt == LC_FMT_F32)
    k_qk_prep<true><<<grid, 32 * wpb, 0, st>>>(a.x, a.pos, a.out_tok, a.out, rows, a.dims.H, a.dims.D, a.dims.d_r,
                                                a.dims.rope_off, a.eps, rt);
  else
    k_qk_prep<false><<<grid, 32 * wpb, 0, st>>>(a.x, a.pos, a.out_tok, a.out, rows, a.dims.H, a.dims.D, a.dims.d_r,
                                                 a.dims.rope_off, a.eps, rt);
  return cudaGetLastError();
}

cudaError_t launch_compress(const lc_compress_args& a, bool per_cta, cudaStream_t st) {
  if (a.max_blocks <= 0 || a.num_seqs <= 0) return cudaSuccess;
  const bool f32 = a.in_fmt == LC_FMT_F32;
  const RopeTable rt = make_rope_table(a.dims.d_r, a.rope_base);
  if (!per_cta) {
    const int wpb = 8;
    const dim3 grid((a.max_blocks + wpb - 1) / wpb, a.num_seqs);
    if (f32) k_compress_warp<true><<<grid, 32 * wpb, 0, st>>>(a, rt);
    else k_compress_warp<false><<<grid, 32 * wpb, 0, st>>>(a, rt);
  } else {
    const dim3 grid(a.max_blocks, a.num_seqs);
    const size_t sm = static_cast<size_t>(8 * a.dims.D + a.m) * sizeof(float);
    if (f32) {
      cudaFuncSetAttribute(k_compress_cta<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
      k_compress_cta<true><<<grid, 256, sm, st>>>(a, rt);
    } else {
      cudaFuncSetAttribute(k_compress_cta<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
      k_compress_cta<false><<<grid, 256, sm, st>>>(a, rt);
    }
  }
  return cudaGetLastError();
}

}  // namespace lc
