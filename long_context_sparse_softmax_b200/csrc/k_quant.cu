// Decode-time maintenance of the lightning indexer's MXFP4 operands.
//
// mxfp4_quantize: rows of FP32 / BF16 values -> OCP MXFP4 (E2M1 elements, one E8M0 scale per
//   32): the indexer runs in FP4 ("解读 DeepSeek V4", "FP4 Quantization-Aware Training": the
//   lightning indexer's QK path is quantised to FP4), so a query's indexer vector is
//   quantised on the GPU every step.
// index_compress: each complete block of m tokens becomes one indexer key, pooled with the
//   block-softmax gate of the KV entries (the indexer scores compressed entries: "解读 DeepSeek
//   V4", CSA section; "DeepSeek-V4 论文分析" §5.3), without RMSNorm or RoPE, then quantised
//   to MXFP4 and written at the entry's row.
//
// Quantisation (OCP Microscaling Formats v1.0): per block of 32 elements the scale is
// X = 2^(floor(log2 amax) - 2) (2 = the largest exponent of E2M1; a zero block takes
// X = 2^0), and each element v / X is converted to E2M1 with round-to-nearest-even and
// saturation at +-6 (cvt.rn.satfinite.e2m1x2.f32).  Zero is always written as code 0.
// Element 2i goes to the low nibble of byte i.
//
// A warp holds 128 consecutive elements, 4 per lane; the 8 lanes of an aligned group hold
// one 32-element block.
#include <cmath>

#include "lc_internal.h"
#include "lc_mxfp4.cuh"
#include "lc_ptx.cuh"

namespace lc {

namespace {

// Quantise the 4 values of this lane (elements 4 lane .. 4 lane + 3 of a 128-element chunk)
// and store their 2 code bytes; lane 8 b stores the scale of block b of the chunk.  Every
// lane of the warp takes part (the block maximum is a shuffle); lanes past the row's end
// (on = false, whole 8-lane groups) store nothing.
__device__ __forceinline__ void mxfp4_store(const float (&v)[4], int lane, bool on, uint8_t* codes, uint8_t* scales) {
  uint32_t sc;
  const uint32_t c = mxfp4_quant4(v, &sc);
  if (!on) return;
  reinterpret_cast<uint16_t*>(codes)[lane] = static_cast<uint16_t>(c);
  if ((lane & 7) == 0) scales[lane >> 3] = static_cast<uint8_t>(sc);
}

template <bool kF32In>
__device__ __forceinline__ void load4(const void* row, int e, float (&v)[4]) {
  if (kF32In) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(row) + e));
    v[0] = f.x;
    v[1] = f.y;
    v[2] = f.z;
    v[3] = f.w;
  } else {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(row) + e));
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
  }
}

}  // namespace

// One warp per row, 8 rows per CTA.
template <bool kF32In>
__global__ void __launch_bounds__(256) k_mxfp4_quantize(lc_mxfp4_quant_args a) {
  // the indexer after this kernel (programmatic dependent launch) may start its set-up and
  // its key loads now; it reads the codes only once this grid has completed
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= a.n_rows) return;
  const size_t esz = kF32In ? 4 : 2;
  const void* src = static_cast<const char*>(a.x) + static_cast<size_t>(row) * a.d * esz;
  for (int c = 0; c < a.d; c += 128) {
    const bool on = c + 4 * lane < a.d;  // d is a multiple of 32: whole 8-lane groups
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (on) load4<kF32In>(src, c + 4 * lane, v);
    mxfp4_store(v, lane, on, a.codes + row * (a.d / 2) + c / 2, a.scales + row * (a.d / 32) + c / 32);
  }
}

// One warp per block (indexer key); grid (ceil(max_blocks / 8), num_seqs).
template <bool kF32In>
__global__ void __launch_bounds__(256) k_index_compress(lc_index_compress_args a) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (i >= __ldg(a.blk_count + b)) return;
  const int m = a.m, d = a.d_I;
  const int j = __ldg(a.blk_first + b) + i;
  const int pos0 = __ldg(a.tok_pos0 + b);
  const int first = j * m;
  if (first < pos0 || first + m > pos0 + __ldg(a.tok_len + b)) {
    if (lane == 0) set_status(a.status, LC_DEV_BAD_BLOCK);
    return;
  }
  const int64_t row0 = __ldg(a.tok_row0 + b) + (first - pos0);
  // gate softmax over the block: lanes hold tokens lane and lane + 32
  const float g0 = lane < m ? __ldg(a.g + row0 + lane) : -INFINITY;
  const float g1 = lane + 32 < m ? __ldg(a.g + row0 + lane + 32) : -INFINITY;
  const float gmax = warp_max(fmaxf(g0, g1));
  float e0 = lane < m ? expf(g0 - gmax) : 0.f;
  float e1 = lane + 32 < m ? expf(g1 - gmax) : 0.f;
  const float esum = warp_sum(e0 + e1);
  e0 /= esum;
  e1 /= esum;
  const size_t esz = kF32In ? 4 : 2;
  const int64_t out_row = __ldg(a.ent_start + b) + j;
  for (int c = 0; c < d; c += 128) {
    const bool on = c + 4 * lane < d;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int t = 0; t < m; ++t) {
      const float al = __shfl_sync(0xffffffffu, t < 32 ? e0 : e1, t & 31);
      if (on) {
        float v[4];
        load4<kF32In>(static_cast<const char*>(a.x) + static_cast<size_t>(row0 + t) * d * esz, c + 4 * lane, v);
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] = fmaf(al, v[u], acc[u]);
      }
    }
    mxfp4_store(acc, lane, on, a.codes + out_row * (d / 2) + c / 2, a.scales + out_row * (d / 32) + c / 32);
  }
}

cudaError_t launch_mxfp4_quantize(const lc_mxfp4_quant_args& a, cudaStream_t st) {
  if (a.n_rows == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((a.n_rows + 7) / 8);
  if (a.in_fmt == LC_FMT_F32) k_mxfp4_quantize<true><<<grid, 256, 0, st>>>(a);
  else k_mxfp4_quantize<false><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_index_compress(const lc_index_compress_args& a, cudaStream_t st) {
  if (a.num_seqs == 0 || a.max_blocks == 0) return cudaSuccess;
  const dim3 grid((a.max_blocks + 7) / 8, a.num_seqs);
  if (a.in_fmt == LC_FMT_F32) k_index_compress<true><<<grid, 256, 0, st>>>(a);
  else k_index_compress<false><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace lc
