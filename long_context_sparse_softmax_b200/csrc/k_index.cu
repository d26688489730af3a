// Lightning-indexer scores: s(p, j) = sum_h w_h * ReLU(<qI[p, h], kI[j]>) for the entries
// j visible to the query at p ("解读 DeepSeek V4", CSA section and "FP4 Quantization-Aware
// Training": the indexer QK path runs in MXFP4; "DeepSeek-V4 论文分析" §5.3, §8.3).
//
// MXFP4 path.  E2M1 values are exactly representable in E4M3 (FP4 -> FP8 is lossless), so
// the codes are widened to E4M3 in shared memory without their scales and fed to FP8
// tensor-core MMAs whose K = 32 is exactly one MX block.  Each product of two E2M1 values
// is a multiple of 1/4 of magnitude <= 36, so a block's dot product (<= 1152) is exact in
// any accumulator with 13 or more significand bits, whatever its internal order.  The
// two E8M0 scales (powers of two) are applied to each block's exact dot product in FP32,
// and the 4 blocks are summed in a fixed order.
//
// FP32 path (small correctness shapes): FP32 FMA in a fixed order, no TF32.
#include "lc_internal.h"

namespace lc {

// Four E2M1 codes (4 nibbles in bits 0..15) -> four E4M3 bytes.
__device__ __forceinline__ uint32_t e2m1x4_to_e4m3x4(uint32_t nib) {
  // E4M3 bytes of the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6
  const uint32_t lo = 0x3C383000u, hi = 0x4C484440u;
  const uint32_t mag = __byte_perm(lo, hi, nib & 0x7777u);
  const uint32_t sign = ((nib & 0x8u) << 4) | ((nib & 0x80u) << 8) | ((nib & 0x800u) << 12) | ((nib & 0x8000u) << 16);
  return mag | sign;
}

// 32 E2M1 codes (16 bytes) -> 32 E4M3 bytes written to dst (16-byte aligned).
__device__ __forceinline__ void widen_block(uint4 c, uint8_t* dst) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = e2m1x4_to_e4m3x4(w[i] & 0xffffu);
    o[2 * i + 1] = e2m1x4_to_e4m3x4(w[i] >> 16);
  }
  reinterpret_cast<uint4*>(dst)[0] = make_uint4(o[0], o[1], o[2], o[3]);
  reinterpret_cast<uint4*>(dst)[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ float e8m0_to_f32(uint8_t e) {
  // 2^(e - 127); codes 1..254 are normal floats, 0 is 2^-127 (subnormal), 255 NaN
  if (e == 0) return 5.877471754111438e-39f;
  if (e == 255) return __int_as_float(0x7fffffff);
  return __int_as_float(static_cast<int>(e) << 23);
}

__device__ __forceinline__ void mma_e4m3_16x8x32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(0.f), "f"(0.f), "f"(0.f),
        "f"(0.f));
}

constexpr int kIdxKeys = 128;       // keys per CTA tile (4 warps x 2 m16 tiles)
constexpr int kIdxMaxHeads = 64;    // heads per pass (8 n8 tiles)

// grid: (query chunks, key tiles); 128 threads.  KB = d_I / 32 MX blocks.
template <int KB>
__global__ void __launch_bounds__(128) k_index_mxfp4(lc_index_args a, int q_chunk) {
  constexpr int DI = KB * 32;
  constexpr int RS = DI + 16;  // padded row stride (bytes): conflict-free fragment loads
  extern __shared__ __align__(16) uint8_t sm[];
  uint8_t* As = sm;                                  // [128][RS] key codes as E4M3
  uint8_t* Bs = As + kIdxKeys * RS;                  // [64][RS] query codes as E4M3
  float* sk = reinterpret_cast<float*>(Bs + kIdxMaxHeads * RS);  // [128][KB]
  float* sq = sk + kIdxKeys * KB;                    // [64][KB]
  float* ws = sq + kIdxMaxHeads * KB;                // [64]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int H = a.H_I;
  const int NT = H >> 3;
  const int j0 = blockIdx.y * kIdxKeys;
  const int qa = blockIdx.x * q_chunk;
  const int qb = min(qa + q_chunk, a.n_q);
  if (qa >= qb) return;

  // the last query of the chunk sees the most entries when the chunk lies in one
  // sequence; otherwise take the max over the chunk
  int nv_max = 0;
  {
    int bq = seq_of_query(a.batch.q_start, a.batch.num_seqs, qa);
    for (int q = qa; q < qb; ++q) {
      while (bq + 1 < a.batch.num_seqs && __ldg(a.batch.q_start + bq + 1) <= q) ++bq;
      const int p = __ldg(a.batch.q_pos0 + bq) + (q - __ldg(a.batch.q_start + bq));
      nv_max = max(nv_max, n_visible(p, a.m, a.W_x, __ldg(a.batch.n_ent + bq)));
    }
  }
  if (j0 >= nv_max) return;

  int b_cur = -1;
  for (int q = qa; q < qb; ++q) {
    const int b = seq_of_query(a.batch.q_start, a.batch.num_seqs, q);
    const int p = __ldg(a.batch.q_pos0 + b) + (q - __ldg(a.batch.q_start + b));
    const int nv = n_visible(p, a.m, a.W_x, __ldg(a.batch.n_ent + b));
    if (j0 >= nv) continue;
    __syncthreads();  // previous query's tiles are no longer read
    if (b != b_cur) {
      // key tile of this sequence: 128 rows x DI codes, widened to E4M3
      const int64_t kbase = __ldg(a.batch.ent_start + b);
      const int n_ent = __ldg(a.batch.n_ent + b);
      for (int u = tid; u < kIdxKeys * KB; u += 128) {
        const int r = u / KB, blk = u % KB;
        const int j = j0 + r;
        uint4 c = make_uint4(0, 0, 0, 0);
        uint8_t e = 127;
        if (j < n_ent) {
          c = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.k) + (kbase + j) * (DI / 2)) + blk);
          e = __ldg(a.k_scale + (kbase + j) * KB + blk);
        }
        widen_block(c, As + r * RS + blk * 32);
        sk[r * KB + blk] = e8m0_to_f32(e);
      }
      b_cur = b;
    }
    // query codes, scales and head weights
    for (int u = tid; u < H * KB; u += 128) {
      const int h = u / KB, blk = u % KB;
      const uint4 c = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.q) +
                                                           (static_cast<int64_t>(q) * H + h) * (DI / 2)) + blk);
      widen_block(c, Bs + h * RS + blk * 32);
      sq[h * KB + blk] = e8m0_to_f32(__ldg(a.q_scale + (static_cast<int64_t>(q) * H + h) * KB + blk));
    }
    for (int h = tid; h < H; h += 128) ws[h] = __ldg(a.w + static_cast<int64_t>(q) * a.w_qstride + h);
    __syncthreads();

    float acc[2][8][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.f;

    const int rbase = warp * 32;
#pragma unroll
    for (int blk = 0; blk < KB; ++blk) {
      uint32_t af[2][4];
      float skr[2][2];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint8_t* r0 = As + (rbase + mt * 16 + g) * RS + blk * 32 + 4 * t;
        const uint8_t* r1 = r0 + 8 * RS;
        af[mt][0] = *reinterpret_cast<const uint32_t*>(r0);
        af[mt][1] = *reinterpret_cast<const uint32_t*>(r1);
        af[mt][2] = *reinterpret_cast<const uint32_t*>(r0 + 16);
        af[mt][3] = *reinterpret_cast<const uint32_t*>(r1 + 16);
        skr[mt][0] = sk[(rbase + mt * 16 + g) * KB + blk];
        skr[mt][1] = sk[(rbase + mt * 16 + g + 8) * KB + blk];
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        if (nt < NT) {
          const uint8_t* c0 = Bs + (nt * 8 + g) * RS + blk * 32 + 4 * t;
          const uint32_t bf[2] = {*reinterpret_cast<const uint32_t*>(c0),
                                  *reinterpret_cast<const uint32_t*>(c0 + 16)};
          const float s0 = sq[(nt * 8 + 2 * t) * KB + blk];
          const float s1 = sq[(nt * 8 + 2 * t + 1) * KB + blk];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            float d[4];
            mma_e4m3_16x8x32(d, af[mt], bf);
            acc[mt][nt][0] = fmaf(d[0], skr[mt][0] * s0, acc[mt][nt][0]);
            acc[mt][nt][1] = fmaf(d[1], skr[mt][0] * s1, acc[mt][nt][1]);
            acc[mt][nt][2] = fmaf(d[2], skr[mt][1] * s0, acc[mt][nt][2]);
            acc[mt][nt][3] = fmaf(d[3], skr[mt][1] * s1, acc[mt][nt][3]);
          }
        }
      }
    }
    // head reduction: sum_h w_h ReLU(acc), over this thread's 2 heads per n-tile, then
    // over the 4 threads sharing a row
    float* srow = a.scores + static_cast<int64_t>(q) * a.score_stride;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      float s_lo = 0.f, s_hi = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        if (nt < NT) {
          const float w0 = ws[nt * 8 + 2 * t], w1 = ws[nt * 8 + 2 * t + 1];
          s_lo = fmaf(w0, fmaxf(acc[mt][nt][0], 0.f), s_lo);
          s_lo = fmaf(w1, fmaxf(acc[mt][nt][1], 0.f), s_lo);
          s_hi = fmaf(w0, fmaxf(acc[mt][nt][2], 0.f), s_hi);
          s_hi = fmaf(w1, fmaxf(acc[mt][nt][3], 0.f), s_hi);
        }
      }
      s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
      s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
      s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
      s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
      if (t == 0) {
        const int jl = j0 + rbase + mt * 16 + g;
        if (jl < nv) srow[jl] = s_lo;
        if (jl + 8 < nv) srow[jl + 8] = s_hi;
      }
    }
  }
}

// FP32 operands: one thread per (query, key); query heads staged in shared memory.
__global__ void __launch_bounds__(128) k_index_f32(lc_index_args a) {
  extern __shared__ float qs[];  // [H_I][d_I] then w [H_I]
  const int q = blockIdx.x;
  const int b = seq_of_query(a.batch.q_start, a.batch.num_seqs, q);
  const int p = __ldg(a.batch.q_pos0 + b) + (q - __ldg(a.batch.q_start + b));
  const int nv = n_visible(p, a.m, a.W_x, __ldg(a.batch.n_ent + b));
  const int j0 = blockIdx.y * blockDim.x;
  if (j0 >= nv) return;
  const int H = a.H_I, DI = a.d_I;
  const float* qg = static_cast<const float*>(a.q) + static_cast<int64_t>(q) * H * DI;
  for (int u = threadIdx.x; u < H * DI; u += blockDim.x) qs[u] = __ldg(qg + u);
  float* wsm = qs + H * DI;
  for (int h = threadIdx.x; h < H; h += blockDim.x) wsm[h] = __ldg(a.w + static_cast<int64_t>(q) * a.w_qstride + h);
  __syncthreads();
  const int j = j0 + threadIdx.x;
  if (j >= nv) return;
  const float4* kr = reinterpret_cast<const float4*>(static_cast<const float*>(a.k) +
                                                     (__ldg(a.batch.ent_start + b) + j) * DI);
  float s = 0.f;
  for (int h = 0; h < H; ++h) {
    const float* qh = qs + h * DI;
    float dot = 0.f;
    for (int i = 0; i < DI / 4; ++i) {
      const float4 kv = __ldg(kr + i);
      dot = fmaf(qh[4 * i + 0], kv.x, dot);
      dot = fmaf(qh[4 * i + 1], kv.y, dot);
      dot = fmaf(qh[4 * i + 2], kv.z, dot);
      dot = fmaf(qh[4 * i + 3], kv.w, dot);
    }
    s = fmaf(wsm[h], fmaxf(dot, 0.f), s);
  }
  a.scores[static_cast<int64_t>(q) * a.score_stride + j] = s;
}

cudaError_t launch_index_scores(const lc_index_args& a, bool decode, cudaStream_t st) {
  if (a.n_q == 0 || a.max_ent == 0) return cudaSuccess;
  if (a.fmt == LC_IDX_F32) {
    const dim3 grid(a.n_q, (a.max_ent + 127) / 128);
    const size_t sm = static_cast<size_t>(a.H_I * a.d_I + a.H_I) * sizeof(float);
    cudaFuncSetAttribute(k_index_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
    k_index_f32<<<grid, 128, sm, st>>>(a);
    return cudaGetLastError();
  }
  if (index_tc_supported(a)) return launch_index_tc(a, decode, st);
  const int q_chunk = decode ? 1 : 32;
  const dim3 grid((a.n_q + q_chunk - 1) / q_chunk, (a.max_ent + kIdxKeys - 1) / kIdxKeys);
  const int KB = a.d_I / 32;
  const size_t rs = static_cast<size_t>(a.d_I + 16);
  const size_t sm = (kIdxKeys + kIdxMaxHeads) * rs + (kIdxKeys + kIdxMaxHeads) * KB * 4 + kIdxMaxHeads * 4;
  switch (KB) {
    case 4:
      cudaFuncSetAttribute(k_index_mxfp4<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
      k_index_mxfp4<4><<<grid, 128, sm, st>>>(a, q_chunk);
      break;
    case 2:
      cudaFuncSetAttribute(k_index_mxfp4<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
      k_index_mxfp4<2><<<grid, 128, sm, st>>>(a, q_chunk);
      break;
    case 8:
      cudaFuncSetAttribute(k_index_mxfp4<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
      k_index_mxfp4<8><<<grid, 128, sm, st>>>(a, q_chunk);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace lc
