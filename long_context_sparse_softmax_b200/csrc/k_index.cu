// Lightning-indexer scores: s(p, j) = sum_h w_h * ReLU(<qI[p, h], kI[j]>) for the entries
// j visible to the query at p ("解读 DeepSeek V4", CSA section and "FP4 Quantization-Aware
// Training": the indexer QK path runs in MXFP4; "DeepSeek-V4 论文分析" §5.3, §8.3).
//
// MXFP4 operands run on the tensor cores (k_index_tc.cu).  This file holds the FP32 path
// of the small correctness workload: FP32 FMA in a fixed order, no TF32.
#include "lc_internal.h"

namespace lc {

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
  if (a.fmt == LC_IDX_MXFP4 || a.fmt == LC_IDX_MXFP4_QBF16) return launch_index_tc(a, decode, st);
  const dim3 grid(a.n_q, (a.max_ent + 127) / 128);
  const size_t sm = static_cast<size_t>(a.H_I * a.d_I + a.H_I) * sizeof(float);
  cudaFuncSetAttribute(k_index_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
  k_index_f32<<<grid, 128, sm, st>>>(a);
  return cudaGetLastError();
}

}  // namespace lc
