// Internal launchers of the CSA / HCA attention library (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>

#include <utility>

#include "lc_common.cuh"

namespace lc {

// cudaLaunchKernelEx with programmatic stream serialization when `pdl` (the kernel may start
// while the previous kernel in the stream runs; it calls griddepcontrol.wait before reading
// that kernel's outputs) and a 1-D thread-block cluster when cluster > 1.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                      int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Streaming multiprocessors of the current device (queried once per device; 148 on B200).
int sm_count();

cudaError_t launch_qk_prep(const lc_qk_prep_args& a, cudaStream_t st);
cudaError_t launch_compress(const lc_compress_args& a, bool per_cta, cudaStream_t st);
cudaError_t launch_mxfp4_quantize(const lc_mxfp4_quant_args& a, cudaStream_t st);
cudaError_t launch_index_compress(const lc_index_compress_args& a, cudaStream_t st);
cudaError_t launch_out_proj(const lc_out_proj_args& a, cudaStream_t st);
cudaError_t launch_index_scores(const lc_index_args& a, bool decode, cudaStream_t st);
cudaError_t launch_topk(const lc_topk_args& a, bool decode, cudaStream_t st);
// idx[q, :] = -1 and count[q] = 0 for every query
cudaError_t launch_empty_selection(int32_t* idx, int32_t* count, int n_q, int k, cudaStream_t st);
cudaError_t launch_attn(const lc_attn_args& a, bool sparse, bool decode, cudaStream_t st);
size_t attn_workspace_bytes(const lc_attn_args& a, bool sparse, bool decode);
size_t attn_image_bytes(const lc_attn_args& a, bool sparse, bool decode);
bool attn_tc_supported(const lc_attn_args& a);
int attn_impl(const lc_attn_args& a);
bool attn_impl_ok(const lc_attn_args& a);
size_t attn_tc_workspace(const lc_attn_args& a, bool sparse, bool decode);
size_t attn_tc_image_bytes(const lc_attn_args& a, bool sparse, bool decode);
cudaError_t launch_attn_tc(const lc_attn_args& a, bool sparse, bool decode, cudaStream_t st, int* n_split);
cudaError_t launch_attn_combine(const lc_attn_args& a, int n_split, cudaStream_t st);
bool attn_tc8_supported(const lc_attn_args& a);
size_t attn_tc8_workspace(const lc_attn_args& a, bool sparse, bool decode);
cudaError_t launch_attn_tc8(const lc_attn_args& a, bool sparse, bool decode, cudaStream_t st, int* n_split);
cudaError_t launch_index_tc(const lc_index_args& a, bool decode, cudaStream_t st);

// Indexer launch shape: key tiles, tiles per CTA, CTAs per query, tensor-memory columns,
// dynamic shared memory.
struct IndexGeom {
  int tiles, tpc, n_chunks;
  uint32_t tmem_cols;
  size_t smem;
};
IndexGeom index_geometry(const lc_index_args& a, bool decode, bool select);
size_t index_topk_workspace(const lc_index_topk_args& a, bool decode);
cudaError_t launch_index_topk(const lc_index_topk_args& a, bool decode, cudaStream_t st);
cudaError_t launch_topk_merge(const lc_index_topk_args& a, int n_chunks, const uint2* cand, const int* cand_cnt,
                              bool decode, cudaStream_t st);

// Sequence of query row q: the b with q_start[b] <= q < q_start[b+1] (binary search).
__device__ __forceinline__ int seq_of_query(const int32_t* __restrict__ q_start, int num_seqs, int q) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(q_start + mid) <= q) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Entries visible to a query at p: j with (j+1)*m - 1 <= p - W_x, clamped to [0, n_ent].
__device__ __forceinline__ int n_visible(int p, int m, int W_x, int n_ent) {
  const int t = p - W_x + 1;
  if (t <= 0) return 0;
  const int v = t / m;
  return v < n_ent ? v : n_ent;
}

}  // namespace lc
