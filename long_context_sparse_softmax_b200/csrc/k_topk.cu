// Top-k selection over each query's visible index scores ("解读 DeepSeek V4", CSA section:
// the lightning indexer picks the top-k compressed entries; "DeepSeek-V4 论文分析" §5.3:
// Top-512 (Flash) / Top-1024 (Pro)).
//
// One CTA per query row.  Scores map to order-preserving 32-bit keys; four 8-bit radix
// passes over a shared-memory histogram find the K-th largest key T and how many of the
// keys equal to T to take.  A final pass in index order keeps every key > T and the first
// `need` keys == T (ties to the lower index), writing indices in ascending order through
// block-wide prefix counts.  Rows of up to kRowCache scores are staged in shared memory
// once; longer rows are re-read from global memory (L2) on each pass.  The result depends
// only on the score values: it is bit-exact and independent of the launch shape.
#include "lc_internal.h"

namespace lc {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kRowCache = 48 * 1024;  // scores held in shared memory (192 KB)

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix count of `flag` over the CTA's threads in thread order.
// Returns the count before this thread; *total receives the CTA total.
__device__ __forceinline__ int block_excl_count(bool flag, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  __syncthreads();  // warp_tot free from its previous use
  if (lane == 0) warp_tot[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    int v = lane < kTopkWarps ? warp_tot[lane] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane < kTopkWarps) warp_tot[lane] = incl - v;  // exclusive
    if (lane == 31) warp_tot[kTopkWarps] = incl;
  }
  __syncthreads();
  *total = warp_tot[kTopkWarps];
  return warp_tot[warp] + in_warp;
}

__global__ void __launch_bounds__(kTopkThreads) k_topk(lc_topk_args a, int use_cache) {
  extern __shared__ uint32_t cache[];  // [kRowCache] keys when the row fits
  __shared__ int hist[256];
  __shared__ int warp_tot[kTopkWarps + 1];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;

  const int q = blockIdx.x;
  const int tid = threadIdx.x;
  const int b = seq_of_query(a.batch.q_start, a.batch.num_seqs, q);
  const int p = __ldg(a.batch.q_pos0 + b) + (q - __ldg(a.batch.q_start + b));
  const int n = n_visible(p, a.m, a.W_x, __ldg(a.batch.n_ent + b));
  const int K = min(a.k, n);
  int32_t* out = a.idx + static_cast<int64_t>(q) * a.k;
  if (tid == 0 && a.count) a.count[q] = K;
  for (int i = K + tid; i < a.k; i += kTopkThreads) out[i] = -1;
  if (K == 0) return;
  if (K == n) {  // every visible entry is selected
    for (int i = tid; i < n; i += kTopkThreads) out[i] = i;
    return;
  }
  const float* row = a.scores + static_cast<int64_t>(q) * a.score_stride;
  const bool cached = use_cache && n <= kRowCache;
  if (cached) {
    for (int i = tid; i < n; i += kTopkThreads) cache[i] = order_key(__ldg(row + i));
  }
  uint32_t prefix = 0, mask = 0;
  int remaining = K;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      const uint32_t u = cached ? cache[i] : order_key(__ldg(row + i));
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 0xffu], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins 255-8l .. 248-8l (descending); find the bin where the count
      // from the top reaches `remaining`
      int c[8];
      int sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * tid - i];
        sum += c[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += v;
      }
      const int excl = incl - sum;
      if (excl < remaining && incl >= remaining) {
        int acc = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc + c[i] >= remaining) {
            s_prefix = prefix | (static_cast<uint32_t>(255 - 8 * tid - i) << shift);
            s_remaining = remaining - acc;
            break;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    remaining = s_remaining;
    mask |= 0xffu << shift;
  }
  // keys > prefix: all taken (K - remaining of them); keys == prefix: first `remaining`
  const uint32_t T = prefix;
  const int need = remaining;
  int eq_seen = 0, written = 0;
  for (int base = 0; base < n && written < K; base += kTopkThreads) {
    const int i = base + tid;
    uint32_t u = 0;
    if (i < n) u = cached ? cache[i] : order_key(__ldg(row + i));
    const bool eq = i < n && u == T;
    int eq_tot;
    const int eq_rank = eq_seen + block_excl_count(eq, warp_tot, &eq_tot);
    const bool sel = i < n && (u > T || (eq && eq_rank < need));
    int sel_tot;
    const int pos = written + block_excl_count(sel, warp_tot, &sel_tot);
    if (sel) out[pos] = i;
    eq_seen += eq_tot;
    written += sel_tot;
  }
}

cudaError_t launch_topk(const lc_topk_args& a, bool /*decode*/, cudaStream_t st) {
  if (a.n_q == 0) return cudaSuccess;
  const int use_cache = a.max_ent <= kRowCache ? 1 : 0;
  const size_t sm = use_cache ? static_cast<size_t>(a.max_ent) * 4 : 0;
  cudaFuncSetAttribute(k_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kRowCache * 4));
  k_topk<<<a.n_q, kTopkThreads, sm, st>>>(a, use_cache);
  return cudaGetLastError();
}

}  // namespace lc
