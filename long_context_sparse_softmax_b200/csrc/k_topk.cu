// Top-k selection over each query's visible index scores ("解读 DeepSeek V4", CSA section:
// the lightning indexer picks the top-k compressed entries; "DeepSeek-V4 论文分析" §5.3:
// Top-512 (Flash) / Top-1024 (Pro)).
//
// One CTA per query row.  Scores map to order-preserving 32-bit keys; four 8-bit radix
// passes over a shared-memory histogram find the K-th largest key T and how many of the
// keys equal to T to take.  A final pass in index order keeps every key > T and the first
// `need` keys == T (ties to the lower index), writing indices in ascending order through
// per-warp counts.  Rows of up to kRowCache scores are staged in shared memory
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

__global__ void __launch_bounds__(kTopkThreads) k_topk(lc_topk_args a, int use_cache) {
  extern __shared__ uint32_t cache[];  // [kRowCache] keys when the row fits
  __shared__ int hist[256];
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
    // 16-byte loads, four in flight per thread (rows start 16-byte aligned: the score
    // stride is a multiple of 4 floats)
    const int n4 = n >> 2;
    const float4* r4 = reinterpret_cast<const float4*>(row);
    for (int base = 0; base < n4; base += 4 * kTopkThreads) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i4 = base + u * kTopkThreads + tid;
        if (i4 < n4) v[u] = __ldg(r4 + i4);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i4 = base + u * kTopkThreads + tid;
        if (i4 < n4) {
          cache[4 * i4 + 0] = order_key(v[u].x);
          cache[4 * i4 + 1] = order_key(v[u].y);
          cache[4 * i4 + 2] = order_key(v[u].z);
          cache[4 * i4 + 3] = order_key(v[u].w);
        }
      }
    }
    for (int i = 4 * n4 + tid; i < n; i += kTopkThreads) cache[i] = order_key(__ldg(row + i));
  }
  uint32_t prefix = 0, mask = 0;
  int remaining = K;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    // scores of one row share their high bits, so in the first passes whole warps often
    // hit one bin: then a single lane adds 32
    for (int base = 0; base < n; base += kTopkThreads) {
      const int i = base + tid;
      int bin = 256;  // not a candidate
      if (i < n) {
        const uint32_t u = cached ? cache[i] : order_key(__ldg(row + i));
        if ((u & mask) == prefix) bin = static_cast<int>((u >> shift) & 0xffu);
      }
      const int b0 = __shfl_sync(0xffffffffu, bin, 0);
      if (__all_sync(0xffffffffu, bin == b0)) {
        if ((tid & 31) == 0 && b0 < 256) atomicAdd(&hist[b0], 32);
      } else if (bin < 256) {
        atomicAdd(&hist[bin], 1);
      }
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
  // keys > T are all taken (K - need of them); of the keys == T the first `need` in index
  // order.  Warp w owns the contiguous segment [w * seg, (w + 1) * seg): it counts its keys
  // > T and == T, the counts of the warps before it give its first tie rank and output
  // slot, and it writes its selections in index order with warp ballots.
  const uint32_t T = prefix;
  const int need = remaining;
  const int lane = tid & 31, warp = tid >> 5;
  const int seg = (n + kTopkWarps - 1) / kTopkWarps;
  const int lo = min(n, warp * seg), hi = min(n, lo + seg);
  int gt_c = 0, eq_c = 0;
  for (int i = lo + lane; i < hi; i += 32) {
    const uint32_t u = cached ? cache[i] : order_key(__ldg(row + i));
    gt_c += u > T;
    eq_c += u == T;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt_c += __shfl_xor_sync(0xffffffffu, gt_c, o);
    eq_c += __shfl_xor_sync(0xffffffffu, eq_c, o);
  }
  __shared__ int s_gt[kTopkWarps], s_eq[kTopkWarps];
  if (lane == 0) {
    s_gt[warp] = gt_c;
    s_eq[warp] = eq_c;
  }
  __syncthreads();
  int eq_rank = 0, pos = 0;
  for (int w = 0; w < warp; ++w) {
    pos += s_gt[w] + min(max(need - eq_rank, 0), s_eq[w]);
    eq_rank += s_eq[w];
  }
  const uint32_t below = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const bool valid = i < hi;
    const uint32_t u = valid ? (cached ? cache[i] : order_key(__ldg(row + i))) : 0u;
    const bool eq = valid && u == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const bool sel = valid && (u > T || (eq && eq_rank + __popc(eqm & below) < need));
    const uint32_t selm = __ballot_sync(0xffffffffu, sel);
    if (sel) out[pos + __popc(selm & below)] = i;
    eq_rank += __popc(eqm);
    pos += __popc(selm);
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
