// Top-k selection over each query's visible index scores ("解读 DeepSeek V4", CSA section:
// the lightning indexer picks the top-k compressed entries; "DeepSeek-V4 论文分析" §5.3:
// Top-512 (Flash) / Top-1024 (Pro)).
//
// A thread-block cluster of C CTAs takes one query row; CTA r holds the r-th of C equal
// segments of the row.  Scores map to order-preserving 32-bit keys, taken relative to the
// row's smallest key.  Radix passes of up to 11 bits find the K-th largest key T and how
// many keys equal to T to take: each CTA builds a 2048-bin histogram of its candidates in
// shared memory, the cluster barrier publishes it, and every CTA sums the C histograms
// over distributed shared memory in rank order, so all CTAs reach the same bin.  When the
// bin the first pass selects holds at most kCand keys of the whole row (the usual case),
// every CTA gathers those keys from the cluster and finishes the selection alone, and each
// rank's counts above and at T follow from the first pass's histograms; otherwise the
// cluster-wide passes continue.  The selection is then every key > T and the first `need`
// keys == T in index order (ties to the lower index), written in ascending index order:
// the CTAs' counts of keys > T and == T give each one its first output slot, and within a
// CTA each warp owns a contiguous piece of the segment.  Segments of up to
// kRowCache keys are staged in shared memory once; longer ones are re-read from global
// memory (L2) on each pass.  The result depends only on the score values: it is bit-exact
// and independent of C and of the launch shape.
#include <cooperative_groups.h>

#include "lc_internal.h"
#include "lc_ptx.cuh"

namespace cg = cooperative_groups;

namespace lc {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kRowCache = 48 * 1024;  // keys held in shared memory per CTA (192 KB)
constexpr int kBins = 2048;
constexpr int kMaxCluster = 8;
constexpr int kCand = kBins;          // candidates gathered after the first pass, at most

// Order-preserving key of a score: larger scores get larger keys.  -0.0 maps to the key
// of +0.0, since the two compare equal (ties between them go to the lower index).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kTopkThreads) k_topk(lc_topk_args a, int use_cache, int decode) {
  extern __shared__ uint32_t cache[];  // [kRowCache] keys of this CTA's segment
  __shared__ int hist[2][kBins];
  __shared__ int s_wsum[kTopkWarps];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  __shared__ int s_cnt[2];  // this CTA's keys > T and == T
  __shared__ int s_gt[kTopkWarps], s_eq[kTopkWarps];
  __shared__ uint32_t s_wmin[kTopkWarps], s_wmax[kTopkWarps];
  __shared__ uint32_t s_range[2];  // this CTA's smallest and largest key
  __shared__ int hist2[kBins];     // histograms of the gathered candidates
  __shared__ int s_bin_total;      // keys of the whole row in the bin just selected
  __shared__ int s_ncand;          // this CTA's keys in the first selected bin
  __shared__ int s_red[kTopkWarps][kMaxCluster];
  __shared__ int s_above[kMaxCluster], s_gtr[kMaxCluster], s_eqr[kMaxCluster];

  cg::cluster_group cl = cg::this_cluster();
  const int C = static_cast<int>(cl.num_blocks());
  const int rank = static_cast<int>(cl.block_rank());
  const int q = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_trigger();
  if (a.pdl) pdl_wait();  // the scores of the indexer before this kernel
  // decode: one query per sequence (q_start[b] = b), no search
  const int b = decode ? q : seq_of_query(a.batch.q_start, a.batch.num_seqs, q);
  const int p = __ldg(a.batch.q_pos0 + b) + (decode ? 0 : q - __ldg(a.batch.q_start + b));
  const int n = n_visible(p, a.m, a.W_x, __ldg(a.batch.n_ent + b));
  const int K = min(a.k, n);
  int32_t* out = a.idx + static_cast<int64_t>(q) * a.k;
  if (rank == 0 && tid == 0 && a.count) a.count[q] = K;
  for (int i = K + rank * kTopkThreads + tid; i < a.k; i += C * kTopkThreads) out[i] = -1;
  if (K == 0) return;  // the whole cluster returns here (K depends on the row only)
  if (K == n) {        // every visible entry is selected
    for (int i = rank * kTopkThreads + tid; i < n; i += C * kTopkThreads) out[i] = i;
    return;
  }
  // this CTA's segment [s0, s1): multiples of 4 keys, so float4 loads stay aligned
  const int segl = ((n + C - 1) / C + 3) & ~3;
  const int s0 = min(n, rank * segl), s1 = min(n, s0 + segl), ns = s1 - s0;
  const float* row = a.scores + static_cast<int64_t>(q) * a.score_stride + s0;
  const bool cached = use_cache != 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  if (cached) {
    // 16-byte loads, four in flight per thread (row and segment starts are 16-byte
    // aligned: the score stride and the segment length are multiples of 4 floats)
    const int n4 = ns >> 2;
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
          const uint32_t k0 = order_key(v[u].x), k1 = order_key(v[u].y), k2 = order_key(v[u].z),
                         k3 = order_key(v[u].w);
          cache[4 * i4 + 0] = k0;
          cache[4 * i4 + 1] = k1;
          cache[4 * i4 + 2] = k2;
          cache[4 * i4 + 3] = k3;
          kmin = min(kmin, min(min(k0, k1), min(k2, k3)));
          kmax = max(kmax, max(max(k0, k1), max(k2, k3)));
        }
      }
    }
    for (int i = 4 * n4 + tid; i < ns; i += kTopkThreads) {
      const uint32_t k0 = order_key(__ldg(row + i));
      cache[i] = k0;
      kmin = min(kmin, k0);
      kmax = max(kmax, k0);
    }
  } else {
    for (int i = tid; i < ns; i += kTopkThreads) {
      const uint32_t k0 = order_key(__ldg(row + i));
      kmin = min(kmin, k0);
      kmax = max(kmax, k0);
    }
  }
  // keys 4 i4 .. 4 i4 + 3 (past ns: don't-cares that the callers mask; they stay inside the
  // cache and inside the score row, whose stride is a multiple of 4)
  auto key4 = [&](int i4) -> uint4 {
    if (cached) return reinterpret_cast<const uint4*>(cache)[i4];
    const float4 f = __ldg(reinterpret_cast<const float4*>(row) + i4);
    return make_uint4(order_key(f.x), order_key(f.y), order_key(f.z), order_key(f.w));
  };
  const int n4 = (ns + 3) >> 2;

  // key range of the whole row (every CTA of the cluster gets the same one)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    s_wmin[warp] = kmin;
    s_wmax[warp] = kmax;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t a0 = 0xffffffffu, b0 = 0u;
    for (int w = 0; w < kTopkWarps; ++w) {
      a0 = min(a0, s_wmin[w]);
      b0 = max(b0, s_wmax[w]);
    }
    s_range[0] = a0;
    s_range[1] = b0;
  }
  cl.sync();
  uint32_t umin = 0xffffffffu, umax = 0u;
  for (int r = 0; r < C; ++r) {
    const uint32_t* rr = cl.map_shared_rank(s_range, r);
    umin = min(umin, rr[0]);
    umax = max(umax, rr[1]);
  }

  // Descending prefix over 2048 bins held two per thread (thread t: bins 2047 - 2t and
  // 2046 - 2t, counts c0 and c1): the bin holding the rem-th largest candidate becomes the
  // next w bits of the prefix; s_prefix / s_remaining / s_bin_total carry the result.
  auto pick_bin = [&](int c0, int c1, int w, uint32_t pf, int rem) {
    const int sm = c0 + c1;
    int incl = sm;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int wv = s_wsum[lane], wi = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += v;
      }
      s_wsum[lane] = wi - wv;  // exclusive over the warps
    }
    __syncthreads();
    const int excl = s_wsum[warp] + incl - sm;
    if (excl < rem && excl + sm >= rem) {
      const bool hi = excl + c0 >= rem;
      const uint32_t bin = static_cast<uint32_t>(hi ? kBins - 1 - 2 * tid : kBins - 2 - 2 * tid);
      s_prefix = (pf << w) | bin;
      s_remaining = hi ? rem - excl : rem - excl - c0;
      s_bin_total = hi ? c0 : c1;
    }
    __syncthreads();
  };
  // sums over the CTA of up to kMaxCluster per-thread counters (result in out[0 .. C))
  auto block_sum = [&](const int (&v)[kMaxCluster], int* out) {
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      if (r >= C) break;
      int x = v[r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (lane == 0) s_red[warp][r] = x;
    }
    __syncthreads();
    if (tid < C) {
      int t = 0;
      for (int w2 = 0; w2 < kTopkWarps; ++w2) t += s_red[w2][tid];
      out[tid] = t;
    }
    __syncthreads();
  };

  // Radix passes over rel = key - umin, < 2^L with L = bit length of the row's key range,
  // 11 bits at a time from the top: the first pass spreads the row over the whole
  // histogram whatever its range, and a row whose keys are all equal needs no pass.
  // pfx holds the bits of rel found so far; `remaining` counts the keys still to take
  // inside the bin they select.
  uint32_t pfx = 0;
  int remaining = K;
  int shift = 32 - __clz(static_cast<int>(umax - umin));
  int pass = 0;
  bool fast = false;  // the candidate path below took over after the first pass
#pragma unroll 1
  while (shift > 0) {
    const int w = min(11, shift);
    const int hi_shift = shift;  // candidates: rel >> hi_shift == pfx
    shift -= w;
    const uint32_t bmask = (1u << w) - 1u;
    int* h = hist[pass & 1];
    for (int i = tid; i < kBins; i += kTopkThreads) h[i] = 0;
    __syncthreads();
    for (int i4 = tid; i4 < n4; i4 += kTopkThreads) {
      const uint4 v = key4(i4);
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t rel = kk[j] - umin;
        const uint32_t top = hi_shift >= 32 ? 0u : rel >> hi_shift;
        if (4 * i4 + j < ns && top == pfx) atomicAdd(&h[(rel >> shift) & bmask], 1);
      }
    }
    cl.sync();  // every CTA's histogram of this pass is complete
    // thread t owns bins 2047 - 2t and 2046 - 2t (descending); sum them over the cluster
    // in rank order
    int v0[kMaxCluster], v1[kMaxCluster];  // every remote load in flight before the sums
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      v0[r] = v1[r] = 0;
      if (r < C) {
        const int* hr = cl.map_shared_rank(h, r);
        v0[r] = hr[kBins - 1 - 2 * tid];
        v1[r] = hr[kBins - 2 - 2 * tid];
      }
    }
    int c0 = 0, c1 = 0;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      c0 += v0[r];
      c1 += v1[r];
    }
    pick_bin(c0, c1, w, pfx, remaining);
    const uint32_t sel = s_prefix & bmask;
    pfx = s_prefix;
    remaining = s_remaining;
    ++pass;
    if (pass == 1 && shift > 0 && s_bin_total <= kCand) {
      // Few keys share the selected bin: every CTA gathers them and finishes the
      // selection alone, with no further cluster-wide histograms.  What each rank holds
      // above the bin comes from this pass's histograms.
      int ab[kMaxCluster];
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r)
        ab[r] = (static_cast<uint32_t>(kBins - 1 - 2 * tid) > sel ? v0[r] : 0) +
                (static_cast<uint32_t>(kBins - 2 - 2 * tid) > sel ? v1[r] : 0);
      block_sum(ab, s_above);
      fast = true;
      break;
    }
  }

  if (fast) {
    // this CTA's keys in the selected bin -> hist[1] (the other ranks read it)
    int* cand = hist[1];
    if (tid == 0) s_ncand = 0;
    __syncthreads();
    for (int i4 = tid; i4 < n4; i4 += kTopkThreads) {
      const uint4 v = key4(i4);
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t rel = kk[j] - umin;
        if (4 * i4 + j < ns && (rel >> shift) == pfx) cand[atomicAdd(&s_ncand, 1)] = static_cast<int>(kk[j]);
      }
    }
    cl.sync();  // every rank's candidates are written; every rank has read the histograms
    // all ranks' candidates, in rank order, into hist[0]
    int* allc = hist[0];
    int cnt[kMaxCluster], off[kMaxCluster];
    int n_all = 0;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      cnt[r] = r < C ? *cl.map_shared_rank(&s_ncand, r) : 0;
      off[r] = n_all;
      n_all += cnt[r];
    }
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      if (r >= C) break;
      const int* rc = cl.map_shared_rank(cand, r);
      for (int i = tid; i < cnt[r]; i += kTopkThreads) allc[off[r] + i] = rc[i];
    }
    // no more reads of other ranks' shared memory; the matching wait comes before exit,
    // so no rank leaves while another still reads its candidates
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
    __syncthreads();
    // the remaining-th largest candidate: radix passes over the bits below the prefix
    while (shift > 0) {
      const int w = min(11, shift);
      const int hi_shift = shift;
      shift -= w;
      const uint32_t bmask = (1u << w) - 1u;
      for (int i = tid; i < kBins; i += kTopkThreads) hist2[i] = 0;
      __syncthreads();
      for (int i = tid; i < n_all; i += kTopkThreads) {
        const uint32_t rel = static_cast<uint32_t>(allc[i]) - umin;
        if ((rel >> hi_shift) == pfx) atomicAdd(&hist2[(rel >> shift) & bmask], 1);
      }
      __syncthreads();
      pick_bin(hist2[kBins - 1 - 2 * tid], hist2[kBins - 2 - 2 * tid], w, pfx, remaining);
      pfx = s_prefix;
      remaining = s_remaining;
    }
    // every rank's keys > T and == T: those above the first bin plus its candidates
    const uint32_t Tc = umin + pfx;
    int gtc[kMaxCluster], eqc[kMaxCluster];
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) gtc[r] = eqc[r] = 0;
    for (int i = tid; i < n_all; i += kTopkThreads) {
      const uint32_t k0 = static_cast<uint32_t>(allc[i]);
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        const bool in = i >= off[r] && i < off[r] + cnt[r];
        gtc[r] += in && k0 > Tc;
        eqc[r] += in && k0 == Tc;
      }
    }
    block_sum(gtc, s_gtr);
    block_sum(eqc, s_eqr);
  }
  const uint32_t T = umin + pfx;
  const int need = remaining;
  // keys > T are all taken (K - need of them); of the keys == T the first `need` in index
  // order.  Counts of the CTAs before this one give its first tie rank and output slot;
  // within the CTA, warp w owns the contiguous piece [w * wseg, (w + 1) * wseg).
  const int wseg4 = (n4 + kTopkWarps - 1) / kTopkWarps;  // in groups of 4 keys
  const int lo4 = min(n4, warp * wseg4), hi4 = min(n4, lo4 + wseg4);
  int gt_c = 0, eq_c = 0;
  for (int i4 = lo4 + lane; i4 < hi4; i4 += 32) {
    const uint4 v = key4(i4);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool valid = 4 * i4 + j < ns;
      gt_c += valid && kk[j] > T;
      eq_c += valid && kk[j] == T;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt_c += __shfl_xor_sync(0xffffffffu, gt_c, o);
    eq_c += __shfl_xor_sync(0xffffffffu, eq_c, o);
  }
  if (lane == 0) {
    s_gt[warp] = gt_c;
    s_eq[warp] = eq_c;
  }
  __syncthreads();
  int eq_rank = 0, pos = 0;
  if (fast) {
    for (int r = 0; r < rank; ++r) {
      const int gr = s_above[r] + s_gtr[r];
      pos += gr + min(max(need - eq_rank, 0), s_eqr[r]);
      eq_rank += s_eqr[r];
    }
  } else {
    if (tid == 0) {
      int g = 0, e = 0;
      for (int w = 0; w < kTopkWarps; ++w) {
        g += s_gt[w];
        e += s_eq[w];
      }
      s_cnt[0] = g;
      s_cnt[1] = e;
    }
    cl.sync();  // every CTA's counts are published
    for (int r = 0; r < rank; ++r) {
      const int* cr = cl.map_shared_rank(s_cnt, r);
      pos += cr[0] + min(max(need - eq_rank, 0), cr[1]);
      eq_rank += cr[1];
    }
  }
  for (int w = 0; w < warp; ++w) {
    pos += s_gt[w] + min(max(need - eq_rank, 0), s_eq[w]);
    eq_rank += s_eq[w];
  }
  if (!fast) cl.sync();  // no CTA leaves while another still reads its counts
  // 128 keys per step, 4 consecutive ones per lane: ties are ranked in index order within
  // the lane, then across the lanes (exclusive warp scans), then across the steps
  for (int base4 = lo4; base4 < hi4; base4 += 32) {
    const int i4 = base4 + lane;
    const uint4 v = i4 < hi4 ? key4(i4) : make_uint4(0, 0, 0, 0);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
    bool gt[4], eq[4];
    int ne = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool valid = i4 < hi4 && 4 * i4 + j < ns;
      gt[j] = valid && kk[j] > T;
      eq[j] = valid && kk[j] == T;
      ne += eq[j];
    }
    int eb = ne;  // inclusive scan of the lanes' tie counts
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, eb, o);
      if (lane >= o) eb += t;
    }
    const int eq_all = __shfl_sync(0xffffffffu, eb, 31);
    eb -= ne;
    bool sel[4];
    int nsel = 0, er = eq_rank + eb;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sel[j] = gt[j] || (eq[j] && er < need);
      er += eq[j];
      nsel += sel[j];
    }
    int sb = nsel;  // inclusive scan of the lanes' selection counts
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, sb, o);
      if (lane >= o) sb += t;
    }
    const int sel_all = __shfl_sync(0xffffffffu, sb, 31);
    int at = pos + sb - nsel;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (sel[j]) out[at++] = s0 + 4 * i4 + j;
    eq_rank += eq_all;
    pos += sel_all;
  }
  if (fast) asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// ---------------------------------------------------------------------------------
// Merge of the fused indexer's candidates (lc_csa_index_topk_* when a query's keys span
// several CTAs).  Range c of query q left cnt[q][c] candidates (order key, entry index) in
// ascending index order in slots c k .. c k + cnt - 1 of the query's [n_chunks][k] block;
// the ranges are disjoint and ascending, so slot order is index order.  One CTA per query
// selects the K largest keys, ties to the lower slot, and writes their indices in slot
// order.  Thread t owns slots t, t + 1024, ... (coalesced loads): up to kMergeRegRounds of
// them in registers, more in shared memory (kMergeCache keys), beyond that re-read from
// global memory on each pass.  The selection is the pair (Tk, Ts): the K-th largest key
// and the slot of the last selected key equal to it; slot s is selected iff key > Tk, or
// key == Tk and s <= Ts.  Radix passes of 11 bits over rel = key - min narrow the bin that
// holds the K-th key until it holds at most kSmallBin keys (usually after one pass); those
// are ranked exactly.  A bin of more than kSmallBin equal keys is ranked in slot order by
// a block-wide scan, as is the output.
constexpr int kMergeThreads = 1024;
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kMergeRegRounds = 8;        // slots per thread held in registers (n_slots <= 8192)
constexpr int kMergeCacheKI = 20 * 1024;  // slots whose key and index fit in shared memory
constexpr int kMergeCacheK = 40 * 1024;   // slots whose key fits in shared memory
constexpr int kMergeMaxChunks = 1024;
constexpr int kSmallBin = 256;
constexpr int kScanRounds = 64;           // slot rounds per block-wide ordering scan
constexpr int kScanPer = kScanRounds * kMergeWarps / kMergeThreads;
constexpr int kBatch = 8;                 // rounds whose global loads are issued together

// exclusive prefix of v over the CTA in thread order; *total gets the sum
__device__ __forceinline__ int scan_cta(int v, int* s_w, int* s_total, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_w[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int x = s_w[lane];
    int xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    s_w[lane] = xi - x;
    if (lane == 31) *s_total = xi;
  }
  __syncthreads();
  const int r = s_w[warp] + incl - v;
  *total = *s_total;
  __syncthreads();
  return r;
}

// R > 0: the slots are held in registers (n_slots <= R * 1024).  R == 0: cache 2 keeps keys
// and indices in shared memory, cache 1 keys only, cache 0 nothing.
template <int R>
__global__ void __launch_bounds__(kMergeThreads) k_topk_merge(int k, int m, int W_x, lc_batch batch,
                                                              const uint2* __restrict__ cand,
                                                              const int* __restrict__ cand_cnt, int n_chunks,
                                                              int32_t* idx, int32_t* count, int decode,
                                                              int cache) {
  static_assert(kMergeWarps == 32, "one warp scans the warp totals");
  static_assert(R * kMergeWarps <= kMergeThreads, "one scan entry per thread");
  extern __shared__ uint32_t kc[];
  __shared__ int s_hist[kBins];
  __shared__ int s_rc[kScanRounds * kMergeWarps];
  __shared__ uint32_t s_lkey[kSmallBin];
  __shared__ int s_lslot[kSmallBin];
  __shared__ int s_cnt[R > 0 ? 1 : kMergeMaxChunks];
  __shared__ int s_w[kMergeWarps];
  __shared__ int s_total, s_lcnt, s_n, s_ts;
  __shared__ int s_pick[3];
  __shared__ uint32_t s_rng[2][kMergeWarps];
  __shared__ uint32_t s_tk;
  const int q = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_trigger();
  for (int i = tid; i < kBins; i += kMergeThreads) s_hist[i] = 0;
  if (tid == 0) {
    s_n = 0;
    s_lcnt = 0;
  }
  // the query's visible entries: step inputs that the indexer does not write
  const int b = decode ? q : seq_of_query(batch.q_start, batch.num_seqs, q);
  const int p = __ldg(batch.q_pos0 + b) + (decode ? 0 : q - __ldg(batch.q_start + b));
  const int nv = n_visible(p, m, W_x, __ldg(batch.n_ent + b));
  const int K = min(k, nv);
  int32_t* out = idx + static_cast<int64_t>(q) * k;
  const int n_slots = n_chunks * k;
  const int J = (n_slots + kMergeThreads - 1) / kMergeThreads;  // rounds of slots
  const uint2* cq = cand + static_cast<int64_t>(q) * n_slots;
  const int* cc = cand_cnt + static_cast<int64_t>(q) * n_chunks;
  const uint32_t lt = (1u << lane) - 1u;
  pdl_wait();  // the indexer's candidates (launched right after it, programmatically)
  // R > 0: every candidate load at once (a slot past its range's count is read and dropped)
  uint2 e0[R > 0 ? R : 1];
  int cn0[R > 0 ? R : 1];
  if constexpr (R > 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int slot = r * kMergeThreads + tid;
      const bool in = K > 0 && slot < n_slots;
      cn0[r] = in ? __ldg(cc + slot / k) : 0;
      e0[r] = in ? __ldg(&cq[slot]) : make_uint2(0u, 0u);
    }
  }
  for (int i = K + tid; i < k; i += kMergeThreads) out[i] = -1;
  if (tid == 0 && count) count[q] = K;
  if (K == 0) return;
  // a range writes at most k candidates (the clamp only matters after a timeout upstream)
  auto held_g = [&](int slot) {
    const int c = slot / k;
    return slot - c * k < min(max(__ldg(cc + c), 0), k);
  };
  uint32_t key[R > 0 ? R : 1];
  int id[R > 0 ? R : 1];
  uint32_t vm = 0;  // R > 0: bit r = round r holds a candidate
  uint32_t* ks = kc;
  int* is = reinterpret_cast<int*>(kc + (cache == 2 ? n_slots : 0));
  uint32_t* vb = kc + (cache == 2 ? 2 * n_slots : cache == 1 ? n_slots : 0);
  // the key of a slot (R == 0) and whether the slot holds a candidate
  auto load = [&](int slot, uint32_t& kk) -> bool {
    if (slot >= n_slots) return false;
    if (cache) {
      kk = ks[slot];
      return (vb[slot >> 5] >> (slot & 31)) & 1u;
    }
    const int c = slot / k;
    if (slot - c * k >= s_cnt[c]) return false;
    kk = __ldg(&cq[slot].x);
    return true;
  };
  // pass 0: the keys (and indices), their range and count
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  int nmine = 0;
  if constexpr (R > 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int slot = r * kMergeThreads + tid;
      const bool v = slot < n_slots && slot % k < min(max(cn0[r], 0), k);
      key[r] = e0[r].x;
      id[r] = static_cast<int>(e0[r].y);
      if (v) {
        vm |= 1u << r;
        kmin = min(kmin, key[r]);
        kmax = max(kmax, key[r]);
        ++nmine;
      }
    }
  } else {
    for (int c = tid; c < n_chunks; c += kMergeThreads) s_cnt[c] = min(max(__ldg(cc + c), 0), k);
#pragma unroll 1
    for (int j0 = 0; j0 < J; j0 += kBatch) {
      uint2 e[kBatch];
      bool v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int slot = (j0 + u) * kMergeThreads + tid;
        v[u] = slot < n_slots && held_g(slot);
        e[u] = v[u] ? __ldg(&cq[slot]) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int slot = (j0 + u) * kMergeThreads + tid;
        if (j0 + u < J) {
          const uint32_t bal = __ballot_sync(0xffffffffu, v[u]);
          if (cache && slot < n_slots) {
            ks[slot] = e[u].x;
            if (cache == 2) is[slot] = static_cast<int>(e[u].y);
            if (lane == 0) vb[slot >> 5] = bal;
          }
        }
        if (v[u]) {
          kmin = min(kmin, e[u].x);
          kmax = max(kmax, e[u].x);
          ++nmine;
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    nmine += __shfl_xor_sync(0xffffffffu, nmine, o);
  }
  if (lane == 0) {
    s_rng[0][warp] = kmin;
    s_rng[1][warp] = kmax;
    atomicAdd(&s_n, nmine);
  }
  __syncthreads();
  uint32_t umin = 0xffffffffu, umax = 0u;
#pragma unroll 8
  for (int w = 0; w < kMergeWarps; ++w) {
    umin = min(umin, s_rng[0][w]);
    umax = max(umax, s_rng[1][w]);
  }
  const int n = s_n;
  // fn(slot, key) for every candidate this thread owns
  auto each = [&](auto fn) {
    if constexpr (R > 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if ((vm >> r) & 1u) fn(r * kMergeThreads + tid, key[r]);
    } else {
#pragma unroll 4
      for (int j = 0; j < J; ++j) {
        const int slot = j * kMergeThreads + tid;
        uint32_t kk;
        if (load(slot, kk)) fn(slot, kk);
      }
    }
  };
  // slot-order ranks of the candidates where pred(slot, key) holds: fn(slot, rank, index)
  // (index: the entry index when it is at hand, else -1)
  auto ordered = [&](auto pred, auto fn) {
    if constexpr (R > 0) {
      uint32_t bal[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int slot = r * kMergeThreads + tid;
        bal[r] = __ballot_sync(0xffffffffu, ((vm >> r) & 1u) && pred(slot, key[r]));
        if (lane == 0) s_rc[r * kMergeWarps + warp] = __popc(bal[r]);
      }
      __syncthreads();
      const int a0 = tid < R * kMergeWarps ? s_rc[tid] : 0;
      int tot;
      const int ex = scan_cta(a0, s_w, &s_total, &tot);
      if (tid < R * kMergeWarps) s_rc[tid] = ex;
      __syncthreads();
#pragma unroll
      for (int r = 0; r < R; ++r)
        if ((bal[r] >> lane) & 1u)
          fn(r * kMergeThreads + tid, s_rc[r * kMergeWarps + warp] + __popc(bal[r] & lt), id[r]);
    } else {
      int carry = 0;
#pragma unroll 1
      for (int j0 = 0; j0 < J; j0 += kScanRounds) {
        const int jn = min(kScanRounds, J - j0);
#pragma unroll 4
        for (int j = 0; j < jn; ++j) {
          const int slot = (j0 + j) * kMergeThreads + tid;
          uint32_t kk = 0;
          const bool pr = load(slot, kk) && pred(slot, kk);
          const uint32_t bal = __ballot_sync(0xffffffffu, pr);
          if (lane == 0) s_rc[j * kMergeWarps + warp] = __popc(bal);
        }
        __syncthreads();
        int av[kScanPer], sum = 0;
#pragma unroll
        for (int i = 0; i < kScanPer; ++i) {
          const int e = kScanPer * tid + i;
          av[i] = e < jn * kMergeWarps ? s_rc[e] : 0;
          sum += av[i];
        }
        int tot;
        int ex = scan_cta(sum, s_w, &s_total, &tot) + carry;
#pragma unroll
        for (int i = 0; i < kScanPer; ++i) {
          const int e = kScanPer * tid + i;
          if (e < jn * kMergeWarps) s_rc[e] = ex;
          ex += av[i];
        }
        __syncthreads();
#pragma unroll 1
        for (int j1 = 0; j1 < jn; j1 += kBatch) {
          int slots[kBatch], ranks[kBatch], ids[kBatch];
          bool picked[kBatch];
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            const int j = j1 + u;
            slots[u] = (j0 + j) * kMergeThreads + tid;
            uint32_t kk = 0;
            picked[u] = j < jn && load(slots[u], kk) && pred(slots[u], kk);
            const uint32_t bal = __ballot_sync(0xffffffffu, picked[u]);
            ranks[u] = j < jn ? s_rc[j * kMergeWarps + warp] + __popc(bal & lt) : 0;
          }
#pragma unroll
          for (int u = 0; u < kBatch; ++u)
            ids[u] = picked[u] ? (cache == 2 ? is[slots[u]] : static_cast<int>(__ldg(&cq[slots[u]].y))) : -1;
#pragma unroll
          for (int u = 0; u < kBatch; ++u)
            if (picked[u]) fn(slots[u], ranks[u], ids[u]);
        }
        carry += tot;
        __syncthreads();
      }
    }
  };
  if (n <= K) {
    // every candidate is taken
    if (tid == 0) {
      s_tk = 0u;
      s_ts = 0x7fffffff;
    }
  } else {
    // radix passes inside the bin (pfx over the bits above `shift`) that holds the K-th
    // largest key; rem = keys still to take inside it, in_bin = keys it holds
    uint32_t pfx = 0;
    int rem = K, in_bin = n;
    int shift = 32 - __clz(static_cast<int>(umax - umin));
    bool zeroed = true;  // the histogram was cleared before the first barrier
#pragma unroll 1
    while (in_bin > kSmallBin && shift > 0) {
      const int w = min(11, shift);
      const int hi = shift;
      shift -= w;
      const uint32_t bmask = (1u << w) - 1u;
      if (!zeroed) {
        for (int i = tid; i < kBins; i += kMergeThreads) s_hist[i] = 0;
        __syncthreads();
      }
      zeroed = false;
      each([&](int, uint32_t kk) {
        const uint32_t rel = kk - umin;
        if ((hi >= 32 ? 0u : rel >> hi) == pfx) atomicAdd(&s_hist[(rel >> shift) & bmask], 1);
      });
      __syncthreads();
      // thread t owns bins 2047 - 2t and 2046 - 2t (descending)
      const int h0 = s_hist[kBins - 1 - 2 * tid], h1 = s_hist[kBins - 2 - 2 * tid];
      int tot;
      const int ex = scan_cta(h0 + h1, s_w, &s_total, &tot);
      if (ex < rem && ex + h0 + h1 >= rem) {
        const bool upper = ex + h0 >= rem;
        s_pick[0] = upper ? kBins - 1 - 2 * tid : kBins - 2 - 2 * tid;
        s_pick[1] = upper ? rem - ex : rem - ex - h0;
        s_pick[2] = upper ? h0 : h1;
      }
      __syncthreads();
      pfx = (pfx << w) | static_cast<uint32_t>(s_pick[0]);
      rem = s_pick[1];
      in_bin = s_pick[2];
    }
    if (in_bin <= kSmallBin) {
      // rank the bin's keys exactly: (key descending, slot ascending)
      each([&](int slot, uint32_t kk) {
        if (shift >= 32 || ((kk - umin) >> shift) == pfx) {
          const int i = atomicAdd(&s_lcnt, 1);
          if (i < kSmallBin) {  // exactly in_bin keys arrive here
            s_lkey[i] = kk;
            s_lslot[i] = slot;
          }
        }
      });
      __syncthreads();
      if (tid < in_bin) {
        const uint32_t ki = s_lkey[tid];
        const int si = s_lslot[tid];
        int r = 0;
        for (int i = 0; i < in_bin; ++i) {
          const uint32_t kj = s_lkey[i];
          r += kj > ki || (kj == ki && s_lslot[i] < si);
        }
        if (r == rem - 1) {
          s_tk = ki;
          s_ts = si;
        }
      }
    } else {
      // more than kSmallBin keys equal to Tk: the rem-th of them in slot order
      const uint32_t T = umin + pfx;
      if (tid == 0) s_tk = T;
      ordered([&](int, uint32_t kk) { return kk == T; },
              [&](int slot, int r, int) {
                if (r == rem - 1) s_ts = slot;
              });
    }
  }
  __syncthreads();
  const uint32_t Tk = s_tk;
  const int Ts = s_ts;
  ordered([&](int slot, uint32_t kk) { return kk > Tk || (kk == Tk && slot <= Ts); },
          [&](int, int r, int e) {
            if (r < K) out[r] = e;
          });
}

cudaError_t launch_topk_merge(const lc_index_topk_args& a, int n_chunks, const uint2* cand, const int* cand_cnt,
                              bool decode, cudaStream_t st) {
  if (n_chunks > kMergeMaxChunks) return cudaErrorInvalidConfiguration;
  const int64_t n_max = static_cast<int64_t>(n_chunks) * a.k;
  if (n_max <= static_cast<int64_t>(kMergeRegRounds) * kMergeThreads)
    return launch_ex(k_topk_merge<kMergeRegRounds>, dim3(a.index.n_q), dim3(kMergeThreads), 0, st, true, 1, a.k,
                     a.index.m, a.index.W_x, a.index.batch, cand, cand_cnt, n_chunks, a.idx, a.count,
                     decode ? 1 : 0, 0);
  const int cache = n_max <= kMergeCacheKI ? 2 : n_max <= kMergeCacheK ? 1 : 0;
  const size_t words = static_cast<size_t>((n_max + 31) / 32);
  const size_t sm = cache == 2 ? static_cast<size_t>(n_max) * 8 + words * 4
                  : cache == 1 ? static_cast<size_t>(n_max) * 4 + words * 4 : 0;
  cudaFuncSetAttribute(k_topk_merge<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       kMergeCacheK * 4 + kMergeCacheK / 8);
  return launch_ex(k_topk_merge<0>, dim3(a.index.n_q), dim3(kMergeThreads), sm, st, true, 1, a.k, a.index.m,
                   a.index.W_x, a.index.batch, cand, cand_cnt, n_chunks, a.idx, a.count, decode ? 1 : 0, cache);
}

__global__ void k_empty_selection(int32_t* idx, int32_t* count, int n_q, int k) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < static_cast<int64_t>(n_q) * k) idx[i] = -1;
  if (count && i < n_q) count[i] = 0;
}

cudaError_t launch_empty_selection(int32_t* idx, int32_t* count, int n_q, int k, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(n_q) * k;
  k_empty_selection<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(idx, count, n_q, k);
  return cudaGetLastError();
}

cudaError_t launch_topk(const lc_topk_args& a, bool decode, cudaStream_t st) {
  if (a.n_q == 0) return cudaSuccess;
  // the largest cluster that keeps the rows within one wave (one 1024-thread CTA per SM),
  // and at least the one whose segments fit the key cache
  int C = 1;
  while (C < kMaxCluster &&
         (static_cast<int64_t>(a.n_q) * 2 * C <= sm_count() || (a.max_ent + C - 1) / C > kRowCache))
    C <<= 1;
  const int segl = ((a.max_ent + C - 1) / C + 3) & ~3;
  const int use_cache = segl <= kRowCache ? 1 : 0;
  const size_t sm = use_cache ? static_cast<size_t>(segl) * 4 : 0;
  cudaFuncSetAttribute(k_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kRowCache * 4));
  const int64_t ctas = static_cast<int64_t>(a.n_q) * C;
  if (ctas > 0x7fffffff) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(kTopkThreads);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k_topk, a, use_cache, decode ? 1 : 0);
}

}  // namespace lc
