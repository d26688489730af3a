// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05, block-scaled FP4).
//
// s(p, j) = sum_h w_h * ReLU(<qI[p, h], kI[j]>) over the entries j visible to the query at
// p ("解读 DeepSeek V4", CSA section and "FP4 Quantization-Aware Training": the indexer QK
// path runs in MXFP4; "DeepSeek-V4 论文分析" §5.3, §8.3).
//
// One MMA tile: A = 128 keys x 128 dims (E2M1, 2 per byte: 64 bytes per key), B = the H_I
// heads of QPC queries (N = QPC * H_I), block scales (E8M0, one per 32 elements) in tensor
// memory, D = 128 x N FP32 in tensor memory.  The tensor core applies the block scales;
// the operands are the caller's bytes, never widened or converted.
//
//   * A tile of 128 consecutive keys is one 2-D bulk tensor copy (TMA) of 8 KB, written
//     with the 64-byte swizzle that is the MMA's K-major SWIZZLE_64B layout (8-row groups
//     512 bytes apart; the second K = 64 step starts 32 bytes into the rows).  The query
//     operand is copied once per CTA into the same layout;
//   * block scales in tensor memory: column c holds, in lane L of every lane quadrant, the
//     four E8M0 bytes (K blocks 0..3) of row (L % 32) + 32 c; the k-th K = 64 MMA reads
//     bytes 2k, 2k + 1 (sf_id = 2k);
//   * warp roles (192 threads): warp 0 loads key tiles (TMA) and their scale words (four
//     tiles ahead, into a register ring; stored as 32 rows x 16 bytes, row L holding the
//     words of keys L, L + 32, L + 64, L + 96) into an 8-stage ring; lane 0 of warp 1 copies a
//     tile's scales into tensor memory (tcgen05.cp 32x128b.warpx4, which fills every
//     lane quadrant) and issues its MMAs into one of three accumulators; warps 2-5 run the
//     epilogue: thread t owns key row t of D (tcgen05.ld 32x32b), so the ReLU-weighted
//     head sum stays in registers (8 partial sums of heads h = k mod 8, added in a fixed
//     order).
//
// The roles meet only at mbarriers.  Every wait is bounded: after ~2^26 polls a role
// records LC_DEV_TIMEOUT in the status word and sets an abort flag that stops the others.
//
// Fused selection (SELECT, lc_csa_index_topk_*): the epilogue keeps the order-preserving
// keys of its range's scores in shared memory (and each thread's key range) instead of
// writing the scores out, and after the last tile its 128 threads select the range's top
// K = min(k, keys in range) exactly, ties to the lower index: radix passes of 11 bits over
// key - min (per-warp histograms) narrow the bin holding the K-th key until it holds at
// most kSmallBin keys, which are ranked exactly (more equal keys than that are ranked in
// index order with warp ballots).  The result is the pair (Tk, Ts): a key is selected iff
// it is above Tk, or equal to it at an offset up to Ts.  Output positions come from
// per-(tile, warp) counts and one scan.  With one CTA per query the selection is the
// answer (indices written ascending); otherwise the CTA writes its K (key, index)
// candidates in index order and k_topk_merge picks the final K among every range's
// candidates.  Every entry of the query's top K is in the top K of its own range, so the
// result equals csa_topk on the scores this kernel computes.  The selection runs once per
// launch, so its loops stay rolled: a taken branch into code not yet fetched stalls on the
// instruction fetch, which unrolled loops with guarded bodies multiply.
#include <cuda.h>

#include "lc_internal.h"
#include "lc_mxfp4.cuh"
#include "lc_ptx.cuh"

namespace lc {

namespace {

constexpr int kKeys = 128;          // keys per tile (MMA M)
constexpr int kDI = 128;            // indexer dims handled here (2 MMAs of K = 64)
constexpr int kRowB = kDI / 2;      // bytes per row
constexpr int kTileB = kKeys * kRowB;
constexpr int kStages = 8;            // key tiles in flight per CTA (2 CTAs per SM: 128 KB)
constexpr int kThreads = 192;
constexpr long kSpin = 1L << 26;
constexpr int kDBuf = 3;            // tensor-memory accumulators
constexpr uint32_t kColSfa = 0;     // offsets past the accumulators
constexpr uint32_t kColSfb = 16;

constexpr int kSelMaxTiles = 64;    // tiles per CTA in the fused-selection mode (32 KB of scores)
constexpr int kSelBins = 2048;
constexpr int kSmallBin = 256;      // the K-th key's first-pass bin is resolved by ranking up to this many

struct IdxBars {
  uint64_t kfull[kStages];   // key tile (expect-tx arrival) and its scale words (32 arrivals) landed
  uint64_t kempty[kStages];  // MMAs of the tile done (commit)
  uint64_t dfull[kDBuf];     // accumulator written (commit)
  uint64_t dempty[kDBuf];    // accumulator read (128 arrivals)
  uint64_t bfull;            // query operand, its scales and the head weights ready (128 arrivals)
  uint64_t fin;              // every MMA complete (commit)
};

// Order-preserving key of a score: larger scores get larger keys; -0.0 maps to +0.0's key.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix of v over the 128 epilogue threads in row order (row = quad * 32 + lane),
// and the total.  Uses named barrier 1; tmp holds 4 ints.
__device__ __forceinline__ int scan128(int v, int quad, int lane, int* tmp, int* total) {
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) tmp[quad] = incl;
  named_bar(1, 128);
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    before += w < quad ? tmp[w] : 0;
    all += tmp[w];
  }
  named_bar(1, 128);
  *total = all;
  return before + incl - v;
}

}  // namespace

// Outputs of the fused selection (k > 0).
struct IdxSelect {
  int k;            // 0: write the score matrix instead
  int n_chunks;     // key-range CTAs per query (gridDim.y)
  uint2* cand;      // n_chunks > 1: [n_q][n_chunks][k] (order key, entry index)
  int* cand_cnt;    // n_chunks > 1: [n_q][n_chunks] candidates written
  int32_t* idx;     // n_chunks == 1: [n_q][k]
  int32_t* count;   // n_chunks == 1: [n_q] or null
};

// grid: (query chunks of QPC queries, key-range chunks); 192 threads.
// Tensor memory: accumulators at columns [k N, (k + 1) N), k < 3; key scales at 3N + {0, 8};
// query scales at 3N + 16 (N / 32 columns).
template <int QPC, bool SELECT>
__global__ void __launch_bounds__(kThreads, 2)
    k_index_tc(const __grid_constant__ CUtensorMap tk, lc_index_args a, int tiles_per_cta, uint32_t tmem_cols,
               int decode, IdxSelect sel) {
  static_assert(!SELECT || QPC == 1, "fused selection takes one query per CTA");
  extern __shared__ __align__(1024) uint8_t smem[];
  const int H = a.H_I;
  const int N = QPC * H;
  uint8_t* As = smem;                                               // [kStages][kTileB], SWIZZLE_64B
  uint8_t* Bs = As + kStages * kTileB;                              // [N rows][64 B], SWIZZLE_64B
  uint32_t* SFs = reinterpret_cast<uint32_t*>(Bs + N * kRowB);      // [kStages][128] key scale words
  float* ws = reinterpret_cast<float*>(SFs + kStages * kKeys);      // [N] head weights
  float* sc = ws + N;                                               // SELECT: [tiles_per_cta][128] scores
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ __align__(8) IdxBars bars;
  __shared__ int s_nv[QPC];
  __shared__ int s_q[QPC];
  __shared__ uint32_t s_qsw[QPC * 64];  // MXFP4_QBF16: each query row's scale word

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();  // the merge / top-k after this kernel may start; it waits for our results
  const int qa = blockIdx.x * QPC;
  if (qa >= a.n_q) return;
  // decode: one query per sequence (q_start[b] = b), no search
  const int b = decode ? qa : seq_of_query(a.batch.q_start, a.batch.num_seqs, qa);
  const int64_t kbase = __ldg(a.batch.ent_start + b);
  const int n_ent = __ldg(a.batch.n_ent + b);
  // queries of this chunk: they must belong to sequence b (prefill: one sequence;
  // decode: QPC = 1)
  if (tid < QPC) {
    const int q = qa + tid;
    int nv = 0;
    if (q < a.n_q && (decode || q < __ldg(a.batch.q_start + b + 1))) {
      const int p = __ldg(a.batch.q_pos0 + b) + (decode ? 0 : q - __ldg(a.batch.q_start + b));
      nv = n_visible(p, a.m, a.W_x, n_ent);
    }
    s_nv[tid] = nv;
    s_q[tid] = q;
  }
  __syncthreads();
  int nv_max = 0;
#pragma unroll
  for (int i = 0; i < QPC; ++i) nv_max = max(nv_max, s_nv[i]);
  const int t_begin = blockIdx.y * tiles_per_cta;
  const int t_end = min(t_begin + tiles_per_cta, (nv_max + kKeys - 1) / kKeys);
  if (t_begin >= t_end) {  // uniform over the CTA: nothing allocated yet
    if constexpr (SELECT) {
      // an empty key range: no candidates (or, alone, an empty selection); written only
      // after the previous kernel, which may still read them, has completed
      if (a.pdl) pdl_wait();
      if (sel.n_chunks > 1) {
        if (tid == 0) sel.cand_cnt[static_cast<int64_t>(qa) * sel.n_chunks + blockIdx.y] = 0;
      } else {
        for (int i = tid; i < sel.k; i += kThreads) sel.idx[static_cast<int64_t>(qa) * sel.k + i] = -1;
        if (tid == 0 && sel.count) sel.count[qa] = 0;
      }
    }
    return;
  }
  const int n_tiles = t_end - t_begin;

  // a caller-set limit counts immediate polls (test_wait), so that a small one runs out
  // for certain; the default counts try_wait polls, which may suspend briefly
  const long spin = a.spin_limit > 0 ? a.spin_limit : kSpin;
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const uint32_t addr = su32(bar);
    for (long it = 0; it < spin; ++it) {
      if (a.spin_limit > 0 ? mbar_probe(addr, parity) : mbar_test(addr, parity)) return true;
      if ((it & 1023) == 1023 && *reinterpret_cast<volatile int*>(&s_abort)) return false;
    }
    set_status(a.status, LC_DEV_TIMEOUT);
    atomicExch(&s_abort, 1);
    return false;
  };
  // before a role ends: the completion of an asynchronous operation it started (a bulk copy
  // landing, its MMAs finishing) - finite on the hardware, so the default limit applies even
  // after an abort; giving up here is reported too
  auto drain = [&](uint64_t* bar, uint32_t parity) {
    const uint32_t addr = su32(bar);
    for (long it = 0; it < kSpin; ++it)
      if (mbar_test(addr, parity)) return;
    set_status(a.status, LC_DEV_TIMEOUT);
  };

  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(&s_tmem)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(su32(&bars.kfull[i]), 1 + 32);
      mbar_init(su32(&bars.kempty[i]), 1);
    }
    for (int i = 0; i < kDBuf; ++i) {
      mbar_init(su32(&bars.dfull[i]), 1);
      mbar_init(su32(&bars.dempty[i]), 128);
    }
    mbar_init(su32(&bars.bfull), 128);
    mbar_init(su32(&bars.fin), 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tk)) : "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = s_tmem;
  const uint32_t col_sfa = kDBuf * N + kColSfa, col_sfb = kDBuf * N + kColSfb;

  if (warp == 0) {
    // ================= loads: key tiles (TMA) and their scale words =================
    // words of tile it: keys lane + 32 c (4-byte aligned: a sequence may start anywhere)
    auto sf_load = [&](int it, uint32_t (&w)[4]) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = (t_begin + it) * kKeys + lane + 32 * c;
        w[c] = j < n_ent ? __ldg(reinterpret_cast<const uint32_t*>(a.k_scale + (kbase + j) * 4)) : 0u;
      }
    };
    // the scale words travel four tiles ahead of their key tile, in a register ring (slot
    // = tile % 4), so no iteration waits for a load it has just issued
    uint32_t sfw[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (u < n_tiles) sf_load(u, sfw[u]);
    bool go = true;
    int issued = 0;  // key tiles whose bulk copy this warp started
    for (int it0 = 0; go && it0 < n_tiles; it0 += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int it = it0 + u;
        if (it >= n_tiles) break;
        const int s = it % kStages;
        const int t = t_begin + it;
        if (it >= kStages && !__all_sync(0xffffffffu, wait(&bars.kempty[s], ((it / kStages) - 1) & 1))) {
          go = false;
          break;
        }
        const uint32_t full = su32(&bars.kfull[s]);
        if (lane == 0) {
          mbar_expect_tx(full, kTileB);
          tma_tile2d(su32(As + s * kTileB), &tk, 0, static_cast<int>(kbase + static_cast<int64_t>(t) * kKeys), full);
        }
        *reinterpret_cast<uint4*>(SFs + s * kKeys + 4 * lane) = make_uint4(sfw[u][0], sfw[u][1], sfw[u][2], sfw[u][3]);
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // the tensor core reads them
        mbar_arrive(full);
        ++issued;
        if (it + 4 < n_tiles) sf_load(it + 4, sfw[u]);
      }
    }
    // every copy this warp started has landed before the CTA goes on (after an abort the
    // shared memory it writes is reused, then released): the last copy into each stage
    if (lane == 0)
      for (int it = max(0, issued - kStages); it < issued; ++it) drain(&bars.kfull[it % kStages], (it / kStages) & 1);
    __syncwarp();
  } else if (warp == 1) {
    // ================= MMA issue (one lane) =================
    if (lane == 0) {
      // E2M1 x E2M1, E8M0 scales, FP32 accumulate, M = 128, N
      const uint32_t idesc0 = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
                              (static_cast<uint32_t>(kKeys >> 4) << 24);
      bool ok = wait(&bars.bfull, 0);
      for (int it = 0; ok && it < n_tiles; ++it) {
        const int s = it % kStages, slot = it % kDBuf, sfs = it & 1;
        ok = wait(&bars.kfull[s], (it / kStages) & 1) &&
             (it < kDBuf || wait(&bars.dempty[slot], ((it / kDBuf) - 1) & 1));
        if (!ok) break;
        fence_after();
        // the tile's key scales: 32 rows of 16 bytes -> lanes 0..31 of every quadrant,
        // columns col_sfa + 8 sfs .. + 3
        {
          uint64_t d = static_cast<uint64_t>((su32(SFs + s * kKeys) >> 4) & 0x3FFF);
          d |= static_cast<uint64_t>(16 >> 4) << 16;   // LBO (one 16-byte column)
          d |= static_cast<uint64_t>(128 >> 4) << 32;  // SBO: next 8 rows
          d |= static_cast<uint64_t>(1) << 46;
          asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n" ::"r"(tm + col_sfa + 8u * sfs), "l"(d));
        }
        const uint32_t a_base = su32(As + s * kTileB), b_base = su32(Bs);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint32_t sfid = 2u * k;
          const uint32_t idesc = idesc0 | (sfid << 29) | (sfid << 4);
          asm volatile(
              "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
              "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(
                  tm + static_cast<uint32_t>(slot * N)),
              "l"(sw64_desc(a_base + k * 32)), "l"(sw64_desc(b_base + k * 32)), "r"(idesc), "r"(k),
              "r"((tm + col_sfa + 8u * sfs) | (sfid << 30)), "r"((tm + col_sfb) | (sfid << 30)));
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
            su32(&bars.dfull[slot])));
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
            su32(&bars.kempty[s])));
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
          su32(&bars.fin)));
      drain(&bars.fin, 0);  // every MMA and scale copy complete before tensor memory is released
    }
  } else {
    // ================= warps 2-5: key scales into tensor memory, epilogue =================
    const int et = tid - 64;                          // 0..127
    const int quad = warp & 3;                        // tensor-memory lane quadrant of this warp
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int row = quad * 32 + lane;                 // key row of D this thread reads
    // the indexer queries may be the previous kernel's output (programmatic dependent
    // launch): the key tiles above stream in meanwhile
    if (a.pdl) pdl_wait();
    // query operand (rows n = i * H + h), head weights, query scales
    if (a.fmt == LC_IDX_MXFP4_QBF16) {
      // the BF16 query rows quantised here, by the rule of the standalone quantiser: a warp
      // takes a row of 128 dims, 4 per lane, into the operand's SW64 layout
      for (int n = et >> 5; n < N; n += 4) {
        const int i = n / H, h = n % H;
        const int q = s_q[i];
        const bool ok = q < a.n_q && s_nv[i] > 0;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (ok) {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(a.q) +
                                                               (static_cast<int64_t>(q) * H + h) * kDI) + lane);
          v[0] = __uint_as_float(u.x << 16);
          v[1] = __uint_as_float(u.x & 0xffff0000u);
          v[2] = __uint_as_float(u.y << 16);
          v[3] = __uint_as_float(u.y & 0xffff0000u);
        }
        uint32_t sc;
        const uint32_t c = mxfp4_quant4(v, &sc);
        *reinterpret_cast<uint16_t*>(Bs + sw64_off(n, lane >> 3) + 2 * (lane & 7)) = static_cast<uint16_t>(c);
        // the row's scale word: block b's byte from lane 8 b
        const uint32_t w = __shfl_sync(0xffffffffu, sc, 0) | (__shfl_sync(0xffffffffu, sc, 8) << 8) |
                           (__shfl_sync(0xffffffffu, sc, 16) << 16) | (__shfl_sync(0xffffffffu, sc, 24) << 24);
        if (lane == 0) s_qsw[n] = ok ? w : 0x7f7f7f7fu;
      }
    } else {
      for (int c = et; c < N * 4; c += 128) {
        const int n = c >> 2, seg = c & 3;
        const int i = n / H, h = n % H;
        const int q = s_q[i];
        const bool ok = q < a.n_q && s_nv[i] > 0;
        const uint8_t* src = static_cast<const uint8_t*>(a.q) + (static_cast<int64_t>(ok ? q : 0) * H + h) * kRowB + seg * 16;
        cp_async16(su32(Bs + sw64_off(n, seg)), src, ok);
      }
    }
    for (int u = et; u < N; u += 128) {
      const int i = u / H, h = u % H;
      ws[u] = __ldg(a.w + static_cast<int64_t>(s_q[i] < a.n_q ? s_q[i] : 0) * a.w_qstride + h);
    }
    if (a.fmt == LC_IDX_MXFP4_QBF16) named_bar(1, 128);  // every row's scale word is in s_qsw
    {
      uint32_t v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int n = lane + 32 * c;
        uint32_t w = 0x7f7f7f7fu;
        if (n < N) {
          if (a.fmt == LC_IDX_MXFP4_QBF16) {
            w = s_qsw[n];
          } else {
            const int i = n / H, h = n % H;
            const int q = s_q[i];
            if (q < a.n_q) w = __ldg(reinterpret_cast<const uint32_t*>(a.q_scale) + static_cast<int64_t>(q) * H + h);
          }
        }
        v[c] = w;
      }
      tmem_st4(tm + lane_off + col_sfb, v[0], v[1], v[2], v[3]);
      if (N > 128) tmem_st4(tm + lane_off + col_sfb + 4, v[4], v[5], v[6], v[7]);
      asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    fence_before();
    mbar_arrive(su32(&bars.bfull));
    __syncwarp();

    // head weights in registers when one query's heads fill the accumulator (H <= 64);
    // the other epilogue warps wrote part of them: wait for all 128 arrivals first
    const bool weights_ok = __all_sync(0xffffffffu, wait(&bars.bfull, 0));
    // SELECT: the range of this thread's valid order keys, kept while the scores come in
    uint32_t sel_kmin = 0xffffffffu, sel_kmax = 0u;
    float wr[64];
    if (QPC == 1) {
#pragma unroll
      for (int k = 0; k < 64; ++k) wr[k] = k < H ? ws[k] : 0.f;
    }
    auto epilogue = [&](int u) -> bool {
      const int slot = u % kDBuf;
      if (!__all_sync(0xffffffffu, wait(&bars.dfull[slot], (u / kDBuf) & 1))) return false;
      fence_after();
      const int j = (t_begin + u) * kKeys + row;
#pragma unroll
      for (int i = 0; i < QPC; ++i) {
        // 8 partial sums (independent FMA chains), added in a fixed order
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int h0 = 0; h0 < H; h0 += 64) {  // H is a multiple of 32, at most 64 here
          uint32_t v[64];
          const uint32_t ta = tm + lane_off + static_cast<uint32_t>(slot * N + i * H + h0);
          const int nh = min(64, H - h0);
          tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          if (nh > 32) tmem_ld32(ta + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
          for (int k = 0; k < 64; ++k)
            if (k < nh) {
              const float w = QPC == 1 ? wr[k] : ws[i * H + h0 + k];
              acc[k & 7] = fmaf(w, fmaxf(__uint_as_float(v[k]), 0.f), acc[k & 7]);
            }
        }
        const float s = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        if constexpr (SELECT) {
          // the order key in place of the score; the selection below reads only keys
          const uint32_t kk = order_key(s);
          reinterpret_cast<uint32_t*>(sc)[u * kKeys + row] = kk;
          if (j < s_nv[0]) {
            sel_kmin = min(sel_kmin, kk);
            sel_kmax = max(sel_kmax, kk);
          }
        }
        else if (j < s_nv[i]) a.scores[static_cast<int64_t>(s_q[i]) * a.score_stride + j] = s;
      }
      fence_before();
      mbar_arrive(su32(&bars.dempty[slot]));
      return true;
    };
    for (int u = 0; weights_ok && u < n_tiles; ++u)
      if (!epilogue(u)) break;

    if constexpr (SELECT) {
      // ================= the range's top K (128 threads; the key ring is idle) =================
      // scratch in the idle key ring (dynamic shared memory, so that the static part stays
      // small enough for two CTAs per SM)
      uint32_t* hist4 = reinterpret_cast<uint32_t*>(As);  // [4][kSelBins] per-warp histograms
      int* s_pre = reinterpret_cast<int*>(hist4 + 4 * kSelBins);                   // [kSelMaxTiles * 4]
      uint32_t* list_key = reinterpret_cast<uint32_t*>(s_pre + kSelMaxTiles * 4);  // [kSmallBin]
      int* list_off = reinterpret_cast<int*>(list_key + kSmallBin);                // [kSmallBin]
      uint32_t (*s_rng)[4] = reinterpret_cast<uint32_t (*)[4]>(list_off + kSmallBin);  // [2][4]
      int* s_tmp = reinterpret_cast<int*>(s_rng + 2);     // [4]
      int* s_pick = s_tmp + 4;                            // [3]
      int* s_cnt = s_pick + 3;                            // [1]
      uint32_t* s_thr = reinterpret_cast<uint32_t*>(s_cnt + 1);  // [2]: Tk, Ts
      const int q = s_q[0];
      const int jbase = t_begin * kKeys;
      const int n_valid = max(0, min(s_nv[0] - jbase, n_tiles * kKeys));
      const int K = min(sel.k, n_valid);
      // the valid offsets are a prefix of the range: this thread's are u * 128 + row, u < nu
      const int nu = n_valid > row ? (n_valid - row + kKeys - 1) / kKeys : 0;
      // the order keys (written in place of the scores by the epilogue).  The loops below
      // stay short: this code runs once per launch, and a taken branch into code not yet
      // fetched stalls on the instruction fetch, so loops unrolled with guarded bodies cost
      // far more here than they save
      const uint32_t* key_s = reinterpret_cast<const uint32_t*>(sc);
      auto key = [&](int u) { return key_s[u * kKeys + row]; };
      uint32_t kmin = sel_kmin, kmax = sel_kmax;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
      }
      if (lane == 0) {
        s_rng[0][quad] = kmin;
        s_rng[1][quad] = kmax;
      }
      if (row == 0) {
        *s_cnt = 0;
        s_thr[0] = 0u;           // every valid key is taken unless a threshold is found
        s_thr[1] = 0x7fffffffu;
      }
      if (K < n_valid) {
        uint4* h4 = reinterpret_cast<uint4*>(hist4);
        for (int i = row; i < kSelBins; i += 128) h4[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      named_bar(1, 128);
      const uint32_t umin = min(min(s_rng[0][0], s_rng[0][1]), min(s_rng[0][2], s_rng[0][3]));
      const uint32_t umax = max(max(s_rng[1][0], s_rng[1][1]), max(s_rng[1][2], s_rng[1][3]));
      // The selection is the pair (Tk, Ts): the K-th largest key and the offset of the last
      // selected key equal to it; offset o is taken iff key > Tk, or key == Tk and o <= Ts.
      // Radix passes of 11 bits over rel = key - umin (histograms kept per warp, summed per
      // bin) narrow the bin of the K-th key until it holds at most kSmallBin keys, usually
      // after one pass; those are ranked exactly (key descending, offset ascending).  A bin
      // of more than kSmallBin equal keys is ranked in offset order.
      if (K < n_valid) {
        uint32_t pfx = 0;
        int rem = K, in_bin = n_valid;
        int shift = 32 - __clz(static_cast<int>(umax - umin));
        bool zeroed = true;
#pragma unroll 1
        while (in_bin > kSmallBin && shift > 0) {
          const int w = min(11, shift);
          const int hi = shift;
          shift -= w;
          const uint32_t bmask = (1u << w) - 1u;
          if (!zeroed) {
            uint4* h4 = reinterpret_cast<uint4*>(hist4);
            for (int i = row; i < kSelBins; i += 128) h4[i] = make_uint4(0u, 0u, 0u, 0u);
            named_bar(1, 128);
          }
          zeroed = false;
#pragma unroll 4
          for (int u = 0; u < nu; ++u) {
              const uint32_t rel = key(u) - umin;
              if ((hi >= 32 ? 0u : rel >> hi) == pfx) atomicAdd(&hist4[quad * kSelBins + ((rel >> shift) & bmask)], 1u);
            }
          named_bar(1, 128);
          // descending: thread `row` owns bins 2047 - 16 row - i, i < 16
          int c[16], sum = 0;
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            const int b0 = kSelBins - 16 * row - 4 * i4 - 4;  // bins b0 .. b0 + 3
            uint4 t = reinterpret_cast<const uint4*>(hist4)[b0 / 4];
#pragma unroll
            for (int w4 = 1; w4 < 4; ++w4) {
              const uint4 x = reinterpret_cast<const uint4*>(hist4 + w4 * kSelBins)[b0 / 4];
              t.x += x.x;
              t.y += x.y;
              t.z += x.z;
              t.w += x.w;
            }
            c[4 * i4] = static_cast<int>(t.w);
            c[4 * i4 + 1] = static_cast<int>(t.z);
            c[4 * i4 + 2] = static_cast<int>(t.y);
            c[4 * i4 + 3] = static_cast<int>(t.x);
            sum += c[4 * i4] + c[4 * i4 + 1] + c[4 * i4 + 2] + c[4 * i4 + 3];
          }
          int tot;
          int run = scan128(sum, quad, lane, s_tmp, &tot);
          if (run < rem && run + sum >= rem) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (run < rem && run + c[i] >= rem) {
                s_pick[0] = kSelBins - 1 - 16 * row - i;
                s_pick[1] = rem - run;
                s_pick[2] = c[i];
              }
              run += c[i];
            }
          }
          named_bar(1, 128);
          pfx = (pfx << w) | static_cast<uint32_t>(s_pick[0]);
          rem = s_pick[1];
          in_bin = s_pick[2];
        }
        if (in_bin <= kSmallBin) {
#pragma unroll 4
          for (int u = 0; u < nu; ++u)
            if (shift >= 32 || ((key(u) - umin) >> shift) == pfx) {
              const int i = atomicAdd(s_cnt, 1);
              if (i < kSmallBin) {  // exactly in_bin keys arrive here
                list_key[i] = key(u);
                list_off[i] = u * kKeys + row;
              }
            }
          named_bar(1, 128);
          for (int i = row; i < in_bin; i += 128) {
            const uint32_t ki = list_key[i];
            const int oi = list_off[i];
            int r = 0;
            for (int j = 0; j < in_bin; ++j) {
              const uint32_t kj = list_key[j];
              r += kj > ki || (kj == ki && list_off[j] < oi);
            }
            if (r == rem - 1) {
              s_thr[0] = ki;
              s_thr[1] = static_cast<uint32_t>(oi);
            }
          }
        } else {
          // every key of the bin equals T: the rem-th of them in offset order (tile, then row)
          const uint32_t T = umin + pfx;
#pragma unroll 1
          for (int u = 0; u < n_tiles; ++u) {
              const uint32_t bal = __ballot_sync(0xffffffffu, u < nu && key(u) == T);
              if (lane == 0) s_pre[u * 4 + quad] = __popc(bal);
            }
          named_bar(1, 128);
          int eq_before = 0;
#pragma unroll 1
          for (int u = 0; u < n_tiles; ++u) {
              const bool eq = u < nu && key(u) == T;
              int rank = eq_before + __popc(__ballot_sync(0xffffffffu, eq) & ((1u << lane) - 1u));
#pragma unroll
              for (int w = 0; w < 4; ++w) rank += w < quad ? s_pre[u * 4 + w] : 0;
              if (eq && rank == rem - 1) {
                s_thr[0] = T;
                s_thr[1] = static_cast<uint32_t>(u * kKeys + row);
              }
              eq_before += s_pre[u * 4] + s_pre[u * 4 + 1] + s_pre[u * 4 + 2] + s_pre[u * 4 + 3];
            }
          named_bar(1, 128);  // s_pre is reused below
        }
        named_bar(1, 128);
      }
      const uint32_t Tk = s_thr[0];
      const int Ts = static_cast<int>(s_thr[1]);
      // output positions in offset order: the selected keys of each (tile, warp), then a
      // scan over the (tile, warp) counts in that order
      uint64_t picks = 0;  // bit u: this thread's key of tile u is selected
#pragma unroll 4
      for (int u = 0; u < n_tiles; ++u) {
          const int off = u * kKeys + row;
          const bool pick = u < nu && (key(u) > Tk || (key(u) == Tk && off <= Ts));
          picks |= static_cast<uint64_t>(pick) << u;
          const uint32_t bal = __ballot_sync(0xffffffffu, pick);
          if (lane == 0) s_pre[u * 4 + quad] = __popc(bal);
        }
      named_bar(1, 128);
      {
        const int ne = n_tiles * 4;  // <= 256: two entries per thread
        const int e0 = 2 * row;
        const int v0 = e0 < ne ? s_pre[e0] : 0, v1 = e0 + 1 < ne ? s_pre[e0 + 1] : 0;
        int tot;
        const int ex = scan128(v0 + v1, quad, lane, s_tmp, &tot);
        if (e0 < ne) s_pre[e0] = ex;
        if (e0 + 1 < ne) s_pre[e0 + 1] = ex + v0;
      }
      named_bar(1, 128);
      const bool alone = sel.n_chunks == 1;
      int32_t* out_idx = alone ? sel.idx + static_cast<int64_t>(q) * sel.k : nullptr;
      uint2* out_c = alone ? nullptr : sel.cand + (static_cast<int64_t>(q) * sel.n_chunks + blockIdx.y) * sel.k;
      const uint32_t lt = (1u << lane) - 1u;
#pragma unroll 4
      for (int u = 0; u < n_tiles; ++u) {
          const bool pick = (picks >> u) & 1u;
          const uint32_t bal = __ballot_sync(0xffffffffu, pick);
          const int pos = s_pre[u * 4 + quad] + __popc(bal & lt);
          if (pick && pos < K) {  // exactly K keys are picked; the guard only matters after a timeout
            const int off = u * kKeys + row;
            if (alone) out_idx[pos] = jbase + off;
            else out_c[pos] = make_uint2(key(u), static_cast<uint32_t>(jbase + off));
          }
        }
      if (alone) {
        for (int i = K + row; i < sel.k; i += 128) out_idx[i] = -1;
        if (row == 0 && sel.count) sel.count[q] = K;
      } else if (row == 0) {
        sel.cand_cnt[static_cast<int64_t>(q) * sel.n_chunks + blockIdx.y] = K;
      }
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tm), "r"(tmem_cols));
}

namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_tiled() {
  static EncodeTiled fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiled>(nullptr);
    return reinterpret_cast<EncodeTiled>(f);
  }();
  return fn;
}

}  // namespace

// Launch shape of the indexer: one query per CTA, each query's keys split into ranges of
// tpc tiles so that the CTAs fill the SMs once in decode (prefill: ranges of 32 tiles).
IndexGeom index_geometry(const lc_index_args& a, bool decode, bool select) {
  IndexGeom g{};
  const int N = a.H_I;
  g.tmem_cols = 32;
  while (g.tmem_cols < static_cast<uint32_t>(kDBuf * N + 24)) g.tmem_cols <<= 1;
  g.tiles = (a.max_ent + kKeys - 1) / kKeys;
  const int per_sm = static_cast<int>(512 / g.tmem_cols);
  if (decode) {
    const int want = max(1, (per_sm * sm_count()) / max(a.n_q, 1));
    g.tpc = max(4, (g.tiles + want - 1) / want);
  } else {
    g.tpc = max(1, min(g.tiles, 32));
  }
  if (select) g.tpc = min(g.tpc, kSelMaxTiles);
  g.tpc = max(g.tpc, 1);
  g.n_chunks = max(1, (g.tiles + g.tpc - 1) / g.tpc);
  size_t sm = static_cast<size_t>(kStages) * kTileB + static_cast<size_t>(N) * kRowB + kStages * kKeys * 4 +
              static_cast<size_t>(N) * 4 + 1024;
  if (select) sm += static_cast<size_t>(g.tpc) * kKeys * 4;
  // no more CTAs per SM than its 512 tensor-memory columns hold, so tcgen05.alloc never
  // waits for another CTA (and no fewer: the static shared memory and the per-CTA
  // reservation fit in the 3 KB left per CTA)
  const size_t cap = 227 * 1024 / per_sm - 3072;
  g.smem = sm < cap ? cap : sm;
  return g;
}

namespace {

bool make_key_map(CUtensorMap* tk, const lc_index_args& a) {
  const EncodeTiled enc = encode_tiled();
  if (!enc) return false;
  // the key codes as a [n_keys, 64 B] tensor; 128-row boxes, 64-byte swizzle; rows past
  // n_keys read as zeros
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kRowB), static_cast<cuuint64_t>(a.n_keys)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kRowB)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kRowB), static_cast<cuuint32_t>(kKeys)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.k), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_index_tc(const lc_index_args& a, bool decode, cudaStream_t st) {
  CUtensorMap tk;
  if (!make_key_map(&tk, a)) return cudaErrorInvalidValue;
  const IndexGeom g = index_geometry(a, decode, false);
  const dim3 grid(a.n_q, g.n_chunks);
  IdxSelect none{};
  cudaFuncSetAttribute(k_index_tc<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(g.smem));
  return launch_ex(k_index_tc<1, false>, grid, dim3(kThreads), g.smem, st, a.pdl != 0, 1, tk, a, g.tpc, g.tmem_cols,
                   decode ? 1 : 0, none);
}

size_t index_topk_workspace(const lc_index_topk_args& a, bool decode) {
  const IndexGeom g = index_geometry(a.index, decode, true);
  if (g.n_chunks <= 1) return 0;
  const size_t rows = static_cast<size_t>(a.index.n_q) * g.n_chunks;
  return (rows * 4 + 15) / 16 * 16 + rows * a.k * sizeof(uint2);
}

cudaError_t launch_index_topk(const lc_index_topk_args& a, bool decode, cudaStream_t st) {
  CUtensorMap tk;
  if (!make_key_map(&tk, a.index)) return cudaErrorInvalidValue;
  const IndexGeom g = index_geometry(a.index, decode, true);
  IdxSelect sel{};
  sel.k = a.k;
  sel.n_chunks = g.n_chunks;
  sel.idx = a.idx;
  sel.count = a.count;
  if (g.n_chunks > 1) {
    const size_t rows = static_cast<size_t>(a.index.n_q) * g.n_chunks;
    sel.cand_cnt = static_cast<int*>(a.workspace);
    sel.cand = reinterpret_cast<uint2*>(static_cast<uint8_t*>(a.workspace) + (rows * 4 + 15) / 16 * 16);
  }
  const dim3 grid(a.index.n_q, g.n_chunks);
  cudaFuncSetAttribute(k_index_tc<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(g.smem));
  cudaError_t e = launch_ex(k_index_tc<1, true>, grid, dim3(kThreads), g.smem, st, a.index.pdl != 0, 1, tk, a.index,
                            g.tpc, g.tmem_cols, decode ? 1 : 0, sel);
  if (e != cudaSuccess || g.n_chunks == 1) return e;
  return launch_topk_merge(a, g.n_chunks, sel.cand, sel.cand_cnt, decode, st);
}

}  // namespace lc
