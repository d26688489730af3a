// CSA sparse / HCA dense attention on the 5th-generation tensor cores (tcgen05, F16 operands,
// FP32 accumulators).
//
// Same mathematics as k_attn.cu ("解读 DeepSeek V4": CSA attends to its top-k compressed
// entries, HCA to all of them, both plus a 128-token window and a per-head sink; V = K =
// the 576-dim entry; "DeepSeek-V4 论文分析" §5.4, §六, §七).  A CTA holds 64 heads of one
// query (they share every key: MQA) and a contiguous range of that query's key slots.
//
// Tiles and tensor memory:
//   * 64-row tiles (the queries' heads, or 64 keys) in shared memory as a grid of 8 x 8
//     F16 core matrices, row group g and dim chunk c at g * 9216 + c * 128.  The same key
//     bytes are the K-major B operand of S = Q K^T and the MN-major A operand V^T of
//     O^T = V^T P^T.  Rows arrive by cp.async: BF16 parts straight into their chunk slots,
//     the E4M3 nope part (16 dims = 16 bytes per piece) raw into the slot of the piece's
//     second chunk.  A conversion pass then widens E4M3 to F16 in place (exact) and rounds
//     BF16 to F16 in place (exact for magnitudes in [2^-14, 65504], which RMS-normalised
//     rows stay within; a value beyond 65504 is reported as LC_DEV_RANGE).  F16 rather than
//     BF16 operands give P 11 significant bits instead of 8.  Dense prefill, given the
//     workspace for it, widens the entries once per call into tiles of this layout
//     (k_attn_f16_tiles); a tile of 64 visible entries is then one bulk copy;
//   * S = Q K^T: M = 64 heads, N = 64 keys, K = 576, two tensor-memory buffers (M = 64
//     layout: row r in lane 32 (r / 16) + r % 16; the 16x32bx2 load gives lanes 0-15 of a
//     warp columns 0-31 and lanes 16-31 columns 32-63 of the same rows);
//   * P = 2^(x - m_h), x = scale * log2(e) * S, with a per-head reference m_h that moves up
//     only when a tile's maximum exceeds it by more than 8; O^T is then rescaled in tensor
//     memory (rare after the first tile: P stays below 2^8).  Masked keys get P = 0.  The
//     row sums add up the F16-rounded P that the MMA multiplies;
//   * O^T = V^T P^T accumulates in tensor memory, dims on lanes: chunks of 128 dims
//     (M = 128) and a last chunk of 64 (M = 64), 64 head columns each.
// The sink joins at the end: M = max(sink, m), Z = e^(sink - M) + l e^(m - M),
// o = O e^(m - M) / Z, lse = M + ln Z.  The output block of a CTA (64 consecutive rows)
// is staged in the freed key stages and written by one bulk copy.  A query's keys may be
// split across CTAs; each split then writes (O, m, l) and k_attn_combine merges them.
//
// Warp roles (320 threads): warps 0-3 load Q, turn S into P and write the output (each
// reaches its own quarter of the tensor-memory lanes); warps 4-7 gather key tiles into a
// two-stage ring; lane 0 of warp 8 issues the S MMAs and lane 0 of warp 9 the O MMAs.  At
// these shapes the tensor pipe takes an MMA in about 35 cycles, but one thread issues one
// only every ~53, so two issuers overlap that cost.  The roles meet only at mbarriers and
// named barriers, and every mbarrier wait is bounded: a role that gives up sets
// LC_DEV_TIMEOUT and an abort flag that stops the others at their next wait; copies and
// MMAs already in flight are waited for (bounded) before the CTA exits.
#include "lc_internal.h"
#include "lc_ptx.cuh"

namespace lc {

namespace {

constexpr int kD = 576;
constexpr int kDR = 64;                   // RoPE dims of the rows this kernel takes
constexpr int kDN = kD - kDR;             // nope dims (E4M3 in E4M3 rows)
constexpr int kTK = 64;                   // keys per tile
constexpr int kNR = 64;                   // heads per CTA
constexpr int kG = 72 * 128;              // bytes per group of 8 rows (72 dim chunks)
constexpr int kTile = 8 * kG;             // bytes of a 64-row tile (Q or keys): 73,728
constexpr int kPBytes = kNR * kTK * 2;    // P^T tile: 8,192
constexpr int kNP = kDN / 16 + kDR / 8;   // pieces per row: 32 nope pieces + 8 RoPE chunks
constexpr int kPI = kNP / 4;              // warp instructions per row group (4 pieces each)
constexpr int kNPair = kD / 16;           // chunk pairs per row (36)
constexpr int kWI = kNPair / 4;           // conversion warp instructions per row group
constexpr long kSpin = 1L << 26;
constexpr uint32_t kWin = 1u << 30;
constexpr int kThreads = 320;
constexpr float kRescale = 8.f;           // log2 headroom before the reference moves
constexpr int kColS = 0;                  // S buffers at columns 0 and 64
constexpr int kColO = 2 * kTK;            // O^T chunk c at 128 + 64 c
constexpr uint32_t kTmemCols = 512;
static_assert(kNP % 4 == 0 && kNPair % 4 == 0 && (kDN / 16) % 4 == 0, "piece grouping");

constexpr size_t kSmem = 3 * static_cast<size_t>(kTile) + kPBytes + 2 * kTK * 4 + kNR * 4;

// 8 E4M3 values -> 8 F16 values, exact (E4M3 is a subset of F16)
__device__ __forceinline__ uint4 e4m3x8_f16x8(uint32_t lo, uint32_t hi) {
  uint32_t o[4];
  const uint32_t w[2] = {lo, hi};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[j] & 0xffffu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[j] >> 16), __NV_E4M3);
    o[2 * j] = static_cast<uint32_t>(a.x) | (static_cast<uint32_t>(a.y) << 16);
    o[2 * j + 1] = static_cast<uint32_t>(b.x) | (static_cast<uint32_t>(b.y) << 16);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// 8 BF16 values -> 8 F16 values (round to nearest; exact for magnitudes in [2^-14, 65504]
// with at most 11 significant bits, which covers every BF16 value there).  `big` is set
// when a value leaves the F16 range.
__device__ __forceinline__ uint4 bf16x8_f16x8(uint4 v, bool& big) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __half2 h = __floats2half2_rn(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u));
    o[j] = *reinterpret_cast<const uint32_t*>(&h);
    big |= ((o[j] & 0x7c00u) == 0x7c00u) | ((o[j] & 0x7c000000u) == 0x7c000000u);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// byte offset of dim chunk c (8 dims) of row r in a 64-row core-matrix tile
__device__ __forceinline__ uint32_t tile_off(int r, int c) { return (r >> 3) * kG + c * 128 + (r & 7) * 16; }

__device__ __forceinline__ void cp16(uint8_t* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(su32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit_wait() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_all;\n" ::: "memory");
}
__device__ __forceinline__ void zero16(uint8_t* dst) { *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0); }

struct RowSrc {  // a row set, by value (no address of a kernel parameter is taken)
  int fmt;
  const uint8_t* x;
  const uint8_t* rope;
};
__device__ __forceinline__ RowSrc row_src(const lc_rows& r) {
  return RowSrc{r.fmt, static_cast<const uint8_t*>(r.x), static_cast<const uint8_t*>(r.rope)};
}

// Piece p of a row: p < 32 = nope dims 16p .. 16p + 15 (chunks 2p, 2p + 1), p >= 32 = RoPE
// chunk p + 32.  One warp instruction covers the 8 rows of a row group and 4 consecutive
// pieces: quarter qq, lane w takes row w and piece 2 (qq / 2) + ((w / 4) ^ qq) % 2 of the
// four, so each quarter writes 8 x 16 bytes on distinct banks and each 32-byte sector of a
// source row is read whole by one instruction.
__device__ __forceinline__ int piece_off(int lane) {
  const int qq = lane >> 3, w = lane & 7;
  return 2 * (qq >> 1) + (((w >> 2) ^ qq) & 1);
}

// Copy phase of a 64-row tile (warp wi of nw).  A BF16 row and the RoPE chunks of an E4M3
// row land in their chunk slots; an E4M3 nope piece lands raw in the slot of its second
// chunk (widened by tile_widen).  row_of(r, src, row) gives row r's source (row < 0: zeros).
template <class RowOf>
__device__ __forceinline__ void tile_copy(uint8_t* tile, int wi, int nw, int lane, RowOf row_of) {
  const int off = piece_off(lane), w = lane & 7;
  for (int k = wi; k < 8 * kPI; k += nw) {
    const int g = k / kPI, p = (k % kPI) * 4 + off, r = g * 8 + w;
    RowSrc rs;
    int64_t row;
    row_of(r, rs, row);
    if (p < kDN / 16) {
      uint8_t* d0 = tile + tile_off(r, 2 * p);
      if (row < 0) {
        zero16(d0);
        zero16(d0 + 128);
      } else if (rs.fmt == LC_FMT_BF16) {
        const uint8_t* src = rs.x + (row * kD + p * 16) * 2;
        cp16(d0, src);
        cp16(d0 + 128, src + 16);
      } else {
        cp16(d0 + 128, rs.x + row * kDN + p * 16);
      }
    } else {
      const int c = p + kDN / 16;
      uint8_t* d0 = tile + tile_off(r, c);
      if (row < 0) zero16(d0);
      else if (rs.fmt == LC_FMT_BF16) cp16(d0, rs.x + (row * kD + c * 8) * 2);
      else cp16(d0, rs.rope + (row * kDR + (c * 8 - kDN)) * 2);
    }
  }
}

// Conversion phase, pair p of a row (chunks 2p, 2p + 1; pairs 32..35 hold the RoPE dims).
// kind(r): 0 = nothing (masked row), 1 = E4M3 row (pairs < 32 are raw E4M3 in the slot of
// their second chunk: widened in place; RoPE pairs are BF16: rounded to F16 in place),
// 2 = BF16 row (every pair rounded to F16 in place).  Each item reads its own slots before
// writing them: no hazard between items.  Four items per thread are loaded before any is
// converted.  Returns whether a BF16 value left the F16 range.
template <class KindOf>
__device__ __forceinline__ bool tile_convert(uint8_t* tile, int wi, int nw, int lane, KindOf kind_of) {
  const int off = piece_off(lane), w = lane & 7;
  bool big = false;
  for (int k0 = wi; k0 < 8 * kWI; k0 += 4 * nw) {
    uint4 v0[4], v1[4];
    uint8_t* d[4];
    int kd[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = k0 + j * nw;
      const int g = k / kWI, p = (k % kWI) * 4 + off, r = g * 8 + w;
      const int kr = k < 8 * kWI ? kind_of(r) : 0;
      // 1: widen raw E4M3, 2: round two BF16 chunks
      kd[j] = kr == 0 ? 0 : (kr == 1 && p < kDN / 16) ? 1 : 2;
      d[j] = tile + tile_off(r, 2 * p);
      if (kd[j] == 1) v1[j] = *reinterpret_cast<const uint4*>(d[j] + 128);
      if (kd[j] == 2) {
        v0[j] = *reinterpret_cast<const uint4*>(d[j]);
        v1[j] = *reinterpret_cast<const uint4*>(d[j] + 128);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (kd[j] == 1) {
        *reinterpret_cast<uint4*>(d[j]) = e4m3x8_f16x8(v1[j].x, v1[j].y);
        *reinterpret_cast<uint4*>(d[j] + 128) = e4m3x8_f16x8(v1[j].z, v1[j].w);
      } else if (kd[j] == 2) {
        *reinterpret_cast<uint4*>(d[j]) = bf16x8_f16x8(v0[j], big);
        *reinterpret_cast<uint4*>(d[j] + 128) = bf16x8_f16x8(v1[j], big);
      }
    }
  }
  return big;
}

__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n" ::"l"(gdst), "r"(su32(ssrc)),
               "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
  asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
}

// one contiguous global -> shared copy, completing `bytes` on the mbarrier (this CTA only)
__device__ __forceinline__ void bulk_load(uint8_t* sdst, const void* gsrc, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   su32(sdst)),
               "l"(gsrc), "r"(bytes), "r"(bar)
               : "memory");
}

}  // namespace

// Dense (HCA) prefill: every query of a sequence reads the same entry rows, so they are
// widened to F16 once per call rather than once per query.  Tile T of the image holds
// entry rows 64 T .. 64 T + 63 (zeros past n_rows) in the core-matrix layout that
// tile_copy + tile_convert leave in shared memory, with the same conversions, so a tile
// loaded from the image is byte for byte the tile a gather would build.  Thread i writes
// the 16 bytes at image offset 16 i: tile T, row group g, dim chunk c, row r8 of the group.
__global__ void __launch_bounds__(256) k_attn_f16_tiles(lc_rows ent, int n_rows, int n_tiles,
                                                         uint8_t* __restrict__ img, int32_t* status) {
  constexpr int kPer = kTile / 16;  // 16-byte items per tile
  const int64_t n_items = static_cast<int64_t>(n_tiles) * kPer;
  const uint8_t* x = static_cast<const uint8_t*>(ent.x);
  const uint8_t* rope = static_cast<const uint8_t*>(ent.rope);
  bool big = false;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_items;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int o = static_cast<int>(i % kPer);
    const int g = o / (8 * (kD / 8)), c = (o / 8) % (kD / 8), r8 = o % 8;
    const int64_t row = (i / kPer) * kTK + g * 8 + r8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row < n_rows) {
      if (ent.fmt == LC_FMT_BF16) {
        v = bf16x8_f16x8(__ldg(reinterpret_cast<const uint4*>(x + (row * kD + c * 8) * 2)), big);
      } else if (c < kDN / 8) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(x + row * kDN + c * 8));
        v = e4m3x8_f16x8(w.x, w.y);
      } else {
        v = bf16x8_f16x8(__ldg(reinterpret_cast<const uint4*>(rope + (row * kDR + (c * 8 - kDN)) * 2)), big);
      }
    }
    reinterpret_cast<uint4*>(img)[i] = v;
  }
  if (big) set_status(status, LC_DEV_RANGE);
}

struct AttnTcGeom {
  int n_split;
  int sps;  // slots per split, multiple of kTK
};

struct TcBars {
  uint64_t qfull;      // Q loaded (128 arrivals)
  uint64_t kfull[2];   // key stage ready (128 arrivals)
  uint64_t kempty[2];  // key stage read by O (commit)
  uint64_t sfull[2];   // S buffer computed (commit)
  uint64_t sempty[2];  // S buffer read (128 arrivals)
  uint64_t pfull;      // P written (128 arrivals)
  uint64_t pempty;     // P read and O updated (commit)
  uint64_t fin;        // every S MMA complete (commit)
  uint64_t fin2;       // every O MMA complete (commit)
};

// grid: one CTA per (query, head group, key split), the split index fastest; 320 threads.
// Partial results of split s go to ws_o rows s * n_q * H + q * H + h (576 floats each) and
// ws_ml[2 ((q * H + h) * n_split + s) + {0, 1}] = (m, l).  img (dense keys only, or null):
// the entries as F16 tiles (k_attn_f16_tiles), img_tiles of them; a tile of 64 visible
// entries that starts on a multiple of 64 in the entry array is then one bulk copy.
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_tc(lc_attn_args a, int sparse, AttnTcGeom geo, float* __restrict__ ws_o, float* __restrict__ ws_ml,
              const uint8_t* __restrict__ img, int img_tiles) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* Qs = smem;                                             // kTile
  uint8_t* Ks = Qs + kTile;                                       // [2][kTile]
  uint8_t* Ps = Ks + 2 * kTile;                                   // kPBytes
  int* kcode = reinterpret_cast<int*>(Ps + kPBytes);              // [2][kTK]
  float* s_f = reinterpret_cast<float*>(kcode + 2 * kTK);         // [kNR] per-head factors
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ __align__(8) TcBars bars;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (a.pdl) pdl_wait();  // the previous kernel's top-k indices (programmatic dependent launch)
  const int n_hg = a.dims.H / kNR;
  const int split = blockIdx.x % geo.n_split;
  const int hg = (blockIdx.x / geo.n_split) % n_hg;
  const int q = blockIdx.x / (geo.n_split * n_hg);
  const int H = a.dims.H;
  const int b = seq_of_query(a.batch.q_start, a.batch.num_seqs, q);
  const int p = __ldg(a.batch.q_pos0 + b) + (q - __ldg(a.batch.q_start + b));
  const int n_ent = __ldg(a.batch.n_ent + b);
  const int nv = n_visible(p, a.m, a.W_x, n_ent);
  const int64_t ent0 = __ldg(a.batch.ent_start + b);
  const int wlo = a.W > 0 ? max(0, p - a.W + 1) : p + 1;
  const int n_first = sparse ? a.k : nv;
  const int n_slots = n_first + (p + 1 - wlo);
  const int s_begin = split * geo.sps;
  const int s_end = min(n_slots, s_begin + geo.sps);
  const int n_tiles = s_end > s_begin ? (s_end - s_begin + kTK - 1) / kTK : 0;
  const int wp0 = a.W > 0 ? __ldg(a.batch.win_pos0 + b) : 0;
  const int wl = a.W > 0 ? __ldg(a.batch.win_len + b) : 0;
  const int64_t wr0 = a.W > 0 ? __ldg(a.batch.win_start + b) : 0;
  const int32_t* idx_row = sparse ? a.idx + static_cast<int64_t>(q) * a.k : nullptr;
  const int64_t row0 = static_cast<int64_t>(q) * H + hg * kNR;  // first output row of the CTA
  // values: all 576 dims (5 O^T chunks), or (v_nope) the 512 non-RoPE dims (chunks 0-3)
  const int n_och = a.v_nope ? 4 : 5;
  const int Dv = a.v_nope ? kDN : kD;

  // bounded wait; gives up (and tells the other roles) after kSpin polls
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const uint32_t addr = su32(bar);
    for (long it = 0; it < kSpin; ++it) {
      if (mbar_test(addr, parity)) return true;
      if ((it & 1023) == 1023 && *reinterpret_cast<volatile int*>(&s_abort)) return false;
    }
    set_status(a.status, LC_DEV_TIMEOUT);
    atomicExch(&s_abort, 1);
    return false;
  };
  // bounded wait that ignores the abort flag: for copies and MMAs already in flight, which
  // must land before the CTA releases its tensor memory and exits
  auto drain = [&](uint64_t* bar, uint32_t parity) {
    const uint32_t addr = su32(bar);
    for (long it = 0; it < kSpin; ++it)
      if (mbar_test(addr, parity)) return;
    set_status(a.status, LC_DEV_TIMEOUT);
  };
  // key slot -> entry index j, kWin | window row, or -1 (masked)
  auto slot_code = [&](int s) -> int {
    if (s >= s_end) return -1;
    if (s < n_first) {
      const int j = sparse ? __ldg(idx_row + s) : s;
      if (j < 0) return -1;
      if (j >= n_ent) {
        set_status(a.status, LC_DEV_BAD_INDEX);
        return -1;
      }
      if (j >= nv) {
        set_status(a.status, LC_DEV_NONVISIBLE);
        return -1;
      }
      return j;
    }
    const int t = wlo + (s - n_first);
    const int rr = t - wp0;
    if (rr < 0 || rr >= wl) {
      set_status(a.status, LC_DEV_WINDOW_RANGE);
      return -1;
    }
    // row of position t within the sequence's window rows (linear, or a ring buffer)
    return static_cast<int>(kWin) | (a.batch.win_ring > 0 ? t % a.batch.win_ring : rr);
  };

  // ---- set-up: tensor memory, barriers ----
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(&s_tmem)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 32) {
    s_abort = 0;
    mbar_init(su32(&bars.qfull), 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(su32(&bars.kfull[i]), 128);
      mbar_init(su32(&bars.kempty[i]), 1);
      mbar_init(su32(&bars.sfull[i]), 1);
      mbar_init(su32(&bars.sempty[i]), 128);
    }
    mbar_init(su32(&bars.pfull), 128);
    mbar_init(su32(&bars.pempty), 1);
    mbar_init(su32(&bars.fin), 1);
    mbar_init(su32(&bars.fin2), 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = s_tmem;

  if (warp >= 4 && warp < 8) {
    // ================= producers: gather + widen key tiles =================
    const int pt = tid - 128, pw = warp - 4;
    const RowSrc src_win = row_src(a.win), src_ent = row_src(a.ent);
    int code_next = pt < kTK ? slot_code(s_begin + pt) : -1;
    int last_bulk0 = -1, last_bulk1 = -1;  // thread pt = 0: the last tile of stage 0 / 1 it bulk-copied
    for (int t = 0; t < n_tiles; ++t) {
      const int st = t & 1;
      // stage st (and its key codes) is free once O(t - 2) is done: that also means the
      // softmax of tile t - 2 has read the codes
      const bool ok = t < 2 || wait(&bars.kempty[st], ((t >> 1) - 1) & 1);
      if (ok && pt < kTK) kcode[st * kTK + pt] = code_next;
      if (named_bar_or(2, 128, !ok)) break;  // the role stops as one
      if (pt < kTK && t + 1 < n_tiles) code_next = slot_code(s_begin + (t + 1) * kTK + pt);
      uint8_t* kt = Ks + st * kTile;
      const int* kc = kcode + st * kTK;
      // dense keys: slot s is entry s, so 64 visible entries from a multiple of 64 in the
      // entry array are one image tile
      const int s0 = s_begin + t * kTK;
      const int64_t e0 = ent0 + s0;
      if (img != nullptr && !sparse && s0 + kTK <= nv && e0 % kTK == 0 && e0 / kTK < img_tiles) {
        if (pt == 0) {
          mbar_expect_tx(su32(&bars.kfull[st]), kTile);  // this thread's arrival, plus the bytes
          bulk_load(kt, img + (e0 / kTK) * kTile, kTile, su32(&bars.kfull[st]));
          (st ? last_bulk1 : last_bulk0) = t;
        } else {
          mbar_arrive(su32(&bars.kfull[st]));
        }
        continue;
      }
      (st ? last_bulk1 : last_bulk0) = -1;  // stage st was released by O(t - 2): its copies have landed
      tile_copy(kt, pw, 4, lane, [&](int r, RowSrc& rs, int64_t& row) {
        const int code = kc[r];
        rs = (code & kWin) ? src_win : src_ent;
        row = code < 0 ? -1 : (code & kWin) ? wr0 + (code & ~kWin) : ent0 + code;
      });
      cp_commit_wait();
      named_bar(2, 128);
      if (tile_convert(kt, pw, 4, lane, [&](int r) {
            const int code = kc[r];
            return code < 0 ? 0 : (!(code & kWin) && src_ent.fmt == LC_FMT_E4M3_BF16) ? 1 : 2;
          }))
        set_status(a.status, LC_DEV_RANGE);
      fence_async_smem();
      mbar_arrive(su32(&bars.kfull[st]));
    }
    // a role that gave up may leave bulk copies in flight: they land (in bounded time,
    // from valid memory) before the CTA's shared memory is released
    if (pt == 0) {
      if (last_bulk0 >= 0) drain(&bars.kfull[0], (last_bulk0 >> 1) & 1);
      if (last_bulk1 >= 0) drain(&bars.kfull[1], (last_bulk1 >> 1) & 1);
    }
  } else if (warp == 8) {
    // ================= S MMA issue (one lane) =================
    if (lane == 0) {
      // F16 operands, FP32 accumulator.  S: M = 64, N = 64, both K-major
      const uint32_t id_s = (1u << 4) | (static_cast<uint32_t>(kTK >> 3) << 17) |
                            (static_cast<uint32_t>(kNR >> 4) << 24);
      const uint64_t dq = cm_desc(su32(Qs), 128, kG);
      // S(ns) once its key stage is full and its S buffer read; S runs at most two tiles
      // ahead of O (the key stage of S(no + 2) is released by O(no))
      bool ok = n_tiles == 0 || wait(&bars.qfull, 0);
      for (int ns = 0; ok && ns < n_tiles; ++ns) {
        const int st = ns & 1;
        ok = wait(&bars.kfull[st], (ns >> 1) & 1) && (ns < 2 || wait(&bars.sempty[st], ((ns >> 1) - 1) & 1));
        if (!ok) break;
        fence_after();
        const uint64_t dk = cm_desc(su32(Ks + st * kTile), 128, kG);
#pragma unroll
        for (int k = 0; k < kD / 16; ++k)
          mma_f16(tm + kColS + st * kTK, dq + k * 16, dk + k * 16, id_s, k > 0);
        mma_commit(su32(&bars.sfull[st]));
      }
      mma_commit(su32(&bars.fin));
      drain(&bars.fin, 0);  // every MMA issued above completes before tensor memory is released
    }
  } else if (warp == 9) {
    // ================= O MMA issue (one lane) =================
    if (lane == 0) {
      // O^T: M = 128 (or 64), N = 64, A (V^T) MN-major, P^T K-major
      const uint32_t id_o128 = (1u << 4) | (1u << 15) |
                               (static_cast<uint32_t>(kNR >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
      const uint32_t id_o64 = (1u << 4) | (1u << 15) |
                              (static_cast<uint32_t>(kNR >> 3) << 17) | (static_cast<uint32_t>(64 >> 4) << 24);
      const uint64_t dp = cm_desc(su32(Ps), 128, (kTK / 8) * 128);
      // O(no) once P(no) is written (its S is then complete)
      for (int no = 0; no < n_tiles; ++no) {
        if (!wait(&bars.pfull, no & 1)) break;
        fence_after();
        // V^T: M = dims (chunk stride 128 B), K = keys (group stride kG)
        const uint64_t dv = cm_desc(su32(Ks + (no & 1) * kTile), kG, 128);
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk)
#pragma unroll
          for (int c = 0; c < 5; ++c)
            if (c < n_och)
              mma_f16(tm + kColO + c * kNR, dv + (c * 2048 + kk * 2 * kG) / 16, dp + kk * 16,
                      c < 4 ? id_o128 : id_o64, (no > 0) || (kk > 0));
        mma_commit(su32(&bars.kempty[no & 1]));
        mma_commit(su32(&bars.pempty));
      }
      mma_commit(su32(&bars.fin2));
      drain(&bars.fin2, 0);  // every O MMA completes before tensor memory is released
    }
  } else {
    // ================= warps 0-3: Q, softmax, epilogue =================
    const int r = warp * 16 + (lane & 15);  // head row (tensor-memory lane 32 w + lane % 16)
    const int hf = lane >> 4;               // which 32 of a tile's 64 keys this thread takes
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale * 1.4426950408889634f;
    if (n_tiles > 0) {
      const RowSrc src_q = row_src(a.q);
      tile_copy(Qs, warp, 4, lane, [&](int rr, RowSrc& rs, int64_t& row) {
        rs = src_q;
        row = row0 + rr;
      });
      cp_commit_wait();
      named_bar(1, 128);
      const int qkind = src_q.fmt == LC_FMT_E4M3_BF16 ? 1 : 2;
      if (tile_convert(Qs, warp, 4, lane, [&](int) { return qkind; })) set_status(a.status, LC_DEV_RANGE);
      fence_async_smem();
      mbar_arrive(su32(&bars.qfull));
    }
    float m_ref = -INFINITY, l_sum = 0.f;  // m_ref is the same in both halves of a row
    bool good = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int st = t & 1;
      const bool okw = wait(&bars.sfull[st], (t >> 1) & 1) && wait(&bars.kfull[st], (t >> 1) & 1);
      if (named_bar_or(1, 128, !okw)) {  // the role stops as one
        good = false;
        break;
      }
      fence_after();
      uint32_t sv[32];
      tmem_ld16x2(tm + lane_off + kColS + st * kTK, sv);
      tmem_wait_ld();
      fence_before();
      mbar_arrive(su32(&bars.sempty[st]));
      const int* kc = kcode + st * kTK + 32 * hf;
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float x = kc[j] >= 0 ? __uint_as_float(sv[j]) * sl2 : -INFINITY;
        sv[j] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const bool need = mx > m_ref + kRescale;
      // P (single buffer) and O are free once O of the previous tile is done
      const bool okp = t == 0 || wait(&bars.pempty, (t - 1) & 1);
      if (named_bar_or(1, 128, !okp)) {
        good = false;
        break;
      }
      const bool any = named_bar_or(1, 128, need && t > 0);
      float f = 1.f;
      if (need) {
        f = m_ref == -INFINITY ? 0.f : exp2f(m_ref - mx);
        l_sum *= f;
        m_ref = mx;
      }
      if (any) {
        // rescale O^T columns (heads) in tensor memory: every lane of all 5 chunks
        if (hf == 0) s_f[r] = f;
        named_bar(1, 128);
        fence_after();
#pragma unroll 1
        for (int c = 0; c < n_och; ++c)
#pragma unroll 1
          for (int hh = 0; hh < kNR; hh += 32) {
            uint32_t ov[32];
            const uint32_t ta = tm + lane_off + kColO + c * kNR + hh;
            tmem_ld32(ta, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * s_f[hh + i]);
            tmem_st32(ta, ov);
          }
        tmem_wait_st();
        named_bar(1, 128);  // s_f is rewritten only after every lane used it
      }
      {
        uint32_t pk[16];
        const float mr = m_ref == -INFINITY ? 0.f : m_ref;  // a row with no key yet: all x = -inf
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          // masked keys: x = -inf, 2^-inf = 0
          const __half2 ph = __floats2half2_rn(ex2(__uint_as_float(sv[j]) - mr), ex2(__uint_as_float(sv[j + 1]) - mr));
          const float2 pf = __half22float2(ph);
          l_sum += pf.x + pf.y;
          pk[j / 2] = *reinterpret_cast<const uint32_t*>(&ph);
        }
        // P^T tile, K-major: head group (r / 8) stride 1024 B, key chunk stride 128 B
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(Ps + (r >> 3) * 1024 + (4 * hf + c) * 128 + (r & 7) * 16) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_async_smem();
      fence_before();
      mbar_arrive(su32(&bars.pfull));
    }
    // ---- epilogue ----
    if (good && n_tiles > 0) good = wait(&bars.pempty, (n_tiles - 1) & 1);
    good = !named_bar_or(1, 128, !good);  // uniform: the tensor-memory loads below are warp-wide
    fence_after();
    const float l_row = l_sum + __shfl_xor_sync(0xffffffffu, l_sum, 16);
    if (hf == 0) {
      const int h = hg * kNR + r;
      if (geo.n_split == 1) {
        const float sk = __ldg(a.sink + h) * 1.4426950408889634f;
        const float M = fmaxf(sk, m_ref);
        const float w = m_ref == -INFINITY ? 0.f : exp2f(m_ref - M);
        const float Z = exp2f(sk - M) + l_row * w;
        s_f[r] = w / Z;
        if (a.lse && good) a.lse[row0 + r] = (M + log2f(Z)) * 0.6931471805599453f;
      } else if (good) {
        const int64_t slot = (row0 + r) * geo.n_split + split;
        ws_ml[2 * slot] = m_ref;
        ws_ml[2 * slot + 1] = l_row;
      }
    }
    named_bar(1, 128);
    if (good) {
      // O rows -> the key stages (free: every MMA is complete), row-major [head][dim]
      const bool f32 = geo.n_split > 1 || a.out_fmt == LC_FMT_F32;
      float* stf = reinterpret_cast<float*>(Ks);
      uint16_t* sth = reinterpret_cast<uint16_t*>(Ks);
      const int ostr = geo.n_split > 1 ? kD : Dv;  // partial rows keep every dim
#pragma unroll 1
      for (int c = 0; c < n_och; ++c) {
        // chunk c < 4: lane L -> dim 128 c + L; chunk 4 (M = 64): lane 32 w + i -> dim 512 + 16 w + i
        const int dim = c < 4 ? c * 128 + warp * 32 + lane : (lane < 16 ? 512 + warp * 16 + lane : -1);
        uint32_t ov[kNR];  // the chunk's 64 head columns, one wait
        if (n_tiles > 0) {
          tmem_ld32(tm + lane_off + kColO + c * kNR, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
          tmem_ld32(tm + lane_off + kColO + c * kNR + 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < kNR; ++i) ov[i] = 0;
        }
        if (dim < 0) continue;
#pragma unroll
        for (int i = 0; i < kNR; ++i) {
          float v = __uint_as_float(ov[i]);
          if (geo.n_split == 1) v *= s_f[i];
          if (f32) stf[i * ostr + dim] = v;
          else sth[i * ostr + dim] = f32_to_bf16_bits(v);
        }
      }
      fence_async_smem();
      named_bar(1, 128);
      if (tid == 0) {
        const uint32_t bytes = kNR * ostr * (f32 ? 4 : 2);
        void* dst;
        if (geo.n_split > 1) dst = ws_o + (static_cast<int64_t>(split) * a.n_q * H + row0) * kD;
        else if (a.out_fmt == LC_FMT_F32) dst = static_cast<float*>(a.out) + row0 * Dv;
        else dst = static_cast<uint16_t*>(a.out) + row0 * Dv;
        bulk_store(dst, Ks, bytes);
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tm), "r"(kTmemCols));
}

// ---------------------------------------------------------------------------------
bool attn_tc_supported(const lc_attn_args& a) {
  if (a.dims.D != kD || a.dims.d_r != kDR || a.dims.H % kNR) return false;
  auto ok = [&](const lc_rows& r) {
    if (r.fmt != LC_FMT_BF16 && r.fmt != LC_FMT_E4M3_BF16) return false;
    if (reinterpret_cast<uintptr_t>(r.x) % 16) return false;
    return r.fmt == LC_FMT_BF16 || reinterpret_cast<uintptr_t>(r.rope) % 16 == 0;
  };
  if (!ok(a.q) || !ok(a.ent) || (a.W > 0 && (a.win.fmt != LC_FMT_BF16 || !ok(a.win)))) return false;
  if (reinterpret_cast<uintptr_t>(a.out) % 16 || reinterpret_cast<uintptr_t>(a.workspace) % 16) return false;
  return a.out_fmt == LC_FMT_BF16 || a.out_fmt == LC_FMT_F32;
}

static AttnTcGeom tc_geometry(const lc_attn_args& a, bool sparse, bool decode) {
  AttnTcGeom g{1, 0};
  const int ns = max((sparse ? a.k : a.max_ent) + a.W, 1);
  const int tiles = (ns + kTK - 1) / kTK;
  g.sps = tiles * kTK;
  const int ctas = a.n_q * (a.dims.H / kNR);
  const int n_sm = sm_count();
  if (decode && ctas < n_sm) {
    // one CTA per SM: split the keys when the (query, head group) pairs leave SMs idle
    const int n = max(1, min(n_sm / max(ctas, 1), tiles));
    const int per = (tiles + n - 1) / n;
    g.n_split = (tiles + per - 1) / per;
    g.sps = per * kTK;
  }
  return g;
}

size_t attn_tc_workspace(const lc_attn_args& a, bool sparse, bool decode) {
  const AttnTcGeom g = tc_geometry(a, sparse, decode);
  if (g.n_split <= 1) return 0;
  const size_t rows = static_cast<size_t>(a.n_q) * a.dims.H * g.n_split;
  return rows * kD * sizeof(float) + rows * 2 * sizeof(float);
}

// Dense prefill: the F16 image of every entry row (n_ent_rows of them, in 64-row tiles),
// built once per call; 0 where it does not apply (CSA, decode, n_ent_rows unknown).
size_t attn_tc_image_bytes(const lc_attn_args& a, bool sparse, bool decode) {
  if (sparse || decode || a.n_ent_rows <= 0) return 0;
  return static_cast<size_t>((a.n_ent_rows + kTK - 1) / kTK) * kTile;
}

cudaError_t launch_attn_tc(const lc_attn_args& a, bool sparse, bool decode, cudaStream_t st, int* n_split_out) {
  const AttnTcGeom g = tc_geometry(a, sparse, decode);
  *n_split_out = g.n_split;
  cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
  float* ws_o = static_cast<float*>(a.workspace);
  float* ws_ml = nullptr;
  if (g.n_split > 1) ws_ml = ws_o + static_cast<size_t>(a.n_q) * a.dims.H * g.n_split * kD;
  const int64_t ctas = static_cast<int64_t>(a.n_q) * (a.dims.H / kNR) * g.n_split;
  if (ctas > 0x7fffffff) return cudaErrorInvalidConfiguration;
  // the image, when the caller's workspace holds it (the prefill variant splits no keys, so
  // the workspace is otherwise unused)
  const size_t img_bytes = g.n_split == 1 ? attn_tc_image_bytes(a, sparse, decode) : 0;
  uint8_t* img = nullptr;
  int img_tiles = 0;
  if (img_bytes > 0 && a.workspace && a.workspace_bytes >= img_bytes &&
      reinterpret_cast<uintptr_t>(a.workspace) % 16 == 0) {
    img = static_cast<uint8_t*>(a.workspace);
    img_tiles = (a.n_ent_rows + kTK - 1) / kTK;
    const int64_t items = static_cast<int64_t>(img_tiles) * (kTile / 16);
    const int64_t want = (items + 255) / 256, cap = 8LL * sm_count();
    const int blocks = static_cast<int>(want < cap ? want : cap);
    k_attn_f16_tiles<<<blocks, 256, 0, st>>>(a.ent, a.n_ent_rows, img_tiles, img, a.status);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_ex(k_attn_tc, dim3(static_cast<unsigned>(ctas)), dim3(kThreads), kSmem, st, a.pdl != 0, 1, a,
                   sparse ? 1 : 0, g, ws_o, ws_ml, static_cast<const uint8_t*>(img), img_tiles);
}

}  // namespace lc
