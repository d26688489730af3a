// CSA sparse / HCA dense attention on the 5th-generation tensor cores with FP8 scores
// (tcgen05; for E4M3 + BF16-RoPE queries and entries, 576 dims, 64 RoPE dims).
//
// Same mathematics as k_attn.cu ("解读 DeepSeek V4": CSA attends to its top-k compressed
// entries, HCA to all of them, both plus a 128-token window and a per-head sink; V = K =
// the 576-dim entry; "DeepSeek-V4 论文分析" §5.4, §六, §七), and the same per-CTA split
// into (query, 64-head group, key range) as k_attn_tc.cu.  What differs is how keys reach
// the tensor core:
//   * entry tiles (64 keys) are gathered by bulk tensor copies (TMA tile::gather4, four rows
//     per copy) into 128-byte-swizzled shared tiles: the E4M3 nope part (4 blocks of 128
//     dims) and the BF16 RoPE part.  The scores of an entry tile need no conversion:
//     S = Qn Kn^T with E4M3 x E4M3 MMAs (kind::f8f6f4; each product is exact in FP32) plus
//     Qr Kr^T with BF16 x BF16 MMAs, both accumulating into one FP32 tensor-memory tile;
//   * V (= K) must be 16-bit for O += P V: converter warps widen each gathered tile to F16
//     (E4M3 -> F16 exact; BF16 -> F16 exact in [2^-14, 65504], else LC_DEV_RANGE) into a
//     core-matrix tile, the MN-major A operand of O^T = V^T P^T (M = 128 dims, a last chunk
//     of 64, N = 64 heads), while the scores of the next tile run;
//   * window tiles come first: their rows are consecutive, so each arrives by nine 2-D bulk
//     tensor copies into the V tile area while the raw stages hold Q converted to BF16;
//     S = Q K^T reads the landed BF16 tile (exact products in FP32), then the tile is
//     widened to F16 in place for O^T = V^T P^T, and the entry gathers begin once every
//     window S is done.
// Softmax, the per-head exponent reference, the sink and the outputs are those of
// k_attn_tc.cu (P in F16, 11 significant bits; row sums of the rounded P).
//
// Warp roles (416 threads): warps 0-3 turn S into P and write the output; warps 4-7
// convert tiles and bring in the window tiles; lane 0 of warp 8 issues the MMAs; warps
// 9-12 compute the key codes and issue the entry-tile gathers, a quarter of each tile per
// warp (a warp issues bulk copies one lane at a time, so four warps issue a tile about
// four times as fast as one).  Every mbarrier wait is bounded: a role that gives up sets
// LC_DEV_TIMEOUT and an abort flag that stops the others at their next wait.
#include <cuda.h>

#include <cooperative_groups.h>

#include "lc_internal.h"
#include "lc_ptx.cuh"

namespace cg = cooperative_groups;

namespace lc {

namespace {

constexpr int kD = 576;
constexpr int kDR = 64;
constexpr int kDN = kD - kDR;
constexpr int kTK = 64;                   // keys per tile
constexpr int kNR = 64;                   // heads per CTA
constexpr int kG = 72 * 128;              // F16 core-matrix tile: bytes per group of 8 rows
constexpr int kTile = 8 * kG;             // F16 tile of 64 rows: 73,728 bytes
constexpr int kBlk = kTK * 128;           // one 128-byte column block of 64 rows (SW128): 8 KB
constexpr int kRawN = 4 * kBlk;           // E4M3 nope part of a tile: 32 KB
constexpr int kRawStage = kRawN + kBlk;   // + BF16 RoPE part: 40 KB
constexpr int kPBytes = kNR * kTK * 2;
constexpr long kSpin = 1L << 26;
constexpr uint32_t kWin = 1u << 30;
constexpr int kThreads = 416;
constexpr int kCopyWarps = 4;            // warps 9 .. 12: key codes and bulk copies
constexpr float kRescale = 8.f;
constexpr int kColS = 0;                  // S buffers at columns 0 and 64
constexpr int kColO = 2 * kTK;            // O^T chunk c at 128 + 64 c
constexpr uint32_t kTmemCols = 512;

// shared memory (dynamic, 1024-byte aligned)
constexpr int kOffQn = 0;                         // Q nope, E4M3, 4 SW128 blocks
constexpr int kOffQr = kOffQn + kRawN;            // Q RoPE, BF16, SW128
constexpr int kOffRaw = kOffQr + kBlk;            // 2 raw stages (window phase: Q in BF16)
constexpr int kOffV = kOffRaw + 2 * kRawStage;    // F16 core-matrix tile
constexpr int kOffP = kOffV + kTile;
constexpr int kOffCode = kOffP + kPBytes;         // [4][kTK] key codes
constexpr int kOffF = kOffCode + 4 * kTK * 4;     // [kNR] per-head factors
constexpr size_t kSmem = kOffF + kNR * 4 + 1024;  // + alignment slack
static_assert(2 * kRawStage >= kTile, "Q in BF16 fits the raw stages");

// 16 E4M3 values -> 16 F16 values (exact)
__device__ __forceinline__ void e4m3x16_f16(uint4 v, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[j] & 0xffffu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[j] >> 16), __NV_E4M3);
    o[2 * j] = static_cast<uint32_t>(a.x) | (static_cast<uint32_t>(a.y) << 16);
    o[2 * j + 1] = static_cast<uint32_t>(b.x) | (static_cast<uint32_t>(b.y) << 16);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}
// 16 E4M3 values -> 16 BF16 values (exact: an E4M3 value has at most 4 significant bits,
// so the upper half of its FP32 bits is its BF16 encoding)
__device__ __forceinline__ void e4m3x16_bf16(uint4 v, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[j] & 0xffffu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[j] >> 16), __NV_E4M3);
    const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&a));
    const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&b));
    o[2 * j] = (__float_as_uint(fa.x) >> 16) | (__float_as_uint(fa.y) & 0xffff0000u);
    o[2 * j + 1] = (__float_as_uint(fb.x) >> 16) | (__float_as_uint(fb.y) & 0xffff0000u);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}
// 8 BF16 values -> 8 F16 values; |value| accumulated (as F16) into `amax`
__device__ __forceinline__ uint4 bf16x8_f16(uint4 v, __half2& amax) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __half2 h = __floats2half2_rn(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u));
    amax = __hmax2(amax, __habs2(h));
    o[j] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ bool f16_inf(__half2 a) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(&a);
  return ((u & 0x7c00u) == 0x7c00u) | ((u & 0x7c000000u) == 0x7c000000u);
}

// byte offset of dim chunk c (8 dims) of row r in the F16 core-matrix tile
__device__ __forceinline__ uint32_t tile_off(int r, int c) { return (r >> 3) * kG + c * 128 + (r & 7) * 16; }


struct Bars {
  uint64_t qfull;      // Q nope + RoPE landed (expect-tx)
  uint64_t kfull[2];   // raw stage landed (expect-tx; one arrival per copy warp)
  uint64_t kempty[2];  // raw stage read by S (commit) and by the converter (1 arrival)
  uint64_t cready[4];  // key codes of a tile written (one arrival per copy warp)
  uint64_t cfree[4];   // key codes of a tile read by the softmax (128 arrivals)
  uint64_t wfull;      // window tile landed in the F16 tile area (expect-tx)
  uint64_t wsdone;     // S of a window tile complete: the tile may be widened in place (commit)
  uint64_t vfull;      // F16 tile ready (1 arrival)
  uint64_t vempty;     // F16 tile read by O (commit)
  uint64_t q16full;    // Q in BF16 ready for the window tiles (1 arrival)
  uint64_t q16free;    // every S that reads Q in BF16 is complete: the raw stages are free (commit)
  uint64_t sfull[2];   // S buffer computed (commit)
  uint64_t sempty[2];  // S buffer read (128 arrivals)
  uint64_t pfull;      // P written (128 arrivals)
  uint64_t pempty;     // P read and O updated (commit)
  uint64_t fin;        // every MMA complete (commit)
};

}  // namespace

struct AttnTc8Geom {
  int n_split;
  int sps;       // slots per split, multiple of kTK
  int win_own;   // 1: the last split takes every window slot, the others the entry slots
  int cluster;   // 1: the splits of a (query, head group) are one thread-block cluster and
                 // merge their partial results over distributed shared memory
};

constexpr int kMaxClusterSplits = 8;
// the receive buffers of the cluster merge (n_split x kNR x ceil(groups / n_split) x 32 floats)
// fit below the key codes, in the dead tiles
static_assert((kD / 32 + kMaxClusterSplits - 1) * kNR * 32 * 4 <= kOffCode, "merge buffers fit");

// grid: one CTA per (query, head group, key split), the split index fastest; 320 threads.
// Partial results of split s go to ws_o rows s * n_q * H + q * H + h (576 floats each) and
// ws_ml[2 ((q * H + h) * n_split + s) + {0, 1}] = (m, l).
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_tc8(const __grid_constant__ CUtensorMap tqn, const __grid_constant__ CUtensorMap tqr,
               const __grid_constant__ CUtensorMap tkn, const __grid_constant__ CUtensorMap tkr,
               const __grid_constant__ CUtensorMap twin, lc_attn_args a,
               int sparse, int decode, AttnTc8Geom geo, float* __restrict__ ws_o, float* __restrict__ ws_ml) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Qn = smem + kOffQn;
  uint8_t* Qr = smem + kOffQr;
  uint8_t* Raw = smem + kOffRaw;
  uint8_t* Vt = smem + kOffV;
  uint8_t* Ps = smem + kOffP;
  int* kcode = reinterpret_cast<int*>(smem + kOffCode);
  float* s_f = reinterpret_cast<float*>(smem + kOffF);
  uint8_t* Q16 = Raw;  // window phase: Q in BF16, core matrices
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ __align__(8) Bars bars;
  __shared__ float2 s_mlall[kMaxClusterSplits][kNR];  // cluster merge: every split's (max, sum) per head
  __shared__ float s_sk[kNR];  // the heads' sinks, log2 units

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_hg = a.dims.H / kNR;
  const int split = blockIdx.x % geo.n_split;
  const int hg = (blockIdx.x / geo.n_split) % n_hg;
  const int q = blockIdx.x / (geo.n_split * n_hg);
  const int H = a.dims.H;
  // decode: one query per sequence (q_start[b] = b), so the per-sequence loads below are
  // independent of one another
  const int b = decode ? q : seq_of_query(a.batch.q_start, a.batch.num_seqs, q);
  const int p = __ldg(a.batch.q_pos0 + b) + (decode ? 0 : q - __ldg(a.batch.q_start + b));
  const int n_ent = __ldg(a.batch.n_ent + b);
  const int nv = n_visible(p, a.m, a.W_x, n_ent);
  const int64_t ent0 = __ldg(a.batch.ent_start + b);
  const int wlo = a.W > 0 ? max(0, p - a.W + 1) : p + 1;
  // window slots start at position wbase: wlo, or, for a ring buffer, wlo rounded down to a
  // multiple of 64, so that every 64-position window tile is 64 consecutive ring rows
  // (positions below wlo are masked)
  const int ring = a.batch.win_ring;
  const int wbase = ring > 0 ? (wlo & ~(kTK - 1)) : wlo;
  const int n_first = sparse ? a.k : nv;
  // the first window slot: right after the entries, or, for a ring, at the next multiple of
  // 64 (the slots between are dead), so that every window tile starts on a 64-position
  // boundary whatever split it falls in
  const int w_slot0 = ring > 0 ? (n_first + kTK - 1) / kTK * kTK : n_first;
  const int n_slots = w_slot0 + (p + 1 - wbase);
  int s_begin, s_end;
  if (!geo.win_own) {
    s_begin = split * geo.sps;
    s_end = min(n_slots, s_begin + geo.sps);
  } else if (split == geo.n_split - 1) {
    s_begin = n_first;
    s_end = n_slots;
  } else {
    s_begin = min(split * geo.sps, n_first);
    s_end = min(s_begin + geo.sps, n_first);
  }
  // entry tiles cover [s_begin, min(s_end, n_first)), window tiles the rest of the range
  const int e_end = min(s_end, n_first);
  const int n_et = e_end > s_begin ? (e_end - s_begin + kTK - 1) / kTK : 0;
  const int w_begin = max(s_begin, w_slot0);
  const int n_wt = s_end > w_begin ? (s_end - w_begin + kTK - 1) / kTK : 0;
  const int n_tiles = n_et + n_wt;
  const int wp0 = a.W > 0 ? __ldg(a.batch.win_pos0 + b) : 0;
  const int wl = a.W > 0 ? __ldg(a.batch.win_len + b) : 0;
  const int64_t wr0 = a.W > 0 ? __ldg(a.batch.win_start + b) : 0;
  const int32_t* idx_row = sparse ? a.idx + static_cast<int64_t>(q) * a.k : nullptr;
  const int64_t row0 = static_cast<int64_t>(q) * H + hg * kNR;
  // values: all 576 dims (5 O^T chunks), or (v_nope) the 512 E4M3 dims (chunks 0-3)
  const int n_och = a.v_nope ? 4 : 5;
  const int Dv = a.v_nope ? kDN : kD;

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
  // first slot of tile t
  // window tiles come first (their rows are on hand while the entry gathers start): tile t
  // is window tile t for t < n_wt, entry tile t - n_wt after that
  auto tile_slot0 = [&](int t) { return t < n_wt ? w_begin + t * kTK : s_begin + (t - n_wt) * kTK; };
  auto tile_slot_end = [&](int t) { return t < n_wt ? s_end : e_end; };
  // key slot -> entry index j, kWin | window row, or -1 (masked)
  auto slot_code = [&](int s, int s_lim) -> int {
    if (s >= s_lim) return -1;
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
    if (s < w_slot0) return -1;  // dead slots before a ring-aligned window
    const int t = wbase + (s - w_slot0);
    if (t < wlo) return -1;  // ring alignment: before the window
    const int rr = t - wp0;
    if (rr < 0 || rr >= wl) {
      set_status(a.status, LC_DEV_WINDOW_RANGE);
      return -1;
    }
    return static_cast<int>(kWin) | (ring > 0 ? t % ring : rr);
  };

  // ---- set-up ----
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(&s_tmem)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 32) {
    s_abort = 0;
    mbar_init(su32(&bars.qfull), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(su32(&bars.kfull[i]), kCopyWarps);
      mbar_init(su32(&bars.kempty[i]), 2);
      mbar_init(su32(&bars.sfull[i]), 1);
      mbar_init(su32(&bars.sempty[i]), 128);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(su32(&bars.cready[i]), kCopyWarps);
      mbar_init(su32(&bars.cfree[i]), 128);
    }
    mbar_init(su32(&bars.wfull), 1);
    mbar_init(su32(&bars.wsdone), 1);
    mbar_init(su32(&bars.vfull), 1);
    mbar_init(su32(&bars.vempty), 1);
    mbar_init(su32(&bars.q16full), 1);
    mbar_init(su32(&bars.q16free), 1);
    mbar_init(su32(&bars.pfull), 128);
    mbar_init(su32(&bars.pempty), 1);
    mbar_init(su32(&bars.fin), 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = s_tmem;
  // cluster: this CTA has started (its shared memory may be written remotely once every
  // CTA of the cluster has arrived here)
  if (geo.cluster) asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");

  if (warp >= 9) {
    // ================= key codes and bulk copies =================
    // Four warps share each tile: a warp issues its bulk copies one lane after another, so
    // the copies of a tile go out about four times faster from four warps than from one.
    // Copy warp cw owns keys 16 cw .. 16 cw + 15 of every tile.
    const int cw = warp - 9;
    if (cw == 0 && lane == 0 && n_tiles > 0) {
      const uint32_t qb = su32(&bars.qfull);
      mbar_expect_tx(qb, kRawN + kBlk);
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) tma_tile2d(su32(Qn + cb * kBlk), &tqn, cb * 128, static_cast<int>(row0), qb);
      tma_tile2d(su32(Qr), &tqr, 0, static_cast<int>(row0), qb);
    }
    int e_last0 = -1, e_last1 = -1;  // lane 0: the last entry tile of stage 0 / 1 this warp copied
    for (int t = 0; t < n_tiles; ++t) {
      const int cb4 = t & 3;
      // the top-k indices may be the previous kernel's output (programmatic dependent
      // launch): the window tiles and Q come in meanwhile
      if (t == n_wt && a.pdl) pdl_wait();
      // the code buffer of tile t - 4 has been read by its softmax
      bool ok = t < 4 || wait(&bars.cfree[cb4], ((t >> 2) - 1) & 1);
      // raw stage of entry tile e: free once S and the conversion of entry tile e - 2 are
      // done; before the first two entry tiles it holds Q in BF16 for the window tiles
      const int e = t - n_wt;
      if (ok && e >= 2) ok = wait(&bars.kempty[e & 1], ((e >> 1) - 1) & 1);
      if (ok && e >= 0 && e < 2 && n_wt > 0) ok = wait(&bars.q16free, 0);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int s0 = tile_slot0(t), s_lim = tile_slot_end(t);
      int* kc = kcode + cb4 * kTK + 16 * cw;
      if (lane < 16) kc[lane] = slot_code(s0 + 16 * cw + lane, s_lim);
      __syncwarp();
      if (lane == 0) mbar_arrive(su32(&bars.cready[cb4]));
      if (e >= 0) {
        const int st = e & 1;
        const uint32_t kb = su32(&bars.kfull[st]);
        if (lane == 0) {
          mbar_expect_tx(kb, kRawStage / kCopyWarps);
          (st ? e_last1 : e_last0) = e;
        }
        __syncwarp();
        if (lane < 4) {
          // rows 4 g .. 4 g + 3 of the tile, g = 4 cw + lane; a masked key reads row 0 (its
          // P is 0)
          const int g = 4 * cw + lane;
          int rr[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int code = kc[4 * lane + u];
            rr[u] = code < 0 ? 0 : static_cast<int>(ent0 + code);
          }
          uint8_t* stage = Raw + st * kRawStage;
#pragma unroll
          for (int cb = 0; cb < 4; ++cb)
            tma_gather4(su32(stage + cb * kBlk + g * 512), &tkn, cb * 128, rr[0], rr[1], rr[2], rr[3], kb);
          tma_gather4(su32(stage + kRawN + g * 512), &tkr, 0, rr[0], rr[1], rr[2], rr[3], kb);
        }
      }
    }
    // a role that gave up may leave copies in flight: they land before the CTA exits (a
    // stage's phase also needs the other copy warps' parts, so this wait is bounded too)
    if (lane == 0) {
      if (e_last0 >= 0) drain(&bars.kfull[0], (e_last0 >> 1) & 1);
      if (e_last1 >= 0) drain(&bars.kfull[1], (e_last1 >> 1) & 1);
      if (cw == 0 && n_tiles > 0) drain(&bars.qfull, 0);
    }
  } else if (warp == 8) {
    // ================= MMA issue (one lane) =================
    if (lane == 0) {
      // S entry: M = 64, N = 64, K-major SW128, E4M3 (kind::f8f6f4) and BF16 (kind::f16)
      const uint32_t id_s8 = (1u << 4) | (static_cast<uint32_t>(kTK >> 3) << 17) | (static_cast<uint32_t>(kNR >> 4) << 24);
      const uint32_t id_sbf = id_s8 | (1u << 7) | (1u << 10);
      // S window: BF16 (id_sbf); O^T: M = 128 (or 64), N = 64, A MN-major, F16
      const uint32_t id_o128 = (1u << 4) | (1u << 15) | (static_cast<uint32_t>(kNR >> 3) << 17) |
                               (static_cast<uint32_t>(128 >> 4) << 24);
      const uint32_t id_o64 = (1u << 4) | (1u << 15) | (static_cast<uint32_t>(kNR >> 3) << 17) |
                              (static_cast<uint32_t>(64 >> 4) << 24);
      const uint64_t dp = cm_desc(su32(Ps), 128, (kTK / 8) * 128);
      const uint64_t dv = cm_desc(su32(Vt), kG, 128);
      int ns = 0, no = 0;
      long idle = 0;
      bool ok = n_tiles == 0 || wait(&bars.qfull, 0);
      while (ok && no < n_tiles) {
        bool progressed = false;
        if (ns < n_tiles && ns <= no + 1) {
          const int sb = ns & 1;
          bool ready = ns < 2 || mbar_probe(su32(&bars.sempty[sb]), ((ns >> 1) - 1) & 1);
          const int e = ns - n_wt;
          if (e >= 0) ready = ready && mbar_probe(su32(&bars.kfull[e & 1]), (e >> 1) & 1);
          else ready = ready && mbar_probe(su32(&bars.q16full), 0) && mbar_probe(su32(&bars.wfull), ns & 1);
          if (ready) {
            fence_after();
            const uint32_t d = tm + kColS + sb * kTK;
            if (e >= 0) {
              const uint32_t st = su32(Raw + (e & 1) * kRawStage);
#pragma unroll
              for (int cb = 0; cb < 4; ++cb)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  mma_f8(d, sw128_desc(su32(Qn) + cb * kBlk + k * 32), sw128_desc(st + cb * kBlk + k * 32), id_s8,
                         cb > 0 || k > 0);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_f16(d, sw128_desc(su32(Qr) + k * 32), sw128_desc(st + kRawN + k * 32), id_sbf, 1);
              mma_commit(su32(&bars.kempty[e & 1]));
            } else {
              // A: Q in BF16 (core matrices); B: the window tile as it landed, BF16, SW128, 64
              // dims per block (each product is exact in FP32, as with F16 operands); the
              // tile is widened to F16 for O only after this S is complete
              const uint64_t dq = cm_desc(su32(Q16), 128, kG);
#pragma unroll
              for (int k = 0; k < kD / 16; ++k)
                mma_f16(d, dq + k * 16, sw128_desc(su32(Vt) + (k >> 2) * kBlk + (k & 3) * 32), id_sbf, k > 0);
              mma_commit(su32(&bars.wsdone));
              if (ns == n_wt - 1) mma_commit(su32(&bars.q16free));
            }
            mma_commit(su32(&bars.sfull[sb]));
            ++ns;
            progressed = true;
          }
        }
        if (no < ns && mbar_probe(su32(&bars.pfull), no & 1) && mbar_probe(su32(&bars.vfull), no & 1)) {
          fence_after();
          if (no >= n_wt) {
#pragma unroll
            for (int kk = 0; kk < kTK / 16; ++kk)
#pragma unroll
              for (int c = 0; c < 5; ++c)
                if (c < n_och)
                  mma_f16(tm + kColO + c * kNR, dv + (c * 2048 + kk * 2 * kG) / 16, dp + kk * 16,
                          c < 4 ? id_o128 : id_o64, (no > 0) || (kk > 0));
          } else {
            // window tile: V^T straight from the SW128 tile (dims along M, 16 keys per step)
#pragma unroll
            for (int kk = 0; kk < kTK / 16; ++kk)
#pragma unroll
              for (int c = 0; c < 5; ++c)
                if (c < n_och)
                  mma_f16(tm + kColO + c * kNR, sw128_mn_desc(su32(Vt) + c * 2 * kBlk + kk * 2048, kBlk),
                          dp + kk * 16, c < 4 ? id_o128 : id_o64, (no > 0) || (kk > 0));
          }
          mma_commit(su32(&bars.vempty));
          mma_commit(su32(&bars.pempty));
          ++no;
          progressed = true;
        }
        if (progressed) {
          idle = 0;
        } else if (++idle >= kSpin) {
          set_status(a.status, LC_DEV_TIMEOUT);
          atomicExch(&s_abort, 1);
          ok = false;
        } else if ((idle & 1023) == 0 && *reinterpret_cast<volatile int*>(&s_abort)) {
          ok = false;
        } else {
          // nothing ready: yield the issue slots this polling loop would take from the
          // converter and softmax warps
          __nanosleep(32);
        }
      }
      mma_commit(su32(&bars.fin));
      drain(&bars.fin, 0);  // every MMA issued above completes before tensor memory is released
    }
  } else if (warp >= 4) {
    // ================= converters: raw or window rows -> F16 tile =================
    const int ct = tid - 128;  // 0..127
    const int r8 = ct & 7;     // row within a group of 8 (one quarter warp: 8 rows, one chunk)
    __half2 amax = __float2half2_rn(0.f);
    bool ok = true;
    int w_last = -1;  // thread ct = 0: the last window tile it copied
    for (int t = 0; ok && t < n_tiles; ++t) {
      if (t < n_wt) {
        // window tile: its rows are consecutive, so it comes as one 64 x 64 BF16 box per 64
        // dims (SW128) straight into the F16 tile area, once O of tile t - 1 is done (these
        // warps wait for every phase of vempty in order; rows past the window are masked by
        // their codes)
        const bool okv = t == 0 || wait(&bars.vempty, (t - 1) & 1);
        if (named_bar_or(2, 128, !okv)) {
          ok = false;
          break;
        }
        if (ct == 0) {
          const uint32_t wb = su32(&bars.wfull);
          mbar_expect_tx(wb, kTile);
          const int t0 = wbase + (tile_slot0(t) - w_slot0);  // first position of the tile
          const int y = static_cast<int>(wr0) + (ring > 0 ? t0 % ring : t0 - wp0);
#pragma unroll
          for (int cb = 0; cb < kD / 64; ++cb) tma_tile2d(su32(Vt + cb * kBlk), &twin, cb * 64, y, wb);
          w_last = t;
        }
      }
      if (t == 0 && n_wt > 0) {
        // Q to BF16 in the raw stages for the window tiles (the entry gathers wait for
        // q16free before they use the raw stages)
        const bool okq = wait(&bars.qfull, 0);
        if (named_bar_or(2, 128, !okq)) {
          ok = false;
          break;
        }
        // 64 rows x (64 E4M3 chunks of 8 + 8 BF16 chunks)
        for (int i = ct; i < kNR * 36; i += 128) {
          const int g = i >> 3, pc = g % 36, r = (g / 36) * 8 + (i & 7);
          if (pc < 32) {  // 16 E4M3 dims: block pc / 8, 16-byte chunk pc % 8 of row r
            const uint4 v = *reinterpret_cast<const uint4*>(Qn + (pc >> 3) * kBlk + sw128_off(r, pc & 7));
            uint4 lo, hi;
            e4m3x16_bf16(v, lo, hi);
            *reinterpret_cast<uint4*>(Q16 + tile_off(r, 2 * pc)) = lo;
            *reinterpret_cast<uint4*>(Q16 + tile_off(r, 2 * pc + 1)) = hi;
          } else {  // 16 RoPE dims (already BF16): chunks 2 (pc - 32), +1 of the SW128 row
            const int j = 2 * (pc - 32);
            *reinterpret_cast<uint4*>(Q16 + tile_off(r, 64 + j)) = *reinterpret_cast<const uint4*>(Qr + sw128_off(r, j));
            *reinterpret_cast<uint4*>(Q16 + tile_off(r, 64 + j + 1)) =
                *reinterpret_cast<const uint4*>(Qr + sw128_off(r, j + 1));
          }
        }
        fence_async_smem();
        named_bar(2, 128);
        if (ct == 0) mbar_arrive(su32(&bars.q16full));
      }
      // the F16 tile is free once O of the previous tile is done; this tile's codes or
      // raw rows have landed
      bool okw = t == 0 || wait(&bars.vempty, (t - 1) & 1);
      const int e = t - n_wt;
      if (e >= 0) okw = okw && wait(&bars.kfull[e & 1], (e >> 1) & 1);
      else  // the window tile is widened in place once its S has read it
        okw = okw && wait(&bars.cready[t & 3], (t >> 2) & 1) && wait(&bars.wsdone, t & 1);
      if (named_bar_or(2, 128, !okw)) {
        ok = false;
        break;
      }
      if (e >= 0) {
        const uint8_t* st = Raw + (e & 1) * kRawStage;
        // 64 keys x 32 E4M3 pieces of 16 dims, then 64 keys x 8 BF16 chunks; a quarter warp
        // takes 8 rows of one piece (its SW128 reads and its core-matrix writes hit
        // distinct banks); the loads of four pieces are issued before any is converted
#pragma unroll 1
        for (int k0 = 0; k0 < kTK * 32 / 128; k0 += 4) {
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int g = (ct + 128 * (k0 + u)) >> 3, pc = g & 31, r = (g >> 5) * 8 + r8;
            v[u] = *reinterpret_cast<const uint4*>(st + (pc >> 3) * kBlk + sw128_off(r, pc & 7));
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int g = (ct + 128 * (k0 + u)) >> 3, pc = g & 31, r = (g >> 5) * 8 + r8;
            uint4 lo, hi;
            e4m3x16_f16(v[u], lo, hi);
            *reinterpret_cast<uint4*>(Vt + tile_off(r, 2 * pc)) = lo;
            *reinterpret_cast<uint4*>(Vt + tile_off(r, 2 * pc + 1)) = hi;
          }
        }
        {
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int g = (ct + 128 * u) >> 3, j = g & 7, r = (g >> 3) * 8 + r8;
            v[u] = *reinterpret_cast<const uint4*>(st + kRawN + sw128_off(r, j));
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int g = (ct + 128 * u) >> 3, j = g & 7, r = (g >> 3) * 8 + r8;
            *reinterpret_cast<uint4*>(Vt + tile_off(r, 64 + j)) = bf16x8_f16(v[u], amax);
          }
        }
      } else {
        // window tile (SW128 BF16: 16-byte chunk i holds 8 dims of row (i / 8) % 64) rounded
        // to F16 in place; rows of masked keys are zeroed
        const int* kc = kcode + (t & 3) * kTK;
#pragma unroll 1
        for (int k0 = 0; k0 < kTile / 16 / 128; k0 += 4) {
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const uint4*>(Vt + (ct + 128 * (k0 + u)) * 16);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = ct + 128 * (k0 + u);
            const int code = kc[(i >> 3) & (kTK - 1)];
            *reinterpret_cast<uint4*>(Vt + i * 16) =
                code < 0 || !(code & kWin) ? make_uint4(0, 0, 0, 0) : bf16x8_f16(v[u], amax);
          }
        }
      }
      fence_async_smem();
      named_bar(2, 128);
      if (ct == 0) {
        mbar_arrive(su32(&bars.vfull));
        if (e >= 0) mbar_arrive(su32(&bars.kempty[e & 1]));
      }
    }
    if (f16_inf(amax)) set_status(a.status, LC_DEV_RANGE);
    if (ct == 0 && w_last >= 0) drain(&bars.wfull, w_last & 1);  // a window copy in flight lands first
  } else {
    // ================= warps 0-3: softmax, epilogue =================
    const int r = warp * 16 + (lane & 15);
    const int hf = lane >> 4;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale * 1.4426950408889634f;
    if (hf == 0) s_sk[r] = __ldg(a.sink + hg * kNR + r) * 1.4426950408889634f;  // read by this thread
    float m_ref = -INFINITY, l_sum = 0.f;
    bool good = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int sb = t & 1;
      const bool okw = wait(&bars.sfull[sb], (t >> 1) & 1) && wait(&bars.cready[t & 3], (t >> 2) & 1);
      if (named_bar_or(1, 128, !okw)) {
        good = false;
        break;
      }
      fence_after();
      uint32_t sv[32];
      tmem_ld16x2(tm + lane_off + kColS + sb * kTK, sv);
      uint32_t live = 0;  // bit j: key 32 hf + j is not masked
      const int* kc = kcode + (t & 3) * kTK + 32 * hf;
#pragma unroll
      for (int j = 0; j < 32; ++j) live |= static_cast<uint32_t>(kc[j] >= 0) << j;
      mbar_arrive(su32(&bars.cfree[t & 3]));
      tmem_wait_ld();
      fence_before();
      mbar_arrive(su32(&bars.sempty[sb]));
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float x = (live >> j) & 1u ? __uint_as_float(sv[j]) * sl2 : -INFINITY;
        sv[j] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const bool need = mx > m_ref + kRescale;
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
        named_bar(1, 128);
      }
      {
        uint32_t pk[16];
        const float mr = m_ref == -INFINITY ? 0.f : m_ref;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const __half2 ph = __floats2half2_rn(ex2(__uint_as_float(sv[j]) - mr), ex2(__uint_as_float(sv[j + 1]) - mr));
          const float2 pf = __half22float2(ph);
          l_sum += pf.x + pf.y;
          pk[j / 2] = *reinterpret_cast<const uint32_t*>(&ph);
        }
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
    good = !named_bar_or(1, 128, !good);
    fence_after();
    const float l_row = l_sum + __shfl_xor_sync(0xffffffffu, l_sum, 16);
    if (geo.cluster) {
      // this split's (max, sum) per head, for the merge over the cluster below
      if (hf == 0) s_mlall[split][r] = make_float2(good ? m_ref : -INFINITY, good ? l_row : 0.f);
    } else if (hf == 0) {
      if (geo.n_split == 1) {
        const float sk = s_sk[r];
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
    if (good && !geo.cluster) {
      // O^T (dims on tensor-memory lanes, heads on columns) straight to global memory:
      // for each head a warp writes 32 consecutive dims, 128 bytes in FP32
      const bool f32 = geo.n_split > 1 || a.out_fmt == LC_FMT_F32;
      const int ostr = geo.n_split > 1 ? kD : Dv;  // partial rows keep every dim
      float* of = nullptr;
      uint16_t* oh = nullptr;
      if (geo.n_split > 1) of = ws_o + (static_cast<int64_t>(split) * a.n_q * H + row0) * kD;
      else if (f32) of = static_cast<float*>(a.out) + row0 * Dv;
      else oh = static_cast<uint16_t*>(a.out) + row0 * Dv;
#pragma unroll 1
      for (int c = 0; c < n_och; ++c) {
        const int dim = c < 4 ? c * 128 + warp * 32 + lane : (lane < 16 ? 512 + warp * 16 + lane : -1);
        uint32_t ov[kNR];
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
          if (f32) of[i * ostr + dim] = v;
          else oh[i * ostr + dim] = f32_to_bf16_bits(v);
        }
      }
    }
  }
  if (geo.cluster) {
    // ================= merge of the key splits over the cluster (every thread) =================
    // Every transfer is a store into another CTA's shared memory (a remote load would wait
    // a round trip).  Split s pushes its (m, l) per head to every split; then each split
    // finds M = max(sink, max_s m_s), Z = e^(sink - M) + sum_s l_s e^(m_s - M) locally,
    // scales its O by e^(m_s - M) / Z and pushes each 32-dim group of it to the split that
    // owns the group (split j owns groups [j gp, (j + 1) gp)), which sums the n_split
    // pieces in split order and writes them out.
    cg::cluster_group cl = cg::this_cluster();
    fence_before();
    __syncthreads();  // this CTA's roles are done: s_mlall[split] is written
    asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory");  // every CTA has started
    if (tid < kNR)
      for (int sp = 0; sp < geo.n_split; ++sp)
        if (sp != split) cl.map_shared_rank(&s_mlall[split][0], sp)[tid] = s_mlall[split][tid];
    cl.sync();  // every split's (m, l) is here; every role of every split is done
    fence_after();
    const int ngr = Dv / 32;
    const int gp = (ngr + geo.n_split - 1) / geo.n_split;
    const int ndj = gp * 32;                       // row length of the receive buffers
    float* recv = reinterpret_cast<float*>(smem);  // [n_split sources][kNR heads][ndj dims]
    if (warp < 4) {
      const int r = warp * 16 + (lane & 15);
      if ((lane >> 4) == 0) {
        const float sk = s_sk[r];
        float M = sk;
        for (int sp = 0; sp < geo.n_split; ++sp) M = fmaxf(M, s_mlall[sp][r].x);
        float Z = exp2f(sk - M);
        for (int sp = 0; sp < geo.n_split; ++sp) {
          const float2 v = s_mlall[sp][r];
          if (v.x != -INFINITY) Z = fmaf(v.y, exp2f(v.x - M), Z);
        }
        const float mo = s_mlall[split][r].x;
        s_f[r] = mo == -INFINITY ? 0.f : exp2f(mo - M) / Z;
        if (split == 0 && a.lse) a.lse[row0 + r] = (M + log2f(Z)) * 0.6931471805599453f;
      }
      named_bar(1, 128);
      const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
      // 32 heads at a time: their factors in registers, so that the stores stream (the
      // compiler cannot tell the factors from the stored rows)
#pragma unroll 1
      for (int hh = 0; hh < kNR; hh += 32) {
        float f[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] = s_f[hh + i];
#pragma unroll 1
        for (int c = 0; c < n_och; ++c) {
          const int dim = c < 4 ? c * 128 + warp * 32 + lane : (lane < 16 ? 512 + warp * 16 + lane : -1);
          uint32_t ov[32];
          if (n_tiles > 0) {
            tmem_ld32(tm + lane_off + kColO + c * kNR + hh, ov);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = 0;
          }
          if (dim < 0) continue;
          const int j = (dim >> 5) / gp;
          float* dst = cl.map_shared_rank(recv, j) + (split * kNR + hh) * ndj + (dim - j * ndj);
#pragma unroll
          for (int i = 0; i < 32; ++i) dst[i * ndj] = __uint_as_float(ov[i]) * f[i];
        }
      }
    }
    cl.sync();  // every split's pieces are in their owners' shared memory
    // this split's dims [d0, d1): the sum over the sources, in split order
    const int d0 = min(Dv, split * ndj), d1 = min(Dv, d0 + ndj);
    const int nq4 = (d1 - d0) / 4;
    for (int it = tid; it < kNR * nq4; it += kThreads) {
      const int h = it / nq4, d4 = 4 * (it - h * nq4);
      float4 acc = *reinterpret_cast<const float4*>(recv + h * ndj + d4);
      for (int sp = 1; sp < geo.n_split; ++sp) {
        const float4 v = *reinterpret_cast<const float4*>(recv + (sp * kNR + h) * ndj + d4);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      const int64_t e = (row0 + h) * Dv + d0 + d4;
      if (a.out_fmt == LC_FMT_F32) {
        *reinterpret_cast<float4*>(static_cast<float*>(a.out) + e) = acc;
      } else {
        const uint32_t lo = static_cast<uint32_t>(f32_to_bf16_bits(acc.x)) | (static_cast<uint32_t>(f32_to_bf16_bits(acc.y)) << 16);
        const uint32_t hi = static_cast<uint32_t>(f32_to_bf16_bits(acc.z)) | (static_cast<uint32_t>(f32_to_bf16_bits(acc.w)) << 16);
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + e) = make_uint2(lo, hi);
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tm), "r"(kTmemCols));
}

// ---------------------------------------------------------------------------------
bool attn_tc8_supported(const lc_attn_args& a) {
  if (a.dims.D != kD || a.dims.d_r != kDR || a.dims.H % kNR || a.n_ent_rows < 1) return false;
  if (a.q.fmt != LC_FMT_E4M3_BF16 || a.ent.fmt != LC_FMT_E4M3_BF16) return false;
  if (a.W > 0 && (a.win.fmt != LC_FMT_BF16 || a.n_win_rows < 1)) return false;
  if (a.batch.win_ring > 0 && a.batch.win_ring % kTK) return false;
  auto al = [](const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; };
  if (!al(a.q.x) || !al(a.q.rope) || !al(a.ent.x) || !al(a.ent.rope) || (a.W > 0 && !al(a.win.x))) return false;
  if (!al(a.out) || !al(a.workspace)) return false;
  if (static_cast<int64_t>(a.n_q) * a.dims.H > 0x7fffffff) return false;
  return a.out_fmt == LC_FMT_BF16 || a.out_fmt == LC_FMT_F32;
}

// Decode splits the keys of each (query, head group) over up to SMs / CTAs splits.  A
// window tile costs about two entry tiles (72 KB of BF16 rows against 40 KB, plus its
// conversion in place), so when the window tiles fit one split that is no longer than the
// entry splits, they get a split of their own.
// Up to kMaxClusterSplits splits form one thread-block cluster and merge over distributed
// shared memory; more splits (few queries) leave partials for k_attn_combine.
static AttnTc8Geom tc8_geometry(const lc_attn_args& a, bool sparse, bool decode) {
  AttnTc8Geom g{1, 0, 0, 0};
  const int ne = sparse ? a.k : a.max_ent;
  // window slots: W, or up to W + 63 when ring-aligned window tiles start before the window
  const bool ring = a.W > 0 && a.batch.win_ring > 0;
  const int wslots = ring ? a.W + kTK - 1 : a.W;
  const int ne_pad = ring ? (ne + kTK - 1) / kTK * kTK : ne;  // window slots start on a tile
  const int ns = max(ne_pad + wslots, 1);
  const int tiles = (ns + kTK - 1) / kTK;
  g.sps = tiles * kTK;
  const int ctas = a.n_q * (a.dims.H / kNR);
  const int n_sm = sm_count();
  if (decode && ctas < n_sm) {
    const int n = max(1, min(n_sm / max(ctas, 1), tiles));
    const int per = (tiles + n - 1) / n;
    g.n_split = (tiles + per - 1) / per;
    g.sps = per * kTK;
    const int te = (ne + kTK - 1) / kTK, tw = (wslots + kTK - 1) / kTK;
    if (a.W > 0 && n >= 2 && te >= 1) {
      const int per_e = (te + n - 2) / (n - 1);
      // cost in entry-tile units: uniform splits put up to one window tile next to `per`
      // tiles; the own-split layout costs max(per_e, 2 tw)
      if (max(per_e, 2 * tw) < per + 1) {
        g.win_own = 1;
        g.sps = per_e * kTK;
        g.n_split = (te + per_e - 1) / per_e + 1;
      }
    }
    g.cluster = g.n_split > 1 && g.n_split <= kMaxClusterSplits;
  }
  return g;
}

size_t attn_tc8_workspace(const lc_attn_args& a, bool sparse, bool decode) {
  const AttnTc8Geom g = tc8_geometry(a, sparse, decode);
  if (g.n_split <= 1 || g.cluster) return 0;
  const size_t rows = static_cast<size_t>(a.n_q) * a.dims.H * g.n_split;
  return rows * kD * sizeof(float) + rows * 2 * sizeof(float);
}

namespace {

using EncodeTiled8 = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled8 encode8() {
  static EncodeTiled8 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiled8>(nullptr);
    return reinterpret_cast<EncodeTiled8>(f);
  }();
  return fn;
}

// a [rows, cols] row-major tensor of `esize`-byte elements, SW128 boxes of box_rows rows
bool make_map(CUtensorMap* m, CUtensorMapDataType ty, const void* base, int64_t rows, int cols, int esize,
              int box_cols, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * esize};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t es[2] = {1, 1};
  return encode8()(m, ty, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn_tc8(const lc_attn_args& a, bool sparse, bool decode, cudaStream_t st, int* n_split_out) {
  if (!encode8()) return cudaErrorNotSupported;
  const AttnTc8Geom g = tc8_geometry(a, sparse, decode);
  *n_split_out = g.cluster ? 1 : g.n_split;  // a cluster merges its splits itself
  const int64_t qrows = static_cast<int64_t>(a.n_q) * a.dims.H;
  CUtensorMap tqn, tqr, tkn, tkr, twin;
  if (!make_map(&tqn, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q.x, qrows, kDN, 1, 128, kNR) ||
      !make_map(&tqr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q.rope, qrows, kDR, 2, 64, kNR) ||
      !make_map(&tkn, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.ent.x, a.n_ent_rows, kDN, 1, 128, 1) ||
      !make_map(&tkr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.ent.rope, a.n_ent_rows, kDR, 2, 64, 1))
    return cudaErrorInvalidValue;
  if (a.W > 0) {
    if (!make_map(&twin, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.win.x, a.n_win_rows, kD, 2, 64, kTK))
      return cudaErrorInvalidValue;
  } else {
    twin = tkr;  // no window tiles: never read
  }
  cudaFuncSetAttribute(k_attn_tc8, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
  float* ws_o = g.cluster ? nullptr : static_cast<float*>(a.workspace);
  float* ws_ml = nullptr;
  if (g.n_split > 1 && !g.cluster) ws_ml = ws_o + static_cast<size_t>(a.n_q) * a.dims.H * g.n_split * kD;
  const int64_t ctas = static_cast<int64_t>(a.n_q) * (a.dims.H / kNR) * g.n_split;
  if (ctas > 0x7fffffff) return cudaErrorInvalidConfiguration;
  return launch_ex(k_attn_tc8, dim3(static_cast<unsigned>(ctas)), dim3(kThreads), kSmem, st, a.pdl != 0,
                   g.cluster ? g.n_split : 1, tqn, tqr, tkn, tkr, twin, a, sparse ? 1 : 0, decode ? 1 : 0, g, ws_o,
                   ws_ml);
}

}  // namespace lc
