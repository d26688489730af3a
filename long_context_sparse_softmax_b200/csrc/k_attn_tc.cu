// CSA sparse / HCA dense attention on the 5th-generation tensor cores (tcgen05, BF16).
//
// Same mathematics as k_attn.cu ("解读 DeepSeek V4": CSA attends to its top-k compressed
// entries, HCA to all of them, both plus a 128-token window and a per-head sink; V = K =
// the 576-dim entry; "DeepSeek-V4 论文分析" §5.4, §六, §七).  The rows of a CTA are NR heads
// of one query, which share every key (MQA).
//
// Tiles and tensor memory:
//   * key tile: 32 keys gathered by index with cp.async (BF16 parts straight into the tile,
//     E4M3 nope parts into a raw area widened to BF16 - exact), laid out as 8 x 8 core
//     matrices: key group g, dim chunk c at g * KG + c * 128.  The same bytes are the
//     K-major B operand of S = Q K^T and the MN-major A operand V^T of O^T = V^T P^T;
//   * S = Q K^T: M = 64 rows (a query's heads; rows past NR are ignored), N = 32, K = 576,
//     in tensor memory (M = 64 layout: row r in lane 32 (r / 16) + r % 16), two buffers;
//   * P = exp(scale * S): the method normalises queries and entries (RMSNorm), so
//     |scale <q, k>| <= |q| |k| / sqrt(D) = sqrt(D) = 24 and the exponent needs no running
//     maximum; a logit above 80 (exp would leave the FP32 range) is reported as
//     LC_DEV_RANGE.  Masked keys get P = 0.  P goes to shared memory (two buffers) as the
//     K-major B operand of the next MMA;
//   * O^T = V^T P^T accumulates in tensor memory, dims on lanes: 5 chunks of 128 dims x NR
//     columns.  Dim 576 of every key is 1, so O^T[576][row] is the row's sum of P.
// The sink joins at the end: Z = e^sink + sum P, o = O / Z, lse = ln Z.  Decode may split
// the keys of a query across CTAs; the splits then go through k_attn_combine.
//
// Warp roles (288 threads): warps 0-3 turn S into P and write the output (each reaches its
// own quarter of the tensor-memory lanes); warps 4-7 gather and widen key tiles into a
// two-stage ring; lane 0 of warp 8 issues the MMAs, S of tile t + 1 ahead of O of tile t
// so that the tensor core works while P is formed.  The roles meet only at mbarriers, and
// every wait is bounded: a role that gives up sets LC_DEV_TIMEOUT and an abort flag that
// stops the others at their next wait.
#include "lc_internal.h"

namespace lc {

namespace {

constexpr int kD = 576;
constexpr int kTK = 32;                      // keys per tile
constexpr int kDC = 73;                      // dim chunks per key group: 72 + the ones chunk
constexpr int kKG = kDC * 128;               // bytes per key group of 8
constexpr int kKTile = (kTK / 8) * kKG;      // bytes per key tile (37,376)
constexpr int kQG = 72 * 128;                // bytes per row group of 8 (Q)
constexpr int kRaw = 512;                    // raw E4M3 bytes per key
constexpr int kStages = 2;
constexpr long kSpin = 1L << 26;
constexpr uint32_t kWin = 1u << 30;
constexpr int kThreads = 288;

__device__ __forceinline__ uint32_t su32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;\n"); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n.reg .b64 st;\nmbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(bar));
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile("{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
               : "=r"(done)
               : "r"(bar), "r"(parity));
  return done != 0;
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n"); }
__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n)); }

__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar));
}

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<64>(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_ld<32>(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld<32>(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n"); }

__device__ __forceinline__ uint4 e4m3x8_bf16x8(uint2 u) {
  const uint32_t w[2] = {u.x, u.y};
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float2 a = e4m3x2_to_f32x2(static_cast<uint16_t>(w[j] & 0xffffu));
    const float2 b = e4m3x2_to_f32x2(static_cast<uint16_t>(w[j] >> 16));
    o[2 * j] = (__float_as_uint(a.x) >> 16) | (__float_as_uint(a.y) & 0xffff0000u);
    o[2 * j + 1] = (__float_as_uint(b.x) >> 16) | (__float_as_uint(b.y) & 0xffff0000u);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// byte offset of dim chunk c (8 dims) of row r in a core-matrix tile with group stride gs
__device__ __forceinline__ uint32_t tile_off(int r, int c, int gs) { return (r >> 3) * gs + c * 128 + (r & 7) * 16; }

}  // namespace

struct AttnTcGeom {
  int n_split;
  int sps;  // slots per split, multiple of kTK
};

// Shared state of one CTA.
struct TcBars {
  uint64_t kfull[kStages];   // producers -> MMA: key stage ready (128 arrivals)
  uint64_t kempty[kStages];  // MMA -> producers: key stage read by O (commit)
  uint64_t sfull[2];         // MMA -> softmax: S buffer computed (commit)
  uint64_t pfull[2];         // softmax -> MMA: P buffer written, S buffer read (128 arrivals)
  uint64_t pempty[2];        // MMA -> softmax: P buffer read by O (commit)
  uint64_t odone;            // MMA -> epilogue: last O complete (commit)
};

// grid: (n_q, head groups * n_split); 288 threads.  NR = heads per CTA (16 or 64).
template <int NR>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_tc(lc_attn_args a, int sparse, AttnTcGeom geo, uint32_t tmem_cols, float* __restrict__ ws_o,
              float* __restrict__ ws_ml) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* Qs = smem;                                        // (NR / 8) * kQG
  uint8_t* Ks = Qs + (NR / 8) * kQG;                         // [kStages][kKTile]
  uint8_t* Raw = Ks + kStages * kKTile;                      // [kStages][kTK][kRaw]
  uint8_t* Ps = Raw + kStages * kTK * kRaw;                  // [2][NR rows][kTK keys] BF16
  int* kcode = reinterpret_cast<int*>(Ps + 2 * NR * kTK * 2);  // [kStages][kTK]
  float* s_l = reinterpret_cast<float*>(kcode + kStages * kTK);  // [NR]
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ __align__(8) TcBars bars;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q = blockIdx.x;
  const int hg = blockIdx.y / geo.n_split, split = blockIdx.y % geo.n_split;
  const int H = a.dims.H, d_r = a.dims.d_r;
  const int d_n = kD - d_r;
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

  // ---- set-up (all threads): tensor memory, barriers, queries, the ones chunk ----
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(&s_tmem)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(su32(&bars.kfull[i]), 128);
      mbar_init(su32(&bars.kempty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(su32(&bars.sfull[i]), 1);
      mbar_init(su32(&bars.pfull[i]), 128);
      mbar_init(su32(&bars.pempty[i]), 1);
    }
    mbar_init(su32(&bars.odone), 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n");
  }
  for (int u = tid; u < NR * 72; u += kThreads) {
    const int r = u / 72, c = u % 72;
    const int h = hg * NR + r;
    uint8_t* dst = Qs + tile_off(r, c, kQG);
    if (h >= H) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      continue;
    }
    const int64_t row = static_cast<int64_t>(q) * H + h;
    if (a.q.fmt == LC_FMT_BF16) cp16(su32(dst), static_cast<const uint16_t*>(a.q.x) + row * kD + c * 8);
    else if (c * 8 < d_n) cp8(su32(Raw + r * kRaw + c * 8), static_cast<const uint8_t*>(a.q.x) + row * d_n + c * 8);
    else cp16(su32(dst), static_cast<const uint16_t*>(a.q.rope) + row * d_r + (c * 8 - d_n));
  }
  for (int u = tid; u < kStages * kTK; u += kThreads) {  // dim 576 = 1, dims 577..583 = 0
    const int st = u / kTK, kr = u % kTK;
    *reinterpret_cast<uint4*>(Ks + st * kKTile + tile_off(kr, 72, kKG)) = make_uint4(0x3F80u, 0, 0, 0);
  }
  cp_commit();
  cp_wait_all();
  __syncthreads();
  if (a.q.fmt == LC_FMT_E4M3_BF16) {
    for (int u = tid; u < NR * (d_n / 8); u += kThreads) {
      const int r = u / (d_n / 8), c = u % (d_n / 8);
      if (hg * NR + r < H)
        *reinterpret_cast<uint4*>(Qs + tile_off(r, c, kQG)) =
            e4m3x8_bf16x8(*reinterpret_cast<const uint2*>(Raw + r * kRaw + c * 8));
    }
  }
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = s_tmem;
  const uint32_t col_o = 2 * kTK;  // S buffers at columns 0 and kTK; O^T chunk c at col_o + c * NR

  if (warp >= 4 && warp < 8) {
    // ================= producers: gather + widen key tiles =================
    const int pt = tid - 128;  // 0..127
    for (int t = 0; t < n_tiles; ++t) {
      const int st = t % kStages;
      const uint32_t ph = (t / kStages) & 1;
      if (!wait(&bars.kempty[st], ph ^ 1)) break;
      if (pt < kTK) {
        const int s = s_begin + t * kTK + pt;
        int code = -1;
        if (s < s_end) {
          if (s < n_first) {
            const int j = sparse ? __ldg(idx_row + s) : s;
            if (j >= 0) {
              if (j >= n_ent) set_status(a.status, LC_DEV_BAD_INDEX);
              else if (j >= nv) set_status(a.status, LC_DEV_NONVISIBLE);
              else code = j;
            }
          } else {
            const int rr = wlo + (s - n_first) - wp0;
            if (rr < 0 || rr >= wl) set_status(a.status, LC_DEV_WINDOW_RANGE);
            else code = static_cast<int>(kWin) | rr;
          }
        }
        kcode[st * kTK + pt] = code;
      }
      named_bar(1, 128);
      uint8_t* kt = Ks + st * kKTile;
      uint8_t* rw = Raw + st * kTK * kRaw;
      for (int u = pt; u < kTK * 72; u += 128) {
        const int kr = u / 72, c = u % 72;
        const int code = kcode[st * kTK + kr];
        uint8_t* dst = kt + tile_off(kr, c, kKG);
        if (code < 0) {
          *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
          continue;
        }
        const lc_rows& rs = (code & kWin) ? a.win : a.ent;
        const int64_t r = (code & kWin) ? wr0 + (code & ~kWin) : ent0 + code;
        if (rs.fmt == LC_FMT_BF16) cp16(su32(dst), static_cast<const uint16_t*>(rs.x) + r * kD + c * 8);
        else if (c * 8 < d_n) cp8(su32(rw + kr * kRaw + c * 8), static_cast<const uint8_t*>(rs.x) + r * d_n + c * 8);
        else cp16(su32(dst), static_cast<const uint16_t*>(rs.rope) + r * d_r + (c * 8 - d_n));
      }
      cp_commit();
      cp_wait_all();
      named_bar(1, 128);
      if (a.ent.fmt == LC_FMT_E4M3_BF16) {
        const int dnc = d_n / 8;
        for (int u = pt; u < kTK * dnc; u += 128) {
          const int kr = u / dnc, c = u % dnc;
          const int code = kcode[st * kTK + kr];
          if (code >= 0 && !(code & kWin))
            *reinterpret_cast<uint4*>(kt + tile_off(kr, c, kKG)) =
                e4m3x8_bf16x8(*reinterpret_cast<const uint2*>(rw + kr * kRaw + c * 8));
        }
      }
      fence_async_smem();
      mbar_arrive(su32(&bars.kfull[st]));
    }
  } else if (warp == 8) {
    // ================= MMA issue (one lane) =================
    if (lane == 0) {
      const uint32_t id_s = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kTK >> 3) << 17) |
                            (static_cast<uint32_t>(64 >> 4) << 24);
      const uint32_t id_o = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) |
                            (static_cast<uint32_t>(NR >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
      const uint32_t qa = su32(Qs);
      auto issue_o = [&](int u) -> bool {  // O^T += V^T P^T for tile u
        const int st = u % kStages, pb = u & 1;
        if (!wait(&bars.pfull[pb], (u >> 1) & 1)) return false;
        fence_after();
        const uint32_t kb = su32(Ks + st * kKTile), pp = su32(Ps + pb * NR * kTK * 2);
#pragma unroll
        for (int c = 0; c < 5; ++c)
#pragma unroll
          for (int k = 0; k < kTK / 16; ++k)
            mma_f16(tm + col_o + c * NR, sdesc(kb + c * 16 * 128 + k * 2 * kKG, kKG, 128),
                    sdesc(pp + k * 256, 128, (kTK / 8) * 128), id_o, (u > 0) || (k > 0));
        mma_commit(su32(&bars.kempty[st]));
        mma_commit(su32(&bars.pempty[pb]));
        return true;
      };
      bool ok = true;
      for (int t = 0; t < n_tiles && ok; ++t) {
        const int st = t % kStages, sb = t & 1;
        ok = wait(&bars.kfull[st], (t / kStages) & 1);
        if (!ok) break;
        fence_after();
        // S buffer sb was last read by the softmax of tile t - 2, which the issue of O(t - 2)
        // waited for
        const uint32_t kb = su32(Ks + st * kKTile);
#pragma unroll 4
        for (int k = 0; k < kD / 16; ++k)
          mma_f16(tm + sb * kTK, sdesc(qa + k * 256, 128, kQG), sdesc(kb + k * 256, 128, kKG), id_s, k > 0);
        mma_commit(su32(&bars.sfull[sb]));
        if (t > 0) ok = issue_o(t - 1);
      }
      if (ok && n_tiles > 0) ok = issue_o(n_tiles - 1);
      mma_commit(su32(&bars.odone));
    }
  } else {
    // ================= softmax: S -> P =================
    const int r = warp * 16 + lane;  // row held by this lane (lanes 0..15 of each quadrant)
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale * 1.4426950408889634f;
    bool range_bad = false;
    for (int t = 0; t < n_tiles; ++t) {
      const int sb = t & 1, st = t % kStages;
      if (!wait(&bars.sfull[sb], (t >> 1) & 1)) break;
      if (!wait(&bars.pempty[sb], ((t >> 1) & 1) ^ 1)) break;
      // acquire the producers' key codes of this stage (the stage cannot have been refilled:
      // that waits for O of this tile, which waits for this P)
      if (!wait(&bars.kfull[st], (t / kStages) & 1)) break;
      fence_after();
      uint32_t sv[kTK];
      tmem_ld<kTK>(tm + lane_off + sb * kTK, sv);
      tmem_wait_ld();
      if (lane < 16 && r < NR) {
        const int* kc = kcode + st * kTK;
        uint32_t pk[kTK / 2];
#pragma unroll
        for (int j = 0; j < kTK; j += 2) {
          const float l0 = __uint_as_float(sv[j]) * sl2, l1 = __uint_as_float(sv[j + 1]) * sl2;
          range_bad |= (l0 > 115.f) | (l1 > 115.f);  // 80 in natural-log units
          const float p0 = kc[j] >= 0 ? exp2f(l0) : 0.f;
          const float p1 = kc[j + 1] >= 0 ? exp2f(l1) : 0.f;
          pk[j / 2] = static_cast<uint32_t>(f32_to_bf16_bits(p0)) | (static_cast<uint32_t>(f32_to_bf16_bits(p1)) << 16);
        }
        uint8_t* pbuf = Ps + sb * NR * kTK * 2;
#pragma unroll
        for (int c = 0; c < kTK / 8; ++c)
          *reinterpret_cast<uint4*>(pbuf + tile_off(r, c, (kTK / 8) * 128)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_async_smem();
      fence_before();
      mbar_arrive(su32(&bars.pfull[sb]));
    }
    if (range_bad) set_status(a.status, LC_DEV_RANGE);
  }

  // ---- epilogue (warps 0-3): chunk c, lane L -> dim 128 c + L; columns -> rows ----
  if (warp < 4) {
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const bool good = n_tiles > 0 && wait(&bars.odone, 0);
    fence_after();
    // row sums: dim 576 = chunk 4, lane 64 (warp 2, lane 0)
    if (warp == 2) {
      uint32_t v[NR];
      if (good) {
        tmem_ld<NR>(tm + lane_off + col_o + 4 * NR, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < NR; ++i) v[i] = 0;
      }
      if (lane == 0)
#pragma unroll
        for (int i = 0; i < NR; ++i) s_l[i] = __uint_as_float(v[i]);
    }
    named_bar(2, 128);
#pragma unroll 1
    for (int c = 0; c < 5; ++c) {
      const int dim = c * 128 + warp * 32 + lane;
      uint32_t v[NR];
      if (good) {
        tmem_ld<NR>(tm + lane_off + col_o + c * NR, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < NR; ++i) v[i] = 0;
      }
      if (dim >= kD) continue;
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        const int h = hg * NR + i;
        if (h >= H) continue;
        const int64_t orow = static_cast<int64_t>(q) * H + h;
        const float ov = __uint_as_float(v[i]);
        if (geo.n_split == 1) {
          const float Z = expf(__ldg(a.sink + h)) + s_l[i];
          const float o = ov / Z;
          if (a.out_fmt == LC_FMT_BF16) static_cast<uint16_t*>(a.out)[orow * kD + dim] = f32_to_bf16_bits(o);
          else static_cast<float*>(a.out)[orow * kD + dim] = o;
          if (dim == 0 && a.lse) a.lse[orow] = logf(Z);
        } else {
          const int64_t slot = orow * geo.n_split + split;
          ws_o[slot * kD + dim] = ov;
          if (dim == 0) {
            ws_ml[2 * slot] = 0.f;  // the exponent reference of every split is 0
            ws_ml[2 * slot + 1] = s_l[i];
          }
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tm), "r"(tmem_cols));
}

// ---------------------------------------------------------------------------------
bool attn_tc_supported(const lc_attn_args& a) {
  if (a.dims.D != kD || a.dims.d_r < 64 || a.dims.d_r % 8 || a.dims.H % 16) return false;
  auto ok = [&](const lc_rows& r) { return r.fmt == LC_FMT_BF16 || r.fmt == LC_FMT_E4M3_BF16; };
  if (!ok(a.q) || !ok(a.ent) || (a.W > 0 && a.win.fmt != LC_FMT_BF16)) return false;
  return a.out_fmt == LC_FMT_BF16 || a.out_fmt == LC_FMT_F32;
}

static AttnTcGeom tc_geometry(const lc_attn_args& a, bool sparse, bool decode) {
  AttnTcGeom g{1, 0};
  const int ns = max((sparse ? a.k : a.max_ent) + a.W, 1);
  const int tiles = (ns + kTK - 1) / kTK;
  g.sps = tiles * kTK;
  if (decode) {
    // one CTA per SM: split the keys only when the (query, head group) pairs leave SMs idle
    const int ctas = a.n_q * (a.dims.H / 16);
    const int want = max(1, 148 / max(ctas, 1));
    const int n = max(1, min(want, tiles / 8));
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

template <int NR>
static cudaError_t launch_tc(const lc_attn_args& a, bool sparse, const AttnTcGeom& g, cudaStream_t st) {
  // the S MMA reads 64 query rows: with NR < 64 the extra rows are the key stages behind Q
  const size_t sm = static_cast<size_t>((NR / 8) * kQG) + kStages * kKTile + kStages * kTK * kRaw +
                    2 * NR * kTK * 2 + kStages * kTK * 4 + NR * 4 + 1024;
  cudaFuncSetAttribute(k_attn_tc<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(2 * kTK + 5 * NR)) cols <<= 1;
  float* ws_o = static_cast<float*>(a.workspace);
  float* ws_ml = nullptr;
  if (g.n_split > 1) ws_ml = ws_o + static_cast<size_t>(a.n_q) * a.dims.H * g.n_split * kD;
  const dim3 grid(a.n_q, (a.dims.H / NR) * g.n_split);
  k_attn_tc<NR><<<grid, kThreads, sm, st>>>(a, sparse ? 1 : 0, g, cols, ws_o, ws_ml);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const lc_attn_args& a, bool sparse, bool decode, cudaStream_t st, int* n_split_out) {
  const AttnTcGeom g = tc_geometry(a, sparse, decode);
  *n_split_out = g.n_split;
  if (decode || a.dims.H % 64) return launch_tc<16>(a, sparse, g, st);
  return launch_tc<64>(a, sparse, g, st);
}

}  // namespace lc
