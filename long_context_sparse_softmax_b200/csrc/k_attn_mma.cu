// Tensor-core CSA sparse / HCA dense attention for 576-dim shared-KV entries (BF16 MMA).
//
// Same mathematics as the reference kernel in k_attn.cu ("解读 DeepSeek V4": CSA attends to
// its top-k compressed entries, HCA to all of them, both plus a 128-token window and a
// per-head sink; V = K = the entry).  The rows of a CTA are heads of ONE query, which all
// share the same keys (MQA), so a key tile is gathered once and feeds every head:
//
//   * key tile: TK keys gathered by index with cp.async.  BF16 data (window rows, the
//     RoPE part of entries) lands directly in the BF16 tile; the E4M3 nope part lands in
//     a raw area and is widened to BF16 in a second pass (E4M3 -> BF16 is exact).  Decode
//     double-buffers the tiles so the next tile's gather overlaps this tile's math;
//   * S = Q K^T on BF16 mma.sync; the D = 576 contraction is split across DS warps and
//     their partial sums are added in a fixed order through shared memory, so every warp
//     of a row tile holds the same S;
//   * online softmax in registers (running max starts at -inf, the sink joins at the end);
//   * O += P V with P from registers and V = the same key tile, each warp owning D/DS
//     output dims.
//
// A CTA covers MT x 16 heads with MT * DS warps: prefill uses 64 heads (MT = 4, DS = 2,
// 64-key tiles), decode 16 heads (MT = 1, DS = 4, 32-key tiles) so that a
// small batch still fills the GPU.  Decode may split a query's keys across CTAs
// (n_split > 1): each writes its unnormalised O, running max and sum to the workspace and
// k_attn_combine merges them with the sink in a fixed order.  The split count depends
// only on the shapes, never on timing.
#include "lc_internal.h"

namespace lc {

constexpr int kAD = 576;          // head dim of this kernel
constexpr int kRS = kAD + 8;      // padded shared row stride (elements): 1168 B, ldmatrix conflict-free
constexpr int kChunks = kAD / 8;  // 16-byte BF16 chunks per row
constexpr int kRawRow = 512;      // bytes of E4M3 nope data staged per key (d_n <= 512)
constexpr int kTileMax = 64;      // largest key tile
constexpr uint32_t kWinFlag = 1u << 30;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  return static_cast<uint32_t>(f32_to_bf16_bits(lo)) | (static_cast<uint32_t>(f32_to_bf16_bits(hi)) << 16);
}

// 8 E4M3 values (8 bytes) -> 8 BF16 values (16 bytes), exact.
__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 u) {
  const uint32_t w[2] = {u.x, u.y};
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float2 a = e4m3x2_to_f32x2(static_cast<uint16_t>(w[j] & 0xffffu));
    const float2 b = e4m3x2_to_f32x2(static_cast<uint16_t>(w[j] >> 16));
    // E4M3 values have <= 4 significant bits: the upper half of the FP32 bits is exact BF16
    o[2 * j] = (__float_as_uint(a.x) >> 16) | (__float_as_uint(a.y) & 0xffff0000u);
    o[2 * j + 1] = (__float_as_uint(b.x) >> 16) | (__float_as_uint(b.y) & 0xffff0000u);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Issue the copies of chunk c (dims 8c .. 8c+7) of row r of a row set into BF16 row `dst`
// (E4M3 nope chunks go to `raw` instead, to be widened later).
__device__ __forceinline__ void gather_chunk(const lc_rows& rs, int64_t r, int d_r, int c, uint16_t* dst,
                                             uint8_t* raw) {
  if (rs.fmt == LC_FMT_BF16) {
    cp16(smem_u32(dst + c * 8), static_cast<const uint16_t*>(rs.x) + r * kAD + c * 8);
  } else {
    const int d_n = kAD - d_r;
    if (c * 8 < d_n) cp8(smem_u32(raw + c * 8), static_cast<const uint8_t*>(rs.x) + r * d_n + c * 8);
    else cp16(smem_u32(dst + c * 8), static_cast<const uint16_t*>(rs.rope) + r * d_r + (c * 8 - d_n));
  }
}

struct AttnGeom {
  int n_split;   // CTAs per (query, head group) along the keys
  int sps;       // slots per split (multiple of the key tile)
};

// grid: (n_q, n_hg * n_split); MT * DS warps; TK keys per tile; NBUF tile buffers.
template <int MT, int DS, int TK, int NBUF>
__global__ void __launch_bounds__(MT * DS * 32, 1)
    k_attn_mma(lc_attn_args a, int sparse, AttnGeom geo, float* __restrict__ ws_o, float* __restrict__ ws_ml) {
  constexpr int NW = MT * DS;
  constexpr int NTHR = NW * 32;
  constexpr int ROWS = MT * 16;
  constexpr int DW = kAD / DS;        // output dims per warp
  constexpr int KS = DW / 16;         // k16 steps of the partial S
  constexpr int NTO = DW / 8;         // n8 tiles of O per warp
  constexpr int NTS = TK / 8;         // n8 tiles of S
  constexpr int SPL = TK / 2;         // partial-S floats per lane
  static_assert(DW % 16 == 0 && NTO % 2 == 0 && TK % 16 == 0 && TK <= kTileMax, "tile shape");
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* Qs = reinterpret_cast<uint16_t*>(smem);                 // [ROWS][kRS]
  uint16_t* Ks = Qs + ROWS * kRS;                                    // [NBUF][TK][kRS]
  uint8_t* Raw = reinterpret_cast<uint8_t*>(Ks + NBUF * TK * kRS);   // [NBUF][TK][kRawRow]
  float* Sx = reinterpret_cast<float*>(Raw + NBUF * TK * kRawRow);   // [NW][SPL][32]
  int* kcode = reinterpret_cast<int*>(Sx + NW * SPL * 32);           // [NBUF][TK]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mt = warp / DS, ds = warp % DS;
  const int g = lane >> 2, t4 = lane & 3;
  const int q = blockIdx.x;
  const int hg = blockIdx.y / geo.n_split, split = blockIdx.y % geo.n_split;
  const int H = a.dims.H, d_r = a.dims.d_r;
  const int b = seq_of_query(a.batch.q_start, a.batch.num_seqs, q);
  const int p = __ldg(a.batch.q_pos0 + b) + (q - __ldg(a.batch.q_start + b));
  const int n_ent = __ldg(a.batch.n_ent + b);
  const int nv = n_visible(p, a.m, a.W_x, n_ent);
  const int64_t ent0 = __ldg(a.batch.ent_start + b);
  const int wlo = a.W > 0 ? max(0, p - a.W + 1) : p + 1;
  const int n_win = p + 1 - wlo;
  const int n_first = sparse ? a.k : nv;           // slots before the window
  const int n_slots = n_first + n_win;
  const int s_begin = split * geo.sps;
  const int s_end = min(n_slots, s_begin + geo.sps);
  const int wp0 = a.W > 0 ? __ldg(a.batch.win_pos0 + b) : 0;
  const int wl = a.W > 0 ? __ldg(a.batch.win_len + b) : 0;
  const int64_t wr0 = a.W > 0 ? __ldg(a.batch.win_start + b) : 0;
  const int32_t* idx_row = sparse ? a.idx + static_cast<int64_t>(q) * a.k : nullptr;
  const int n_tiles = s_end > s_begin ? (s_end - s_begin + TK - 1) / TK : 0;

  // slot -> key code: entry index j, kWinFlag | window row, or -1 (masked)
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
    const int rr = wlo + (s - n_first) - wp0;
    if (rr < 0 || rr >= wl) {
      set_status(a.status, LC_DEV_WINDOW_RANGE);
      return -1;
    }
    return static_cast<int>(kWinFlag) | rr;
  };
  // codes of tile t into kcode[buf] (call, then __syncthreads, then issue)
  auto tile_codes = [&](int t, int buf) {
    if (tid < TK) kcode[buf * TK + tid] = slot_code(s_begin + t * TK + tid);
  };
  // cp.async gather of tile t into buffer buf (codes already in kcode[buf])
  auto tile_issue = [&](int buf) {
    uint16_t* kb = Ks + buf * TK * kRS;
    uint8_t* rb = Raw + buf * TK * kRawRow;
    for (int u = tid; u < TK * kChunks; u += NTHR) {
      const int kr = u / kChunks, c = u % kChunks;
      const int code = kcode[buf * TK + kr];
      uint16_t* dst = kb + kr * kRS;
      if (code < 0) reinterpret_cast<uint4*>(dst)[c] = make_uint4(0, 0, 0, 0);
      else if (code & kWinFlag) gather_chunk(a.win, wr0 + (code & ~kWinFlag), d_r, c, dst, rb + kr * kRawRow);
      else gather_chunk(a.ent, ent0 + code, d_r, c, dst, rb + kr * kRawRow);
    }
  };
  // widen the E4M3 nope part of buffer buf (after its copies landed)
  auto tile_widen = [&](int buf) {
    if (a.ent.fmt != LC_FMT_E4M3_BF16) return;
    const int dnc = (kAD - d_r) / 8;
    uint16_t* kb = Ks + buf * TK * kRS;
    const uint8_t* rb = Raw + buf * TK * kRawRow;
    for (int u = tid; u < TK * dnc; u += NTHR) {
      const int kr = u / dnc, c = u % dnc;
      const int code = kcode[buf * TK + kr];
      if (code >= 0 && !(code & kWinFlag))
        reinterpret_cast<uint4*>(kb + kr * kRS)[c] =
            e4m3x8_to_bf16x8(*reinterpret_cast<const uint2*>(rb + kr * kRawRow + c * 8));
    }
  };

  // queries of this head group (cp.async into Qs, E4M3 nope through Raw buffer 0)
  {
    for (int u = tid; u < ROWS * kChunks; u += NTHR) {
      const int r = u / kChunks, c = u % kChunks;
      const int h = hg * ROWS + r;
      uint16_t* dst = Qs + r * kRS;
      if (h < H) gather_chunk(a.q, static_cast<int64_t>(q) * H + h, d_r, c, dst, Raw + r * kRawRow);
      else reinterpret_cast<uint4*>(dst)[c] = make_uint4(0, 0, 0, 0);
    }
    cp_commit();
    cp_wait<0>();
    __syncthreads();
    if (a.q.fmt == LC_FMT_E4M3_BF16) {
      const int dnc = (kAD - d_r) / 8;
      for (int u = tid; u < ROWS * dnc; u += NTHR) {
        const int r = u / dnc, c = u % dnc;
        if (hg * ROWS + r < H)
          reinterpret_cast<uint4*>(Qs + r * kRS)[c] = e4m3x8_to_bf16x8(*reinterpret_cast<const uint2*>(Raw + r * kRawRow + c * 8));
      }
    }
    __syncthreads();  // Raw buffer 0 is free again
  }

  float o[NTO][4];
#pragma unroll
  for (int i = 0; i < NTO; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  const float sl2 = a.scale * 1.4426950408889634f;  // logits in log2 units

  if (n_tiles > 0) {
    tile_codes(0, 0);
    __syncthreads();
    tile_issue(0);
    cp_commit();
  }
  for (int t = 0; t < n_tiles; ++t) {
    const int buf = NBUF == 2 ? (t & 1) : 0;
    if (NBUF == 2) {
      // prefetch tile t + 1 into the other buffer (its last reader finished at the end
      // of the previous iteration)
      if (t + 1 < n_tiles) {
        tile_codes(t + 1, buf ^ 1);
        __syncthreads();
        tile_issue(buf ^ 1);
      }
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    tile_widen(buf);
    __syncthreads();
    const uint16_t* Kb = Ks + buf * TK * kRS;
    const int* kv = kcode + buf * TK;

    // partial S over this warp's dims: 16 rows x TK keys
    float sacc[NTS][4];
#pragma unroll
    for (int i = 0; i < NTS; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
    const uint32_t qa = smem_u32(Qs + (mt * 16 + (lane & 15)) * kRS + ds * DW + (lane >> 4) * 8);
    const uint32_t kb = smem_u32(Kb + ((lane >> 4) * 8 + (lane & 7)) * kRS + ds * DW + ((lane >> 3) & 1) * 8);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(qa + ks * 32, a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < NTS / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + np * 16 * kRS * 2 + ks * 32, b0, b1, b2, b3);
        mma_bf16(sacc[2 * np], a0, a1, a2, a3, b0, b1);
        mma_bf16(sacc[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // add the DS partial sums in a fixed order (every warp of the row tile gets the same S)
    float* mine = Sx + warp * SPL * 32;
#pragma unroll
    for (int i = 0; i < NTS; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) mine[(i * 4 + j) * 32 + lane] = sacc[i][j];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < NTS; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v = Sx[(mt * DS + 0) * SPL * 32 + (i * 4 + j) * 32 + lane];
#pragma unroll
        for (int d = 1; d < DS; ++d) v += Sx[(mt * DS + d) * SPL * 32 + (i * 4 + j) * 32 + lane];
        sacc[i][j] = v;
      }
    // online softmax (log2 units); masked keys get -inf
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < NTS; ++i) {
      const bool v0 = kv[i * 8 + 2 * t4] >= 0, v1 = kv[i * 8 + 2 * t4 + 1] >= 0;
      sacc[i][0] = v0 ? sacc[i][0] * sl2 : -INFINITY;
      sacc[i][1] = v1 ? sacc[i][1] * sl2 : -INFINITY;
      sacc[i][2] = v0 ? sacc[i][2] * sl2 : -INFINITY;
      sacc[i][3] = v1 ? sacc[i][3] * sl2 : -INFINITY;
      tmax[0] = fmaxf(tmax[0], fmaxf(sacc[i][0], sacc[i][1]));
      tmax[1] = fmaxf(tmax[1], fmaxf(sacc[i][2], sacc[i][3]));
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
    }
    float corr[2], mref[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float mn = fmaxf(m_run[r], tmax[r]);
      corr[r] = (m_run[r] == -INFINITY) ? 0.f : exp2f(m_run[r] - mn);
      mref[r] = (mn == -INFINITY) ? 0.f : mn;
      m_run[r] = mn;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < NTS; ++i) {
      sacc[i][0] = exp2f(sacc[i][0] - mref[0]);
      sacc[i][1] = exp2f(sacc[i][1] - mref[0]);
      sacc[i][2] = exp2f(sacc[i][2] - mref[1]);
      sacc[i][3] = exp2f(sacc[i][3] - mref[1]);
      rs[0] += sacc[i][0] + sacc[i][1];
      rs[1] += sacc[i][2] + sacc[i][3];
    }
    l_run[0] = l_run[0] * corr[0] + rs[0];
    l_run[1] = l_run[1] * corr[1] + rs[1];
#pragma unroll
    for (int i = 0; i < NTO; ++i) {
      o[i][0] *= corr[0];
      o[i][1] *= corr[0];
      o[i][2] *= corr[1];
      o[i][3] *= corr[1];
    }
    // O += P V over the TK keys, this warp's dims
#pragma unroll
    for (int kk = 0; kk < TK / 16; ++kk) {
      const uint32_t pa0 = pack_bf16(sacc[2 * kk][0], sacc[2 * kk][1]);
      const uint32_t pa1 = pack_bf16(sacc[2 * kk][2], sacc[2 * kk][3]);
      const uint32_t pa2 = pack_bf16(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]);
      const uint32_t pa3 = pack_bf16(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3]);
      const uint32_t vb =
          smem_u32(Kb + (kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * kRS + ds * DW + (lane >> 4) * 8);
#pragma unroll
      for (int np = 0; np < NTO / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + np * 32, b0, b1, b2, b3);
        mma_bf16(o[2 * np], pa0, pa1, pa2, pa3, b0, b1);
        mma_bf16(o[2 * np + 1], pa0, pa1, pa2, pa3, b2, b3);
      }
    }
    __syncthreads();  // this tile's buffers and Sx are free
    if (NBUF == 1 && t + 1 < n_tiles) {
      tile_codes(t + 1, 0);
      __syncthreads();
      tile_issue(0);
      cp_commit();
    }
  }

  // row sums over the 4 threads of a row
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
  }
  const int hr0 = hg * ROWS + mt * 16 + g;  // head of row g (row g + 8 is hr0 + 8)
  if (geo.n_split == 1) {
    // join the sink and normalise: M = max(sink, m), Z = e^(sink-M) + l e^(m-M)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int h = hr0 + 8 * r;
      if (h >= H) continue;
      const float sk = __ldg(a.sink + h) * 1.4426950408889634f;
      const float M = fmaxf(sk, m_run[r]);
      const float wl_ = (m_run[r] == -INFINITY) ? 0.f : exp2f(m_run[r] - M);
      const float Z = exp2f(sk - M) + l_run[r] * wl_;
      const float f = wl_ / Z;
      const int64_t orow = static_cast<int64_t>(q) * H + h;
      if (a.out_fmt == LC_FMT_BF16) {
        uint32_t* op = reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(a.out) + orow * kAD + ds * DW + 2 * t4);
#pragma unroll
        for (int i = 0; i < NTO; ++i) op[i * 4] = pack_bf16(o[i][2 * r] * f, o[i][2 * r + 1] * f);
      } else {
        float2* op = reinterpret_cast<float2*>(static_cast<float*>(a.out) + orow * kAD + ds * DW + 2 * t4);
#pragma unroll
        for (int i = 0; i < NTO; ++i) op[i * 4] = make_float2(o[i][2 * r] * f, o[i][2 * r + 1] * f);
      }
      if (a.lse && ds == 0 && t4 == 0) a.lse[orow] = (M + log2f(Z)) * 0.6931471805599453f;
    }
  } else {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int h = hr0 + 8 * r;
      if (h >= H) continue;
      const int64_t slot = (static_cast<int64_t>(q) * H + h) * geo.n_split + split;
      const int64_t orow = static_cast<int64_t>(split) * a.n_q * H + static_cast<int64_t>(q) * H + h;
      float2* op = reinterpret_cast<float2*>(ws_o + orow * kAD + ds * DW + 2 * t4);
#pragma unroll
      for (int i = 0; i < NTO; ++i) op[i * 4] = make_float2(o[i][2 * r], o[i][2 * r + 1]);
      if (ds == 0 && t4 == 0) {
        ws_ml[2 * slot] = m_run[r];
        ws_ml[2 * slot + 1] = l_run[r];
      }
    }
  }
}

// Merge the key splits of each (query, head) with the sink, in split order.  Split c of
// row (q * H + h) left its unnormalised O at ws_o row c * n_q * H + q * H + h and its
// (max, sum) at ws_ml[2 ((q * H + h) * n_split + c)].  One thread per (row, 4 dims): the
// loads of all splits are independent, so they are in flight together.
constexpr int kCombineThreads = 256;
constexpr int kQuads = kAD / 4;  // float4 groups per row

// S > 0: exactly S splits, every load issued before any arithmetic (one memory round trip);
// S = 0: any split count, one split after another.  Both add the splits in split order.
template <int S>
__global__ void __launch_bounds__(kCombineThreads) k_attn_combine(lc_attn_args a, int n_split,
                                                                  const float* __restrict__ ws_o,
                                                                  const float* __restrict__ ws_ml) {
  const int64_t rows = static_cast<int64_t>(a.n_q) * a.dims.H;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x;
  if (t >= rows * kQuads) return;
  const int64_t row = t / kQuads;
  const int c4 = static_cast<int>(t % kQuads);
  const int h = static_cast<int>(row % a.dims.H);
  const float sk = __ldg(a.sink + h) * 1.4426950408889634f;
  const float2* ml = reinterpret_cast<const float2*>(ws_ml) + row * n_split;
  const float4* src = reinterpret_cast<const float4*>(ws_o) + row * kQuads + c4;
  const int64_t split_stride = rows * kQuads;
  float M = sk, Z;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  if constexpr (S > 0) {
    float2 mc[S];
    float4 v[S];
#pragma unroll
    for (int c = 0; c < S; ++c) {
      mc[c] = __ldg(ml + c);
      v[c] = __ldg(src + c * split_stride);
    }
#pragma unroll
    for (int c = 0; c < S; ++c) M = fmaxf(M, mc[c].x);
    Z = exp2f(sk - M);
#pragma unroll
    for (int c = 0; c < S; ++c) {
      const float w = mc[c].x == -INFINITY ? 0.f : exp2f(mc[c].x - M);
      Z = fmaf(mc[c].y, w, Z);
      o.x = fmaf(v[c].x, w, o.x);
      o.y = fmaf(v[c].y, w, o.y);
      o.z = fmaf(v[c].z, w, o.z);
      o.w = fmaf(v[c].w, w, o.w);
    }
  } else {
    for (int c = 0; c < n_split; ++c) M = fmaxf(M, __ldg(ml + c).x);
    Z = exp2f(sk - M);
#pragma unroll 4
    for (int c = 0; c < n_split; ++c) {
      const float2 mc = __ldg(ml + c);
      const float4 v = __ldg(src + c * split_stride);
      const float w = mc.x == -INFINITY ? 0.f : exp2f(mc.x - M);
      Z = fmaf(mc.y, w, Z);
      o.x = fmaf(v.x, w, o.x);
      o.y = fmaf(v.y, w, o.y);
      o.z = fmaf(v.z, w, o.z);
      o.w = fmaf(v.w, w, o.w);
    }
  }
  const float inv = 1.f / Z;
  if (a.out_fmt == LC_FMT_BF16) {
    uint2 pk;
    pk.x = pack_bf16(o.x * inv, o.y * inv);
    pk.y = pack_bf16(o.z * inv, o.w * inv);
    reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + row * kAD)[c4] = pk;
  } else {
    reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * kAD)[c4] =
        make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
  }
  if (a.lse && c4 == 0) a.lse[row] = (M + log2f(Z)) * 0.6931471805599453f;
}

static unsigned combine_blocks(const lc_attn_args& a) {
  const int64_t n = static_cast<int64_t>(a.n_q) * a.dims.H * kQuads;
  return static_cast<unsigned>((n + kCombineThreads - 1) / kCombineThreads);
}

static void combine_launch(const lc_attn_args& a, int n_split, const float* ws_o, const float* ws_ml,
                           cudaStream_t st) {
  const unsigned g = combine_blocks(a);
  switch (n_split) {
    case 2: k_attn_combine<2><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 3: k_attn_combine<3><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 4: k_attn_combine<4><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 5: k_attn_combine<5><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 6: k_attn_combine<6><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 7: k_attn_combine<7><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    case 8: k_attn_combine<8><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
    default: k_attn_combine<0><<<g, kCombineThreads, 0, st>>>(a, n_split, ws_o, ws_ml); break;
  }
}

// ---------------------------------------------------------------------------------
// launch configuration
// ---------------------------------------------------------------------------------
constexpr int kTkPrefill = 64;
constexpr int kTkDecode = 32;

bool attn_mma_supported(const lc_attn_args& a) {
  if (a.dims.D != kAD || a.dims.d_r % 8 || a.dims.d_r < 64 || a.dims.H % 16) return false;
  auto ok_rows = [&](const lc_rows& r) {
    return r.fmt == LC_FMT_BF16 || (r.fmt == LC_FMT_E4M3_BF16 && a.dims.d_r > 0);
  };
  if (!ok_rows(a.q) || !ok_rows(a.ent) || (a.W > 0 && a.win.fmt != LC_FMT_BF16)) return false;
  return a.out_fmt == LC_FMT_BF16 || a.out_fmt == LC_FMT_F32;
}

static int max_slots(const lc_attn_args& a, bool sparse) {
  return (sparse ? a.k : a.max_ent) + a.W;
}

AttnGeom attn_geometry(const lc_attn_args& a, bool sparse, bool decode) {
  AttnGeom g{1, 0};
  const int tk = decode ? kTkDecode : kTkPrefill;
  const int ns = max(max_slots(a, sparse), 1);
  const int tiles = (ns + tk - 1) / tk;
  if (decode) {
    // fill ~2 CTAs per SM, but keep >= 8 key tiles (256 keys) per split so that the
    // partial results a split writes stay small next to the keys it reads
    const int ctas = a.n_q * (a.dims.H / 16);
    const int want = (2 * 148 + ctas - 1) / max(ctas, 1);
    int n = min(want, max(1, tiles / 8));
    n = max(1, min(n, tiles));
    const int per = (tiles + n - 1) / n;
    g.n_split = (tiles + per - 1) / per;
    g.sps = per * tk;
  } else {
    g.sps = tiles * tk;
  }
  return g;
}

size_t attn_mma_workspace(const lc_attn_args& a, bool sparse, bool decode) {
  const AttnGeom g = attn_geometry(a, sparse, decode);
  if (g.n_split <= 1) return 0;
  const size_t rows = static_cast<size_t>(a.n_q) * a.dims.H * g.n_split;
  return rows * kAD * sizeof(float) + rows * 2 * sizeof(float);
}

template <int MT, int DS, int TK, int NBUF>
static cudaError_t launch_mma(const lc_attn_args& a, bool sparse, const AttnGeom& g, cudaStream_t st) {
  constexpr int ROWS = MT * 16;
  const size_t sm = static_cast<size_t>(ROWS + NBUF * TK) * kRS * 2 + static_cast<size_t>(NBUF) * TK * kRawRow +
                    static_cast<size_t>(MT * DS) * (TK / 2) * 32 * 4 + NBUF * TK * 4;
  cudaFuncSetAttribute(k_attn_mma<MT, DS, TK, NBUF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(sm));
  const int n_hg = (a.dims.H + ROWS - 1) / ROWS;
  float* ws_o = static_cast<float*>(a.workspace);
  float* ws_ml = nullptr;
  if (g.n_split > 1) {
    const size_t rows = static_cast<size_t>(a.n_q) * a.dims.H * g.n_split;
    ws_ml = ws_o + rows * kAD;
  }
  const dim3 grid(a.n_q, n_hg * g.n_split);
  k_attn_mma<MT, DS, TK, NBUF><<<grid, MT * DS * 32, sm, st>>>(a, sparse ? 1 : 0, g, ws_o, ws_ml);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || g.n_split == 1) return e;
  combine_launch(a, g.n_split, ws_o, ws_ml, st);
  return cudaGetLastError();
}

// Merge step for the key splits of the tensor-core kernel (workspace: partial O, then
// (max, sum) pairs).
cudaError_t launch_attn_combine(const lc_attn_args& a, int n_split, cudaStream_t st) {
  float* ws_o = static_cast<float*>(a.workspace);
  float* ws_ml = ws_o + static_cast<size_t>(a.n_q) * a.dims.H * n_split * kAD;
  combine_launch(a, n_split, ws_o, ws_ml, st);
  return cudaGetLastError();
}

cudaError_t launch_attn_mma(const lc_attn_args& a, bool sparse, bool decode, cudaStream_t st) {
  const AttnGeom g = attn_geometry(a, sparse, decode);
  // decode: one buffer of 32 keys keeps the CTA at 80 KB of shared memory, two per SM
  if (decode) return launch_mma<1, 4, kTkDecode, 1>(a, sparse, g, st);
  if (a.dims.H % 64) return launch_mma<1, 4, kTkPrefill, 1>(a, sparse, g, st);
  return launch_mma<4, 2, kTkPrefill, 1>(a, sparse, g, st);
}

}  // namespace lc
