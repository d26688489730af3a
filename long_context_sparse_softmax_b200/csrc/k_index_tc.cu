// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05, block-scaled FP4).
//
// s(p, j) = sum_h w_h * ReLU(<qI[p, h], kI[j]>) over the entries j visible to the query at
// p ("解读 DeepSeek V4", CSA section and "FP4 Quantization-Aware Training": the indexer QK
// path runs in MXFP4; "DeepSeek-V4 论文分析" §5.3, §8.3).
//
// One MMA tile: A = 128 keys x d_I (K-major E2M1, 2 per byte) in shared memory, B = the H_I
// heads of QPC queries (N = QPC * H_I <= 256), block scales (E8M0, one per 32 elements) in
// tensor memory, D = 128 x N FP32 in tensor memory.  The tensor core applies the block
// scales; the operands are the caller's bytes, never widened or converted.
//
//   * shared layout: no-swizzle K-major core matrices, 8 rows x 16 bytes each, 128 bytes
//     apart along K (LBO) and 512 bytes apart along rows (SBO); a 128 x 128 FP4 tile is 8 KB;
//   * scale factors in tensor memory: column c holds, in lane L (all four lane quadrants),
//     the four E8M0 bytes (K blocks 0..3) of row (L % 32) + 32 c; the k-th K = 64 MMA reads
//     bytes 2k, 2k+1 (sf_id = 2k);
//   * key tiles stream through three shared buffers with cp.async, two tiles ahead;
//   * epilogue: thread t of the 128 owns key row t of D (tcgen05.ld 32x32b), so the
//     ReLU-weighted head sum stays in registers, in a fixed order.
//
// Every wait on the tensor core is bounded: after ~2^26 polls the kernel records
// LC_DEV_TIMEOUT in the status word, stops issuing work, and releases its tensor memory.
#include "lc_internal.h"

namespace lc {

namespace {

constexpr int kKeys = 128;          // keys per tile (MMA M)
constexpr int kDI = 128;            // indexer dims handled here (2 MMAs of K = 64)
constexpr int kRowB = kDI / 2;      // bytes per row
constexpr int kTileB = kKeys * kRowB;
constexpr int kStages = 3;
constexpr long kSpinLimit = 1L << 26;

__device__ __forceinline__ uint32_t su32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// byte offset of (row, byte) in the core-matrix layout
__device__ __forceinline__ uint32_t cm_off(int r, int b) {
  return (r >> 3) * 512 + (b >> 4) * 128 + (r & 7) * 16 + (b & 15);
}

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  uint64_t d = static_cast<uint64_t>((addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(128 >> 4) << 16;   // LBO: next core matrix along K
  d |= static_cast<uint64_t>(512 >> 4) << 32;   // SBO: next 8-row group
  d |= static_cast<uint64_t>(1) << 46;          // descriptor version for sm_100
  return d;                                     // base offset 0, no swizzle
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  uint32_t done = 0;
  for (long it = 0; it < kSpinLimit; ++it) {
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity));
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n"); }

__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace

// grid: (query chunks of QPC queries, key-range chunks); 128 threads.
// TMEM columns: D [0, N), SFA [N, N + 4), SFB [N + 8, N + 8 + N / 32).
template <int QPC>
__global__ void __launch_bounds__(128) k_index_tc(lc_index_args a, int tiles_per_cta, uint32_t tmem_cols) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int H = a.H_I;
  const int N = QPC * H;
  uint8_t* As = smem;                                               // [kStages][kTileB]
  uint8_t* Bs = As + kStages * kTileB;                              // [N rows][64 B] core matrices
  uint32_t* SFs = reinterpret_cast<uint32_t*>(Bs + N * kRowB);      // [kStages][128] key scale words
  float* ws = reinterpret_cast<float*>(SFs + kStages * kKeys);      // [N] head weights
  __shared__ uint32_t s_tmem;
  __shared__ __align__(8) uint64_t s_mbar;
  __shared__ int s_nv[QPC];
  __shared__ int s_q[QPC];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qa = blockIdx.x * QPC;
  if (qa >= a.n_q) return;
  const int b = seq_of_query(a.batch.q_start, a.batch.num_seqs, qa);
  const int64_t kbase = __ldg(a.batch.ent_start + b);
  const int n_ent = __ldg(a.batch.n_ent + b);
  // queries of this chunk: they must belong to sequence b (prefill: one sequence;
  // decode: QPC = 1)
  int nv_max = 0;
  if (tid < QPC) {
    const int q = qa + tid;
    int nv = 0;
    if (q < a.n_q && q < __ldg(a.batch.q_start + b + 1)) {
      const int p = __ldg(a.batch.q_pos0 + b) + (q - __ldg(a.batch.q_start + b));
      nv = n_visible(p, a.m, a.W_x, n_ent);
    }
    s_nv[tid] = nv;
    s_q[tid] = q;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < QPC; ++i) nv_max = max(nv_max, s_nv[i]);
  const int t_begin = blockIdx.y * tiles_per_cta;
  const int t_end = min(t_begin + tiles_per_cta, (nv_max + kKeys - 1) / kKeys);
  if (t_begin >= t_end) return;

  // query operand B (rows n = i * H + h), its scales, head weights
  for (int c = tid; c < N * 4; c += 128) {
    const int n = c >> 2, seg = c & 3;
    const int i = n / H, h = n % H;
    const int q = s_q[i];
    const bool ok = q < a.n_q && s_nv[i] > 0;
    const uint8_t* src = static_cast<const uint8_t*>(a.q) + (static_cast<int64_t>(ok ? q : 0) * H + h) * kRowB + seg * 16;
    cp_async16(su32(Bs + cm_off(n, seg * 16)), src, ok);
  }
  for (int u = tid; u < N; u += 128) {
    const int i = u / H, h = u % H;
    ws[u] = __ldg(a.w + static_cast<int64_t>(s_q[i] < a.n_q ? s_q[i] : 0) * a.w_qstride + h);
  }
  cp_async_commit();

  auto load_tile = [&](int t, int stage) {
    const int j0 = t * kKeys;
    uint8_t* dst = As + stage * kTileB;
    for (int c = tid; c < kKeys * 4; c += 128) {
      const int r = c >> 2, seg = c & 3;
      const int j = j0 + r;
      const bool ok = j < n_ent;
      const uint8_t* src = static_cast<const uint8_t*>(a.k) + (kbase + (ok ? j : 0)) * kRowB + seg * 16;
      cp_async16(su32(dst + cm_off(r, seg * 16)), src, ok);
    }
    {  // the 4 scale bytes of key row tid (4-byte aligned: a sequence may start anywhere)
      const int j = j0 + tid;
      const bool ok = j < n_ent;
      const uint8_t* src = a.k_scale + (kbase + (ok ? j : 0)) * 4;
      cp_async4(su32(SFs + stage * kKeys + tid), src, ok);
    }
  };

  // tensor memory
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(&s_tmem)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(su32(&s_mbar)));
    asm volatile("fence.mbarrier_init.release.cluster;\n");
  }
  load_tile(t_begin, 0);
  cp_async_commit();
  if (t_begin + 1 < t_end) load_tile(t_begin + 1, 1);
  cp_async_commit();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = s_tmem;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t col_sfa = static_cast<uint32_t>(N), col_sfb = static_cast<uint32_t>(N + 8);

  // query scales -> tensor memory (lane L of every quadrant, column c: row (L % 32) + 32 c)
  {
    uint32_t v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int n = lane + 32 * c;
      uint32_t w = 0x7f7f7f7fu;
      if (n < N) {
        const int i = n / H, h = n % H;
        const int q = s_q[i];
        if (q < a.n_q) w = __ldg(reinterpret_cast<const uint32_t*>(a.q_scale) + static_cast<int64_t>(q) * H + h);
      }
      v[c] = w;
    }
    tmem_st4(tm + lane_off + col_sfb, v[0], v[1], v[2], v[3]);
    if (N > 128) tmem_st4(tm + lane_off + col_sfb + 4, v[4], v[5], v[6], v[7]);
  }

  // instruction descriptor: E2M1 x E2M1, E8M0 scales, FP32 accumulate, M = 128, N
  const uint32_t idesc0 = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
                          (static_cast<uint32_t>(kKeys >> 4) << 24);
  bool alive = true;
  uint32_t phase = 0;
  for (int t = t_begin; t < t_end; ++t) {
    const int it = t - t_begin;
    const int stage = it % kStages;
    if (t + 2 < t_end) load_tile(t + 2, (it + 2) % kStages);
    cp_async_commit();
    cp_async_wait<2>();  // tile t (and B) landed
    asm volatile("fence.proxy.async.shared::cta;\n");
    __syncthreads();
    // key scales of this tile -> tensor memory
    {
      const uint32_t* sf = SFs + stage * kKeys;
      tmem_st4(tm + lane_off + col_sfa, sf[lane], sf[lane + 32], sf[lane + 64], sf[lane + 96]);
      asm volatile("tcgen05.wait::st.sync.aligned;\n");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0 && alive) {
      const uint32_t a_base = su32(As + stage * kTileB), b_base = su32(Bs);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint32_t sfid = 2u * k;
        const uint32_t idesc = idesc0 | (sfid << 29) | (sfid << 4);
        const uint64_t da = smem_desc(a_base + k * 256), db = smem_desc(b_base + k * 256);
        asm volatile(
            "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(tm),
            "l"(da), "l"(db), "r"(idesc), "r"(k), "r"((tm + col_sfa) | (sfid << 30)), "r"((tm + col_sfb) | (sfid << 30)));
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
          su32(&s_mbar)));
    }
    if (alive && !mbar_wait(su32(&s_mbar), phase)) {
      alive = false;
      set_status(a.status, LC_DEV_TIMEOUT);
    }
    phase ^= 1u;
    tc_fence_after();
    if (alive) {
      // epilogue: this thread's key row, the H columns of each query
      const int j = t * kKeys + tid;
#pragma unroll
      for (int i = 0; i < QPC; ++i) {
        float s = 0.f;
        for (int h0 = 0; h0 < H; h0 += 32) {
          float v[32];
          tmem_ld32(tm + lane_off + static_cast<uint32_t>(i * H + h0), v);
#pragma unroll
          for (int u = 0; u < 32; ++u) s = fmaf(ws[i * H + h0 + u], fmaxf(v[u], 0.f), s);
        }
        if (j < s_nv[i]) a.scores[static_cast<int64_t>(s_q[i]) * a.score_stride + j] = s;
      }
    }
    tc_fence_before();
    __syncthreads();  // D and the tile's buffers are free again
  }
  cp_async_wait<0>();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tm), "r"(tmem_cols));
}

bool index_tc_supported(const lc_index_args& a) {
  return a.fmt == LC_IDX_MXFP4 && a.d_I == kDI && a.H_I % 32 == 0 && a.H_I <= 256;
}

cudaError_t launch_index_tc(const lc_index_args& a, bool decode, cudaStream_t st) {
  const int H = a.H_I;
  int qpc = 1;
  if (!decode && a.batch.num_seqs == 1) qpc = (H <= 64) ? 2 : 1;
  const int N = qpc * H;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(N + 16)) cols <<= 1;
  const int tiles = (a.max_ent + kKeys - 1) / kKeys;
  const int n_qc = (a.n_q + qpc - 1) / qpc;
  // decode: split each query's keys so that ~4 CTAs run per SM
  int tpc = tiles;
  if (decode) {
    const int want = max(1, (4 * 148 + n_qc - 1) / n_qc);
    tpc = max(4, (tiles + want - 1) / want);
  } else {
    tpc = max(1, min(tiles, 16));
  }
  const dim3 grid(n_qc, (tiles + tpc - 1) / tpc);
  size_t sm = static_cast<size_t>(kStages) * kTileB + static_cast<size_t>(N) * kRowB + kStages * kKeys * 4 +
              static_cast<size_t>(N) * 4;
  // ask for enough shared memory that no more CTAs share an SM than its 512 tensor-memory
  // columns hold, so tcgen05.alloc never has to wait for another CTA
  const size_t per_sm = 227 * 1024;
  const size_t cap = per_sm / (512 / cols) - 2048;
  if (sm < cap) sm = cap;
  switch (qpc) {
    case 1:
      cudaFuncSetAttribute(k_index_tc<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
      k_index_tc<1><<<grid, 128, sm, st>>>(a, tpc, cols);
      break;
    case 2:
      cudaFuncSetAttribute(k_index_tc<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
      k_index_tc<2><<<grid, 128, sm, st>>>(a, tpc, cols);
      break;
    default:
      cudaFuncSetAttribute(k_index_tc<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
      k_index_tc<4><<<grid, 128, sm, st>>>(a, tpc, cols);
      break;
  }
  return cudaGetLastError();
}

}  // namespace lc
