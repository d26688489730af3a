// Grouped output projection of the attention heads (10100.com analysis §三.1: CSA and HCA
// both use a grouped output projection to cut its cost).  The H heads of a query are split
// into G groups of H / G consecutive heads; group g projects the concatenation of its heads'
// outputs, K = (H / G) Dv values, to its own d_g output dims with its own weights:
//   y[n, g d_g + c] = sum_k x[n, g K + k] W_g[k, c].
// That is one GEMM per group (M = queries, N = d_g, K); a dense projection of all H Dv
// values would cost G times as much.
//
// tcgen05 kind::f16 (BF16 x BF16, FP32 accumulate in tensor memory).  One CTA per
// 128 x 128 output tile of one group; K in steps of 64 through a 6-stage ring of 2-D bulk
// tensor copies (TMA, 128-byte swizzle: A = 128 query rows x 64 values of x, B = 128 output
// rows x 64 values of W_g^T).  Warp 0 loads, lane 0 of warp 1 issues four K = 16 MMAs per
// stage, warps 2-5 read the accumulator (thread t owns query row t of the tile) and store
// the rows.  Rows past n_q and columns past d_g are computed on zero-filled or neighbouring
// operands and never stored.  Every wait is bounded (LC_DEV_TIMEOUT).
#include <cuda.h>

#include "lc_internal.h"
#include "lc_ptx.cuh"

namespace lc {

namespace {

constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kStages = 6;
constexpr int kTileA = kBM * kBK * 2;  // 16 KB
constexpr int kTileB = kBN * kBK * 2;  // 16 KB
constexpr int kThreads = 192;
constexpr long kSpin = 1L << 26;
constexpr size_t kSmem = static_cast<size_t>(kStages) * (kTileA + kTileB) + 1024;

struct ProjBars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t done;
};

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    k_out_proj(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw, lc_out_proj_args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* As = smem;
  uint8_t* Bs = smem + kStages * kTileA;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ __align__(8) ProjBars bars;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * kBN, g = blockIdx.z;
  const int K = (a.H / a.G) * a.Dv;
  const int nk = K / kBK;

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

  if (warp == 1) tmem_alloc(su32(&s_tmem), kBN);
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(su32(&bars.full[i]), 1);
      mbar_init(su32(&bars.empty[i]), 1);
    }
    mbar_init(su32(&bars.done), 1);
    fence_mbar_init();
    prefetch_tensormap(&tx);
    prefetch_tensormap(&tw);
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % kStages;
        if (kt >= kStages && !wait(&bars.empty[s], ((kt / kStages) - 1) & 1)) break;
        const uint32_t full = su32(&bars.full[s]);
        mbar_expect_tx(full, kTileA + kTileB);
        tma_tile2d(su32(As + s * kTileA), &tx, g * K + kt * kBK, m0, full);
        tma_tile2d(su32(Bs + s * kTileB), &tw, kt * kBK, g * a.d_g + n0, full);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // BF16 x BF16 -> FP32, A and B K-major, M = 128, N = 128
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                             (static_cast<uint32_t>(kBM >> 4) << 24);
      bool ok = true;
      for (int kt = 0; ok && kt < nk; ++kt) {
        const int s = kt % kStages;
        ok = wait(&bars.full[s], (kt / kStages) & 1);
        if (!ok) break;
        fence_after();
        const uint32_t ab = su32(As + s * kTileA), bb = su32(Bs + s * kTileB);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          mma_f16(tm, sw128_desc(ab + k * 32), sw128_desc(bb + k * 32), idesc, kt > 0 || k > 0);
        mma_commit(su32(&bars.empty[s]));
      }
      mma_commit(su32(&bars.done));
    }
  } else {
    // warps 2-5: thread -> accumulator row (lane quadrant of the warp)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const bool ok = wait(&bars.done, 0);
    fence_after();
    const int n = m0 + row;
    const int64_t ybase = static_cast<int64_t>(n) * a.G * a.d_g + static_cast<int64_t>(g) * a.d_g + n0;
#pragma unroll 1
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tm + lane_off + c0, v);
      tmem_wait_ld();
      if (!ok || n >= a.n_q) continue;
      if (a.out_fmt == LC_FMT_F32) {
        float* y = static_cast<float*>(a.y) + ybase + c0;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (n0 + c0 + i < a.d_g) y[i] = __uint_as_float(v[i]);
      } else {
        uint16_t* y = static_cast<uint16_t*>(a.y) + ybase + c0;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (n0 + c0 + i < a.d_g) y[i] = f32_to_bf16_bits(__uint_as_float(v[i]));
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tm, kBN);
}

namespace {

using EncodeTiledP = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledP encode_p() {
  static EncodeTiledP fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledP>(nullptr);
    return reinterpret_cast<EncodeTiledP>(f);
  }();
  return fn;
}

// [rows, cols] BF16 row-major, 64 x 128 boxes, 128-byte swizzle; rows past the end read as 0
bool bf16_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {kBK, 128};
  const cuuint32_t es[2] = {1, 1};
  return encode_p()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_out_proj(const lc_out_proj_args& a, cudaStream_t st) {
  if (a.n_q == 0) return cudaSuccess;
  if (!encode_p()) return cudaErrorNotSupported;
  const int64_t K = static_cast<int64_t>(a.H / a.G) * a.Dv;
  CUtensorMap tx, tw;
  if (!bf16_map(&tx, a.x, a.n_q, static_cast<int64_t>(a.H) * a.Dv) ||
      !bf16_map(&tw, a.w, static_cast<int64_t>(a.G) * a.d_g, K))
    return cudaErrorInvalidValue;
  const dim3 grid((a.n_q + kBM - 1) / kBM, (a.d_g + kBN - 1) / kBN, a.G);
  cudaFuncSetAttribute(k_out_proj, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
  k_out_proj<<<grid, kThreads, kSmem, st>>>(tx, tw, a);
  return cudaGetLastError();
}

}  // namespace lc
