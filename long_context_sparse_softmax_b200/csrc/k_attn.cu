// CSA sparse attention and HCA dense attention with sliding window and attention sink
// ("解读 DeepSeek V4": CSA attends only to the top-k compressed entries, HCA densely to all
// heavily compressed entries, both joined with a 128-token sliding window; an attention
// sink lets a head attend to nothing.  "DeepSeek-V4 论文分析" §5.4, §六, §七, §8.4).
//
// For a query at p and head h, keys = selected (CSA) or all visible (HCA) entries, then
// the window rows for positions max(0, p-W+1) .. p; values are the same rows.
//   l = scale <q_h, key>, running max M starts at the sink logit, Z at e^0 = 1;
//   o = sum e^(l-M) key / Z, lse = M + ln Z.
//
// Reference kernel: one warp per (query, head), online softmax over the keys in order,
// 8 dims per lane group.  Used for small shapes and as the baseline the tensor-core
// kernels are checked against.
#include "lc_internal.h"

namespace lc {

constexpr int kAttnGroups = 4;  // D <= 1024

struct OnlineSoftmax {
  float m, z;
  Vec8 o[kAttnGroups];
};

__device__ __forceinline__ void attend_row(OnlineSoftmax& st, const Vec8 (&q)[kAttnGroups], const lc_rows& rows,
                                           int64_t r, int D, int d_r, int lane, float scale) {
  const int G = D >> 3;
  Vec8 v[kAttnGroups];
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < kAttnGroups; ++i) {
    const int g = lane + kWarp * i;
    if (g < G) {
      v[i] = load8_rows(rows, r, D, d_r, g << 3);
#pragma unroll
      for (int u = 0; u < 8; ++u) dot = fmaf(q[i].v[u], v[i].v[u], dot);
    }
  }
  const float l = scale * warp_sum(dot);
  float cw, ew;  // weight of the old state, weight of this key
  if (l > st.m) {
    cw = expf(st.m - l);
    ew = 1.f;
    st.m = l;
  } else {
    cw = 1.f;
    ew = expf(l - st.m);
  }
  st.z = fmaf(st.z, cw, ew);
#pragma unroll
  for (int i = 0; i < kAttnGroups; ++i) {
    const int g = lane + kWarp * i;
    if (g < G)
#pragma unroll
      for (int u = 0; u < 8; ++u) st.o[i].v[u] = fmaf(st.o[i].v[u], cw, ew * v[i].v[u]);
  }
}

// grid: (n_q, ceil(H / 8)); 8 warps, one head each.
__global__ void __launch_bounds__(256) k_attn_ref(lc_attn_args a, int sparse) {
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int q = blockIdx.x;
  const int H = a.dims.H, D = a.dims.D, d_r = a.dims.d_r;
  if (a.pdl) asm volatile("griddepcontrol.wait;\n" ::: "memory");  // the previous kernel's top-k
  if (h >= H) return;
  const int b = seq_of_query(a.batch.q_start, a.batch.num_seqs, q);
  const int p = __ldg(a.batch.q_pos0 + b) + (q - __ldg(a.batch.q_start + b));
  const int n_ent = __ldg(a.batch.n_ent + b);
  const int nv = n_visible(p, a.m, a.W_x, n_ent);
  const int64_t ent0 = __ldg(a.batch.ent_start + b);
  const int G = D >> 3;
  const int64_t qrow = static_cast<int64_t>(q) * H + h;
  Vec8 qv[kAttnGroups];
#pragma unroll
  for (int i = 0; i < kAttnGroups; ++i) {
    const int g = lane + kWarp * i;
    if (g < G) qv[i] = load8_rows(a.q, qrow, D, d_r, g << 3);
  }
  OnlineSoftmax st;
  st.m = __ldg(a.sink + h);
  st.z = 1.f;
#pragma unroll
  for (int i = 0; i < kAttnGroups; ++i)
#pragma unroll
    for (int u = 0; u < 8; ++u) st.o[i].v[u] = 0.f;

  if (sparse) {
    const int32_t* ir = a.idx + static_cast<int64_t>(q) * a.k;
    for (int s = 0; s < a.k; ++s) {
      const int j = __ldg(ir + s);
      if (j < 0) continue;
      if (j >= n_ent) {
        if (lane == 0) set_status(a.status, LC_DEV_BAD_INDEX);
        continue;
      }
      if (j >= nv) {
        if (lane == 0) set_status(a.status, LC_DEV_NONVISIBLE);
        continue;
      }
      attend_row(st, qv, a.ent, ent0 + j, D, d_r, lane, a.scale);
    }
  } else {
    for (int j = 0; j < nv; ++j) attend_row(st, qv, a.ent, ent0 + j, D, d_r, lane, a.scale);
  }
  if (a.W > 0) {
    const int wp0 = __ldg(a.batch.win_pos0 + b), wl = __ldg(a.batch.win_len + b);
    const int64_t wr0 = __ldg(a.batch.win_start + b);
    const int ring = a.batch.win_ring;
    for (int t = max(0, p - a.W + 1); t <= p; ++t) {
      const int r = t - wp0;
      if (r < 0 || r >= wl) {
        if (lane == 0) set_status(a.status, LC_DEV_WINDOW_RANGE);
        continue;
      }
      attend_row(st, qv, a.win, wr0 + (ring > 0 ? t % ring : r), D, d_r, lane, a.scale);
    }
  }
  const float inv = 1.f / st.z;
  lc_rows out;
  out.fmt = a.out_fmt;
  out.x = a.out;
  out.rope = nullptr;
  // values: every dim, or (v_nope) the non-RoPE dims, written in logical order
  const int rope_off = a.dims.rope_off;
  const int Dv = a.v_nope ? D - d_r : D;
#pragma unroll
  for (int i = 0; i < kAttnGroups; ++i) {
    const int g = lane + kWarp * i;
    if (g < G) {
      int d = g << 3;
      if (a.v_nope) {
        if (d >= rope_off && d < rope_off + d_r) continue;
        if (d >= rope_off + d_r) d -= d_r;
      }
      Vec8 o;
#pragma unroll
      for (int u = 0; u < 8; ++u) o.v[u] = st.o[i].v[u] * inv;
      store8(out, qrow, Dv, 0, d, o);
    }
  }
  if (a.lse && lane == 0) a.lse[qrow] = st.m + logf(st.z);
}

// The kernel a call runs.  AUTO (and TC) take the tcgen05 kernels where they apply
// (576-dim rows with 64 RoPE dims, 64-head groups, 16-byte aligned buffers): the
// E4M3-score kernel where queries and entries are E4M3 + BF16 RoPE, else the F16-operand
// kernel (BF16 queries).  Every other shape (the FP32 workload, other head dims) runs on
// the reference kernel above, which REF also forces.
static bool tc_any(const lc_attn_args& a) { return attn_tc8_supported(a) || attn_tc_supported(a); }

int attn_impl(const lc_attn_args& a) {
  if (a.impl == LC_IMPL_REF) return LC_IMPL_REF;
  if (a.impl == LC_IMPL_TC) return LC_IMPL_TC;
  return tc_any(a) ? LC_IMPL_TC : LC_IMPL_REF;
}

bool attn_impl_ok(const lc_attn_args& a) { return attn_impl(a) == LC_IMPL_REF || tc_any(a); }

size_t attn_workspace_bytes(const lc_attn_args& a, bool sparse, bool decode) {
  if (attn_impl(a) != LC_IMPL_TC) return 0;
  // the formats decide between the two tcgen05 kernels (buffer alignment is validated
  // separately), so the size is known before the buffers are
  lc_attn_args t = a;
  t.out = nullptr;
  t.workspace = nullptr;
  if (attn_tc8_supported(t)) return attn_tc8_workspace(a, sparse, decode);
  return attn_tc_supported(t) ? attn_tc_workspace(a, sparse, decode) : 0;
}

// The optional prefill workspace: the F16 image of the entries that the F16-operand kernel
// reads instead of widening each query's tiles (dense keys, BF16 queries).
size_t attn_image_bytes(const lc_attn_args& a, bool sparse, bool decode) {
  if (attn_impl(a) != LC_IMPL_TC) return 0;
  lc_attn_args t = a;
  t.out = nullptr;
  t.workspace = nullptr;
  if (attn_tc8_supported(t) || !attn_tc_supported(t)) return 0;
  return attn_tc_image_bytes(a, sparse, decode);
}

cudaError_t launch_attn(const lc_attn_args& a, bool sparse, bool decode, cudaStream_t st) {
  if (a.n_q == 0) return cudaSuccess;
  if (attn_impl(a) == LC_IMPL_TC) {
    int n_split = 1;
    const bool fp8 = attn_tc8_supported(a);
    cudaError_t e = fp8 ? launch_attn_tc8(a, sparse, decode, st, &n_split) : launch_attn_tc(a, sparse, decode, st, &n_split);
    if (e != cudaSuccess || n_split == 1) return e;
    return launch_attn_combine(a, n_split, st);
  }
  const dim3 grid(a.n_q, (a.dims.H + 7) / 8);
  return launch_ex(k_attn_ref, grid, dim3(256), 0, st, a.pdl != 0, 1, a, sparse ? 1 : 0);
}

}  // namespace lc
