// C ABI of the CSA / HCA attention library: host-side validation, then one launch (or a
// short fixed sequence of launches) on the caller's stream.  See include/lc.h.
#include <atomic>
#include <cstdint>

#include "lc_internal.h"

namespace lc {

int sm_count() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

}  // namespace lc

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lc_status check_dims(const lc_dims& d) {
  if (d.D < 8 || d.D > 1024 || d.D % 8) return LC_ERR_ARG;
  if (d.d_r < 0 || d.d_r > d.D || d.d_r % 8 || d.d_r > 2 * lc::kMaxRopePairs) return LC_ERR_ARG;
  if (d.rope_off < 0 || d.rope_off % 8 || d.rope_off + d.d_r > d.D) return LC_ERR_ARG;
  if (d.H < 1) return LC_ERR_ARG;
  return LC_OK;
}

lc_status check_rows(const lc_rows& r, const lc_dims& d, bool need) {
  if (r.fmt != LC_FMT_F32 && r.fmt != LC_FMT_BF16 && r.fmt != LC_FMT_E4M3_BF16) return LC_ERR_ARG;
  if (!need) return LC_OK;
  if (!r.x) return LC_ERR_ARG;
  if (!aligned16(r.x)) return LC_ERR_ALIGN;
  if (r.fmt == LC_FMT_E4M3_BF16) {
    if (d.d_r <= 0 || d.rope_off != d.D - d.d_r || !r.rope) return LC_ERR_ARG;
    if (!aligned16(r.rope)) return LC_ERR_ALIGN;
  }
  return LC_OK;
}

lc_status check_batch(const lc_batch& b, bool ents, bool window) {
  if (b.num_seqs < 1) return LC_ERR_ARG;
  if (!b.q_start || !b.q_pos0) return LC_ERR_ARG;
  if (ents && (!b.ent_start || !b.n_ent)) return LC_ERR_ARG;
  if (window && (!b.win_start || !b.win_pos0 || !b.win_len)) return LC_ERR_ARG;
  return LC_OK;
}

lc_status launched(cudaError_t e) { return e == cudaSuccess ? LC_OK : LC_ERR_LAUNCH; }

#define LC_TRY(x)                      \
  do {                                 \
    const lc_status s_ = (x);          \
    if (s_ != LC_OK) return s_;        \
  } while (0)

lc_status qk_prep(const lc_qk_prep_args* a, void* stream) {
  if (!a) return LC_ERR_ARG;
  LC_TRY(check_dims(a->dims));
  if (a->in_fmt != LC_FMT_F32 && a->in_fmt != LC_FMT_BF16) return LC_ERR_ARG;
  if (a->n_tok < 0) return LC_ERR_ARG;
  const bool need = a->n_tok > 0;
  LC_TRY(check_rows(a->out, a->dims, need));
  if (need && (!a->x || !a->pos)) return LC_ERR_ARG;
  if (need && !aligned16(a->x)) return LC_ERR_ALIGN;
  return launched(lc::launch_qk_prep(*a, static_cast<cudaStream_t>(stream)));
}

lc_status compress(const lc_compress_args* a, void* stream, bool hca) {
  if (!a) return LC_ERR_ARG;
  LC_TRY(check_dims(a->dims));
  if (hca ? (a->m < 64 || a->m > 1024 || a->m % 32) : (a->m < 1 || a->m > 64)) return LC_ERR_ARG;
  if (a->in_fmt != LC_FMT_F32 && a->in_fmt != LC_FMT_BF16) return LC_ERR_ARG;
  if (a->num_seqs < 0 || a->max_blocks < 0) return LC_ERR_ARG;
  const bool need = a->num_seqs > 0 && a->max_blocks > 0;
  LC_TRY(check_rows(a->out, a->dims, need));
  if (need && (!a->x || !a->g || !a->tok_row0 || !a->tok_pos0 || !a->tok_len || !a->blk_first ||
               !a->blk_count || !a->ent_start))
    return LC_ERR_ARG;
  if (need && !aligned16(a->x)) return LC_ERR_ALIGN;
  return launched(lc::launch_compress(*a, hca, static_cast<cudaStream_t>(stream)));
}

// Validation shared by the indexer calls; `scores` says whether a score matrix is written.
lc_status check_index(const lc_index_args* a, bool decode, bool scores) {
  if (!a) return LC_ERR_ARG;
  if (a->n_q < 0 || a->max_ent < 0 || a->m < 1 || a->W_x < 0) return LC_ERR_ARG;
  if (a->H_I < 1) return LC_ERR_ARG;
  if (a->fmt == LC_IDX_F32) {
    if (a->d_I < 4 || a->d_I % 4 || a->d_I > 256 || a->H_I * a->d_I > 16384) return LC_ERR_UNSUPPORTED;
  } else if (a->fmt == LC_IDX_MXFP4 || a->fmt == LC_IDX_MXFP4_QBF16) {
    // the tensor-core kernel: 128 dims (two K = 64 block-scaled MMAs), 32 or 64 heads
    if (a->d_I != 128 || (a->H_I != 32 && a->H_I != 64)) return LC_ERR_UNSUPPORTED;
  } else {
    return LC_ERR_ARG;
  }
  if (a->w_qstride != 0 && a->w_qstride != a->H_I) return LC_ERR_ARG;
  if (scores && (a->score_stride < a->max_ent || a->score_stride % 4)) return LC_ERR_ARG;
  if (decode && a->n_q != a->batch.num_seqs) return LC_ERR_ARG;
  if (a->n_q == 0 || a->max_ent == 0) return LC_OK;
  LC_TRY(check_batch(a->batch, true, false));
  if (!a->q || !a->k || !a->w || (scores && !a->scores)) return LC_ERR_ARG;
  const bool mx = a->fmt == LC_IDX_MXFP4 || a->fmt == LC_IDX_MXFP4_QBF16;
  if (mx && (!a->k_scale || a->n_keys < 1 || a->n_keys >= (int64_t{1} << 31))) return LC_ERR_ARG;
  if (a->fmt == LC_IDX_MXFP4 && !a->q_scale) return LC_ERR_ARG;
  if (mx && (reinterpret_cast<uintptr_t>(a->k_scale) & 3u)) return LC_ERR_ALIGN;
  if (a->fmt == LC_IDX_MXFP4 && (reinterpret_cast<uintptr_t>(a->q_scale) & 3u)) return LC_ERR_ALIGN;
  if (!aligned16(a->q) || !aligned16(a->k) || (scores && !aligned16(a->scores))) return LC_ERR_ALIGN;
  return LC_OK;
}

lc_status mxfp4_quantize(const lc_mxfp4_quant_args* a, void* stream) {
  if (!a) return LC_ERR_ARG;
  if (a->n_rows < 0 || a->d < 32 || a->d > 1024 || a->d % 32) return LC_ERR_ARG;
  if (a->in_fmt != LC_FMT_F32 && a->in_fmt != LC_FMT_BF16) return LC_ERR_ARG;
  if (a->n_rows == 0) return LC_OK;
  if (!a->x || !a->codes || !a->scales) return LC_ERR_ARG;
  if (!aligned16(a->x) || (reinterpret_cast<uintptr_t>(a->codes) & 15u) || (reinterpret_cast<uintptr_t>(a->scales) & 3u))
    return LC_ERR_ALIGN;
  return launched(lc::launch_mxfp4_quantize(*a, static_cast<cudaStream_t>(stream)));
}

lc_status index_compress(const lc_index_compress_args* a, void* stream) {
  if (!a) return LC_ERR_ARG;
  if (a->d_I < 32 || a->d_I > 256 || a->d_I % 32 || a->m < 1 || a->m > 64) return LC_ERR_ARG;
  if (a->in_fmt != LC_FMT_F32 && a->in_fmt != LC_FMT_BF16) return LC_ERR_ARG;
  if (a->num_seqs < 0 || a->max_blocks < 0) return LC_ERR_ARG;
  if (a->num_seqs == 0 || a->max_blocks == 0) return LC_OK;
  if (!a->x || !a->g || !a->tok_row0 || !a->tok_pos0 || !a->tok_len || !a->blk_first || !a->blk_count ||
      !a->ent_start || !a->codes || !a->scales)
    return LC_ERR_ARG;
  if (!aligned16(a->x) || (reinterpret_cast<uintptr_t>(a->codes) & 15u) || (reinterpret_cast<uintptr_t>(a->scales) & 3u))
    return LC_ERR_ALIGN;
  return launched(lc::launch_index_compress(*a, static_cast<cudaStream_t>(stream)));
}

lc_status out_proj(const lc_out_proj_args* a, void* stream) {
  if (!a) return LC_ERR_ARG;
  if (a->n_q < 0 || a->H < 1 || a->G < 1 || a->H % a->G || a->Dv < 1 || a->d_g < 16 || a->d_g % 16) return LC_ERR_ARG;
  if (a->out_fmt != LC_FMT_F32 && a->out_fmt != LC_FMT_BF16) return LC_ERR_ARG;
  if ((static_cast<int64_t>(a->H / a->G) * a->Dv) % 64) return LC_ERR_UNSUPPORTED;
  if (a->n_q == 0) return LC_OK;
  if (!a->x || !a->w || !a->y) return LC_ERR_ARG;
  if (!aligned16(a->x) || !aligned16(a->w) || !aligned16(a->y)) return LC_ERR_ALIGN;
  return launched(lc::launch_out_proj(*a, static_cast<cudaStream_t>(stream)));
}

lc_status index_scores(const lc_index_args* a, void* stream, bool decode) {
  LC_TRY(check_index(a, decode, true));
  if (a->n_q == 0 || a->max_ent == 0) return LC_OK;
  return launched(lc::launch_index_scores(*a, decode, static_cast<cudaStream_t>(stream)));
}

lc_status index_topk(const lc_index_topk_args* a, void* stream, bool decode) {
  if (!a) return LC_ERR_ARG;
  if (a->k < 1 || a->k > 2048) return LC_ERR_ARG;
  LC_TRY(check_index(&a->index, decode, false));
  if (a->index.fmt != LC_IDX_MXFP4 && a->index.fmt != LC_IDX_MXFP4_QBF16) return LC_ERR_UNSUPPORTED;
  if (a->index.n_q == 0) return LC_OK;
  if (!a->idx) return LC_ERR_ARG;
  if (a->index.max_ent > 0 && lc::index_geometry(a->index, decode, true).n_chunks > 1024) return LC_ERR_UNSUPPORTED;
  const size_t need = a->index.max_ent > 0 ? lc::index_topk_workspace(*a, decode) : 0;
  if (need > 0 && (!a->workspace || a->workspace_bytes < need)) return LC_ERR_WORKSPACE;
  if (need > 0 && !aligned16(a->workspace)) return LC_ERR_ALIGN;
  if (a->index.max_ent == 0) {
    // no entries anywhere: every query selects nothing
    return launched(lc::launch_empty_selection(a->idx, a->count, a->index.n_q, a->k, static_cast<cudaStream_t>(stream)));
  }
  return launched(lc::launch_index_topk(*a, decode, static_cast<cudaStream_t>(stream)));
}

lc_status topk(const lc_topk_args* a, void* stream, bool decode) {
  if (!a) return LC_ERR_ARG;
  if (a->n_q < 0 || a->k < 1 || a->max_ent < 0 || a->m < 1 || a->W_x < 0) return LC_ERR_ARG;
  if (a->score_stride < a->max_ent || a->score_stride % 4) return LC_ERR_ARG;
  if (decode && a->n_q != a->batch.num_seqs) return LC_ERR_ARG;
  if (a->n_q == 0) return LC_OK;
  LC_TRY(check_batch(a->batch, true, false));
  if (!a->scores || !a->idx) return LC_ERR_ARG;
  if (!aligned16(a->scores)) return LC_ERR_ALIGN;
  return launched(lc::launch_topk(*a, decode, static_cast<cudaStream_t>(stream)));
}

lc_status attn(const lc_attn_args* a, void* stream, bool sparse, bool decode) {
  if (!a) return LC_ERR_ARG;
  LC_TRY(check_dims(a->dims));
  if (a->n_q < 0 || a->m < 1 || a->W < 0 || a->W_x < 0 || a->max_ent < 0) return LC_ERR_ARG;
  if (a->out_fmt != LC_FMT_F32 && a->out_fmt != LC_FMT_BF16) return LC_ERR_ARG;
  if (a->batch.win_ring < 0 || (a->batch.win_ring > 0 && a->batch.win_ring < a->W)) return LC_ERR_ARG;
  if (a->v_nope != 0 && (a->v_nope != 1 || a->dims.d_r <= 0)) return LC_ERR_ARG;
  if (sparse && a->k < 1) return LC_ERR_ARG;
  if (decode && a->n_q != a->batch.num_seqs) return LC_ERR_ARG;
  if (a->impl != LC_IMPL_AUTO && a->impl != LC_IMPL_TC && a->impl != LC_IMPL_REF) return LC_ERR_ARG;
  if (!lc::attn_impl_ok(*a)) return LC_ERR_UNSUPPORTED;
  if (a->n_q == 0) return LC_OK;
  LC_TRY(check_rows(a->q, a->dims, true));
  LC_TRY(check_rows(a->ent, a->dims, a->max_ent > 0));
  LC_TRY(check_rows(a->win, a->dims, a->W > 0));
  LC_TRY(check_batch(a->batch, true, a->W > 0));
  if (!a->sink || !a->out || (sparse && !a->idx)) return LC_ERR_ARG;
  if (!aligned16(a->out)) return LC_ERR_ALIGN;
  const size_t need = lc::attn_workspace_bytes(*a, sparse, decode);
  if (need > 0 && (!a->workspace || a->workspace_bytes < need)) return LC_ERR_WORKSPACE;
  if (need > 0 && !aligned16(a->workspace)) return LC_ERR_ALIGN;
  return launched(lc::launch_attn(*a, sparse, decode, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

lc_status lc_qk_prep_prefill(const lc_qk_prep_args* a, void* stream) { return qk_prep(a, stream); }
lc_status lc_qk_prep_decode(const lc_qk_prep_args* a, void* stream) { return qk_prep(a, stream); }

lc_status lc_csa_compress_prefill(const lc_compress_args* a, void* stream) { return compress(a, stream, false); }
lc_status lc_csa_compress_decode(const lc_compress_args* a, void* stream) { return compress(a, stream, false); }
lc_status lc_hca_compress_prefill(const lc_compress_args* a, void* stream) { return compress(a, stream, true); }
lc_status lc_hca_compress_decode(const lc_compress_args* a, void* stream) { return compress(a, stream, true); }

lc_status lc_csa_index_scores_prefill(const lc_index_args* a, void* stream) { return index_scores(a, stream, false); }
lc_status lc_csa_index_scores_decode(const lc_index_args* a, void* stream) { return index_scores(a, stream, true); }

lc_status lc_mxfp4_quantize(const lc_mxfp4_quant_args* a, void* stream) { return mxfp4_quantize(a, stream); }
lc_status lc_grouped_out_proj(const lc_out_proj_args* a, void* stream) { return out_proj(a, stream); }
lc_status lc_csa_index_compress_prefill(const lc_index_compress_args* a, void* stream) { return index_compress(a, stream); }
lc_status lc_csa_index_compress_decode(const lc_index_compress_args* a, void* stream) { return index_compress(a, stream); }

lc_status lc_csa_index_topk_prefill(const lc_index_topk_args* a, void* stream) { return index_topk(a, stream, false); }
lc_status lc_csa_index_topk_decode(const lc_index_topk_args* a, void* stream) { return index_topk(a, stream, true); }
size_t lc_csa_index_topk_workspace_bytes(const lc_index_topk_args* a, int32_t decode) {
  if (!a || a->index.n_q <= 0 || a->index.max_ent <= 0 || a->k < 1) return 0;
  return lc::index_topk_workspace(*a, decode != 0);
}

lc_status lc_csa_topk_prefill(const lc_topk_args* a, void* stream) { return topk(a, stream, false); }
lc_status lc_csa_topk_decode(const lc_topk_args* a, void* stream) { return topk(a, stream, true); }

lc_status lc_csa_sparse_attn_prefill(const lc_attn_args* a, void* stream) { return attn(a, stream, true, false); }
lc_status lc_csa_sparse_attn_decode(const lc_attn_args* a, void* stream) { return attn(a, stream, true, true); }
lc_status lc_hca_attn_prefill(const lc_attn_args* a, void* stream) { return attn(a, stream, false, false); }
lc_status lc_hca_attn_decode(const lc_attn_args* a, void* stream) { return attn(a, stream, false, true); }

// Workspace of the decode variant (the prefill variant needs none).
size_t lc_csa_sparse_attn_workspace_bytes(const lc_attn_args* a) {
  return a ? lc::attn_workspace_bytes(*a, true, true) : 0;
}
size_t lc_hca_attn_workspace_bytes(const lc_attn_args* a) {
  return a ? lc::attn_workspace_bytes(*a, false, true) : 0;
}
// Optional workspace of the HCA prefill variant (the F16 image of the entries).
size_t lc_hca_attn_prefill_workspace_bytes(const lc_attn_args* a) {
  return a ? lc::attn_image_bytes(*a, false, false) : 0;
}

const char* lc_version(void) { return "lc 0.1.0 (CSA/HCA attention, sm_100a)"; }

const char* lc_status_string(lc_status s) {
  switch (s) {
    case LC_OK: return "LC_OK";
    case LC_ERR_ARG: return "LC_ERR_ARG: invalid argument";
    case LC_ERR_ALIGN: return "LC_ERR_ALIGN: buffer not 16-byte aligned";
    case LC_ERR_UNSUPPORTED: return "LC_ERR_UNSUPPORTED: no kernel for this format/shape";
    case LC_ERR_WORKSPACE: return "LC_ERR_WORKSPACE: workspace missing or too small";
    case LC_ERR_LAUNCH: return "LC_ERR_LAUNCH: CUDA launch failed";
    case LC_ERR_TOO_LARGE: return "LC_ERR_TOO_LARGE: needs more scratch than the static array holds";
    default: return "unknown lc_status";
  }
}

size_t lc_struct_size(int32_t which) {
  switch (which) {
    case 0: return sizeof(lc_rows);
    case 1: return sizeof(lc_dims);
    case 2: return sizeof(lc_batch);
    case 3: return sizeof(lc_qk_prep_args);
    case 4: return sizeof(lc_compress_args);
    case 5: return sizeof(lc_index_args);
    case 6: return sizeof(lc_topk_args);
    case 7: return sizeof(lc_attn_args);
    case 8: return sizeof(lc_index_topk_args);
    case 9: return sizeof(lc_mxfp4_quant_args);
    case 10: return sizeof(lc_index_compress_args);
    case 11: return sizeof(lc_out_proj_args);
    default: return 0;
  }
}

}  // extern "C"
