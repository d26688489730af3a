/*
 * lc.h — C ABI of the CSA / HCA long-context attention path for NVIDIA B200 (sm_100a).
 *
 * The method (DeepSeek-V4 hybrid attention, as described on the pages
 * "解读 DeepSeek V4" (llm-tech.com.cn), "DeepSeek-V4 论文分析" (ai.kenelite.com) and the
 * 10100.com technical analysis):
 *   - Compressed Sparse Attention (CSA): every m = 4 tokens of KV are compressed into
 *     one entry; a lightning indexer scores the entries per query; the query attends to
 *     its top-k entries (512 / 1024), a 128-token sliding window of raw tokens and an
 *     attention sink.
 *   - Heavily Compressed Attention (HCA): m' = 128, dense attention over every entry
 *     plus the same window and sink.
 *   - RMSNorm on queries and KV entries; partial RoPE; KV entries keep the RoPE dims in
 *     BF16 and the rest in FP8 (E4M3); the indexer runs in FP4 (MXFP4).
 *
 * Readings this library takes where the pages are silent:
 *   gate:    alpha = softmax(g) over the m tokens of a block (one FP32 logit per token),
 *            entry = RMSNorm(sum alpha_t x_t), then RoPE at the block's last position.
 *   norm:    RMSNorm with unit weight over all D dims, eps given per call (1e-6 default).
 *   RoPE:    interleaved pairs (2i, 2i+1) of the d_r RoPE dims, angle pos * base^(-2i/d_r).
 *   indexer: s(p, j) = sum_h w_h * ReLU(<qI[p, h], kI[j]>), w_h >= 0.
 *   window:  raw tokens max(0, p-W+1) .. p (prepared with RMSNorm + RoPE like queries).
 *   visible: entry j is visible to a query at p iff (j+1)*m - 1 <= p - W_x and j < n_ent;
 *            W_x = W keeps window and entries disjoint (default), W_x = 0 lets them overlap.
 *   values:  V = K = the full D-dim entry (shared-KV MQA); output D dims per head.
 *   sink:    one logit per head in the softmax denominator only (unscaled).
 *   top-k:   K = min(k, n_vis) best scores, ties to the lower index, written in
 *            ascending index order and padded with -1.
 *
 * Conventions
 *   - Every pointer inside an args struct is a DEVICE pointer unless its comment says
 *     host.  The caller allocates every input, output and workspace buffer and owns the
 *     stream; the library allocates nothing, keeps no global state, never synchronises.
 *     Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Host-side validation failures return an LC_ERR_* code and launch nothing.
 *     LC_ERR_LAUNCH reports a CUDA launch error (cudaGetLastError after the launch).
 *   - Conditions only the device can see (an index out of range, a window row that is
 *     not present, a block whose tokens are not given) are skipped by the kernel and
 *     reported by OR-ing LC_DEV_* bits into *status when `status` is non-NULL.
 *   - Row layouts are dense and row-major.  A query tensor [n_q, H, D] is n_q*H rows.
 *   - Buffers must be 16-byte aligned (LC_ERR_ALIGN otherwise).
 *   - Each operation has a _prefill and a _decode entry point taking the same struct.
 *     Prefill: one sequence, many queries (num_seqs == 1).  Decode: one query per
 *     sequence (q_start[b] = b).  The variant picks the kernel tiling; results agree.
 */
#ifndef LC_H_
#define LC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t lc_status;
enum {
  LC_OK = 0,
  LC_ERR_ARG = 1,          /* a null pointer, a size out of range, inconsistent shapes */
  LC_ERR_ALIGN = 2,        /* a buffer not 16-byte aligned */
  LC_ERR_UNSUPPORTED = 3,  /* a format / shape combination the library has no kernel for */
  LC_ERR_WORKSPACE = 4,    /* workspace missing or smaller than *_workspace_bytes() */
  LC_ERR_LAUNCH = 5,       /* the CUDA launch failed */
  LC_ERR_TOO_LARGE = 6     /* the call needs more scratch than the allocation-free entry
                              point's fixed array holds */
};

/* Bits OR-ed into *status by the kernels. */
enum {
  LC_DEV_BAD_INDEX = 1,    /* a top-k index outside [0, n_ent(b)) other than -1: skipped */
  LC_DEV_WINDOW_RANGE = 2, /* a window position outside the given window rows: skipped */
  LC_DEV_BAD_BLOCK = 4,    /* a block whose tokens are not in the given token rows: skipped */
  LC_DEV_NONVISIBLE = 8,   /* a selected entry not visible to its query: skipped */
  LC_DEV_TIMEOUT = 16,     /* a bounded wait on the tensor core gave up: results of that
                              CTA are missing (never expected; reported, not hung) */
  LC_DEV_RANGE = 32        /* an attention logit above 80: the inputs were not
                              RMS-normalised as the method prescribes */
};

/* Row storage formats. */
enum {
  LC_FMT_F32 = 0,          /* one FP32 array [n, D] */
  LC_FMT_BF16 = 1,         /* one BF16 array [n, D] */
  LC_FMT_E4M3_BF16 = 2     /* nope dims E4M3 [n, D - d_r] + RoPE dims BF16 [n, d_r] */
};

/* Lightning-indexer operand formats. */
enum {
  LC_IDX_F32 = 0,          /* FP32 [.., d_I] */
  LC_IDX_MXFP4 = 3,        /* OCP MXFP4: E2M1 codes [.., d_I/2] (element 2i in the low
                              nibble, 2i+1 in the high nibble) + E8M0 scales [.., d_I/32] */
  LC_IDX_MXFP4_QBF16 = 4   /* keys as LC_IDX_MXFP4; queries BF16 [.., d_I], quantised to
                              MXFP4 inside the call by the rule of lc_mxfp4_quantize (the
                              same bytes); q_scale is not read */
};

/* Rows of D logical dims.  In LC_FMT_E4M3_BF16 the logical order is the D - d_r nope
 * dims followed by the d_r RoPE dims, and rope_off (lc_dims) must equal D - d_r. */
typedef struct lc_rows {
  int32_t fmt;
  int32_t reserved;
  void* x;                 /* F32/BF16 rows, or the E4M3 nope part */
  void* rope;              /* E4M3_BF16: BF16 RoPE part [n, d_r]; otherwise NULL */
} lc_rows;

typedef struct lc_dims {
  int32_t D;               /* dims per row (multiple of 8, <= 1024) */
  int32_t d_r;             /* RoPE dims (multiple of 8, <= min(D, 128)) */
  int32_t rope_off;        /* first RoPE dim inside a row (multiple of 8) */
  int32_t H;               /* heads per query token (rows per token) */
} lc_dims;

/* Ragged batch descriptor: device arrays, one entry per sequence. */
typedef struct lc_batch {
  int32_t num_seqs;
  int32_t win_ring;         /* host value.  0: window position t of b is row
                               win_start[b] + (t - win_pos0[b]).  R > 0: the window rows of b
                               are a ring buffer of R rows, position t in row
                               win_start[b] + t mod R (R >= W; the tensor-core kernels take
                               R a multiple of 64).  Either way positions win_pos0[b] ..
                               win_pos0[b] + win_len[b] - 1 are present. */
  const int32_t* q_start;   /* [num_seqs + 1] queries of b are q_start[b] .. q_start[b+1]-1 */
  const int32_t* q_pos0;    /* [num_seqs] position of the first query of b; query i of b
                               sits at q_pos0[b] + (i - q_start[b]) */
  const int64_t* ent_start; /* [num_seqs] row of entry 0 (and indexer key 0) of b */
  const int32_t* n_ent;     /* [num_seqs] entries stored for b */
  const int64_t* win_start; /* [num_seqs] row of the first window row of b */
  const int32_t* win_pos0;  /* [num_seqs] position of that row */
  const int32_t* win_len;   /* [num_seqs] window rows present for b */
} lc_batch;

/* ---------------------------------------------------------------------------------
 * qk_prep — RMSNorm over the D dims, RoPE on the RoPE dims at the token's position,
 * cast to out.fmt.  Used for queries (H heads share a position) and for window tokens
 * (H = 1).  Pages: 10100.com analysis §三.1 "辅助优化" (RMSNorm on queries/KV entries,
 * partial RoPE).
 * ------------------------------------------------------------------------------- */
typedef struct lc_qk_prep_args {
  lc_dims dims;
  int32_t n_tok;           /* tokens; rows = n_tok * H */
  int32_t in_fmt;          /* LC_FMT_F32 or LC_FMT_BF16 */
  const void* x;           /* [n_tok, H, D] raw rows */
  const int32_t* pos;      /* [n_tok] position of each token */
  const int64_t* out_tok;  /* optional [n_tok]: token t writes rows out_tok[t]*H .. +H-1
                              of `out` (e.g. its slot in a window cache); NULL: rows t*H.. */
  lc_rows out;             /* output rows */
  float eps;               /* RMSNorm epsilon */
  float rope_base;         /* RoPE base (10000) */
  int32_t* status;         /* optional */
} lc_qk_prep_args;

lc_status lc_qk_prep_prefill(const lc_qk_prep_args* a, void* stream);
lc_status lc_qk_prep_decode(const lc_qk_prep_args* a, void* stream);

/* ---------------------------------------------------------------------------------
 * csa_compress / hca_compress — for each requested complete block j of sequence b
 * (tokens j*m .. j*m + m - 1): alpha = softmax(g over the block), c = sum alpha_t x_t,
 * entry = RoPE(RMSNorm(c), (j+1)*m - 1), cast to out.fmt, written to row
 * ent_start[b] + j.  Pages: "解读 DeepSeek V4" CSA (m = 4) and HCA (m' = 128) sections;
 * "DeepSeek-V4 论文分析" §5.2 (learned per-token contribution weights, not an average).
 * csa_compress takes 1 <= m <= 64; hca_compress takes 64 <= m <= 1024, m % 32 == 0.
 * Prefill: blk_first = 0, blk_count = L / m.  Decode: the block the newest token closed.
 * ------------------------------------------------------------------------------- */
typedef struct lc_compress_args {
  lc_dims dims;            /* H unused */
  int32_t m;
  int32_t num_seqs;
  int32_t in_fmt;          /* LC_FMT_F32 or LC_FMT_BF16 */
  int32_t max_blocks;      /* host value: max over b of blk_count[b] */
  const void* x;           /* raw token rows [*, D] */
  const float* g;          /* gate logit of each token row */
  const int64_t* tok_row0; /* [num_seqs] row of the token at position tok_pos0[b] */
  const int32_t* tok_pos0; /* [num_seqs] */
  const int32_t* tok_len;  /* [num_seqs] consecutive token rows present for b */
  const int32_t* blk_first;/* [num_seqs] first block to compress */
  const int32_t* blk_count;/* [num_seqs] blocks to compress */
  const int64_t* ent_start;/* [num_seqs] row of entry 0 of b in `out` */
  lc_rows out;
  float eps;
  float rope_base;
  int32_t* status;
} lc_compress_args;

lc_status lc_csa_compress_prefill(const lc_compress_args* a, void* stream);
lc_status lc_csa_compress_decode(const lc_compress_args* a, void* stream);
lc_status lc_hca_compress_prefill(const lc_compress_args* a, void* stream);
lc_status lc_hca_compress_decode(const lc_compress_args* a, void* stream);

/* ---------------------------------------------------------------------------------
 * csa_index_scores — lightning indexer: for each query (position p, sequence b) and
 * each visible entry j < n_vis(p), scores[q, j] = sum_h w_h * ReLU(<qI[q,h], kI[j]>).
 * Columns j >= n_vis(p) are not written.  Pages: "解读 DeepSeek V4" CSA section and
 * "FP4 Quantization-Aware Training" (indexer QK path in MXFP4); "DeepSeek-V4 论文分析"
 * §5.3 and §8.3.
 * FP32 operands are computed with FP32 FMA (no TF32).  MXFP4 operands are exact
 * products accumulated in FP32.
 * ------------------------------------------------------------------------------- */
typedef struct lc_index_args {
  int32_t n_q;
  int32_t H_I;             /* indexer heads (F32: H_I * d_I <= 16384; MXFP4: 32 or 64) */
  int32_t d_I;             /* indexer dims (F32: multiple of 4, <= 256; MXFP4: 128) */
  int32_t fmt;             /* LC_IDX_F32, LC_IDX_MXFP4 or LC_IDX_MXFP4_QBF16 */
  const void* q;           /* F32 [n_q, H_I, d_I], MXFP4 codes [n_q, H_I, d_I/2] or (MXFP4_QBF16)
                              BF16 [n_q, H_I, d_I] */
  const uint8_t* q_scale;  /* MXFP4: [n_q, H_I, d_I/32], 4-byte aligned; else unused */
  const void* k;           /* F32 [n_keys, d_I] or MXFP4 codes [n_keys, d_I/2] */
  const uint8_t* k_scale;  /* MXFP4: [n_keys, d_I/32], 4-byte aligned */
  int64_t n_keys;          /* rows of k and k_scale (every ent_start[b] + n_ent[b] <= n_keys);
                              MXFP4 requires it: the tensor-core path reads whole 128-key
                              tiles by bulk copy and must not read past the arrays */
  const float* w;          /* head weights, >= 0: [H_I], or [n_q, H_I] if w_qstride = H_I */
  int32_t w_qstride;       /* 0 (shared) or H_I */
  int32_t m;
  int32_t W_x;
  int32_t max_ent;         /* host value: max over b of n_ent[b] */
  lc_batch batch;          /* q_start, q_pos0, ent_start, n_ent */
  float* scores;           /* [n_q, score_stride] */
  int64_t score_stride;    /* >= max_ent, multiple of 4 */
  int32_t* status;
  int32_t spin_limit;      /* polls a bounded wait of the MXFP4 kernel makes before it gives up
                              (LC_DEV_TIMEOUT, results undefined, every copy and MMA in flight
                              drained before the CTA exits); 0: the default (~2^26) */
  int32_t pdl;             /* 1: programmatic dependent launch - the MXFP4 call may start while
                              the kernel before it in the stream still runs, and reads q and
                              q_scale only after that kernel completes; every other input must
                              be complete before that kernel starts.  0: ordinary ordering */
} lc_index_args;

lc_status lc_csa_index_scores_prefill(const lc_index_args* a, void* stream);
lc_status lc_csa_index_scores_decode(const lc_index_args* a, void* stream);

/* ---------------------------------------------------------------------------------
 * csa_topk — per query: K = min(k, n_vis(p)) largest scores among columns
 * 0 .. n_vis(p) - 1, ties to the lower index; idx[q, 0..K-1] ascending, the rest -1;
 * count[q] = K.  Pages: "解读 DeepSeek V4" CSA section; "DeepSeek-V4 论文分析" §5.3
 * (Top-512 Flash / Top-1024 Pro).  Bit-exact: the result depends only on the scores.
 * ------------------------------------------------------------------------------- */
typedef struct lc_topk_args {
  int32_t n_q;
  int32_t k;               /* 1 .. 2048 */
  int32_t m;
  int32_t W_x;
  int32_t max_ent;         /* host value */
  int32_t pdl;             /* 1: may start while the kernel before it in the stream (the
                              indexer) runs; reads the scores only after it completes */
  const float* scores;     /* [n_q, score_stride], 16-byte aligned */
  int64_t score_stride;    /* >= max_ent, multiple of 4 */
  lc_batch batch;          /* q_start, q_pos0, n_ent */
  int32_t* idx;            /* [n_q, k] */
  int32_t* count;          /* [n_q] or NULL */
  int32_t* status;
} lc_topk_args;

lc_status lc_csa_topk_prefill(const lc_topk_args* a, void* stream);
lc_status lc_csa_topk_decode(const lc_topk_args* a, void* stream);

/* ---------------------------------------------------------------------------------
 * csa_index_topk — the lightning indexer and the top-k selection fused: the same
 * scores as csa_index_scores and the same selection as csa_topk (K = min(k, n_vis(p))
 * largest, ties to the lower index, idx ascending and padded with -1, count[q] = K), but
 * the score matrix is never written.  Pages: "解读 DeepSeek V4" CSA section (the indexer
 * exists to pick the top-k entries); "DeepSeek-V4 论文分析" §5.3.
 * Each indexer CTA keeps the scores of its key range on chip and selects its own top K
 * exactly (every entry of the global top K is in the top K of its range); when a
 * query's keys span several CTAs, a merge kernel selects the final K from the ranges'
 * candidates.  The result is bit-identical to csa_index_scores followed by csa_topk.
 * MXFP4 operands only (d_I = 128, H_I = 32 or 64); k <= 2048.  The workspace holds the
 * candidates: lc_csa_index_topk_workspace_bytes(a) bytes, 16-byte aligned (0 when every
 * query's keys fit one CTA).
 * ------------------------------------------------------------------------------- */
typedef struct lc_index_topk_args {
  lc_index_args index;     /* scores and score_stride are ignored (nothing is written) */
  int32_t k;               /* 1 .. 2048 */
  int32_t reserved;
  int32_t* idx;            /* [n_q, k] */
  int32_t* count;          /* [n_q] or NULL */
  void* workspace;
  size_t workspace_bytes;
} lc_index_topk_args;

lc_status lc_csa_index_topk_prefill(const lc_index_topk_args* a, void* stream);
lc_status lc_csa_index_topk_decode(const lc_index_topk_args* a, void* stream);
size_t lc_csa_index_topk_workspace_bytes(const lc_index_topk_args* a, int32_t decode);

/* ---------------------------------------------------------------------------------
 * mxfp4_quantize — rows of FP32 / BF16 values to OCP MXFP4 (Microscaling Formats v1.0):
 * per block of 32 elements the E8M0 scale X = 2^(floor(log2 amax) - 2) (a zero block takes
 * 2^0) and each element v / X converted to E2M1 with round-to-nearest-even, saturating at
 * +-6; zero is code 0.  Element 2i goes to the low nibble of byte i.  Used for the
 * indexer queries of each step.  Pages: "解读 DeepSeek V4", "FP4 Quantization-Aware
 * Training" (the lightning indexer's QK path runs in FP4).
 * ------------------------------------------------------------------------------- */
typedef struct lc_mxfp4_quant_args {
  int64_t n_rows;
  int32_t d;               /* elements per row: multiple of 32, <= 1024 */
  int32_t in_fmt;          /* LC_FMT_F32 or LC_FMT_BF16 */
  const void* x;           /* [n_rows, d] */
  uint8_t* codes;          /* [n_rows, d/2] */
  uint8_t* scales;         /* [n_rows, d/32] */
} lc_mxfp4_quant_args;

lc_status lc_mxfp4_quantize(const lc_mxfp4_quant_args* a, void* stream);

/* ---------------------------------------------------------------------------------
 * csa_index_compress — for each requested complete block j of sequence b, the
 * lightning-indexer key of entry j: the raw indexer-key rows of the block's m tokens
 * pooled with the same block-softmax gate as the KV entries (alpha = softmax(g over the
 * block), k = sum alpha_t k_t; no RMSNorm, no RoPE), quantised to MXFP4 as
 * lc_mxfp4_quantize does, written at row ent_start[b] + j of codes / scales.  Prefill:
 * every block; decode: the block the newest token closed.  Pages: "解读 DeepSeek V4" CSA
 * section (the indexer scores the compressed entries) and FP4 QAT section;
 * "DeepSeek-V4 论文分析" §5.3, §8.3.
 * ------------------------------------------------------------------------------- */
typedef struct lc_index_compress_args {
  int32_t d_I;             /* key dims: multiple of 32, <= 256 */
  int32_t m;               /* 1 .. 64 */
  int32_t num_seqs;
  int32_t in_fmt;          /* raw key rows: LC_FMT_F32 or LC_FMT_BF16 */
  int32_t max_blocks;      /* host value: max over b of blk_count[b] */
  int32_t reserved;
  const void* x;           /* raw indexer-key rows of the tokens [*, d_I] */
  const float* g;          /* gate logit of each token row (the KV entries' gates) */
  const int64_t* tok_row0; /* as in lc_compress_args */
  const int32_t* tok_pos0;
  const int32_t* tok_len;
  const int32_t* blk_first;
  const int32_t* blk_count;
  const int64_t* ent_start;
  uint8_t* codes;          /* [*, d_I/2] */
  uint8_t* scales;         /* [*, d_I/32] */
  int32_t* status;         /* optional: LC_DEV_BAD_BLOCK */
} lc_index_compress_args;

lc_status lc_csa_index_compress_prefill(const lc_index_compress_args* a, void* stream);
lc_status lc_csa_index_compress_decode(const lc_index_compress_args* a, void* stream);

/* ---------------------------------------------------------------------------------
 * csa_sparse_attn / hca_attn — for each query at p and head h, softmax attention over
 *   CSA: the selected entries idx[q, :] (-1 skipped), HCA: every visible entry,
 * joined with the window rows for positions max(0, p-W+1) .. p and the sink logit
 * sink[h]:  l = scale * <q_h, key>, M = max(sink_h, max l),
 * Z = e^(sink_h - M) + sum e^(l - M), o = sum e^(l - M) key / Z, lse = M + ln Z.
 * Pages: "解读 DeepSeek V4" CSA / HCA sections and "其他架构细节" (attention sink);
 * "DeepSeek-V4 论文分析" §5.4, §六, §七 and §8.4 (sparse core attention).
 * out: [n_q, H, D] in out_fmt (F32 or BF16); lse: [n_q, H] FP32 (optional).
 * The decode variant may split the keys of each query across CTAs; it then needs a
 * workspace of lc_*_workspace_bytes(a) bytes.  The prefill variants need none.  The HCA
 * prefill variant takes an optional one of lc_hca_attn_prefill_workspace_bytes(a) bytes
 * (16-byte aligned; 0 when it does not apply): with BF16 queries it then widens the
 * entries to F16 once per call instead of once per query, and reads each 64 visible
 * entries that start on a multiple of 64 in the entry array as one bulk copy.  The
 * results are the same either way; a smaller workspace is not an error.
 * ------------------------------------------------------------------------------- */
typedef struct lc_attn_args {
  lc_dims dims;
  int32_t n_q;
  int32_t k;               /* CSA: columns of idx; HCA: ignored */
  int32_t m;
  int32_t W;
  int32_t W_x;
  int32_t max_ent;         /* host value: max over b of n_ent[b] */
  float scale;             /* softmax scale (1/sqrt(D)) */
  int32_t out_fmt;         /* LC_FMT_F32 or LC_FMT_BF16 */
  lc_rows q;               /* [n_q * H] prepared queries */
  lc_rows ent;             /* compressed entries */
  lc_rows win;             /* prepared window rows (LC_FMT_F32 or LC_FMT_BF16) */
  const int32_t* idx;      /* CSA: [n_q, k] entry index within the sequence, -1 = none */
  const float* sink;       /* [H] */
  lc_batch batch;
  void* out;               /* [n_q, H, D] */
  float* lse;              /* [n_q, H] or NULL */
  void* workspace;
  size_t workspace_bytes;
  int32_t* status;
  int32_t impl;            /* LC_IMPL_AUTO (0): the tensor-core kernels where they apply,
                              else the reference kernel; LC_IMPL_TC or LC_IMPL_REF force one
                              (LC_ERR_UNSUPPORTED if it cannot run the shape); other values
                              are LC_ERR_ARG */
  int32_t n_ent_rows;      /* rows of ent (every ent_start[b] + n_ent[b] <= n_ent_rows), or 0 if
                              unknown; the FP8 tensor-core kernel reads entries by bulk tensor
                              copies and needs it */
  int32_t n_win_rows;      /* rows of win (every win_start[b] + win_len[b] <= n_win_rows), or 0
                              if unknown; with W > 0 the FP8 tensor-core kernel reads window
                              rows by bulk tensor copies and needs it */
  int32_t v_nope;          /* 0: the values are the whole D-dim key rows (out [n_q, H, D]);
                              1: the values are the D - d_r non-RoPE dims of each key row, in
                              logical order (out [n_q, H, D - d_r]); needs d_r > 0 */
  int32_t pdl;             /* 1: may start while the kernel before it in the stream (the top-k)
                              runs, and reads idx only after that kernel completes; every other
                              input must be complete before that kernel starts */
} lc_attn_args;

/* Attention kernels. */
enum {
  LC_IMPL_AUTO = 0,
  LC_IMPL_TC = 2,          /* tcgen05 tiles, accumulators in tensor memory (576-dim entries,
                              64 RoPE dims, heads in groups of 64): E4M3 scores from
                              bulk-copied tiles where queries and entries are E4M3 + BF16 RoPE
                              and n_ent_rows (and, with W > 0, n_win_rows) is set, else every
                              operand widened to F16 (BF16 queries) */
  LC_IMPL_REF = 3          /* one warp per (query, head), FP32 CUDA cores (any shape; the
                              FP32 workload) */
};

lc_status lc_csa_sparse_attn_prefill(const lc_attn_args* a, void* stream);
lc_status lc_csa_sparse_attn_decode(const lc_attn_args* a, void* stream);
lc_status lc_hca_attn_prefill(const lc_attn_args* a, void* stream);
lc_status lc_hca_attn_decode(const lc_attn_args* a, void* stream);

size_t lc_csa_sparse_attn_workspace_bytes(const lc_attn_args* a);
size_t lc_hca_attn_workspace_bytes(const lc_attn_args* a);
/* F16 image of the n_ent_rows entry rows (needs n_ent_rows > 0), or 0 */
size_t lc_hca_attn_prefill_workspace_bytes(const lc_attn_args* a);

/* ---------------------------------------------------------------------------------
 * lc_csa_sparse_attn_decode_static — lc_csa_sparse_attn_decode for callers that cannot
 * allocate device memory when they call: hosts that give all device memory to their own
 * allocator up front and forbid any other allocation, and latency-bound serving loops
 * that must not pay for the device-wide synchronisation cudaMalloc can imply.  The pages
 * have no counterpart; it is a property of this library's interface.
 *
 * Same arguments and results as lc_csa_sparse_attn_decode, except that a->workspace and
 * a->workspace_bytes are ignored: the scratch is a fixed array of
 * lc_csa_sparse_attn_decode_static_capacity() bytes (16 MiB) compiled into the library,
 * held on every device that loads the library until the process exits.  The call
 * allocates and frees nothing.
 *   - If the call needs more scratch than the array holds (lc_csa_sparse_attn_workspace_bytes
 *     above the capacity), it returns LC_ERR_TOO_LARGE before touching the device.
 *   - The first call on a device, with that device current, looks up the array's device
 *     address (cudaGetSymbolAddress) and keeps it; make that first call before any stream
 *     capture on the device.
 *   - Every call on a device shares the one array.  Calls whose executions overlap on the
 *     GPU (different streams, or other threads) race on it and give wrong results: order
 *     them on one stream or serialise them.  Nothing carries over from one call to the
 *     next: every scratch word a call reads, the same call has written first, except
 *     after a bounded wait gave up (LC_DEV_TIMEOUT in *status): the outputs of that call
 *     are then undefined and may mix in an earlier call's partial results.
 * ------------------------------------------------------------------------------- */
lc_status lc_csa_sparse_attn_decode_static(const lc_attn_args* a, void* stream);
size_t lc_csa_sparse_attn_decode_static_capacity(void);

/* ---------------------------------------------------------------------------------
 * grouped_out_proj — the grouped output projection of the attention heads: the H heads of
 * a query form G groups of H/G consecutive heads, and group g projects the concatenation
 * of its heads' outputs (K = (H/G) Dv values) to its own d_g output dims:
 *   y[n, g d_g + c] = sum_k x[n, g K + k] W_g[k, c],  0 <= c < d_g.
 * Pages: 10100.com analysis §三.1 (CSA and HCA use a grouped output projection to reduce
 * its cost).  BF16 operands, FP32 accumulation on the tensor cores.
 * ------------------------------------------------------------------------------- */
typedef struct lc_out_proj_args {
  int32_t n_q;             /* queries */
  int32_t H;               /* heads per query (H % G == 0) */
  int32_t Dv;              /* output dims per head of the attention */
  int32_t G;               /* groups */
  int32_t d_g;             /* output dims per group: multiple of 16 */
  int32_t out_fmt;         /* LC_FMT_F32 or LC_FMT_BF16 */
  const void* x;           /* [n_q, H, Dv] BF16: the attention output ((H/G) Dv a multiple of 64) */
  const void* w;           /* [G, d_g, (H/G) Dv] BF16: W_g transposed (row c of group g holds the
                              weights of output c) */
  void* y;                 /* [n_q, G d_g] */
  int32_t* status;         /* optional: LC_DEV_TIMEOUT */
} lc_out_proj_args;

lc_status lc_grouped_out_proj(const lc_out_proj_args* a, void* stream);

/* Library version string (static storage). */
const char* lc_version(void);
/* Name of a status code (static storage). */
const char* lc_status_string(lc_status s);
/* sizeof of the args structs, for bindings to check their mirrors:
 * 0 lc_rows, 1 lc_dims, 2 lc_batch, 3 lc_qk_prep_args, 4 lc_compress_args,
 * 5 lc_index_args, 6 lc_topk_args, 7 lc_attn_args, 8 lc_index_topk_args,
 * 9 lc_mxfp4_quant_args, 10 lc_index_compress_args, 11 lc_out_proj_args; other values
 * return 0. */
size_t lc_struct_size(int32_t which);

#ifdef __cplusplus
}
#endif

#endif /* LC_H_ */
