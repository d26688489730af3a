"""CPU oracle for the CSA / HCA long-context attention path.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline may import this module.  The library never calls it, and the two share no
code: this file has its own number-format codecs, its own RMSNorm / RoPE / pooling /
scoring / selection / softmax, and reads only numpy arrays of raw storage bits.

Plain numpy in float64.  Every step is written the way the method states it, with no
blocking, fusion or reordering beyond what the definition allows; library primitives
(matrix products, sorts, exp/log/sin/cos) serve as steps.  The method is the hybrid
attention of DeepSeek-V4 as the pages describe it:

* CSA: every m = 4 tokens of KV become one entry by a learned (gated) weighting, not
  an average; a lightning indexer scores the entries for each query; the query keeps
  the top-k (512 Flash / 1024 Pro) and attends only to those, joined with a 128-token
  sliding window of raw tokens and an attention sink ("解读 DeepSeek V4", sections
  "Compressed Sparse Attention (CSA)" and "其他架构细节"; "DeepSeek-V4 论文分析",
  §5.1-§5.3 and §二 model table).
* HCA: m' = 128, dense attention over every entry, same window and sink
  ("解读 DeepSeek V4", "Heavily Compressed Attention (HCA)"; "DeepSeek-V4 论文分析", §六).
* RMSNorm on queries and KV entries, partial RoPE, attention sink (10100.com article,
  §三.1 混合注意力架构, "辅助优化" bullet).
* KV entries store the RoPE dims in BF16 and the rest in FP8; the indexer runs in FP4
  ("解读 DeepSeek V4", "其他架构细节"; "DeepSeek-V4 论文分析", §8.2-§8.3).

The pages leave the gate form, indexer score form, norm epsilon, RoPE layout and the
window/compressed overlap open.  The readings taken (each one a parameter here):
gate = softmax over the block of one scalar logit per token, pooled over the raw
tokens before RMSNorm; indexer score s = sum_h w_h ReLU(<qI_h, kI>); RMSNorm with unit
weight and eps = 1e-6 over all D dims; RoPE on interleaved pairs of the RoPE dims with
base 10000, at the token's position (an entry at its block's last position); an entry
is visible to a query at p iff its last token is at or before p - W_x, with W_x = W
(window and compressed entries disjoint) or W_x = 0 (overlap); V = K = the full entry.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

FMT_F32 = 0
FMT_BF16 = 1
FMT_E4M3_BF16 = 2
IDX_F32 = 0
IDX_MXFP4 = 3

RMS_EPS = 1e-6
ROPE_BASE = 10000.0
E4M3_MAX = 448.0


# =====================================================================================
# Number formats (decoded exactly into float64; encoded with round-to-nearest-even)
# =====================================================================================
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """BF16 is the upper half of an IEEE binary32: shift the 16 bits up and reinterpret."""
    u = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def _round_to_grid(v: np.ndarray, mant_bits: int, min_exp: int) -> np.ndarray:
    """Round |v| to the binary grid with `mant_bits` fraction bits, exponent >= min_exp.

    For |v| in [2^e, 2^(e+1)) the spacing is 2^(e - mant_bits); below 2^min_exp the
    spacing stays 2^(min_exp - mant_bits) (subnormals).  np.rint rounds half to even,
    and since the grid spacing is a power of two, |v| / spacing is exact.
    """
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))        # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, min_exp)
    q = np.ldexp(1.0, e - mant_bits)
    return np.rint(a / q) * q


def f64_to_bf16(v: np.ndarray) -> np.ndarray:
    """float64 -> BF16 bits (int16), round to nearest even (8 significant bits)."""
    v = np.asarray(v, dtype=np.float64)
    r = _round_to_grid(v, 7, -126)
    r = np.where(v < 0, -r, r)
    assert np.all(np.isfinite(r)) and np.all(np.abs(r) < 3.3e38)
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16).view(np.int16)


def _e4m3_table() -> np.ndarray:
    """Values of all 256 E4M3 codes (OCP 8-bit floating point, E4M3: bias 7, no infinity,
    S.1111.111 is NaN, max 448)."""
    t = np.empty(256, dtype=np.float64)
    for b in range(256):
        s = -1.0 if b & 0x80 else 1.0
        E = (b >> 3) & 0xF
        M = b & 0x7
        if E == 0xF and M == 0x7:
            t[b] = np.nan
        elif E == 0:
            t[b] = s * (M / 8.0) * 2.0 ** -6
        else:
            t[b] = s * (1.0 + M / 8.0) * 2.0 ** (E - 7)
    return t


E4M3_TABLE = _e4m3_table()
_E4M3_POS = E4M3_TABLE[:127]          # codes 0x00..0x7E: 0 .. 448, strictly increasing


def e4m3_to_f64(bits: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(bits).astype(np.uint8)]


def f64_to_e4m3(v: np.ndarray) -> np.ndarray:
    """float64 -> E4M3 bits (uint8): round to nearest even, saturating at +-448."""
    v = np.asarray(v, dtype=np.float64)
    r = np.minimum(_round_to_grid(v, 3, -6), E4M3_MAX)
    code = np.searchsorted(_E4M3_POS, r).astype(np.uint8)
    assert np.array_equal(_E4M3_POS[code], r)
    return np.where(v < 0, code | np.uint8(0x80), code).astype(np.uint8)


def e2m1_to_f64(nib: np.ndarray) -> np.ndarray:
    """E2M1 (OCP MX v1.0 FP4): sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0."""
    n = np.asarray(nib).astype(np.int64) & 0xF
    s = np.where(n & 0x8, -1.0, 1.0)
    E = (n >> 1) & 0x3
    M = (n & 0x1).astype(np.float64)
    mag = np.where(E == 0, 0.5 * M, (1.0 + 0.5 * M) * np.ldexp(1.0, E - 1))
    return s * mag


def e8m0_to_f64(bits: np.ndarray) -> np.ndarray:
    """E8M0 scale (OCP MX v1.0): 2^(code - 127); code 255 is NaN."""
    b = np.asarray(bits).astype(np.int64)
    return np.where(b == 255, np.nan, np.ldexp(1.0, b - 127))


def mxfp4_to_f64(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """MXFP4 [..., d]: element 2i in the low nibble of byte i, 2i+1 in the high nibble;
    one E8M0 scale per 32 consecutive elements."""
    c = np.asarray(codes).astype(np.uint8)
    lo = e2m1_to_f64(c & 0xF)
    hi = e2m1_to_f64(c >> 4)
    el = np.stack([lo, hi], axis=-1).reshape(*c.shape[:-1], c.shape[-1] * 2)
    sc = e8m0_to_f64(scales)
    return el * np.repeat(sc, 32, axis=-1)


# =====================================================================================
# Rows in the storage formats: [n, D] logical dims (nope dims first in the split form)
# =====================================================================================
def rows_to_f64(fmt: int, x: np.ndarray, rope: Optional[np.ndarray] = None) -> np.ndarray:
    if fmt == FMT_F32:
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if fmt == FMT_BF16:
        return bf16_to_f64(x)
    if fmt == FMT_E4M3_BF16:
        return np.concatenate([e4m3_to_f64(x), bf16_to_f64(rope)], axis=-1)
    raise ValueError(fmt)


def rows_from_f64(fmt: int, y: np.ndarray, d_n: int):
    """Cast float64 rows to a storage format.  Returns (x, rope-or-None)."""
    if fmt == FMT_F32:
        return y.astype(np.float32), None
    if fmt == FMT_BF16:
        return f64_to_bf16(y), None
    if fmt == FMT_E4M3_BF16:
        return f64_to_e4m3(y[..., :d_n]), f64_to_bf16(y[..., d_n:])
    raise ValueError(fmt)


def rope_lo(fmt: int, D: int, d_r: int, rope_off: int) -> int:
    """First RoPE dim in logical order: the split format keeps RoPE dims last."""
    return D - d_r if fmt == FMT_E4M3_BF16 else rope_off


# =====================================================================================
# The method's steps
# =====================================================================================
def rms_norm(x: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """RMSNorm with unit weight over the last axis: x / sqrt(mean(x^2) + eps)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope(y: np.ndarray, pos, lo: int, d_r: int, base: float = ROPE_BASE) -> np.ndarray:
    """Partial rotary embedding: dims lo..lo+d_r-1 in interleaved pairs (lo+2i, lo+2i+1)
    turned by the angle pos * base^(-2i/d_r).  `pos` broadcasts against y[..., 0]."""
    out = np.array(y, dtype=np.float64, copy=True)
    i = np.arange(d_r // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * i / d_r)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    a = y[..., lo + 0:lo + d_r:2]
    b = y[..., lo + 1:lo + d_r:2]
    out[..., lo + 0:lo + d_r:2] = a * c - b * s
    out[..., lo + 1:lo + d_r:2] = a * s + b * c
    return out


def qk_prep(x: np.ndarray, pos, lo: int, d_r: int, eps: float = RMS_EPS,
            base: float = ROPE_BASE) -> np.ndarray:
    """Query / window-token preparation: RMSNorm over the row, then RoPE at its position.

    x: [n, H, D] (or [n, D]) float64; pos: [n] (shared by the heads of a token)."""
    y = rms_norm(x, eps)
    p = np.asarray(pos)
    if x.ndim == 3:
        p = p[:, None]
    return rope(y, p, lo, d_r, base)


def pool_block(x_blk: np.ndarray, g_blk: np.ndarray) -> np.ndarray:
    """Gated pooling of one block: alpha = softmax(g over the block); c = sum_t alpha_t x_t."""
    e = np.exp(g_blk - np.max(g_blk))
    alpha = e / np.sum(e)
    return alpha @ x_blk


def compress(x: np.ndarray, g: np.ndarray, m: int, lo: int, d_r: int, first_block: int = 0,
             tok_pos0: int = 0, n_blocks: Optional[int] = None, eps: float = RMS_EPS,
             base: float = ROPE_BASE) -> np.ndarray:
    """Compress complete blocks of m tokens into one entry each.

    x: [T, D] float64 raw token KV rows for positions tok_pos0 .. tok_pos0 + T - 1;
    g: [T] gate logits.  Block j covers positions j*m .. j*m + m - 1; its entry is the
    gated pool, RMS-normalised, then RoPE'd at the block's last position (j+1)*m - 1.
    Returns [n_blocks, D] float64 for blocks first_block .. first_block + n_blocks - 1.
    """
    if n_blocks is None:
        n_blocks = (tok_pos0 + x.shape[0]) // m - first_block
    out = np.empty((n_blocks, x.shape[1]), dtype=np.float64)
    for i in range(n_blocks):
        j = first_block + i
        r0 = j * m - tok_pos0
        assert r0 >= 0 and r0 + m <= x.shape[0], "block outside the given token rows"
        c = pool_block(x[r0:r0 + m], g[r0:r0 + m])
        out[i] = rope(rms_norm(c, eps), (j + 1) * m - 1, lo, d_r, base)
    return out


def n_visible(p: int, m: int, W_x: int, n_ent: int) -> int:
    """Entries visible to a query at position p: j with (j+1)*m - 1 <= p - W_x, j < n_ent."""
    return int(min(max((p - W_x + 1) // m, 0), n_ent))


def index_scores(qI: np.ndarray, kI: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Lightning-indexer score of every key for one query:
    s_j = sum_h w_h * ReLU(<qI_h, kI_j>).   qI [H_I, d_I], kI [n, d_I], w [H_I]."""
    dots = kI @ qI.T                         # [n, H_I]
    return np.maximum(dots, 0.0) @ w


def score_error_bound(qI: np.ndarray, kI: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Worst-case |fl32(s_j) - s_j| for any FP32 evaluation order of the score
    (Higham, Accuracy and Stability of Numerical Algorithms, eq. 3.5):
    gamma_n * sum_h w_h sum_i |qI_hi kI_ji|, with n = d_I + H_I + 1 and u = 2^-24."""
    u = 2.0 ** -24
    n = qI.shape[1] + qI.shape[0] + 1
    gamma = n * u / (1 - n * u)
    return gamma * (np.abs(kI) @ np.abs(qI).T) @ np.abs(w)


def topk(s: np.ndarray, k: int) -> np.ndarray:
    """Top-k over one row of visible scores: the K = min(k, n) largest, ties to the
    lower index (sort by (-s, j)), returned in ascending index order."""
    n = s.shape[0]
    K = min(k, n)
    order = np.lexsort((np.arange(n), -s))    # primary key -s, then j
    return np.sort(order[:K]).astype(np.int64)


def window_positions(p: int, W: int) -> range:
    """Raw tokens a query at p attends to through the sliding window."""
    return range(max(0, p - W + 1), p + 1)


def attend(q: np.ndarray, keys: np.ndarray, sink: np.ndarray, scale: float, v_dims=None):
    """Softmax attention of H heads over a shared key set plus a per-head sink.

    q [H, D]; keys [n, D]; the values are the same rows, or their dims v_dims (an index
    array: the V = non-RoPE-dims variant); sink [H] (a logit in the denominator only,
    unscaled).  l = scale * <q_h, key>; M = max(sink_h, max l);
    Z = e^(sink_h - M) + sum e^(l - M); o = sum e^(l - M) v / Z; lse = M + ln Z.
    """
    logits = scale * (q @ keys.T)                               # [H, n]
    M = np.maximum(sink, logits.max(axis=1) if keys.shape[0] else -np.inf)
    e = np.exp(logits - M[:, None])
    Z = np.exp(sink - M) + e.sum(axis=1)
    values = keys if v_dims is None else keys[:, v_dims]
    o = (e @ values) / Z[:, None]
    return o, M + np.log(Z)


def nope_dims(D: int, lo: int, d_r: int) -> np.ndarray:
    """The non-RoPE dims of a D-dim row whose RoPE dims are lo .. lo + d_r - 1, in order
    (the values of the variant that leaves the RoPE part out of V)."""
    return np.concatenate([np.arange(0, lo), np.arange(lo + d_r, D)])


def sparse_attn_query(q: np.ndarray, entries: np.ndarray, idx: Sequence[int], win_rows: np.ndarray,
                      win_pos0: int, p: int, W: int, sink: np.ndarray, scale: float, v_dims=None):
    """CSA core attention for one query at position p: keys = the selected entries
    (index -1 = padding, skipped) joined with the window tokens p-W+1..p and the sink.
    win_rows holds prepped window rows for positions win_pos0, win_pos0 + 1, ...
    v_dims: the value dims (None: the whole rows)."""
    sel = [int(j) for j in idx if j >= 0]
    wp = [t - win_pos0 for t in window_positions(p, W)]
    assert all(0 <= r < win_rows.shape[0] for r in wp), "window row missing"
    D = entries.shape[1]
    keys = np.concatenate([entries[sel].reshape(len(sel), D), win_rows[wp].reshape(len(wp), D)], axis=0)
    return attend(q, keys, sink, scale, v_dims)


def hca_attn_query(q: np.ndarray, entries: np.ndarray, n_vis: int, win_rows: np.ndarray,
                   win_pos0: int, p: int, W: int, sink: np.ndarray, scale: float, v_dims=None):
    """HCA attention: every visible entry is selected, no indexer."""
    return sparse_attn_query(q, entries, range(n_vis), win_rows, win_pos0, p, W, sink, scale, v_dims)


def grouped_out_proj(o: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Grouped output projection (10100.com analysis §三.1): the H heads of each query form G
    groups of H/G consecutive heads; group g maps the concatenation of its heads' outputs
    (K = (H/G) Dv values) to its own d_g outputs with its own weights W_g [K, d_g].
    o [n, H, Dv]; w [G, K, d_g] -> [n, G d_g] (group g's outputs at columns g d_g ..)."""
    n, H, Dv = o.shape
    G, K, d_g = w.shape
    Hg = H // G
    assert Hg * G == H and Hg * Dv == K
    return np.concatenate([o[:, g * Hg:(g + 1) * Hg, :].reshape(n, K) @ w[g] for g in range(G)], axis=1)


# =====================================================================================
# Decode-time cache maintenance
# =====================================================================================
E2M1_POS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])   # codes 0..7


def f64_to_e2m1(v: np.ndarray) -> np.ndarray:
    """float64 -> E2M1 codes (uint8, 4 bits): the nearest E2M1 value, ties to the even
    code, saturating at +-6 (OCP MX v1.0 conversion with saturation).  Zero is code 0
    whatever the sign of the input."""
    a = np.minimum(np.abs(np.asarray(v, dtype=np.float64)), 6.0)
    d = np.abs(a[..., None] - E2M1_POS)                      # distance to each magnitude
    best = d.min(axis=-1, keepdims=True)
    cand = d == best                                           # one or two nearest codes
    codes = np.arange(8)
    # among the nearest, the even code (two nearest neighbours differ in the last bit)
    even = cand & (codes % 2 == 0)
    pick = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))
    neg = (np.asarray(v) < 0) & (pick > 0)
    return (pick | (neg.astype(np.int64) << 3)).astype(np.uint8)


def f64_to_mxfp4(v: np.ndarray):
    """float64 [..., d] (d a multiple of 32) -> MXFP4 (codes uint8 [..., d/2] with element 2i
    in the low nibble, E8M0 scales uint8 [..., d/32]), OCP MX v1.0: per block of 32 the
    shared scale is X = 2^(floor(log2 amax) - 2), 2 being the largest exponent of E2M1; a
    block of zeros takes X = 2^0; each element is v / X converted to E2M1."""
    v = np.asarray(v, dtype=np.float64)
    d = v.shape[-1]
    assert d % 32 == 0
    blk = v.reshape(*v.shape[:-1], d // 32, 32)
    amax = np.abs(blk).max(axis=-1)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))          # amax = f 2^ex, f in [0.5, 1)
    e = np.where(amax > 0, ex - 1 - 2, 0)
    e = np.clip(e, -127, 127)
    el = f64_to_e2m1(blk / np.ldexp(1.0, e)[..., None]).reshape(*v.shape)
    codes = (el[..., 0::2] | (el[..., 1::2] << 4)).astype(np.uint8)
    return codes, (e + 127).astype(np.uint8)


def pool_index_keys(k_raw: np.ndarray, g: np.ndarray, m: int, first_block: int = 0, tok_pos0: int = 0,
                    n_blocks: Optional[int] = None) -> np.ndarray:
    """Lightning-indexer keys of complete blocks: the same gated pooling as the KV entries
    (alpha = softmax(g over the block), k = sum alpha_t k_t), with no RMSNorm and no RoPE
    (the indexer operands are given directly).  k_raw [T, d_I] for positions
    tok_pos0 .. tok_pos0 + T - 1; returns [n_blocks, d_I] float64."""
    if n_blocks is None:
        n_blocks = (tok_pos0 + k_raw.shape[0]) // m - first_block
    out = np.empty((n_blocks, k_raw.shape[1]), dtype=np.float64)
    for i in range(n_blocks):
        r0 = (first_block + i) * m - tok_pos0
        assert r0 >= 0 and r0 + m <= k_raw.shape[0], "block outside the given token rows"
        out[i] = pool_block(k_raw[r0:r0 + m], g[r0:r0 + m])
    return out


def ring_slot(pos, R: int):
    """Window ring buffer of R rows: the prepared row of position `pos` lives in slot pos mod R."""
    return np.asarray(pos) % R


def window_from_ring(ring: np.ndarray, p: int, W: int) -> np.ndarray:
    """Window rows of a query at p (positions max(0, p-W+1) .. p) read from a ring buffer of
    R >= W rows, in position order."""
    ts = list(window_positions(p, W))
    return ring[ring_slot(np.array(ts, dtype=np.int64), ring.shape[0])] if ts else ring[:0]


# =====================================================================================
# Numbers a test needs about a result
# =====================================================================================
def ulp_e4m3(v: np.ndarray) -> np.ndarray:
    """Spacing of the E4M3 grid at |v|."""
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    return np.ldexp(1.0, np.maximum(ex - 1, -6) - 3)


def ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    return np.ldexp(1.0, np.maximum(ex - 1, -126) - 7)


def rms(x: np.ndarray) -> float:
    return float(np.sqrt(np.mean(np.asarray(x, dtype=np.float64) ** 2)))


__all__ = [n for n in dir() if not n.startswith("_")]
