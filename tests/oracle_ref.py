"""Test-side glue: run the oracle on a workload's inputs (host copies of the very tensors
the library receives) and compare library outputs with it.

Acceptance (stated per workload class):
  * stored entries / window rows / queries: within one step of the storage format's grid
    (the library rounds an FP32 value, the oracle a float64 one; they can land on the
    two sides of a rounding midpoint), FP32 within 1e-5;
  * index scores: within the FP32 evaluation error bound of the score;
  * top-k on identical scores: bit-exact; end to end, FP32 inputs: identical wherever the
    k-th / (k+1)-th score gap exceeds the error bound; FP4 inputs: the selected sets may
    differ only in entries whose oracle score lies within 1e-2 |s_k| of the k-th score;
  * attention: max-abs error <= 1e-4 (FP32 outputs) or <= 2e-2 x RMS of each head's
    oracle output (BF16 outputs), for every (query, head) row: stage-wise on the oracle's
    own intermediates, and end to end on the library's own intermediates; the oracle's
    result on those differs from its result on its own by at most perturbation_bound().
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import numpy as np
import torch

from oracle import lc_oracle as O
from oracle import pipeline as P
from long_context_sparse_softmax_b200 import workloads as wl

ATTN_TOL_F32 = 1e-4
ATTN_TOL_REL_BF16 = 2e-2
TOPK_FP4_BAND = 1e-2


def np_(t):
    return None if t is None else t.detach().cpu().numpy()


def idx_operand_np(op: Dict[str, torch.Tensor], rows=None):
    d = {k: np_(v if rows is None else v[rows]) for k, v in op.items()}
    return d


# Absolute error of the library's FP32 evaluation of a normalised row value (|v| <= sqrt(D)):
# a few FP32 roundings of terms of size <= 24.  RoPE's a*c - b*s can cancel to a value
# much smaller than its terms, so this error is absolute, not relative to the result.
FP32_EVAL_ABS = 1e-5


def stored_close(fmt: int, got_f64: np.ndarray, exp_f64: np.ndarray, d_n: int) -> np.ndarray:
    """Per-element acceptance of stored rows: the two pre-rounding values differ by at most
    the FP32 evaluation error, so the stored values differ by at most that plus one grid
    step of the storage format (taken at the larger magnitude)."""
    mag = np.maximum(np.abs(got_f64), np.abs(exp_f64))
    ev = FP32_EVAL_ABS * np.maximum(1.0, np.abs(exp_f64))
    if fmt == O.FMT_F32:
        tol = ev
    elif fmt == O.FMT_BF16:
        tol = O.ulp_bf16(mag) + ev
    else:
        tol = np.concatenate([O.ulp_e4m3(mag[..., :d_n]), O.ulp_bf16(mag[..., d_n:])], -1) + ev
    return np.abs(got_f64 - exp_f64) <= tol


# A stored value can differ from the oracle's only where the pre-rounding value lies within
# the FP32 evaluation error (~1e-6 relative) of a rounding midpoint: a rare event.  A
# systematic shift (a wrong scale, a wrong rounding mode) would move many values by one
# grid step and still pass the per-element check, so the fraction of differing values is
# bounded too.
MAX_FLIP_FRACTION = 1e-3


def stored_check(fmt: int, got_f64: np.ndarray, exp_f64: np.ndarray, d_n: int, what: str) -> float:
    ok = stored_close(fmt, got_f64, exp_f64, d_n)
    assert ok.all(), f"{what}: {(~ok).sum()} elements beyond one grid step"
    n_diff = int(np.sum(got_f64 != exp_f64))
    frac = n_diff / got_f64.size if got_f64.size else 0.0
    if fmt != O.FMT_F32:
        assert n_diff <= MAX_FLIP_FRACTION * got_f64.size + 3, \
            f"{what}: {n_diff} of {got_f64.size} stored values differ from the oracle's"
    return frac


def mxfp4_check(lib_codes, lib_scales, orc_codes, orc_scales, what: str) -> float:
    """Acceptance of MXFP4 values the path computed from FP32 intermediates (pooled indexer
    keys): each element within one E2M1 grid step (at the larger of the two block scales,
    which differ only where the block maximum sits at a power of two) of the oracle's,
    and few elements differing at all.  Returns the fraction that differ."""
    dl = O.mxfp4_to_f64(lib_codes, lib_scales)
    do = O.mxfp4_to_f64(orc_codes, orc_scales)
    X = np.repeat(np.exp2(np.maximum(lib_scales, orc_scales).astype(np.float64) - 127), 32, axis=-1)
    mag = np.maximum(np.abs(dl), np.abs(do)) / X
    step = np.where(mag < 2, 0.5, np.where(mag < 4, 1.0, 2.0)) * X
    ok = np.abs(dl - do) <= step + FP32_EVAL_ABS * np.abs(do)
    assert ok.all(), f"{what}: {(~ok).sum()} elements beyond one grid step"
    n_diff = int(np.sum(dl != do))
    assert n_diff <= MAX_FLIP_FRACTION * dl.size + 32, f"{what}: {n_diff} of {dl.size} values differ"
    return n_diff / dl.size if dl.size else 0.0


def rows_np(fmt: int, r: Dict[str, torch.Tensor], sel=None) -> np.ndarray:
    x = r["x"] if sel is None else r["x"][sel]
    rope = r.get("rope")
    if rope is not None and sel is not None:
        rope = rope[sel]
    return O.rows_to_f64(fmt, np_(x), np_(rope))


def write_rows(r: Dict[str, torch.Tensor], fmt: int, y: np.ndarray, d_n: int, sel) -> None:
    """Write float64 rows (cast to the storage format) into library buffer rows `sel`."""
    x, rope = O.rows_from_f64(fmt, y, d_n)
    dev = r["x"].device
    r["x"][sel] = torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    if rope is not None:
        r["rope"][sel] = torch.from_numpy(np.ascontiguousarray(rope)).to(dev)


def out_np(run, q_sel: Sequence[int]) -> np.ndarray:
    s = run.spec
    o = run.out.view(-1, s.H, s.Dv)[torch.as_tensor(list(q_sel), device=run.out.device)]
    o = np_(o)
    return o.astype(np.float64) if s.out_f32 else O.bf16_to_f64(o)


def attn_ok(got: np.ndarray, exp: np.ndarray, out_f32: bool):
    """Acceptance of one query's attention output [H, D].

    FP32 output: max-abs error <= 1e-4.  BF16 output: for each head, max-abs error over
    its D-dim output vector <= 2e-2 x that vector's RMS.  (An RMS pooled over heads of
    very different magnitude - one sharp head next to diffuse ones - would reject the
    exact result rounded to BF16 itself, whose error reaches 2^-9 |o|.)
    Returns (ok, worst err, its tolerance)."""
    if got.size == 0:
        return True, 0.0, 1.0
    if out_f32:
        err = float(np.max(np.abs(got - exp)))
        return err <= ATTN_TOL_F32, err, ATTN_TOL_F32
    err_h = np.max(np.abs(got - exp), axis=-1)
    tol_h = ATTN_TOL_REL_BF16 * np.sqrt(np.mean(exp * exp, axis=-1))
    ratio = np.where(tol_h > 0, err_h / np.where(tol_h > 0, tol_h, 1.0), np.where(err_h > 0, np.inf, 0.0))
    h = int(np.argmax(ratio))
    return bool(np.all(err_h <= tol_h)), float(err_h[h]), float(tol_h[h])


def perturbation_bound(q_a: np.ndarray, keys_a: np.ndarray, q_b: np.ndarray, keys_b: np.ndarray,
                       sink: np.ndarray, scale: float, v_dims=None) -> np.ndarray:
    """Bound on |attend(q_b, keys_b) - attend(q_a, keys_a)| per output element [H, D], for
    two inputs with the same keys in the same order whose values differ slightly (the
    library's stored intermediates against the oracle's, one storage grid step apart).

    With logit changes |dl_k| <= L (per head, computed exactly here), every softmax weight
    moves by a factor in [e^-2L, e^2L], so with p, o the weights and output on input a:
      |o_b - o_a| <= e^2L sum_k p_k |v_b,k - v_a,k| + (e^2L - 1) (sum_k p_k |v_a,k - o_a| + p_sink |o_a|).
    """
    la = scale * (q_a @ keys_a.T)
    lb = scale * (q_b @ keys_b.T)
    L = np.max(np.abs(lb - la), axis=1) if keys_a.shape[0] else np.zeros(q_a.shape[0])
    o_a, lse = O.attend(q_a, keys_a, sink, scale, v_dims)
    p = np.exp(la - lse[:, None])                        # [H, n]
    p_sink = np.exp(sink - lse)                          # [H]
    va = keys_a if v_dims is None else keys_a[:, v_dims]
    vb = keys_b if v_dims is None else keys_b[:, v_dims]
    dv = np.abs(vb - va)                                 # [n, Dv]
    g = np.exp(2 * L)[:, None]
    spread = np.empty_like(o_a)
    for h in range(o_a.shape[0]):
        spread[h] = p[h] @ np.abs(va - o_a[h])
    bound = g * (p @ dv) + (g - 1) * (spread + p_sink[:, None] * np.abs(o_a))
    return bound * (1 + 1e-9) + 1e-12


def attn_err_in_ulps(got: np.ndarray, exp: np.ndarray, out_f32: bool) -> float:
    """Largest error in units of the output format's grid step at that value (reported,
    not asserted: the tensor-core path rounds the softmax weights to BF16 before P V)."""
    if got.size == 0:
        return 0.0
    mag = np.maximum(np.abs(got), np.abs(exp))
    step = np.full(mag.shape, 2.0 ** -23) * np.maximum(mag, 1e-30) if out_f32 else O.ulp_bf16(mag)
    return float(np.max(np.abs(got - exp) / np.maximum(step, 1e-30)))


def topk_sets_ok(got_idx: np.ndarray, exp_idx: np.ndarray, s_oracle: np.ndarray, k: int, fp32: bool,
                 bound: np.ndarray = None):
    """End-to-end selection check for one query.  Returns (ok, n_diff, reason)."""
    g = set(int(v) for v in got_idx if v >= 0)
    e = set(int(v) for v in exp_idx if v >= 0)
    if g == e:
        return True, 0, ""
    diff = g ^ e
    K = len(e)
    if len(g) != K:
        return False, len(diff), "count differs"
    order = np.lexsort((np.arange(s_oracle.shape[0]), -s_oracle))
    s_k = s_oracle[order[K - 1]]
    if fp32:
        # only allowed where the oracle's k-th/(k+1)-th gap is within the FP32 error bound
        if K < s_oracle.shape[0]:
            s_k1 = s_oracle[order[K]]
            b = bound[order[K - 1]] + bound[order[K]]
            if s_k - s_k1 <= b and all(abs(s_oracle[j] - s_k) <= 2 * b for j in diff):
                return True, len(diff), "within error bound"
        return False, len(diff), "fp32 selection differs"
    band = TOPK_FP4_BAND * abs(s_k)
    bad = [j for j in diff if abs(s_oracle[j] - s_k) > band]
    return (not bad), len(diff), ("" if not bad else f"{len(bad)} entries outside band")


class OraclePrefill:
    """Oracle of a prefill workload, for a sample of its queries (local indices)."""

    def __init__(self, inp, q_sel: Sequence[int], W_x: int = None, entries=True):
        s: wl.Spec = inp["spec"]
        self.s = s
        self.sink = np_(inp["sink"]).astype(np.float64)
        self.v_dims = O.nope_dims(s.D, s.rope_off, s.d_r) if s.v_nope else None
        self.W_x = s.W if W_x is None else W_x
        self.q_sel = list(q_sel)
        self.pos = [s.q_first + i for i in self.q_sel]
        lo, d_r, d_n = s.rope_off, s.d_r, s.d_n
        x_bits = np_(inp["x"])
        self.x_bits = x_bits
        g = np_(inp["g"]).astype(np.float64)
        if entries:
            xfun = lambda r0, n: P.raw_rows(s.raw_fmt, x_bits[r0:r0 + n])
            self.ent_f, self.ent_x, self.ent_r = P.entries_from_tokens(xfun, g, s.m, lo, d_r, s.kv_fmt, d_n)
            if self.ent_f.size == 0:
                self.ent_f = np.zeros((0, s.D))
        # window rows needed by the sampled queries
        need = sorted(set(t for p in self.pos for t in O.window_positions(p, s.W)))
        self.win_pos = np.array(need, dtype=np.int64)
        if need:
            raw = P.raw_rows(s.raw_fmt, x_bits[self.win_pos])
            self.win_f, _, _ = P.stored(s.win_fmt, O.qk_prep(raw, self.win_pos, lo, d_r), d_n)
        else:
            self.win_f = np.zeros((0, s.D))
        self.win_row = {int(t): i for i, t in enumerate(need)}
        # queries
        qr = P.raw_rows(s.raw_fmt, np_(inp["q_raw"][torch.as_tensor(self.q_sel, device=inp["q_raw"].device)]))
        self.q_f, _, _ = P.stored(s.q_fmt, O.qk_prep(qr, np.array(self.pos), lo, d_r), d_n)
        if s.is_csa:
            sel_t = torch.as_tensor(self.q_sel, device=inp["q_raw"].device)
            if s.idx_fmt == O.IDX_MXFP4:
                # the path quantises the raw indexer queries and pools + quantises the keys
                self.qI_codes, self.qI_scales = O.f64_to_mxfp4(O.bf16_to_f64(np_(inp["qI_raw"][sel_t])))
                self.qI = O.mxfp4_to_f64(self.qI_codes, self.qI_scales)
                pooled = O.pool_index_keys(O.bf16_to_f64(np_(inp["kI_raw"])), g, s.m)
                self.kI_codes, self.kI_scales = O.f64_to_mxfp4(pooled.reshape(-1, s.d_I))
                self.kI = O.mxfp4_to_f64(self.kI_codes, self.kI_scales)
            else:
                self.qI = P.indexer_f64(s.idx_fmt, idx_operand_np(inp["qI"], sel_t))
                self.kI = P.indexer_f64(s.idx_fmt, idx_operand_np(inp["kI"]))
            self.w = np_(inp["w"]).astype(np.float64)

    def scores(self, i: int, kI: np.ndarray = None):
        """Visible scores of sampled query i, and their FP32 error bound (on the oracle's
        indexer keys, or on the decoded keys `kI` of another path)."""
        p = self.pos[i]
        kI = self.kI if kI is None else kI
        w = self.w[self.q_sel[i]] if self.s.w_per_query else self.w
        s, n_vis = P.visible_scores(self.qI[i], kI, w, p, self.s.m, self.W_x)
        return s, O.score_error_bound(self.qI[i], kI[:n_vis], w)

    def select(self, i: int, s_vis: np.ndarray = None):
        if s_vis is None:
            s_vis, _ = self.scores(i)
        return O.topk(s_vis, self.s.k)

    def window_block(self, p: int, win: np.ndarray = None):
        """(position of the first row, rows) of the window rows of positions
        max(0, p-W+1) .. p, taken from `win` (rows for self.win_pos; default the oracle's)."""
        win = self.win_f if win is None else win
        ts = list(O.window_positions(p, self.s.W))
        if not ts:
            return p + 1, np.zeros((0, self.s.D))
        return ts[0], win[[self.win_row[t] for t in ts]]

    def attend(self, i: int, idx: Sequence[int], q: np.ndarray = None, ent: np.ndarray = None,
               win: np.ndarray = None):
        """Attention of sampled query i through the oracle's own CSA / HCA query functions.
        q, ent, win default to the oracle's stored intermediates; another path's stored
        intermediates in the same layouts may be given instead."""
        s = self.s
        p = self.pos[i]
        q = self.q_f[i] if q is None else q
        ent = self.ent_f if ent is None else ent
        w0, wr = self.window_block(p, win)
        if s.is_csa:
            return O.sparse_attn_query(q, ent, idx, wr, w0, p, s.W, self.sink, s.scale, self.v_dims)
        n_vis = O.n_visible(p, s.m, self.W_x, ent.shape[0])
        return O.hca_attn_query(q, ent, n_vis, wr, w0, p, s.W, self.sink, s.scale, self.v_dims)

    def keys(self, i: int, idx: Sequence[int], ent: np.ndarray = None, win: np.ndarray = None):
        """The key rows attend() uses for sampled query i, in its order (for the
        perturbation bound)."""
        s = self.s
        p = self.pos[i]
        ent = self.ent_f if ent is None else ent
        _, wr = self.window_block(p, win)
        sel = [int(j) for j in idx if j >= 0] if s.is_csa else list(range(O.n_visible(p, s.m, self.W_x, ent.shape[0])))
        return np.concatenate([ent[sel].reshape(len(sel), s.D), wr], 0)


class OracleDecode:
    """Oracle of a decode step: one query per sequence on the given cache."""

    def __init__(self, inp, W_x: int = None):
        s: wl.Spec = inp["spec"]
        self.s = s
        self.W_x = s.W if W_x is None else W_x
        self.sink = np_(inp["sink"]).astype(np.float64)
        self.v_dims = O.nope_dims(s.D, s.rope_off, s.d_r) if s.v_nope else None
        lo, d_r, d_n = s.rope_off, s.d_r, s.d_n
        B = s.num_seqs
        self.n_c = list(inp["n_c"])
        self.ent_start = [int(v) for v in np_(inp["batch"]["ent_start"])]
        cache = inp["cache"]
        self.ent_f = O.rows_to_f64(s.kv_fmt, np_(cache["x"]), np_(cache.get("rope")))
        # decode-time compression of the block the newest token closed
        xt = np_(inp["x_tail"])
        gt = np_(inp["g_tail"]).astype(np.float64)
        self.blk_count = [int(v) for v in np_(inp["blk_count"])]
        self.new_entry = {}
        for b, L in enumerate(s.seq_lens):
            if self.blk_count[b]:
                j = L // s.m - 1
                y = O.compress(P.raw_rows(s.raw_fmt, xt[b]), gt[b], s.m, lo, d_r, first_block=j,
                               tok_pos0=L - s.m, n_blocks=1)
                f, _, _ = P.stored(s.kv_fmt, y, d_n)
                self.new_entry[b] = f[0]
                self.ent_f[self.ent_start[b] + j] = f[0]
        # window rows in position order (read through the ring when the cache is one), with
        # the newest token prepared from x_new
        self.win_f = O.rows_to_f64(s.win_fmt, np_(inp["win"])).reshape(B, s.W, s.D)
        if s.ring:
            for b, L in enumerate(s.seq_lens):
                p0 = max(0, L - s.W)
                self.win_f[b] = self.win_f[b][O.ring_slot(np.arange(p0, p0 + s.W), s.W)]
        xn = P.raw_rows(s.raw_fmt, np_(inp["x_new"]))
        self.pos = [L - 1 for L in s.seq_lens]
        newrow, _, _ = P.stored(s.win_fmt, O.qk_prep(xn, np.array(self.pos), lo, d_r), d_n)
        self.win_pos0 = [max(0, L - s.W) for L in s.seq_lens]
        self.win_len = [min(s.W, L) for L in s.seq_lens]
        for b in range(B):
            self.win_f[b, self.win_len[b] - 1] = newrow[b]
        self.new_win = newrow
        qr = P.raw_rows(s.raw_fmt, np_(inp["q_raw"]))
        self.q_f, _, _ = P.stored(s.q_fmt, O.qk_prep(qr, np.array(self.pos), lo, d_r), d_n)
        if s.is_csa:
            kI_np = idx_operand_np(inp["kI"])
            self.new_key = {}
            if s.idx_fmt == O.IDX_MXFP4:
                # the step quantises the query's raw indexer rows ...
                self.qI_codes, self.qI_scales = O.f64_to_mxfp4(O.bf16_to_f64(np_(inp["qI_raw"])))
                self.qI = O.mxfp4_to_f64(self.qI_codes, self.qI_scales)
                # ... and pools + quantises the indexer key of the block the newest token closed
                kt = O.bf16_to_f64(np_(inp["kI_tail"]))
                kI_np = {k: v.copy() for k, v in kI_np.items()}
                for b, L in enumerate(s.seq_lens):
                    if self.blk_count[b]:
                        j = L // s.m - 1
                        key = O.pool_index_keys(kt[b], gt[b], s.m, first_block=j, tok_pos0=L - s.m, n_blocks=1)
                        c, sc = O.f64_to_mxfp4(key)
                        r = self.ent_start[b] + j
                        kI_np["codes"][r], kI_np["scales"][r] = c[0], sc[0]
                        self.new_key[b] = (r, c[0], sc[0])
            else:
                self.qI = P.indexer_f64(s.idx_fmt, idx_operand_np(inp["qI"]))
            self.kI_np = kI_np
            self.w = np_(inp["w"]).astype(np.float64)

    def kI(self, b: int, kI_np=None):
        """Decoded indexer keys of sequence b (the oracle's, or another path's kI_np)."""
        kI_np = self.kI_np if kI_np is None else kI_np
        n0, n = self.ent_start[b], self.n_c[b]
        s = self.s
        if s.idx_fmt == O.IDX_F32:
            return kI_np["f32"][n0:n0 + n].astype(np.float64)
        return O.mxfp4_to_f64(kI_np["codes"][n0:n0 + n], kI_np["scales"][n0:n0 + n])

    def scores(self, b: int, kI_np=None):
        kI = self.kI(b, kI_np)
        w = self.w[b] if self.s.w_per_query else self.w
        s, n_vis = P.visible_scores(self.qI[b], kI, w, self.pos[b], self.s.m, self.W_x)
        return s, O.score_error_bound(self.qI[b], kI[:n_vis], w)

    def entries(self, b: int):
        return self.ent_f[self.ent_start[b]:self.ent_start[b] + self.n_c[b]]

    def window_rows(self, b: int, win: np.ndarray = None):
        """The window rows present for sequence b (positions win_pos0[b] ..), from `win`
        ([B, W, D]; default the oracle's)."""
        win = self.win_f if win is None else win
        return win[b][:self.win_len[b]]

    def attend(self, b: int, idx: Sequence[int], q: np.ndarray = None, ent: np.ndarray = None,
               win: np.ndarray = None):
        """Attention of sequence b's query through the oracle's own CSA / HCA query
        functions.  q ([H, D]), ent (all entry rows) and win ([B, W, D]) default to the
        oracle's stored intermediates; another path's may be given instead."""
        s = self.s
        p = self.pos[b]
        q = self.q_f[b] if q is None else q
        ent = self.ent_f if ent is None else ent
        e = ent[self.ent_start[b]:self.ent_start[b] + self.n_c[b]]
        wr = self.window_rows(b, win)
        if s.is_csa:
            return O.sparse_attn_query(q, e, idx, wr, self.win_pos0[b], p, s.W, self.sink, s.scale, self.v_dims)
        n_vis = O.n_visible(p, s.m, self.W_x, self.n_c[b])
        return O.hca_attn_query(q, e, n_vis, wr, self.win_pos0[b], p, s.W, self.sink, s.scale, self.v_dims)

    def keys(self, b: int, idx: Sequence[int], ent: np.ndarray = None, win: np.ndarray = None):
        """The key rows attend() uses for sequence b, in its order."""
        s = self.s
        p = self.pos[b]
        ent = self.ent_f if ent is None else ent
        e = ent[self.ent_start[b]:self.ent_start[b] + self.n_c[b]]
        sel = [int(j) for j in idx if j >= 0] if s.is_csa else list(range(O.n_visible(p, s.m, self.W_x, self.n_c[b])))
        wr = self.window_rows(b, win)
        ts = [t - self.win_pos0[b] for t in O.window_positions(p, s.W)]
        return np.concatenate([e[sel].reshape(len(sel), s.D), wr[ts].reshape(len(ts), s.D)], 0)
