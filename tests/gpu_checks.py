"""Stage-by-stage and end-to-end comparison of a library run with the oracle (GPU tests).

Every stage is checked twice where it makes sense:
  * stage-wise: the stage's inputs are the oracle's own values (written into the library's
    buffers), so the comparison isolates that kernel;
  * end to end: the library's whole path against the oracle's whole path.  Every stored
    intermediate is within one storage grid step of the oracle's (stored_check), the
    selection is within the stated band (topk_sets_ok), and the attention output of every
    (query, head) row is within the attention tolerance of the oracle evaluated on the
    library's own intermediates and selection.  Where the selection agrees, the oracle's
    results on the two sets of intermediates must differ by no more than
    perturbation_bound(); the worst error against the oracle's own path is reported.
"""
from __future__ import annotations

import json
import os

from typing import Sequence

import numpy as np
import torch

from oracle import lc_oracle as O
from long_context_sparse_softmax_b200 import runner
from long_context_sparse_softmax_b200 import workloads as wl
from tests.oracle_ref import (OracleDecode, OraclePrefill, attn_err_in_ulps, attn_ok, mxfp4_check, np_, out_np,
                              perturbation_bound, rows_np, stored_check, topk_sets_ok, write_rows)


# lse = ln Z with Z = e^sink + sum_k e^l_k.  FP32 path: FP32 rounding only.  BF16 paths:
# the tensor-core kernels round each e^l_k to BF16 (relative 2^-9) before summing it, so
# ln Z can move by 2^-9 from that rounding, and by as much again from the accumulation.
LSE_TOL_F32 = 1e-4
LSE_TOL_BF16 = 2.0 ** -8


def _sync():
    torch.cuda.synchronize()


def _separate_index_topk(run, rep) -> None:
    """A step with the fused index + top-k leaves its selection in run.idx.  Run the
    separate indexer and top-k calls on the same inputs (they fill run.scores, which the
    checks below compare with the oracle, and run.idx again): the fused selection must be
    bit-identical to top-k of those scores."""
    if not run.spec.is_csa or not run.fused:
        return
    fused_idx, fused_cnt = run.idx.clone(), run.count.clone()
    run.index()
    run.topk()
    _sync()
    assert run.read_status() == 0
    assert torch.equal(fused_idx, run.idx), \
        f"fused index+top-k differs from the separate calls in {int((fused_idx != run.idx).any(1).sum())} rows"
    assert torch.equal(fused_cnt, run.count)
    rep["fused_topk_rows_identical"] = int(fused_idx.shape[0])


def check_prefill(spec: wl.Spec, q_sel: Sequence[int] = None, W_x: int = None, report=None, impl: int = 0):
    """Run a prefill workload through the library and compare it with the oracle on the
    queries q_sel (local indices; all queries if None)."""
    dev = "cuda"
    inp = wl.make_prefill(spec, dev)
    run = runner.Prefill(inp, dev, W_x, impl)
    run.step()
    _sync()
    assert run.read_status() == 0, f"device status {run.read_status()}"
    rep = {} if report is None else report
    _separate_index_topk(run, rep)
    q_sel = list(range(spec.n_q)) if q_sel is None else list(q_sel)
    orc = OraclePrefill(inp, q_sel, W_x)
    d_n = spec.d_n

    # compression
    n_c = inp["n_c"]
    lib_ent = rows_np(spec.kv_fmt, run.ent)[:n_c]
    rep["entries_flip_frac"] = stored_check(spec.kv_fmt, lib_ent, orc.ent_f, d_n, "entries")

    # window rows the sampled queries use
    lib_win = orc.win_f
    if orc.win_pos.size:
        sel = torch.as_tensor(orc.win_pos - inp["win_pos0"], device=dev)
        lib_win = rows_np(spec.win_fmt, run.win, sel)
        rep["window_flip_frac"] = stored_check(spec.win_fmt, lib_win, orc.win_f, d_n, "window rows")

    # queries (rows of all heads of the sampled queries)
    qrows = torch.as_tensor([i * spec.H + h for i in q_sel for h in range(spec.H)], device=dev)
    lib_q = rows_np(spec.q_fmt, run.q, qrows).reshape(len(q_sel), spec.H, spec.D)
    rep["query_flip_frac"] = stored_check(spec.q_fmt, lib_q, orc.q_f, d_n, "queries")

    e2e_out = out_np(run, q_sel)
    sel_t = torch.as_tensor(q_sel, device=dev)
    e2e_idx = np_(run.idx[sel_t]) if spec.is_csa else None

    exp_idx = {}
    orc_idx = {}
    if spec.is_csa:
        scores_gpu = np_(run.scores[sel_t])
        lib_kI = None
        if spec.idx_fmt == wl.IDX_MXFP4:
            # indexer queries quantised by the standalone quantiser (exact inputs: bit-exact;
            # the indexer forms the same bytes itself, see test_gpu_index_topk), keys pooled
            # and quantised by the path (FP32 pooling: within one grid step)
            run.quant_q()
            _sync()
            assert np.array_equal(np_(run.qI["codes"][sel_t]), orc.qI_codes), "quantised indexer query codes"
            assert np.array_equal(np_(run.qI["scales"][sel_t]), orc.qI_scales), "quantised indexer query scales"
            kc, ks = np_(run.kI["codes"][:n_c]), np_(run.kI["scales"][:n_c])
            rep["index_keys_flip_frac"] = mxfp4_check(kc, ks, orc.kI_codes, orc.kI_scales, "indexer keys")
            lib_kI = O.mxfp4_to_f64(kc, ks)
        s_or = {}
        n_diff = 0
        for i, q in enumerate(q_sel):
            # scores on the path's own indexer operands; the selection against the oracle's
            s, bnd = orc.scores(i, lib_kI)
            s_o, bnd_o = orc.scores(i) if lib_kI is not None else (s, bnd)
            s_or[i] = s
            g = scores_gpu[i, :s.shape[0]].astype(np.float64)
            assert np.all(np.abs(g - s) <= bnd), f"scores of query {q}: max err {np.max(np.abs(g - s))}"
            exp_idx[i] = O.topk(s_o, spec.k)
            orc_idx[i] = exp_idx[i]
            ok_i, nd, why = topk_sets_ok(e2e_idx[i], exp_idx[i], s_o, spec.k, spec.fp32, bnd_o)
            assert ok_i, f"top-k of query {q}: {why}"
            n_diff += nd
        rep["topk_e2e_set_diff"] = n_diff
        # top-k stage-wise: identical FP32 scores on both sides -> bit-exact
        for i, q in enumerate(q_sel):
            row = torch.full((run.scores.shape[1],), float("nan"), dtype=torch.float32)
            row[:s_or[i].shape[0]] = torch.from_numpy(s_or[i].astype(np.float32))
            run.scores[q] = row.to(dev)
        run.topk()
        _sync()
        got_idx = np_(run.idx[sel_t])
        for i, q in enumerate(q_sel):
            exp = O.topk(s_or[i].astype(np.float32).astype(np.float64), spec.k)
            e = -np.ones(spec.k, dtype=np.int64)
            e[:exp.shape[0]] = exp
            assert np.array_equal(got_idx[i], e), f"top-k (identical scores) of query {q} differs"
            exp_idx[i] = exp
        assert np.array_equal(np_(run.count[sel_t]), [len(exp_idx[i]) for i in range(len(q_sel))])

    # attention, stage-wise on the oracle's inputs
    write_rows(run.ent, spec.kv_fmt, orc.ent_f, d_n, slice(0, n_c))
    if orc.win_pos.size:
        write_rows(run.win, spec.win_fmt, orc.win_f, d_n,
                   torch.as_tensor(orc.win_pos - inp["win_pos0"], device=dev))
    write_rows(run.q, spec.q_fmt, orc.q_f.reshape(-1, spec.D), d_n, qrows)
    if spec.is_csa:
        rows_idx = np.full((len(q_sel), spec.k), -1, dtype=np.int32)
        for i in range(len(q_sel)):
            rows_idx[i, :exp_idx[i].shape[0]] = exp_idx[i]
        run.idx[sel_t] = torch.from_numpy(rows_idx).to(dev)
    run.attn()
    _sync()
    assert run.read_status() == 0
    got = out_np(run, q_sel)
    got_lse = np_(run.lse.view(-1, spec.H)[sel_t])
    worst = 0.0
    e2e = _E2E(spec)
    for i, q in enumerate(q_sel):
        o, lse = orc.attend(i, exp_idx.get(i))
        ok_i, err, tol = attn_ok(got[i], o, spec.out_f32)
        worst = max(worst, _ratio(err, tol))
        assert ok_i, f"attention (oracle inputs) query {q}: err {err} > tol {tol}"
        rep["attn_max_err_ulps"] = max(rep.get("attn_max_err_ulps", 0.0), attn_err_in_ulps(got[i], o, spec.out_f32))
        np.testing.assert_allclose(got_lse[i], lse, rtol=0, atol=LSE_TOL_F32 if spec.out_f32 else LSE_TOL_BF16)
        # end to end: every row of the library's own pipeline
        lib_idx = e2e_idx[i] if spec.is_csa else None
        e2e.add(f"query {q}", e2e_out[i],
                lambda idx, **kw: orc.attend(i, idx, **kw), lambda idx, **kw: orc.keys(i, idx, **kw),
                orc.q_f[i], lib_q[i], lib_ent, lib_win, lib_idx, orc_idx.get(i), orc.sink)
    rep["attn_worst_err_over_tol"] = worst
    e2e.verdict(rep, len(q_sel))
    return rep


def _ratio(err, tol):
    return err / tol if tol > 0 else (0.0 if err == 0 else float("inf"))


class _E2E:
    """End-to-end attention check over the queries of one run (see the module docstring)."""

    def __init__(self, spec):
        self.spec = spec
        self.rows = self.queries = self.bounded = 0
        self.worst_own = self.worst_path = self.worst_bound = 0.0

    def add(self, what, out, attend, keys, q_orc, q_lib, ent_lib, win_lib, idx_lib, idx_orc, sink):
        s = self.spec
        # the library's output against the method applied to the library's own
        # intermediates and selection: every (query, head) row within the tolerance
        o_lib, _ = attend(idx_lib, q=q_lib, ent=ent_lib, win=win_lib)
        ok, err, tol = attn_ok(out, o_lib, s.out_f32)
        assert ok, f"attention (end to end) {what}: err {err} > tol {tol}"
        self.worst_own = max(self.worst_own, _ratio(err, tol))
        self.rows += out.shape[0]
        self.queries += 1
        # the oracle's own whole path, and how far the library's intermediates move it
        o_orc, _ = attend(idx_orc)
        _, err2, tol2 = attn_ok(out, o_orc, s.out_f32)
        self.worst_path = max(self.worst_path, _ratio(err2, tol2))
        same_sel = not s.is_csa or np.array_equal(np.asarray([v for v in idx_lib if v >= 0]), np.asarray(idx_orc))
        if same_sel:
            b = perturbation_bound(q_orc, keys(idx_orc), q_lib, keys(idx_lib, ent=ent_lib, win=win_lib), sink, s.scale,
                                   O.nope_dims(s.D, s.rope_off, s.d_r) if s.v_nope else None)
            d = np.abs(o_lib - o_orc)
            assert np.all(d <= b), f"attention (end to end) {what}: intermediates move the result by " \
                                   f"{np.max(d - b)} beyond their perturbation bound"
            self.worst_bound = max(self.worst_bound, float(np.max(d / b)))
            self.bounded += 1

    def verdict(self, rep, n_queries):
        assert self.queries == n_queries, "every query is compared end to end"
        rep["attn_e2e_rows_checked"] = self.rows
        rep["attn_e2e_worst_err_over_tol"] = self.worst_own
        rep["attn_e2e_queries_same_selection"] = f"{self.bounded}/{self.queries}"
        rep["attn_e2e_worst_shift_over_bound"] = self.worst_bound
        rep["attn_e2e_worst_err_over_tol_vs_oracle_path"] = self.worst_path


def save_report(name: str, rep: dict) -> None:
    """Write a test's report dict to $LC_TEST_REPORT_DIR/<name>.json when that is set."""
    d = os.environ.get("LC_TEST_REPORT_DIR")
    if d:
        os.makedirs(d, exist_ok=True)
        with open(os.path.join(d, name + ".json"), "w") as f:
            json.dump(rep, f, indent=1, default=float)


def check_decode(spec: wl.Spec, W_x: int = None, report=None, impl: int = 0):
    dev = "cuda"
    inp = wl.make_decode(spec, dev)
    run = runner.Decode(inp, dev, W_x, impl)
    run.step()
    _sync()
    assert run.read_status() == 0, f"device status {run.read_status()}"
    rep = {} if report is None else report
    _separate_index_topk(run, rep)
    orc = OracleDecode(inp, W_x)
    B = spec.num_seqs
    d_n = spec.d_n

    # decode-time compression of the closed block
    lib_ent = orc.ent_f.copy()
    for b, f in orc.new_entry.items():
        r = orc.ent_start[b] + spec.seq_lens[b] // spec.m - 1
        got = rows_np(spec.kv_fmt, run.ent, torch.as_tensor([r], device=dev))[0]
        stored_check(spec.kv_fmt, got[None], f[None], d_n, f"decode compression of sequence {b}")
        lib_ent[r] = got
    # newest window rows
    got = rows_np(spec.win_fmt, run.win, run.win_slot)
    rep["window_flip_frac"] = stored_check(spec.win_fmt, got, orc.new_win, d_n, "newest window rows")
    lib_win = orc.win_f.copy()
    for b in range(B):
        lib_win[b, orc.win_len[b] - 1] = got[b]
    # queries
    lib_q = rows_np(spec.q_fmt, run.q).reshape(B, spec.H, spec.D)
    rep["query_flip_frac"] = stored_check(spec.q_fmt, lib_q, orc.q_f, d_n, "queries")

    e2e_out = out_np(run, range(B))
    exp_idx = {}
    orc_idx = {}
    if spec.is_csa:
        e2e_idx = np_(run.idx)
        scores_gpu = np_(run.scores)
        lib_kI = None
        if spec.idx_fmt == wl.IDX_MXFP4:
            run.quant_q()
            _sync()
            assert np.array_equal(np_(run.qI["codes"]), orc.qI_codes), "quantised indexer query codes"
            assert np.array_equal(np_(run.qI["scales"]), orc.qI_scales), "quantised indexer query scales"
            lib_kI = {"codes": np_(run.kI["codes"]), "scales": np_(run.kI["scales"])}
            for b, (r, c, sc) in orc.new_key.items():
                mxfp4_check(lib_kI["codes"][r:r + 1], lib_kI["scales"][r:r + 1], c[None], sc[None],
                            f"indexer key of the block sequence {b} closed")
        s_or = {}
        n_diff = 0
        for b in range(B):
            s, bnd = orc.scores(b, lib_kI)
            s_o, bnd_o = orc.scores(b) if lib_kI is not None else (s, bnd)
            s_or[b] = s
            g = scores_gpu[b, :s.shape[0]].astype(np.float64)
            assert np.all(np.abs(g - s) <= bnd), f"scores of sequence {b}: max err {np.max(np.abs(g - s))}"
            exp_idx[b] = O.topk(s_o, spec.k)
            orc_idx[b] = exp_idx[b]
            ok_b, nd, why = topk_sets_ok(e2e_idx[b], exp_idx[b], s_o, spec.k, spec.fp32, bnd_o)
            assert ok_b, f"top-k of sequence {b}: {why}"
            n_diff += nd
        rep["topk_e2e_set_diff"] = n_diff
        s32 = torch.full_like(run.scores, float("nan"))
        for b in range(B):
            s32[b, :s_or[b].shape[0]] = torch.from_numpy(s_or[b].astype(np.float32)).to(dev)
        run.scores.copy_(s32)
        run.topk()
        _sync()
        got_idx = np_(run.idx)
        for b in range(B):
            exp = O.topk(s_or[b].astype(np.float32).astype(np.float64), spec.k)
            e = -np.ones(spec.k, dtype=np.int64)
            e[:exp.shape[0]] = exp
            assert np.array_equal(got_idx[b], e), f"top-k (identical scores) of sequence {b}"
            exp_idx[b] = exp
    # attention stage-wise: oracle's window rows, queries, indices (the cache is shared input)
    write_rows(run.win, spec.win_fmt, orc.new_win, d_n, run.win_slot)
    for b, f in orc.new_entry.items():
        r = orc.ent_start[b] + spec.seq_lens[b] // spec.m - 1
        write_rows(run.ent, spec.kv_fmt, f[None], d_n, slice(r, r + 1))
    write_rows(run.q, spec.q_fmt, orc.q_f.reshape(-1, spec.D), d_n, slice(0, B * spec.H))
    if spec.is_csa:
        idx_t = torch.full_like(run.idx, -1)
        for b in range(B):
            idx_t[b, :exp_idx[b].shape[0]] = torch.from_numpy(exp_idx[b].astype(np.int32)).to(dev)
        run.idx.copy_(idx_t)
    run.attn()
    _sync()
    assert run.read_status() == 0
    got = out_np(run, range(B))
    got_lse = np_(run.lse.view(B, spec.H))
    worst = 0.0
    e2e = _E2E(spec)
    for b in range(B):
        o, lse = orc.attend(b, exp_idx.get(b))
        ok_b, err, tol = attn_ok(got[b], o, spec.out_f32)
        worst = max(worst, _ratio(err, tol))
        assert ok_b, f"attention (oracle inputs) sequence {b}: err {err} > tol {tol}"
        rep["attn_max_err_ulps"] = max(rep.get("attn_max_err_ulps", 0.0), attn_err_in_ulps(got[b], o, spec.out_f32))
        np.testing.assert_allclose(got_lse[b], lse, rtol=0, atol=LSE_TOL_F32 if spec.out_f32 else LSE_TOL_BF16)
        lib_idx = e2e_idx[b] if spec.is_csa else None
        e2e.add(f"sequence {b}", e2e_out[b],
                lambda idx, **kw: orc.attend(b, idx, **kw), lambda idx, **kw: orc.keys(b, idx, **kw),
                orc.q_f[b], lib_q[b], lib_ent, lib_win, lib_idx, orc_idx.get(b), orc.sink)
    rep["attn_worst_err_over_tol"] = worst
    e2e.verdict(rep, B)
    return rep
