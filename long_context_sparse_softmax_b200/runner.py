"""Drive a workload through the C ABI: allocate the path's buffers with torch (device
memory only) and issue the library calls in the method's order.

Prefill (one sequence): prepare queries and window tokens -> compress the context ->
[CSA: index scores -> top-k] -> attention.  Decode (one query per sequence, on a
cache): prepare the query and the newest token's window row, compress the block the
newest token closed, [CSA: index -> top-k] -> attention.  With MXFP4 indexer operands the
index and top-k stages run fused (lc_csa_index_topk_*: no score matrix) unless the run is
built with fused=False, or the choice is left open and the fused call's merge would take
more than FUSED_MAX_CANDIDATES candidates per query; the separate calls stay available as
index() and topk().

Nothing here computes any part of the method; every step is a kernel of liblc.so.
"""
from __future__ import annotations

import functools
from typing import Dict, Optional

import torch

from . import (AttnArgs, Batch, CompressArgs, Dims, IndexArgs, IndexCompressArgs, IndexTopkArgs, Mxfp4QuantArgs,
               QkPrepArgs, Rows, TopkArgs,
               LC_FMT_BF16, LC_FMT_E4M3_BF16, LC_FMT_F32, LC_IDX_F32, LC_IDX_MXFP4, LC_IDX_MXFP4_QBF16,
               lc_csa_compress_decode, lc_csa_compress_prefill, lc_csa_index_scores_decode,
               lc_csa_index_scores_prefill, lc_csa_index_topk_decode, lc_csa_index_topk_prefill,
               lc_csa_index_topk_workspace_bytes, lc_csa_index_compress_decode, lc_csa_index_compress_prefill,
               lc_mxfp4_quantize, lc_csa_sparse_attn_decode, lc_csa_sparse_attn_prefill,
               lc_csa_sparse_attn_workspace_bytes, lc_csa_topk_decode, lc_csa_topk_prefill,
               lc_hca_attn_decode, lc_hca_attn_prefill, lc_hca_attn_prefill_workspace_bytes, lc_hca_attn_workspace_bytes,
               lc_hca_compress_decode, lc_hca_compress_prefill, lc_qk_prep_decode, lc_qk_prep_prefill)
from . import workloads as wl

RMS_EPS = 1e-6
ROPE_BASE = 10000.0


def ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def alloc_rows(fmt: int, n: int, D: int, d_r: int, device) -> Dict[str, torch.Tensor]:
    if fmt == LC_FMT_F32:
        return {"x": torch.empty(n, D, dtype=torch.float32, device=device)}
    if fmt == LC_FMT_BF16:
        return {"x": torch.empty(n, D, dtype=torch.int16, device=device)}
    return {"x": torch.empty(n, D - d_r, dtype=torch.uint8, device=device),
            "rope": torch.empty(n, d_r, dtype=torch.int16, device=device)}


def rows(fmt: int, r: Dict[str, torch.Tensor]) -> Rows:
    return Rows(fmt, 0, ptr(r["x"]), ptr(r.get("rope")))


def batch(bd: Dict[str, torch.Tensor]) -> Batch:
    return Batch(int(bd["n_ent"].numel()), int(bd.get("win_ring", 0)), ptr(bd["q_start"]), ptr(bd["q_pos0"]),
                 ptr(bd["ent_start"]),
                 ptr(bd["n_ent"]), ptr(bd["win_start"]), ptr(bd["win_pos0"]), ptr(bd["win_len"]))


def _round4(n: int) -> int:
    return max(4, (n + 3) // 4 * 4)


class _Common:
    # side stages in groups: a group runs in order on one side stream (its stages share
    # inputs); groups run concurrently with one another and with the main stages
    SIDE_GROUPS = (("qk_prep_q",), ("qk_prep_win",), ("compress", "index_compress"))

    def dag(self):
        """The step as (side groups, main, after).  The side groups (query and window
        preparation, compression) and `main` (decode: indexer query quantisation; index
        scores -> top-k) share no buffers that one writes and the other reads in the same step, so
        they may run concurrently; `after` (attention) needs all of them.  In prefill the
        indexer keys are compressed on the main stream: the indexer reads them."""
        st = dict(self.stages())
        main_names = ("index_compress",) if not self.spec.is_decode else ()
        main_names += ("quant_q", "index", "topk", "index_topk")
        side = [[(n, st[n]) for n in grp if n in st and n not in main_names] for grp in self.SIDE_GROUPS]
        side = [g for g in side if g]
        main = [(n, st[n]) for n in main_names if n in st]
        return side, main, [("attn", st["attn"])]

    def host_inputs(self):
        """The device tensors a step reads that a caller refills from the host each step,
        by the stage that first reads them: {stage: [tensors]}.  Tensors that stages on
        different streams share are listed under "_fork" (copied before the fork)."""
        inp, s = self.inp, self.spec
        raw = s.is_csa and s.idx_fmt == wl.IDX_MXFP4
        qI = ([inp["qI_raw"]] if raw else list(inp["qI"].values())) if s.is_csa else []
        if s.is_decode:
            h = {"qk_prep_q": [inp["q_raw"]], "qk_prep_win": [inp["x_new"]],
                 "compress": [inp["x_tail"], inp["g_tail"]]}
            if raw:
                h["index_compress"] = [inp["kI_tail"]]
        else:
            h = {"qk_prep_q": [inp["q_raw"]], "_fork": [inp["x"], inp["g"]]}
            if raw:
                h["index_compress"] = [inp["kI_raw"]]
        if qI:
            h["quant_q" if raw and not self.q_in_call else ("index_topk" if self.fused else "index")] = qI
        return h

    def host_outputs(self):
        """The step's results a caller reads back: attention output and lse."""
        return [self.out, self.lse]

    def _indexer_buffers(self, n_q: int, n_keys: int, decode: bool):
        """Indexer operands the step reads: in MXFP4 the queries quantised by the step's
        quant_q stage and, in prefill, the compressed keys that the step's own kernels
        write; or the given FP32 operands.  The indexer can quantise BF16 queries itself
        (LC_IDX_MXFP4_QBF16, q_in_call), but the separate quantiser measured faster in both
        steps: in decode its short kernel lets the side-stream kernels take their SMs before
        the indexer fills every SM (in-call: decode step 103 against 92 us), and in prefill
        each query's rows would be quantised once per key range (in-call: index 27.8 against
        19.3 ms)."""
        s, inp, dev = self.spec, self.inp, self.device
        if s.idx_fmt != wl.IDX_MXFP4:
            self.qI, self.kI = inp["qI"], inp["kI"]
            return
        u8 = dict(dtype=torch.uint8, device=dev)
        self.qI = {"codes": torch.empty(n_q, s.H_I, s.d_I // 2, **u8), "scales": torch.empty(n_q, s.H_I, s.d_I // 32, **u8)}
        if decode:
            self.kI = inp["kI"]
        else:
            self.kI = {"codes": torch.empty(max(n_keys, 1), s.d_I // 2, **u8),
                       "scales": torch.empty(max(n_keys, 1), s.d_I // 32, **u8)}
        self.a_quant_q = Mxfp4QuantArgs(n_q * s.H_I, s.d_I, LC_FMT_BF16, ptr(inp["qI_raw"]), ptr(self.qI["codes"]),
                                        ptr(self.qI["scales"]))

    def _index_compress_args(self, x_raw, g, c: Dict[str, torch.Tensor], num_seqs: int, max_blocks: int,
                             blk_first, blk_count, ent_start) -> IndexCompressArgs:
        s = self.spec
        return IndexCompressArgs(s.d_I, s.m, num_seqs, LC_FMT_BF16, max_blocks, 0, ptr(x_raw), ptr(g),
                                 ptr(c["tok_row0"]), ptr(c["tok_pos0"]), ptr(c["tok_len"]), ptr(blk_first),
                                 ptr(blk_count), ptr(ent_start), ptr(self.kI["codes"]), ptr(self.kI["scales"]),
                                 ptr(self.status))

    def quant_q(self, stream=None):
        """The indexer queries in MXFP4 by the standalone quantiser (a decode stage)."""
        lc_mxfp4_quantize(self.a_quant_q, stream)

    def _index_stages(self):
        """The indexer and top-k stages of a step.  On the main stream each follows another
        kernel of the step whose outputs alone it reads after that kernel completes, so it
        is launched programmatically (its set-up and the loads of its other inputs overlap
        the previous kernel): the indexer after the query quantisation (unless it quantises
        them itself: then the kernel before it may write its keys, and it launches in plain
        order), the top-k after the indexer, and the attention (see stages()) after the
        top-k.  Called on their own, the stages launch in plain stream order."""
        pdl_index = self.spec.idx_fmt == wl.IDX_MXFP4 and not self.q_in_call  # after quant_q
        if self.fused:
            return [("index_topk", functools.partial(self.index_topk, pdl=pdl_index))]
        return [("index", functools.partial(self.index, pdl=pdl_index)), ("topk", functools.partial(self.topk, pdl=True))]

    def step_overlapped(self, main, side, on_stage=None, io=None):
        """One step on several streams: the side stages fork from `main` (stage i on
        side[i % len(side)]; `side` is one stream or a list) and join it before
        attention.  on_stage(name, stream, fn) may wrap each launch (e.g. with timing
        events).  io = (h2d, d2h) adds the host copies: h2d maps a stage (or "_fork") to
        (device, pinned host) pairs copied on that stage's stream just before it, so an
        upload overlaps the stages before it (the main stream's uploads go first, before
        the fork); d2h holds (pinned host, device) pairs copied on `main` after attention."""
        import torch
        sd, mn, af = self.dag()
        sides = list(side) if isinstance(side, (list, tuple)) else [side]
        launch = on_stage or (lambda name, stream, fn: fn(stream))
        h2d, d2h = io if io is not None else ({}, [])

        copied = set()

        def run(name, stream, fn):
            if h2d.get(name) and name not in copied:
                with torch.cuda.stream(stream):
                    for d, h in h2d[name]:
                        d.copy_(h, non_blocking=True)
            launch(name, stream, fn)
        # uploads for the critical path go first, before the fork: the side streams' larger
        # uploads (query rows) queue behind them on the copy engine instead of in front
        with torch.cuda.stream(main):
            for name in ["_fork"] + [n for n, _ in mn]:
                for d, h in h2d.get(name, []):
                    d.copy_(h, non_blocking=True)
                copied.add(name)
        fork = torch.cuda.Event()
        fork.record(main)
        used = sides[:min(len(sd), len(sides))]
        for st in used:
            st.wait_event(fork)
        # the critical path is enqueued first, so its CTAs take the SMs before the side
        # streams' do
        for n, f in mn:
            run(n, main, f)
        for i, grp in enumerate(sd):
            for n, f in grp:
                run(n, sides[i % len(sides)], f)
        for st in used:
            join = torch.cuda.Event()
            join.record(st)
            main.wait_event(join)
        for n, f in af:
            run(n, main, f)
        if d2h:
            with torch.cuda.stream(main):
                for h, d in d2h:
                    h.copy_(d, non_blocking=True)

    def _index_args(self, n_q: int, max_ent: int, scores: torch.Tensor) -> IndexArgs:
        s, inp = self.spec, self.inp
        qI, kI = self.qI, self.kI
        mx = s.idx_fmt == wl.IDX_MXFP4
        if mx and self.q_in_call:
            fmt, q, q_scale = LC_IDX_MXFP4_QBF16, ptr(inp["qI_raw"]), None
        elif mx:
            fmt, q, q_scale = LC_IDX_MXFP4, ptr(qI["codes"]), ptr(qI["scales"])
        else:
            fmt, q, q_scale = LC_IDX_F32, ptr(qI["f32"]), None
        return IndexArgs(n_q, s.H_I, s.d_I, fmt, q, q_scale,
                         ptr(kI["codes"] if mx else kI["f32"]), ptr(kI.get("scales")),
                         (kI["codes"] if mx else kI["f32"]).shape[0], ptr(inp["w"]), s.H_I if s.w_per_query else 0, s.m,
                         self.W_x, max_ent, self.batch,
                         ptr(scores), scores.shape[1], ptr(self.status))

    # The fused index + top-k call is the default while its merge takes at most this many
    # candidates per query (they then stay in registers: measured faster than the separate
    # score matrix and top-k); past it the separate calls are faster (measured on B200:
    # 32 ranges x 1024 candidates merged in about 43 us against a 40 us separate top-k).
    FUSED_MAX_CANDIDATES = 8192

    def _choose_fused(self, fused_arg, n_q: int):
        """Keep the fused call unless the caller left the choice open and its merge would
        take more than FUSED_MAX_CANDIDATES candidates per query (the workspace holds them:
        n_chunks x k pairs of 8 bytes per query)."""
        if fused_arg is None and self.fused:
            per_query = self.a_index_topk.workspace_bytes // (8 * max(n_q, 1))
            if per_query > self.FUSED_MAX_CANDIDATES:
                self.fused = False

    def _index_topk_args(self, n_q: int, max_ent: int, decode: bool) -> IndexTopkArgs:
        """Fused index + top-k into idx / count (the buffers the separate top-k call writes
        and attention reads)."""
        s = self.spec
        a = IndexTopkArgs()
        a.index = self._index_args(n_q, max_ent, self.scores)
        a.index.scores, a.index.score_stride = None, 0
        a.k = s.k
        a.idx, a.count = ptr(self.idx), ptr(self.count)
        ws = lc_csa_index_topk_workspace_bytes(a, decode)
        self.ws_topk = torch.empty(max(ws, 16), dtype=torch.uint8, device=self.device)
        a.workspace, a.workspace_bytes = ptr(self.ws_topk), ws
        return a

    def _topk_args(self, n_q: int, max_ent: int) -> TopkArgs:
        s = self.spec
        return TopkArgs(n_q, s.k, s.m, self.W_x, max_ent, 0, ptr(self.scores), self.scores.shape[1], self.batch,
                        ptr(self.idx), ptr(self.count), ptr(self.status))

    def _attn_args(self, n_q: int, max_ent: int, sparse: bool, prefill: bool = False) -> AttnArgs:
        s = self.spec
        a = AttnArgs()
        a.dims = self.dims
        a.n_q, a.k, a.m, a.W, a.W_x, a.max_ent = n_q, (s.k if sparse else 0), s.m, s.W, self.W_x, max_ent
        a.scale = s.scale
        a.out_fmt = LC_FMT_F32 if s.out_f32 else LC_FMT_BF16
        a.q = rows(s.q_fmt, self.q)
        a.ent = rows(s.kv_fmt, self.ent)
        a.win = rows(s.win_fmt, self.win)
        a.idx = ptr(self.idx) if sparse else None
        a.sink = ptr(self.inp["sink"])
        a.batch = self.batch
        a.out = ptr(self.out)
        a.lse = ptr(self.lse)
        a.status = ptr(self.status)
        a.impl = self.impl
        a.n_ent_rows = int(next(iter(self.ent.values())).shape[0])
        a.n_win_rows = int(self.win["x"].shape[0])
        a.v_nope = 1 if s.v_nope else 0
        if sparse:
            ws = lc_csa_sparse_attn_workspace_bytes(a)
        elif prefill:  # optional: the entries widened to F16 once per call
            ws = lc_hca_attn_prefill_workspace_bytes(a)
        else:
            ws = lc_hca_attn_workspace_bytes(a)
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=self.device)
        a.workspace, a.workspace_bytes = ptr(self.workspace), ws
        return a

    def read_status(self) -> int:
        return int(self.status.item())


class Prefill(_Common):
    """One sequence of L raw tokens; queries at q_first .. q_first + n_q - 1."""

    def __init__(self, inp: Dict[str, object], device="cuda", W_x: Optional[int] = None, impl: int = 0,
                 fused: Optional[bool] = None):
        s: wl.Spec = inp["spec"]
        self.impl = impl
        self.spec, self.inp, self.device = s, inp, device
        self.fused = s.is_csa and s.idx_fmt == wl.IDX_MXFP4 if fused is None else fused
        self.q_in_call = False  # the quant_q stage quantises them (see _indexer_buffers)
        self.W_x = s.W if W_x is None else W_x
        L, n_c = inp["L"], inp["n_c"]
        self.dims = Dims(s.D, s.d_r, s.rope_off, s.H)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.ent = alloc_rows(s.kv_fmt, max(n_c, 1), s.D, s.d_r, device)
        n_win = int(inp["win_pos"].numel())
        self.win = alloc_rows(s.win_fmt, n_win, s.D, s.d_r, device)
        self.q = alloc_rows(s.q_fmt, s.n_q * s.H, s.D, s.d_r, device)
        self.batch = batch(inp["batch"])
        i32 = dict(dtype=torch.int32, device=device)
        i64 = dict(dtype=torch.int64, device=device)
        self._cmp = {"tok_row0": torch.zeros(1, **i64), "tok_pos0": torch.zeros(1, **i32),
                     "tok_len": torch.tensor([L], **i32), "blk_first": torch.zeros(1, **i32),
                     "blk_count": torch.tensor([n_c], **i32), "ent_start": torch.zeros(1, **i64)}
        c = self._cmp
        self.a_compress = CompressArgs(Dims(s.D, s.d_r, s.rope_off, 1), s.m, 1, s.raw_fmt, n_c, ptr(inp["x"]),
                                       ptr(inp["g"]), ptr(c["tok_row0"]), ptr(c["tok_pos0"]), ptr(c["tok_len"]),
                                       ptr(c["blk_first"]), ptr(c["blk_count"]), ptr(c["ent_start"]),
                                       rows(s.kv_fmt, self.ent), RMS_EPS, ROPE_BASE, ptr(self.status))
        self.a_prep_q = QkPrepArgs(self.dims, s.n_q, s.raw_fmt, ptr(inp["q_raw"]), ptr(inp["q_pos"]), None,
                                   rows(s.q_fmt, self.q), RMS_EPS, ROPE_BASE, ptr(self.status))
        x_win = inp["x"][inp["win_pos0"]:]
        self.a_prep_win = QkPrepArgs(Dims(s.D, s.d_r, s.rope_off, 1), n_win, s.raw_fmt, ptr(x_win),
                                     ptr(inp["win_pos"]), None, rows(s.win_fmt, self.win), RMS_EPS, ROPE_BASE,
                                     ptr(self.status))
        self.out = torch.empty(s.n_q * s.H, s.Dv, dtype=torch.float32 if s.out_f32 else torch.int16, device=device)
        self.lse = torch.empty(s.n_q * s.H, dtype=torch.float32, device=device)
        if s.is_csa:
            self._indexer_buffers(s.n_q, n_c, False)
            if s.idx_fmt == wl.IDX_MXFP4:
                self.a_index_compress = self._index_compress_args(inp["kI_raw"], inp["g"], c, 1, n_c, c["blk_first"],
                                                                  c["blk_count"], c["ent_start"])
            self.scores = torch.empty(s.n_q, _round4(n_c), dtype=torch.float32, device=device)
            self.idx = torch.empty(s.n_q, s.k, dtype=torch.int32, device=device)
            self.count = torch.empty(s.n_q, dtype=torch.int32, device=device)
            self.a_index = self._index_args(s.n_q, n_c, self.scores)
            self.a_topk = self._topk_args(s.n_q, n_c)
            if self.fused:
                self.a_index_topk = self._index_topk_args(s.n_q, n_c, False)
                self._choose_fused(fused, s.n_q)
        else:
            self.idx = None
        self.a_attn = self._attn_args(s.n_q, n_c, s.is_csa, prefill=True)

    def prep_queries(self, stream=None):
        lc_qk_prep_prefill(self.a_prep_q, stream)

    def prep_window(self, stream=None):
        lc_qk_prep_prefill(self.a_prep_win, stream)

    def compress(self, stream=None):
        (lc_csa_compress_prefill if self.spec.is_csa else lc_hca_compress_prefill)(self.a_compress, stream)

    def index_compress(self, stream=None):
        lc_csa_index_compress_prefill(self.a_index_compress, stream)

    # pdl: launch programmatically after the previous kernel of the step (see stages())
    def index(self, stream=None, pdl=False):
        self.a_index.pdl = int(pdl)
        lc_csa_index_scores_prefill(self.a_index, stream)

    def topk(self, stream=None, pdl=False):
        self.a_topk.pdl = int(pdl)
        lc_csa_topk_prefill(self.a_topk, stream)

    def index_topk(self, stream=None, pdl=False):
        self.a_index_topk.index.pdl = int(pdl)
        lc_csa_index_topk_prefill(self.a_index_topk, stream)

    def attn(self, stream=None, pdl=False):
        self.a_attn.pdl = int(pdl)
        (lc_csa_sparse_attn_prefill if self.spec.is_csa else lc_hca_attn_prefill)(self.a_attn, stream)

    def stages(self):
        s = self.spec
        st = [("qk_prep_q", self.prep_queries), ("qk_prep_win", self.prep_window), ("compress", self.compress)]
        if s.is_csa:
            if s.idx_fmt == wl.IDX_MXFP4:
                st += [("index_compress", self.index_compress)]
                if not self.q_in_call:
                    st += [("quant_q", self.quant_q)]
            st += self._index_stages()
        return st + [("attn", functools.partial(self.attn, pdl=s.is_csa))]

    def step(self, stream=None):
        for _, f in self.stages():
            f(stream)


class Decode(_Common):
    """B sequences, one query each at L_b - 1, on an existing cache (see workloads.make_decode)."""

    def __init__(self, inp: Dict[str, object], device="cuda", W_x: Optional[int] = None, impl: int = 0,
                 fused: Optional[bool] = None):
        s: wl.Spec = inp["spec"]
        self.impl = impl
        self.spec, self.inp, self.device = s, inp, device
        self.fused = s.is_csa and s.idx_fmt == wl.IDX_MXFP4 if fused is None else fused
        self.q_in_call = False  # the quant_q stage quantises them (see _indexer_buffers)
        self.W_x = s.W if W_x is None else W_x
        B = s.num_seqs
        n_c = inp["n_c"]
        max_ent = max(n_c)
        self.dims = Dims(s.D, s.d_r, s.rope_off, s.H)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.ent = inp["cache"]
        self.win = {"x": inp["win"]}
        self.q = alloc_rows(s.q_fmt, B * s.H, s.D, s.d_r, device)
        self.batch = batch(inp["batch"])
        i32 = dict(dtype=torch.int32, device=device)
        i64 = dict(dtype=torch.int64, device=device)
        L = s.seq_lens
        self._cmp = {"tok_row0": torch.tensor([b * s.m for b in range(B)], **i64),
                     "tok_pos0": torch.tensor([Lb - s.m for Lb in L], **i32),
                     "tok_len": torch.tensor([s.m] * B, **i32)}
        c = self._cmp
        self.a_compress = CompressArgs(Dims(s.D, s.d_r, s.rope_off, 1), s.m, B, s.raw_fmt, 1, ptr(inp["x_tail"]),
                                       ptr(inp["g_tail"]), ptr(c["tok_row0"]), ptr(c["tok_pos0"]), ptr(c["tok_len"]),
                                       ptr(inp["blk_first"]), ptr(inp["blk_count"]), ptr(inp["batch"]["ent_start"]),
                                       rows(s.kv_fmt, self.ent), RMS_EPS, ROPE_BASE, ptr(self.status))
        self.a_prep_q = QkPrepArgs(self.dims, B, s.raw_fmt, ptr(inp["q_raw"]), ptr(inp["q_pos"]), None,
                                   rows(s.q_fmt, self.q), RMS_EPS, ROPE_BASE, ptr(self.status))
        # the newest token's window row: its ring slot, or the last row of the linear window
        self.win_slot = torch.tensor([b * s.W + ((Lb - 1) % s.W if s.ring else Lb - 1 - max(0, Lb - s.W))
                                      for b, Lb in enumerate(L)], **i64)
        self.a_prep_win = QkPrepArgs(Dims(s.D, s.d_r, s.rope_off, 1), B, s.raw_fmt, ptr(inp["x_new"]),
                                     ptr(inp["q_pos"]), ptr(self.win_slot), rows(s.win_fmt, self.win), RMS_EPS,
                                     ROPE_BASE, ptr(self.status))
        self.out = torch.empty(B * s.H, s.Dv, dtype=torch.float32 if s.out_f32 else torch.int16, device=device)
        self.lse = torch.empty(B * s.H, dtype=torch.float32, device=device)
        if s.is_csa:
            self._indexer_buffers(B, sum(n_c), True)
            if s.idx_fmt == wl.IDX_MXFP4:
                self.a_index_compress = self._index_compress_args(inp["kI_tail"], inp["g_tail"], c, B, 1,
                                                                  inp["blk_first"], inp["blk_count"],
                                                                  inp["batch"]["ent_start"])
            self.scores = torch.empty(B, _round4(max_ent), dtype=torch.float32, device=device)
            self.idx = torch.empty(B, s.k, dtype=torch.int32, device=device)
            self.count = torch.empty(B, dtype=torch.int32, device=device)
            self.a_index = self._index_args(B, max_ent, self.scores)
            self.a_topk = self._topk_args(B, max_ent)
            if self.fused:
                self.a_index_topk = self._index_topk_args(B, max_ent, True)
                self._choose_fused(fused, B)
        else:
            self.idx = None
        self.a_attn = self._attn_args(B, max_ent, s.is_csa)

    def prep_queries(self, stream=None):
        lc_qk_prep_decode(self.a_prep_q, stream)

    def prep_window(self, stream=None):
        lc_qk_prep_decode(self.a_prep_win, stream)

    def compress(self, stream=None):
        (lc_csa_compress_decode if self.spec.is_csa else lc_hca_compress_decode)(self.a_compress, stream)

    def index_compress(self, stream=None):
        lc_csa_index_compress_decode(self.a_index_compress, stream)

    # pdl: launch programmatically after the previous kernel of the step (see stages())
    def index(self, stream=None, pdl=False):
        self.a_index.pdl = int(pdl)
        lc_csa_index_scores_decode(self.a_index, stream)

    def topk(self, stream=None, pdl=False):
        self.a_topk.pdl = int(pdl)
        lc_csa_topk_decode(self.a_topk, stream)

    def index_topk(self, stream=None, pdl=False):
        self.a_index_topk.index.pdl = int(pdl)
        lc_csa_index_topk_decode(self.a_index_topk, stream)

    def attn(self, stream=None, pdl=False):
        self.a_attn.pdl = int(pdl)
        (lc_csa_sparse_attn_decode if self.spec.is_csa else lc_hca_attn_decode)(self.a_attn, stream)

    def stages(self):
        s = self.spec
        st = [("qk_prep_q", self.prep_queries), ("qk_prep_win", self.prep_window), ("compress", self.compress)]
        if s.is_csa:
            if s.idx_fmt == wl.IDX_MXFP4:
                st += [("index_compress", self.index_compress)]
                if not self.q_in_call:
                    st += [("quant_q", self.quant_q)]
            st += self._index_stages()
        return st + [("attn", functools.partial(self.attn, pdl=s.is_csa))]

    def step(self, stream=None):
        for _, f in self.stages():
            f(stream)


def capture_step(runs, main, side, on_stage=None, io=None):
    """Record one overlapped step of every run in `runs` as a CUDA graph (on_stage, if
    given, is called as on_stage(run index, stage name, stream, launch); io, if given,
    holds each run's (h2d, d2h) host copies, see step_overlapped).

    The library calls are made once, during capture; `graph.replay()` then launches the
    same kernels with the same arguments on the current stream, with the fork onto `side`
    and the join before attention kept as graph edges.  Each run's buffers and arguments
    are fixed at capture: refill the input tensors in place between replays.  Make one
    eager step first, so that one-time set-up (kernel attributes, the no-allocation
    scratch address) happens outside the capture."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=main):
        for i, r in enumerate(runs):
            r.step_overlapped(main, side, None if on_stage is None else
                              (lambda name, st, fn, i=i: on_stage(i, name, st, fn)),
                              None if io is None else io[i])
    return g


def make_run(spec: wl.Spec, device="cuda", W_x: Optional[int] = None):
    if spec.is_decode:
        return Decode(wl.make_decode(spec, device), device, W_x)
    return Prefill(wl.make_prefill(spec, device), device, W_x)
