"""Context-parallel CSA prefill: one sequence's tokens split over ranks (one process per GPU).

The 10100.com analysis lists context parallelism for the compressed attention among
DeepSeek-V4's infrastructure pieces (§三 infra list); the pages give no scheme, so this
one follows the method's data flow:

* rank r owns the block-aligned token range [t0_r, t1_r) (``partition``): its raw KV rows,
  gates, raw indexer-key rows, and the queries at those positions;
* each rank compresses its own complete blocks into KV entries and indexer keys
  (lc_csa_compress_prefill, lc_csa_index_compress_prefill), written at their global entry
  rows of a buffer padded to world x blocks-per-rank rows;
* one all-gather per array gives every rank every entry and indexer key (the only
  collective on the data path);
* the window rows of a rank's first queries reach back W - 1 tokens into the previous
  rank's range: that rank sends those raw rows (``DistComm.halo``, point to point), and
  each rank prepares the window rows of [t0_r - W + 1, t1_r) itself;
* each rank then runs the quantised indexer, the fused top-k and the sparse attention for
  its own queries over the gathered entries.

Every kernel is the library's; this module only allocates buffers, moves rows between
ranks and issues the C-ABI calls.  The rank-to-rank moves go through a `comm` object:
``DistComm`` (torch.distributed: NCCL over NVLink on GPUs, gloo on CPU) or, to run all
ranks in one process on one device, ``LocalComm``, whose ranks are stepped phase by phase
so that no kernel waits for another rank's.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import torch

from . import (AttnArgs, Batch, CompressArgs, Dims, IndexCompressArgs, IndexArgs, IndexTopkArgs, Mxfp4QuantArgs,
               QkPrepArgs, Rows, LC_FMT_BF16, LC_FMT_E4M3_BF16, LC_IDX_MXFP4, lc_csa_compress_prefill,
               lc_csa_index_compress_prefill, lc_csa_index_topk_prefill, lc_csa_index_topk_workspace_bytes,
               lc_csa_sparse_attn_prefill, lc_mxfp4_quantize, lc_qk_prep_prefill)
from . import workloads as wl

RMS_EPS = 1e-6
ROPE_BASE = 10000.0


def partition(L: int, m: int, world: int) -> Tuple[List[Tuple[int, int]], int]:
    """Token ranges [t0, t1) of the ranks and the blocks per rank nb: rank r owns blocks
    r nb .. (r + 1) nb - 1 (the last rank fewer, and the tokens past the last complete
    block).  Every range starts on a block boundary, so each block lies in one rank."""
    n_blk = L // m
    nb = max(1, -(-n_blk // world))
    ranges = []
    for r in range(world):
        t0 = min(L, r * nb * m)
        t1 = L if r == world - 1 else min(L, (r + 1) * nb * m)
        ranges.append((t0, t1))
    return ranges, nb


def halo_range(t0: int, W: int) -> Tuple[int, int]:
    """Positions [h0, t0) whose raw rows a rank starting at t0 needs from earlier ranks for
    the windows of its first queries."""
    return max(0, t0 - W + 1), t0


class DistComm:
    """Rank-to-rank moves over torch.distributed (the default process group)."""

    def __init__(self):
        import torch.distributed as dist
        self.dist = dist
        self.rank = dist.get_rank()
        self.world = dist.get_world_size()

    def all_gather_rows(self, full: torch.Tensor, nb: int) -> None:
        """full [world * nb, ...]: every rank's rows [r nb, (r + 1) nb) to every rank."""
        parts = list(full.split(nb, dim=0))
        local = parts[self.rank].clone()
        self.dist.all_gather(parts, local)

    def halo(self, send_rows: torch.Tensor, n_recv: int) -> torch.Tensor:
        """Send this rank's last rows to the next rank; receive n_recv rows from the previous
        one (rank 0 receives nothing)."""
        recv = torch.empty((n_recv,) + tuple(send_rows.shape[1:]), dtype=send_rows.dtype, device=send_rows.device)
        reqs = []
        if self.rank + 1 < self.world and send_rows.shape[0] > 0:
            reqs.append(self.dist.isend(send_rows.contiguous(), self.rank + 1))
        if self.rank > 0 and n_recv > 0:
            reqs.append(self.dist.irecv(recv, self.rank - 1))
        for req in reqs:
            req.wait()
        return recv


class LocalComm:
    """All ranks in one process: moves are copies between the ranks' buffers."""

    def __init__(self, ranks: Sequence["CpPrefillRank"]):
        self.ranks = list(ranks)

    def all_gather(self, name: str, nb: int) -> None:
        bufs = [r.gathered[name] for r in self.ranks]
        for r, src in enumerate(bufs):
            rows = src[r * nb:(r + 1) * nb]
            for dst in bufs:
                if dst is not src:
                    dst[r * nb:(r + 1) * nb].copy_(rows)


def _i32(v, dev):
    return torch.tensor(list(v), dtype=torch.int32, device=dev)


def _i64(v, dev):
    return torch.tensor(list(v), dtype=torch.int64, device=dev)


class CpPrefillRank:
    """One rank of a context-parallel CSA prefill (MXFP4 indexer, E4M3 + BF16 entries).

    local: this rank's inputs — x [t1 - t0, D] raw BF16 rows, g [t1 - t0] gates, kI_raw
    [t1 - t0, d_I], q_raw [t1 - t0, H, D], qI_raw [t1 - t0, H_I, d_I] (every position of the
    range is a query), sink [H], w [H_I]."""

    def __init__(self, spec: wl.Spec, L: int, rank: int, world: int, local: Dict[str, torch.Tensor], device):
        s = spec
        assert s.is_csa and not s.is_decode and s.idx_fmt == LC_IDX_MXFP4 and s.kv_fmt == LC_FMT_E4M3_BF16
        self.spec, self.L, self.rank, self.world, self.device = s, L, rank, world, device
        ranges, nb = partition(L, s.m, world)
        # a window reaches back W - 1 tokens: the halo must come from the previous rank alone
        assert all(t1 - t0 >= s.W - 1 for t0, t1 in ranges[:-1]), "ranges shorter than the window's halo"
        self.t0, self.t1 = ranges[rank]
        self.nb = nb
        self.n_c = L // s.m
        n_tok = self.t1 - self.t0
        self.h0, _ = halo_range(self.t0, s.W)
        self.local = local
        dev = device
        u8 = dict(dtype=torch.uint8, device=dev)
        rows = world * nb
        # entries and indexer keys at their global rows, padded to world x nb rows
        self.gathered = {
            "nope": torch.zeros(rows, s.d_n, **u8),
            "rope": torch.zeros(rows, s.d_r, dtype=torch.int16, device=dev),
            "kI_codes": torch.zeros(rows, s.d_I // 2, **u8),
            "kI_scales": torch.zeros(rows, s.d_I // 32, **u8),
        }
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        # the window rows of positions [h0, t1): raw halo rows first, then this rank's rows
        self.win_raw = torch.empty(self.t1 - self.h0, s.D, dtype=torch.int16, device=dev)
        self.win = torch.empty(self.t1 - self.h0, s.D, dtype=torch.int16, device=dev)
        self.q = {"x": torch.empty(n_tok * s.H, s.d_n, **u8),
                  "rope": torch.empty(n_tok * s.H, s.d_r, dtype=torch.int16, device=dev)}
        self.qI = {"codes": torch.empty(n_tok, s.H_I, s.d_I // 2, **u8),
                   "scales": torch.empty(n_tok, s.H_I, s.d_I // 32, **u8)}
        self.idx = torch.empty(n_tok, s.k, dtype=torch.int32, device=dev)
        self.count = torch.empty(n_tok, dtype=torch.int32, device=dev)
        self.out = torch.empty(n_tok * s.H, s.Dv, dtype=torch.int16, device=dev)
        self.lse = torch.empty(n_tok * s.H, dtype=torch.float32, device=dev)
        self._args()

    # ------------------------------------------------------------------ arguments
    def _args(self):
        s, dev, loc = self.spec, self.device, self.local
        n_tok = self.t1 - self.t0
        j0, j1 = self.t0 // s.m, self.t1 // s.m
        self._keep = []

        def keep(t):
            self._keep.append(t)
            return t.data_ptr()
        ent = Rows(LC_FMT_E4M3_BF16, 0, self.gathered["nope"].data_ptr(), self.gathered["rope"].data_ptr())
        cmp = dict(tok_row0=keep(_i64([0], dev)), tok_pos0=keep(_i32([self.t0], dev)), tok_len=keep(_i32([n_tok], dev)),
                   blk_first=keep(_i32([j0], dev)), blk_count=keep(_i32([j1 - j0], dev)), ent_start=keep(_i64([0], dev)))
        self.n_blk = j1 - j0
        self.a_compress = CompressArgs(Dims(s.D, s.d_r, s.rope_off, 1), s.m, 1, LC_FMT_BF16, max(self.n_blk, 0),
                                       loc["x"].data_ptr(), loc["g"].data_ptr(), cmp["tok_row0"], cmp["tok_pos0"],
                                       cmp["tok_len"], cmp["blk_first"], cmp["blk_count"], cmp["ent_start"], ent,
                                       RMS_EPS, ROPE_BASE, self.status.data_ptr())
        self.a_index_compress = IndexCompressArgs(s.d_I, s.m, 1, LC_FMT_BF16, max(self.n_blk, 0), 0,
                                                  loc["kI_raw"].data_ptr(), loc["g"].data_ptr(), cmp["tok_row0"],
                                                  cmp["tok_pos0"], cmp["tok_len"], cmp["blk_first"], cmp["blk_count"],
                                                  cmp["ent_start"], self.gathered["kI_codes"].data_ptr(),
                                                  self.gathered["kI_scales"].data_ptr(), self.status.data_ptr())
        pos_q = keep(torch.arange(self.t0, self.t1, dtype=torch.int32, device=dev))
        self.a_prep_q = QkPrepArgs(Dims(s.D, s.d_r, s.rope_off, s.H), n_tok, LC_FMT_BF16, loc["q_raw"].data_ptr(), pos_q,
                                   None, Rows(LC_FMT_E4M3_BF16, 0, self.q["x"].data_ptr(), self.q["rope"].data_ptr()),
                                   RMS_EPS, ROPE_BASE, self.status.data_ptr())
        pos_w = keep(torch.arange(self.h0, self.t1, dtype=torch.int32, device=dev))
        self.a_prep_win = QkPrepArgs(Dims(s.D, s.d_r, s.rope_off, 1), self.t1 - self.h0, LC_FMT_BF16,
                                     self.win_raw.data_ptr(), pos_w, None, Rows(LC_FMT_BF16, 0, self.win.data_ptr(), None),
                                     RMS_EPS, ROPE_BASE, self.status.data_ptr())
        self.a_quant_q = Mxfp4QuantArgs(n_tok * s.H_I, s.d_I, LC_FMT_BF16, loc["qI_raw"].data_ptr(),
                                        self.qI["codes"].data_ptr(), self.qI["scales"].data_ptr())
        bd = Batch(1, 0, keep(_i32([0, n_tok], dev)), keep(_i32([self.t0], dev)), keep(_i64([0], dev)),
                   keep(_i32([self.n_c], dev)), keep(_i64([0], dev)), keep(_i32([self.h0], dev)),
                   keep(_i32([self.t1 - self.h0], dev)))
        self.batch = bd
        ia = IndexArgs(n_tok, s.H_I, s.d_I, LC_IDX_MXFP4, self.qI["codes"].data_ptr(), self.qI["scales"].data_ptr(),
                       self.gathered["kI_codes"].data_ptr(), self.gathered["kI_scales"].data_ptr(),
                       self.gathered["kI_codes"].shape[0], loc["w"].data_ptr(), 0, s.m, s.W, max(self.n_c, 1), bd,
                       None, 0, self.status.data_ptr())
        self.a_index_topk = IndexTopkArgs(ia, s.k, 0, self.idx.data_ptr(), self.count.data_ptr(), None, 0)
        ws = lc_csa_index_topk_workspace_bytes(self.a_index_topk, False)
        self.ws_topk = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
        self.a_index_topk.workspace, self.a_index_topk.workspace_bytes = self.ws_topk.data_ptr(), ws
        a = AttnArgs()
        a.dims = Dims(s.D, s.d_r, s.rope_off, s.H)
        a.n_q, a.k, a.m, a.W, a.W_x, a.max_ent = n_tok, s.k, s.m, s.W, s.W, self.n_c
        a.scale = s.scale
        a.out_fmt = LC_FMT_BF16
        a.q = Rows(LC_FMT_E4M3_BF16, 0, self.q["x"].data_ptr(), self.q["rope"].data_ptr())
        a.ent = ent
        a.win = Rows(LC_FMT_BF16, 0, self.win.data_ptr(), None)
        a.idx = self.idx.data_ptr()
        a.sink = loc["sink"].data_ptr()
        a.batch = bd
        a.out, a.lse = self.out.data_ptr(), self.lse.data_ptr()
        a.status = self.status.data_ptr()
        a.n_ent_rows = self.gathered["nope"].shape[0]
        a.n_win_rows = self.win.shape[0]
        a.v_nope = 1 if s.v_nope else 0
        self.a_attn = a

    # ------------------------------------------------------------------ phases
    def compress_local(self, stream=None):
        """Phase 1: this rank's blocks -> entries and indexer keys at their global rows; its
        queries prepared and quantised."""
        if self.n_blk > 0:
            lc_csa_compress_prefill(self.a_compress, stream)
            lc_csa_index_compress_prefill(self.a_index_compress, stream)
        if self.t1 > self.t0:
            lc_qk_prep_prefill(self.a_prep_q, stream)
            lc_mxfp4_quantize(self.a_quant_q, stream)

    def halo_send_rows(self) -> torch.Tensor:
        """The raw rows the next rank needs for its first windows: this rank's last W - 1."""
        n = min(self.spec.W - 1, self.t1 - self.t0)
        return self.local["x"][self.t1 - self.t0 - n:]

    def set_halo(self, rows: torch.Tensor, stream=None):
        """Phase 2 (after the halo exchange): the window's raw rows [h0, t1), then their
        preparation."""
        nh = self.t0 - self.h0
        if nh:
            self.win_raw[:nh].copy_(rows[rows.shape[0] - nh:])
        self.win_raw[nh:].copy_(self.local["x"])
        lc_qk_prep_prefill(self.a_prep_win, stream)

    def attend(self, stream=None):
        """Phase 3 (after the all-gather): index + top-k and attention of this rank's queries."""
        if self.t1 > self.t0:
            lc_csa_index_topk_prefill(self.a_index_topk, stream)
            lc_csa_sparse_attn_prefill(self.a_attn, stream)


def local_inputs(inp: Dict[str, object], t0: int, t1: int) -> Dict[str, torch.Tensor]:
    """Rank slice of a whole-sequence prefill input (wl.make_prefill with q_first = 0 and
    n_q = L): the rows of positions [t0, t1)."""
    return {"x": inp["x"][t0:t1].contiguous(), "g": inp["g"][t0:t1].contiguous(),
            "kI_raw": inp["kI_raw"][t0:t1].contiguous(), "q_raw": inp["q_raw"][t0:t1].contiguous(),
            "qI_raw": inp["qI_raw"][t0:t1].contiguous(), "sink": inp["sink"], "w": inp["w"]}


def run_dist(rank_state: CpPrefillRank, comm: DistComm, stream=None) -> None:
    """One context-parallel prefill step of this process's rank: every rank makes the
    same collective calls in the same order."""
    r = rank_state
    r.compress_local(stream)
    n_recv = r.t0 - r.h0
    halo = comm.halo(r.halo_send_rows(), n_recv)
    r.set_halo(halo, stream)
    for name in ("nope", "rope", "kI_codes", "kI_scales"):
        comm.all_gather_rows(r.gathered[name], r.nb)
    r.attend(stream)


def run_local(ranks: Sequence[CpPrefillRank], stream=None) -> None:
    """The same step with every rank in this process (one device), phase by phase."""
    comm = LocalComm(ranks)
    for r in ranks:
        r.compress_local(stream)
    for i, r in enumerate(ranks):
        prev = ranks[i - 1].halo_send_rows() if i > 0 else r.local["x"][:0]
        r.set_halo(prev, stream)
    for name in ("nope", "rope", "kI_codes", "kI_scales"):
        comm.all_gather(name, ranks[0].nb)
    for r in ranks:
        r.attend(stream)
