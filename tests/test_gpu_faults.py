"""Device-side failure paths, made on the host (no GPU fault, trap or hang is involved).

* Bad selections: a top-k index past the sequence's entries (pointing, in the buffer, at
  the next sequence's rows, so even a missing check would read valid memory), an index of
  an entry the query cannot see yet, and window rows the caller did not provide.  The
  attention skips those keys, reports LC_DEV_BAD_INDEX, LC_DEV_NONVISIBLE and
  LC_DEV_WINDOW_RANGE, and its output equals the oracle's over the remaining keys.
* A bounded wait that runs out: the indexer called with a spin limit of one poll gives up
  at its first wait, reports LC_DEV_TIMEOUT, drains its bulk copies and MMAs, and
  returns; the same call with the default limit then gives the usual scores (the context
  is still usable)."""
import numpy as np
import pytest
import torch

import long_context_sparse_softmax_b200 as lc
from long_context_sparse_softmax_b200 import runner
from long_context_sparse_softmax_b200 import workloads as wl
from oracle import lc_oracle as O
from tests.oracle_ref import OracleDecode, attn_ok, np_, out_np, rows_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("impl", [2, 3], ids=["tcgen05", "reference"])
def test_bad_indices_and_missing_window_rows_are_skipped_and_reported(impl):
    s = wl.shrink(wl.CSA_DECODE, name="faults", seed=91, seq_lens=(3000, 2051, 4096, 1500), k=64)
    inp = wl.make_decode(s, "cuda")
    run = runner.Decode(inp, "cuda", impl=impl)
    run.step()
    torch.cuda.synchronize()
    assert run.read_status() == 0
    orc = OracleDecode(inp)
    idx = np_(run.idx).copy()
    n_c = inp["n_c"]
    pos = [L - 1 for L in s.seq_lens]
    nv = [O.n_visible(p, s.m, s.W, n) for p, n in zip(pos, n_c)]
    # sequence 0: an index past its entries (inside sequence 1's rows of the buffer)
    idx[0, 3] = n_c[0] + 5
    # sequence 1: an entry not visible yet (in the window's span)
    idx[1, 7] = nv[1] + 2
    assert nv[1] + 2 < n_c[1]
    run.idx.copy_(torch.from_numpy(idx))
    # sequence 2: the last 5 window positions (the newest tokens) are missing
    win_len = np_(inp["batch"]["win_len"]).copy()
    win_len[2] -= 5
    inp["batch"]["win_len"].copy_(torch.from_numpy(win_len))
    run.status.zero_()
    run.attn()
    torch.cuda.synchronize()
    st = run.read_status()
    assert st & lc.LC_DEV_BAD_INDEX and st & lc.LC_DEV_NONVISIBLE and st & lc.LC_DEV_WINDOW_RANGE
    assert not st & lc.LC_DEV_TIMEOUT
    got = out_np(run, range(s.num_seqs))
    # the oracle over the remaining keys, on the library's own prepared rows
    lib_q = rows_np(s.q_fmt, run.q).reshape(s.num_seqs, s.H, s.D)
    for b in range(s.num_seqs):
        sel = [int(j) for j in idx[b] if 0 <= j < nv[b]]
        ent = orc.entries(b)
        wr = orc.window_rows(b)
        ts = [t for t in O.window_positions(pos[b], s.W) if t - orc.win_pos0[b] < win_len[b]]
        keys = np.concatenate([ent[sel], wr[[t - orc.win_pos0[b] for t in ts]]], 0)
        o, _ = O.attend(lib_q[b], keys, orc.sink, s.scale)
        ok, err, tol = attn_ok(got[b], o, False)
        assert ok, f"sequence {b}: err {err} > tol {tol}"


@pytest.mark.parametrize("fused", [False, True], ids=["scores", "fused_topk"])
def test_indexer_wait_limit_runs_out_cleanly(fused):
    s = wl.shrink(wl.CSA_DECODE, name="timeout", seed=92, seq_lens=(20000, 9000, 33000), k=256)
    run = runner.Decode(wl.make_decode(s, "cuda"), "cuda", fused=fused)
    run.step()
    run.index()
    torch.cuda.synchronize()
    assert run.read_status() == 0
    scores, idx = run.scores.clone(), run.idx.clone()
    args = run.a_index_topk.index if fused else run.a_index
    for attempt in range(3):
        args.spin_limit = 1
        run.status.zero_()
        run.scores.fill_(float("nan"))
        run.index_topk() if fused else run.index()
        torch.cuda.synchronize()
        assert run.read_status() & lc.LC_DEV_TIMEOUT, "a one-poll wait limit must run out"
        args.spin_limit = 0
        run.status.zero_()
        run.index_topk() if fused else run.index()
        torch.cuda.synchronize()
        assert run.read_status() == 0
        if fused:
            assert torch.equal(run.idx, idx)
        else:
            for b, L in enumerate(s.seq_lens):  # the visible columns (the rest is never written)
                n = O.n_visible(L - 1, s.m, s.W, L // s.m)
                assert torch.equal(run.scores[b, :n], scores[b, :n])
