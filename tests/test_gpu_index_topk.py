"""Fused lightning indexer + top-k (lc_csa_index_topk_*), through the C ABI.

The fused call never writes the score matrix: each indexer CTA selects the top K of its
own key range on chip and, when a query's keys span several CTAs, a merge kernel picks
the final K from the ranges' candidates.  Its selection must be bit-identical to the
oracle's top-k (ties to the lower index) of the scores the separate indexer call
computes on the same inputs.  Cases: ragged decode batches whose keys span many CTAs
(and a few that fit one), top-k 512 and 1024, fewer visible entries than k, no visible
entry, prefill queries whose keys span several CTAs, and rows of tied scores (identical
keys, all-zero queries, a few distinct keys repeated)."""
import numpy as np
import pytest
import torch

from long_context_sparse_softmax_b200 import runner
from long_context_sparse_softmax_b200 import workloads as wl
from oracle import lc_oracle as O

pytestmark = pytest.mark.gpu


def _visible(run):
    s = run.spec
    if s.is_decode:
        return [O.n_visible(L - 1, s.m, run.W_x, n) for L, n in zip(s.seq_lens, run.inp["n_c"])]
    return [O.n_visible(s.q_first + i, s.m, run.W_x, run.inp["n_c"]) for i in range(s.n_q)]


def _check(run):
    """Fused selection (a whole step: the indexer operands are quantised and pooled by
    the step's own kernels) against the oracle's top-k of the separate call's scores."""
    k = run.spec.k
    run.step()
    torch.cuda.synchronize()
    fused = run.idx.cpu().numpy()
    cnt = run.count.cpu().numpy()
    run.index()
    torch.cuda.synchronize()
    assert run.read_status() == 0
    scores = run.scores.cpu().numpy()
    nv = _visible(run)
    for q, n in enumerate(nv):
        exp = O.topk(scores[q, :n].astype(np.float64), k)
        e = -np.ones(k, dtype=np.int64)
        e[:exp.shape[0]] = exp
        assert np.array_equal(fused[q].astype(np.int64), e), f"query {q} (n_vis {n}): fused top-{k} differs"
        assert cnt[q] == exp.shape[0]
    return nv


def _decode(seq_lens, k, seed, edit=None):
    s = wl.shrink(wl.CSA_DECODE, name=f"index_topk_decode_{seed}", seed=seed, seq_lens=tuple(seq_lens), k=k)
    inp = wl.make_decode(s, "cuda")
    if edit:
        edit(inp)
    return runner.Decode(inp, "cuda", fused=True)


def test_fused_decode_ragged_many_ranges():
    run = _decode((131072, 20000, 513, 600, 1, 130, 4096 * 9 + 7, 65536), 512, 81)
    nv = _check(run)
    assert min(nv) == 0 and max(nv) > 4 * 4096  # an empty row and rows spanning several CTAs


def test_fused_decode_topk_1024_long_rows():
    _check(_decode((262144, 100000, 5000, 1030 * 4 + 128), 1024, 82))


def test_fused_decode_identical_keys_take_the_lowest_indices():
    def same_keys(inp):
        for t in inp["kI"].values():
            t[:] = t[0]
    run = _decode((50000, 30000, 7000), 512, 83, same_keys)
    _check(run)
    idx = run.idx.cpu().numpy()
    assert np.array_equal(idx[0], np.arange(512))  # every score equal: the first K entries


def test_fused_decode_zero_queries_tie_everywhere():
    def zero_q(inp):
        inp["qI_raw"].zero_()
    _check(_decode((40000, 9000), 512, 84, zero_q))


def test_fused_decode_few_distinct_keys_tie_at_the_threshold():
    def few_keys(inp):
        for t in inp["kI"].values():
            n = t.shape[0]
            pick = torch.arange(n, device=t.device) % 7
            t[:] = t[pick]
    _check(_decode((60000, 33333, 4096 * 3), 1024, 85, few_keys))


def test_fused_prefill_queries_spanning_several_ranges():
    s = wl.shrink(wl.CSA_PREFILL, name="index_topk_prefill", seed=86, seq_lens=(20000,), H=16, k=1024,
                  q_first=20000 - 200, n_q=200)
    run = runner.Prefill(wl.make_prefill(s, "cuda"), "cuda", fused=True)
    _check(run)
    s2 = wl.shrink(wl.CSA_PREFILL, name="index_topk_prefill_early", seed=87, seq_lens=(3000,), H=16, k=256,
                   q_first=0, n_q=3000)
    _check(runner.Prefill(wl.make_prefill(s2, "cuda"), "cuda", fused=True))


def test_indexer_quantises_queries_like_the_quantiser():
    """The MXFP4 indexer call quantises its BF16 queries itself (LC_IDX_MXFP4_QBF16): its
    scores must be bit-identical to those of the same call fed the standalone quantiser's
    codes and scales (LC_IDX_MXFP4), in decode and in prefill, including queries that
    quantise to zero blocks and to saturated codes."""
    import long_context_sparse_softmax_b200 as lc

    def both(run, decode, n_q, width):
        run.step()     # every operand the indexer reads (prefill: its compressed keys)
        run.quant_q()  # the standalone quantiser's codes and scales, into run.qI
        torch.cuda.synchronize()
        outs = []
        for fmt in (lc.LC_IDX_MXFP4_QBF16, lc.LC_IDX_MXFP4):
            a = type(run.a_index).from_buffer_copy(run.a_index)
            a.fmt, a.pdl = fmt, 0
            if fmt == lc.LC_IDX_MXFP4_QBF16:
                a.q, a.q_scale = run.inp["qI_raw"].data_ptr(), None
            else:
                a.q, a.q_scale = run.qI["codes"].data_ptr(), run.qI["scales"].data_ptr()
            sc = torch.full_like(run.scores, float("nan"))
            a.scores = sc.data_ptr()
            (lc.lc_csa_index_scores_decode if decode else lc.lc_csa_index_scores_prefill)(a, None)
            outs.append(sc)
        torch.cuda.synchronize()
        assert run.read_status() == 0
        for q in range(n_q):
            n = width(q)
            assert torch.equal(outs[0][q, :n], outs[1][q, :n]), f"query {q}: in-call quantisation differs"

    def spiky(inp):
        # BF16 bits (int16): edit through float32 and back, truncating to BF16
        x = inp["qI_raw"]
        f = (x.to(torch.int32) << 16).view(torch.float32)
        f[0, 0, :32] = 0.0              # a zero block
        f[0, 1, 5] *= 4000.0            # a block whose other values round to 0
        f[1, 2, :] *= 1e-3
        x.copy_((f.view(torch.int32) >> 16).to(torch.int16))

    s = wl.shrink(wl.CSA_DECODE, name="qbf16_decode", seed=88, seq_lens=(9000, 20000, 513), k=256)
    inp = wl.make_decode(s, "cuda")
    spiky(inp)
    run = runner.Decode(inp, "cuda", fused=False)
    nv = _visible(run)
    both(run, True, len(nv), lambda q: nv[q])
    sp = wl.shrink(wl.CSA_PREFILL, name="qbf16_prefill", seed=89, seq_lens=(3000,), H=16, k=256, q_first=0,
                   n_q=700)
    runp = runner.Prefill(wl.make_prefill(sp, "cuda"), "cuda", fused=False)
    nvp = _visible(runp)
    both(runp, False, len(nvp), lambda q: nvp[q])
