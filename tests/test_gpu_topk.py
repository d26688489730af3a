"""Top-k on crafted score rows, through the C ABI, bit-exact against the oracle.

The kernel finds the K-th largest key by radix passes.  When few keys share the bin the
first pass selects, every CTA of the row's cluster gathers them and finishes alone;
otherwise the cluster-wide passes continue.  The rows here drive both paths:
  * spread scores: the first bin holds a few dozen keys (gathered path);
  * a dense band plus outliers: the band fills one first-pass bin (cluster-wide passes);
  * a handful of distinct values: long runs of ties at the threshold (ties go to the
    lower index);
  * a constant row: no pass at all;
  * ragged rows, including rows with fewer visible scores than k.
Every row is checked for the exact index list and the count."""
import numpy as np
import pytest
import torch

import long_context_sparse_softmax_b200 as lc
from oracle import lc_oracle as O

pytestmark = pytest.mark.gpu

M, W_X = 4, 128


def _rows(kind: str, n: int, rng: np.random.Generator) -> np.ndarray:
    if kind == "spread":
        return (rng.standard_normal(n) * 10.0).astype(np.float32)
    if kind == "band":
        s = (5.0 + rng.random(n) * 1e-4).astype(np.float32)  # one first-pass bin
        n_out = min(40, n // 2)
        s[rng.choice(n, n_out, replace=False)] = 100.0 + rng.random(n_out).astype(np.float32)
        return s
    if kind == "ties":
        return (np.round(rng.standard_normal(n) * 3.0) / 4.0).astype(np.float32)
    if kind == "const":
        return np.full(n, 1.5, dtype=np.float32)
    raise ValueError(kind)


def _run(rows, k: int):
    """Rows of visible scores (one decode sequence each) -> (indices [B, k], counts [B])."""
    B = len(rows)
    n_ent = [len(r) for r in rows]
    stride = (max(max(n_ent), 1) + 3) // 4 * 4
    dev = "cuda"
    scores = torch.full((B, stride), float("nan"), dtype=torch.float32)
    for b, r in enumerate(rows):
        scores[b, :len(r)] = torch.from_numpy(r)
    scores = scores.to(dev)
    i32 = dict(dtype=torch.int32, device=dev)
    i64 = dict(dtype=torch.int64, device=dev)
    q_start = torch.arange(B + 1, **i32)
    # the query of sequence b sits far enough past its last entry to see all of them
    q_pos0 = torch.tensor([M * n + W_X for n in n_ent], **i32)
    ent_start = torch.zeros(B, **i64)
    n_ent_t = torch.tensor(n_ent, **i32)
    idx = torch.empty(B, k, **i32)
    count = torch.empty(B, **i32)
    status = torch.zeros(1, **i32)
    batch = lc.Batch(B, 0, q_start.data_ptr(), q_pos0.data_ptr(), ent_start.data_ptr(), n_ent_t.data_ptr(),
                     None, None, None)
    a = lc.TopkArgs(B, k, M, W_X, max(n_ent), 0, scores.data_ptr(), stride, batch, idx.data_ptr(),
                    count.data_ptr(), status.data_ptr())
    lc.lc_csa_topk_decode(a, None)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return idx.cpu().numpy(), count.cpu().numpy()


def _check(rows, k: int):
    got, cnt = _run(rows, k)
    for b, r in enumerate(rows):
        exp = O.topk(r.astype(np.float64), k)
        e = -np.ones(k, dtype=np.int64)
        e[:exp.shape[0]] = exp
        assert np.array_equal(got[b].astype(np.int64), e), f"row {b}: top-{k} differs"
        assert cnt[b] == exp.shape[0]


@pytest.mark.parametrize("B", [8, 32])
@pytest.mark.parametrize("kind", ["spread", "band", "ties", "const"])
def test_topk_row_kinds(kind, B):
    """8 rows give clusters of 8 CTAs, 32 rows clusters of 4."""
    rng = np.random.default_rng(7 + B)
    _check([_rows(kind, 32736, rng) for _ in range(B)], 512)


def test_topk_mixed_and_ragged_rows():
    rng = np.random.default_rng(11)
    kinds = ["spread", "band", "ties", "const"]
    lens = [32736, 20001, 513, 300, 7, 1, 65536, 4099]
    rows = [_rows(kinds[i % 4], n, rng) for i, n in enumerate(lens)]
    _check(rows, 512)
    _check(rows, 1024)


def test_topk_signed_zeros_tie_by_index():
    """-0.0 and +0.0 compare equal: at the threshold they are ties, taken by lower index
    whatever their sign bits."""
    rng = np.random.default_rng(13)
    n = 5000
    r = np.zeros(n, dtype=np.float32)
    r[rng.random(n) < 0.5] = np.float32(-0.0)
    pos = rng.choice(n, 200, replace=False)
    r[pos] = np.abs(rng.standard_normal(200)).astype(np.float32) + 0.5
    neg = rng.choice(np.setdiff1d(np.arange(n), pos), 300, replace=False)
    r[neg] = -np.abs(rng.standard_normal(300)).astype(np.float32) - 0.5
    assert np.signbit(r[r == 0]).any() and (~np.signbit(r[r == 0])).any()
    _check([r, r[::-1].copy()], 512)
