"""Pins of the oracle's method steps against things other than itself: torch library
routines (rms_norm, scaled_dot_product_attention, stable sort), closed forms, brute
force on tiny inputs, and the invariants the method must satisfy."""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import lc_oracle as O
from oracle import pipeline as P
from long_context_sparse_softmax_b200 import workloads as wl

RNG = np.random.default_rng(1234)


# ------------------------------------------------------------------ RMSNorm / RoPE
def test_rms_norm_matches_torch():
    x = RNG.standard_normal((7, 3, 576))
    ref = F.rms_norm(torch.tensor(x), (576,), eps=O.RMS_EPS).numpy()
    np.testing.assert_allclose(O.rms_norm(x), ref, rtol=1e-14, atol=0)


def test_rms_norm_bound_keeps_fp8_in_range():
    """|y_d| <= sqrt(D) after RMSNorm (one coordinate carries all the energy at most),
    so the E4M3 cast of a normalised 576-dim row never saturates (sqrt(576) = 24 < 448)."""
    x = np.zeros((1, 576))
    x[0, 5] = 1e4
    y = O.rms_norm(x)
    assert np.max(np.abs(y)) <= np.sqrt(576) + 1e-9
    y2 = O.rms_norm(RNG.standard_normal((100, 576)) * 50)
    assert np.max(np.abs(y2)) <= np.sqrt(576)


def test_rope_preserves_norm_and_leaves_other_dims():
    y = RNG.standard_normal((5, 576))
    pos = np.array([0, 1, 1000, 131071, 1048575])
    r = O.rope(y, pos, 512, 64)
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(y, axis=1), rtol=1e-13)
    assert np.array_equal(r[:, :512], y[:, :512])
    assert np.array_equal(O.rope(y, np.zeros(5), 512, 64), y)


def test_rope_first_pair_closed_form():
    """Pair 0 has frequency base^0 = 1: it turns by exactly `pos` radians; pair i by
    pos * 10000^(-2i/d_r)."""
    y = np.zeros((1, 128))
    y[0, 0] = 1.0
    y[0, 2 * 5] = 1.0
    p = 7.0
    r = O.rope(y, np.array([p]), 0, 64)
    assert np.allclose(r[0, 0:2], [np.cos(p), np.sin(p)], atol=1e-15)
    f5 = 10000.0 ** (-2 * 5 / 64)
    assert np.allclose(r[0, 10:12], [np.cos(p * f5), np.sin(p * f5)], atol=1e-15)


def test_rope_relative_position():
    """<RoPE(q, p1), RoPE(k, p2)> depends only on p1 - p2."""
    q = RNG.standard_normal(64)
    k = RNG.standard_normal(64)
    a = O.rope(q[None], np.array([1000]), 0, 64) @ O.rope(k[None], np.array([900]), 0, 64).T
    b = O.rope(q[None], np.array([100]), 0, 64) @ O.rope(k[None], np.array([0]), 0, 64).T
    np.testing.assert_allclose(a, b, rtol=1e-9)


# ------------------------------------------------------------------ compression
def test_equal_gates_give_mean_pooling():
    x = RNG.standard_normal((4, 576))
    np.testing.assert_allclose(O.pool_block(x, np.full(4, 0.3)), x.mean(0), rtol=1e-13)


def test_dominant_gate_selects_its_token():
    x = RNG.standard_normal((128, 64))
    g = np.full(128, -40.0)
    g[77] = 40.0
    np.testing.assert_allclose(O.pool_block(x, g), x[77], rtol=1e-12, atol=1e-30)


def test_gate_weights_closed_form():
    x = np.eye(4)
    g = np.array([0.0, np.log(2.0), np.log(3.0), np.log(4.0)])
    np.testing.assert_allclose(O.pool_block(x, g), np.array([1, 2, 3, 4]) / 10.0, rtol=1e-14)


def test_pooling_comes_before_rmsnorm():
    """The entry is RMSNorm of the gated pool, not the pool of normalised tokens: two
    tokens of different norms with equal gates (closed form, no RoPE dims).  With
    x1 = 2 e0 and x2 = 6 e1 the pool is e0 + 3 e1, whose RMS over D dims is sqrt(10 / D);
    normalising each token first would give equal weights on e0 and e1 instead."""
    D = 64
    x = np.zeros((2, D))
    x[0, 0] = 2.0
    x[1, 1] = 6.0
    e = O.compress(x, np.zeros(2), 2, 0, 0)
    r = np.sqrt(10.0 / D + O.RMS_EPS)
    expect = np.zeros(D)
    expect[0], expect[1] = 1.0 / r, 3.0 / r
    np.testing.assert_allclose(e[0], expect, rtol=1e-14, atol=0)
    assert abs(e[0, 1] / e[0, 0] - 3.0) < 1e-12


def test_block_entry_is_roped_at_its_last_position():
    """A block of identical tokens pools to that token; its entry equals the token
    prepared at position (j+1)m - 1."""
    m, j = 4, 9
    t = RNG.standard_normal(576)
    x = np.tile(t, (m * (j + 1), 1))
    g = RNG.standard_normal(m * (j + 1))
    e = O.compress(x, g, m, 512, 64)
    np.testing.assert_allclose(e[j], O.qk_prep(t[None], np.array([(j + 1) * m - 1]), 512, 64)[0], rtol=1e-12)


def test_m1_compression_equals_window_preparation():
    """m = 1: every token is its own block, so compression equals RMSNorm + RoPE of the
    token at its own position (the window-row preparation)."""
    x = RNG.standard_normal((50, 128))
    g = RNG.standard_normal(50)
    np.testing.assert_allclose(O.compress(x, g, 1, 0, 64), O.qk_prep(x, np.arange(50), 0, 64), rtol=1e-13)


def test_only_complete_blocks_are_compressed():
    x = RNG.standard_normal((4 * 5 + 3, 64))
    e = O.compress(x, RNG.standard_normal(23), 4, 0, 32)
    assert e.shape[0] == 5


# ------------------------------------------------------------------ visibility
@pytest.mark.parametrize("m,W", [(4, 128), (128, 128), (4, 0), (1, 16)])
def test_n_visible_brute_force(m, W):
    for p in list(range(0, 600)) + [131071, 1048575]:
        for n_ent in (5, 10**6):
            brute = sum(1 for j in range(min(n_ent, p // m + 2)) if (j + 1) * m - 1 <= p - W)
            assert O.n_visible(p, m, W, n_ent) == brute


def test_tiny_config_visibility_numbers():
    """L = 1024, m = 4, W = 128: the last query sees 224 entries; the first entry
    becomes visible at p = 131."""
    assert O.n_visible(1023, 4, 128, 256) == 224
    assert O.n_visible(130, 4, 128, 256) == 0
    assert O.n_visible(131, 4, 128, 256) == 1


# ------------------------------------------------------------------ indexer
def test_index_scores_brute_force():
    H_I, d_I, n = 3, 8, 11
    q = RNG.standard_normal((H_I, d_I))
    k = RNG.standard_normal((n, d_I))
    w = RNG.random(H_I)
    s = O.index_scores(q, k, w)
    for j in range(n):
        tot = 0.0
        for h in range(H_I):
            dot = 0.0
            for i in range(d_I):
                dot += q[h, i] * k[j, i]
            tot += w[h] * (dot if dot > 0 else 0.0)
        assert abs(s[j] - tot) <= 1e-12 * (1 + abs(tot))


def test_index_single_head_unit_weight_is_relu_dot():
    q = RNG.standard_normal((1, 64))
    k = RNG.standard_normal((40, 64))
    np.testing.assert_allclose(O.index_scores(q, k, np.ones(1)), np.maximum(k @ q[0], 0), rtol=1e-14)


def test_index_nonnegative_weights_commute_with_relu():
    """w >= 0 => w * ReLU(x) = ReLU(w * x)."""
    q = RNG.standard_normal((4, 16))
    k = RNG.standard_normal((9, 16))
    w = RNG.random(4)
    alt = np.maximum((k @ q.T) * w, 0).sum(1)
    np.testing.assert_allclose(O.index_scores(q, k, w), alt, rtol=1e-13)


def test_score_error_bound_covers_fp32_evaluation():
    q = RNG.standard_normal((64, 128)).astype(np.float32)
    k = RNG.standard_normal((500, 128)).astype(np.float32)
    w = RNG.random(64).astype(np.float32)
    exact = O.index_scores(q.astype(np.float64), k.astype(np.float64), w.astype(np.float64))
    f32 = (np.maximum(k @ q.T, np.float32(0)) @ w).astype(np.float64)
    bound = O.score_error_bound(q.astype(np.float64), k.astype(np.float64), w.astype(np.float64))
    assert np.all(np.abs(f32 - exact) <= bound)


# ------------------------------------------------------------------ top-k
@pytest.mark.parametrize("k", [1, 5, 64, 200])
def test_topk_matches_stable_sorts(k):
    s = RNG.integers(0, 12, 150).astype(np.float64)   # many ties
    got = O.topk(s, k)
    _, order = torch.sort(-torch.tensor(s), stable=True)
    ref = np.sort(order.numpy()[:min(k, 150)])
    assert np.array_equal(got, ref)
    ref2 = np.sort(np.argsort(-s, kind="stable")[:min(k, 150)])
    assert np.array_equal(got, ref2)


def test_topk_takes_all_when_k_exceeds_visible():
    s = RNG.standard_normal(10)
    assert np.array_equal(O.topk(s, 64), np.arange(10))
    assert O.topk(np.zeros(0), 8).shape == (0,)


def test_topk_ties_go_to_lower_index():
    s = np.zeros(100)
    assert np.array_equal(O.topk(s, 7), np.arange(7))
    s[[3, 50, 90]] = 1.0
    assert np.array_equal(O.topk(s, 4), [0, 3, 50, 90])


# ------------------------------------------------------------------ attention
def _sdpa_with_sink(q, keys, sink, scale):
    """torch SDPA (float64) with the sink as an extra key whose value is zero and whose
    logit is supplied through the additive mask."""
    H, D = q.shape
    n = keys.shape[0]
    K = torch.cat([torch.zeros(1, D, dtype=torch.float64), torch.tensor(keys)], 0)
    mask = torch.zeros(H, 1, n + 1, dtype=torch.float64)
    mask[:, 0, 0] = torch.tensor(sink)
    Qt = torch.tensor(q)[:, None, :]
    o = F.scaled_dot_product_attention(Qt, K.expand(H, n + 1, D), K.expand(H, n + 1, D),
                                       attn_mask=mask, scale=scale)
    logits = scale * (torch.tensor(q) @ torch.tensor(keys).T)
    lse = torch.logsumexp(torch.cat([torch.tensor(sink)[:, None], logits], 1), 1)
    return o[:, 0].numpy(), lse.numpy()


def test_attend_matches_sdpa_with_sink():
    H, D, n = 8, 128, 37
    q = RNG.standard_normal((H, D)) * 3
    keys = RNG.standard_normal((n, D))
    sink = RNG.standard_normal(H)
    o, lse = O.attend(q, keys, sink, 1 / np.sqrt(D))
    ro, rl = _sdpa_with_sink(q, keys, sink, 1 / np.sqrt(D))
    np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, rl, rtol=1e-13)


def test_softmax_weights_with_sink_sum_to_one():
    H, D, n = 4, 64, 20
    q = RNG.standard_normal((H, D)) * 5
    keys = RNG.standard_normal((n, D))
    sink = RNG.standard_normal(H) * 3
    _, lse = O.attend(q, keys, sink, 0.125)
    tot = np.exp(sink - lse) + np.exp(0.125 * (q @ keys.T) - lse[:, None]).sum(1)
    np.testing.assert_allclose(tot, 1.0, rtol=1e-14)


def test_one_key_plus_sink_closed_form():
    """o = sigmoid(l - sink) * v for a single key."""
    q = RNG.standard_normal((3, 16))
    v = RNG.standard_normal((1, 16))
    sink = RNG.standard_normal(3)
    o, _ = O.attend(q, v, sink, 0.25)
    l = 0.25 * (q @ v[0])
    np.testing.assert_allclose(o, (1 / (1 + np.exp(-(l - sink))))[:, None] * v, rtol=1e-13)


def test_no_keys_gives_zero_output_and_sink_lse():
    o, lse = O.attend(np.ones((2, 4)), np.zeros((0, 4)), np.array([0.5, -1.0]), 1.0)
    assert np.all(o == 0) and np.array_equal(lse, [0.5, -1.0])


def _tiny_prefill(L=96, D=32, d_r=16, H=4, m=4, W=16, seed=5):
    r = np.random.default_rng(seed)
    return dict(x=r.standard_normal((L, D)), g=r.standard_normal(L), q=r.standard_normal((L, H, D)),
                sink=r.standard_normal(H), L=L, D=D, d_r=d_r, H=H, m=m, W=W)


def _csa_query(t, p, k, m=None, W=None, W_x=None, qI=None, kI=None, w=None):
    m = t["m"] if m is None else m
    W = t["W"] if W is None else W
    W_x = W if W_x is None else W_x
    ent = O.compress(t["x"], t["g"], m, 0, t["d_r"])
    win = O.qk_prep(t["x"], np.arange(t["L"]), 0, t["d_r"])
    q = O.qk_prep(t["q"][p:p + 1], np.array([p]), 0, t["d_r"])[0]
    n_vis = O.n_visible(p, m, W_x, ent.shape[0])
    if qI is None:
        idx = np.arange(min(n_vis, k))
    else:
        idx = O.topk(O.index_scores(qI[p], kI[:n_vis], w), k)
    return O.sparse_attn_query(q, ent, idx, win, 0, p, W, t["sink"], 1 / np.sqrt(t["D"]))


def test_m1_full_topk_is_full_causal_attention_with_sink():
    """m = 1 and k >= p + 1: compressed entries are the prepared tokens before the window
    and the window holds the rest, so CSA is full causal attention plus the sink."""
    t = _tiny_prefill()
    win = O.qk_prep(t["x"], np.arange(t["L"]), 0, t["d_r"])
    for p in (0, 5, 16, 17, 50, 95):
        o, lse = _csa_query(t, p, k=10**6, m=1)
        q = O.qk_prep(t["q"][p:p + 1], np.array([p]), 0, t["d_r"])[0]
        ro, rl = _sdpa_with_sink(q, win[:p + 1], t["sink"], 1 / np.sqrt(t["D"]))
        np.testing.assert_allclose(o, ro, rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(lse, rl, rtol=1e-12)


def test_large_k_csa_equals_hca_style_dense():
    """k >= number of visible entries: CSA equals dense attention over the visible
    compressed entries plus the window (what HCA computes)."""
    t = _tiny_prefill(seed=6)
    r = np.random.default_rng(8)
    qI = r.standard_normal((t["L"], 2, 8))
    kI = r.standard_normal((t["L"] // t["m"], 8))
    w = r.random(2)
    ent = O.compress(t["x"], t["g"], t["m"], 0, t["d_r"])
    win = O.qk_prep(t["x"], np.arange(t["L"]), 0, t["d_r"])
    for p in (20, 40, 95):
        o, lse = _csa_query(t, p, k=1000, qI=qI, kI=kI, w=w)
        q = O.qk_prep(t["q"][p:p + 1], np.array([p]), 0, t["d_r"])[0]
        n_vis = O.n_visible(p, t["m"], t["W"], ent.shape[0])
        ho, hl = O.hca_attn_query(q, ent, n_vis, win, 0, p, t["W"], t["sink"], 1 / np.sqrt(t["D"]))
        np.testing.assert_allclose(o, ho, rtol=1e-13)
        np.testing.assert_allclose(lse, hl, rtol=1e-13)


def test_causality_future_tokens_and_open_blocks_do_not_matter():
    t = _tiny_prefill(seed=9)
    p = 61  # block 15 (tokens 60..63) is still open at p = 61
    o1, l1 = _csa_query(t, p, k=8)
    t2 = dict(t)
    t2["x"] = t["x"].copy()
    t2["g"] = t["g"].copy()
    t2["x"][p + 1:] = np.random.default_rng(1).standard_normal(t["x"][p + 1:].shape)
    t2["g"][p + 1:] = 100.0
    o2, l2 = _csa_query(t2, p, k=8)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=0)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=0)


def test_causality_is_violated_by_a_visible_change():
    """Control for the test above: changing a token the query does see changes o."""
    t = _tiny_prefill(seed=9)
    p = 61
    o1, _ = _csa_query(t, p, k=8)
    t2 = dict(t)
    t2["x"] = t["x"].copy()
    t2["x"][p] += 1.0
    o2, _ = _csa_query(t2, p, k=8)
    assert np.max(np.abs(o1 - o2)) > 1e-3


def test_overlap_and_disjoint_readings_coincide_without_window():
    t = _tiny_prefill(seed=10)
    for p in (3, 30, 95):
        a = _csa_query(t, p, k=1000, W=0, W_x=0)
        b = _csa_query(t, p, k=1000, W=0)
        np.testing.assert_allclose(a[0], b[0])


def test_window_and_entries_are_disjoint_under_default_reading():
    """Under the default reading no token reaches the query through both paths: every
    visible entry ends before the window starts."""
    for m in (4, 128):
        for p in range(0, 2000, 7):
            n_vis = O.n_visible(p, m, 128, 10**6)
            if n_vis:
                assert n_vis * m - 1 < max(0, p - 128 + 1)


# ------------------------------------------------------------------ pages' shapes
def test_workload_shapes_follow_the_pages():
    gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "v4_attention_shapes.json")))
    assert wl.CSA_DECODE.m == gold["csa_m"] and wl.CSA_PREFILL.m == gold["csa_m"]
    assert wl.HCA_PREFILL.m == gold["hca_m"] and wl.MIXED_HCA.m == gold["hca_m"]
    assert wl.CSA_DECODE.k == gold["topk_flash"] and wl.CSA_PREFILL.k == gold["topk_pro"]
    for s in (wl.TINY_CSA_PREFILL, wl.CSA_DECODE, wl.HCA_PREFILL, wl.CSA_PREFILL, wl.MIXED_CSA):
        assert s.W == gold["window"]
    assert wl.HCA_PREFILL.seq_lens[0] // wl.HCA_PREFILL.m == 8192


def test_mixed_lengths_are_in_range():
    assert len(wl.MIXED_CSA.seq_lens) == 8
    assert all(524288 <= L <= 1048576 for L in wl.MIXED_CSA.seq_lens)


# ------------------------------------------------------------------ decode-time cache maintenance
def test_index_key_pooling_closed_forms():
    """Indexer keys use the entries' gate: equal gates give the mean, a dominant gate its
    token, weights e^g / sum e^g in closed form; no normalisation or rotation."""
    k = RNG.standard_normal((8, 128))
    np.testing.assert_allclose(O.pool_index_keys(k, np.zeros(8), 4), [k[:4].mean(0), k[4:].mean(0)], rtol=1e-13)
    g = np.array([0.0, np.log(2.0), np.log(3.0), np.log(4.0)])
    np.testing.assert_allclose(O.pool_index_keys(np.eye(4), g, 4)[0], np.array([1, 2, 3, 4]) / 10.0, rtol=1e-14)
    g2 = np.full(8, -50.0)
    g2[6] = 50.0
    np.testing.assert_allclose(O.pool_index_keys(k, g2, 4, first_block=1, tok_pos0=0, n_blocks=1)[0], k[6],
                               rtol=1e-12, atol=1e-30)


@pytest.mark.parametrize("R,W", [(128, 128), (192, 128), (16, 16)])
def test_window_ring_equals_the_linear_window(R, W):
    """Rows appended one position at a time into slot pos mod R give, for every query
    position, the same window rows as the linear history."""
    n = 3 * R + 5
    rows = RNG.standard_normal((n, 8))
    ring = np.zeros((R, 8))
    for p in range(n):
        ring[O.ring_slot(p, R)] = rows[p]
        got = O.window_from_ring(ring, p, W)
        assert np.array_equal(got, rows[max(0, p - W + 1):p + 1])


# ------------------------------------------------------------------ values without the RoPE dims
def test_nope_values_match_sdpa_and_the_full_value_output():
    """V = the non-RoPE dims: torch SDPA with those value columns, and exactly the non-RoPE
    columns of the full-V output (same weights)."""
    H, D, n, lo, d_r = 8, 128, 41, 64, 64
    q = RNG.standard_normal((H, D)) * 2
    keys = RNG.standard_normal((n, D))
    sink = RNG.standard_normal(H)
    vd = O.nope_dims(D, lo, d_r)
    assert np.array_equal(vd, np.arange(64))
    o, lse = O.attend(q, keys, sink, 1 / np.sqrt(D), vd)
    full, lse_f = O.attend(q, keys, sink, 1 / np.sqrt(D))
    np.testing.assert_allclose(o, full[:, vd], rtol=1e-13, atol=1e-15)
    assert np.array_equal(lse, lse_f)
    K = torch.cat([torch.zeros(1, D, dtype=torch.float64), torch.tensor(keys)], 0)
    V = K[:, torch.tensor(vd)]
    mask = torch.zeros(H, 1, n + 1, dtype=torch.float64)
    mask[:, 0, 0] = torch.tensor(sink)
    ref = F.scaled_dot_product_attention(torch.tensor(q)[:, None, :], K.expand(H, n + 1, D),
                                         V.expand(H, n + 1, len(vd)), attn_mask=mask, scale=1 / np.sqrt(D))
    np.testing.assert_allclose(o, ref[:, 0].numpy(), rtol=1e-12, atol=1e-14)
    # RoPE dims first in the row (the FP32 layout): the value dims are the rest
    assert np.array_equal(O.nope_dims(128, 0, 64), np.arange(64, 128))


# ------------------------------------------------------------------ grouped output projection
def test_grouped_projection_is_a_block_diagonal_dense_projection():
    """Grouped projection = the dense projection of the concatenated head outputs by the
    block-diagonal matrix of the groups' weights (scipy's block_diag, numpy matmul)."""
    from scipy.linalg import block_diag
    n, H, Dv, G, d_g = 5, 8, 6, 4, 3
    o = RNG.standard_normal((n, H, Dv))
    w = RNG.standard_normal((G, (H // G) * Dv, d_g))
    ref = o.reshape(n, H * Dv) @ block_diag(*w)
    np.testing.assert_allclose(O.grouped_out_proj(o, w), ref, rtol=1e-13, atol=1e-13)
    # one group is the dense projection
    w1 = RNG.standard_normal((1, H * Dv, 7))
    np.testing.assert_allclose(O.grouped_out_proj(o, w1), o.reshape(n, -1) @ w1[0], rtol=1e-13)
