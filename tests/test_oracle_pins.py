"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks the oracle against something the model-doc page fixes (its worked mask example),
a closed form, an invariant, or a textbook/library routine (torch's fp64 scaled-dot-product
attention, numpy sorting and means). They are chosen so that a plausible slip (a wrong pair
layout or frequency in RoPE, a window off by one, a missing sink term, a forward rotation of the
output instead of the inverse, a wrong sign of the indexer head weights) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import OracleParams

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mask_layout_example.json")
NEG = -1e300  # a sink this low contributes exp(-inf) = 0 to the normaliser


def rng(seed):
    return np.random.default_rng(seed)


def sdpa_explicit(qrot, keys, scale):
    """Plain softmax attention of one query over an explicit key list (K = V), via torch's
    fp64 scaled_dot_product_attention. qrot [H,D], keys [nk,D] -> [H,D]."""
    H, D = qrot.shape
    q = torch.from_numpy(qrot).reshape(1, H, 1, D)
    k = torch.from_numpy(keys).reshape(1, 1, -1, D).expand(1, H, -1, D)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, k, scale=scale)
    return o.reshape(H, D).numpy()


# ------------------------------------------------------------------------------------------------
# RoPE
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("i", [0, 1, 5, 7])
def test_rope_closed_form_one_hot(i):
    D, R, theta, pos = 48, 16, 10000.0, 37.0
    x = np.zeros(D)
    x[D - R + 2 * i] = 1.0
    y = oracle.rope(x, R, theta, pos)
    phi = pos * theta ** (-2.0 * i / R)
    expect = np.zeros(D)
    expect[D - R + 2 * i] = math.cos(phi)
    expect[D - R + 2 * i + 1] = math.sin(phi)
    np.testing.assert_allclose(y, expect, atol=1e-14)
    # second member of the pair turns towards -sin
    x = np.zeros(D)
    x[D - R + 2 * i + 1] = 1.0
    y = oracle.rope(x, R, theta, pos)
    assert abs(y[D - R + 2 * i] + math.sin(phi)) < 1e-14
    assert abs(y[D - R + 2 * i + 1] - math.cos(phi)) < 1e-14


def test_rope_leaves_non_rope_channels_and_preserves_norm():
    r = rng(1)
    x = r.standard_normal(64)
    y = oracle.rope(x, 16, 10000.0, 1234.0)
    np.testing.assert_array_equal(y[:48], x[:48])
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12
    np.testing.assert_allclose(oracle.rope(y, 16, 10000.0, -1234.0), x, atol=1e-12)
    np.testing.assert_array_equal(oracle.rope(x, 0, 10000.0, 99.0), x)


def test_rope_dot_product_depends_on_distance_only():
    r = rng(2)
    a, b = r.standard_normal(32), r.standard_normal(32)
    d1 = oracle.rope(a, 32, 160000.0, 1000.0) @ oracle.rope(b, 32, 160000.0, 990.0)
    d2 = oracle.rope(a, 32, 160000.0, 77.0) @ oracle.rope(b, 32, 160000.0, 67.0)
    assert abs(d1 - d2) < 1e-11


# ------------------------------------------------------------------------------------------------
# Compressor
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("S,m,N", [(16, 8, 2), (17, 4, 4), (3, 4, 0), (256, 4, 64)])
def test_entry_count(S, m, N):
    x = rng(3).standard_normal((1, S, 4))
    assert oracle.compress(x, np.ones(4), np.zeros(2 * m), m, 2 * m).shape == (1, N, 4)


@pytest.mark.parametrize("S,m,N", [(8192, 4, 2048), (32768, 128, 256), (131072, 4, 32768)])
def test_entry_count_of_the_workloads(S, m, N):
    # u = 0 keeps this cheap; only the count matters here
    x = np.zeros((1, S, 1))
    assert oracle.compress(x, np.zeros(1), np.zeros(m if m > 4 else 2 * m), m,
                           m if m > 4 else 2 * m).shape[1] == N


def test_zero_gate_is_window_mean_csa():
    S, m, L, C = 40, 4, 8, 6
    x = rng(4).standard_normal((2, S, C))
    pool = oracle.compress(x, np.zeros(C), np.zeros(L), m, L)
    for b in range(2):
        for w in range(S // m):
            lo, hi = max(0, (w - 1) * m), (w + 1) * m
            np.testing.assert_allclose(pool[b, w], x[b, lo:hi].mean(0), atol=1e-14)


def test_zero_gate_is_window_mean_hca():
    S, m, C = 50, 8, 5
    x = rng(5).standard_normal((1, S, C))
    pool = oracle.compress(x, np.zeros(C), np.zeros(m), m, m)
    for w in range(S // m):
        np.testing.assert_allclose(pool[0, w], x[0, w * m:(w + 1) * m].mean(0), atol=1e-14)


@pytest.mark.parametrize("offset,row_of", [(4, lambda w, m: w * m),
                                           (7, lambda w, m: (w + 1) * m - 1),
                                           (5, lambda w, m: w * m + 1)])
def test_one_hot_bias_selects_one_window_offset_csa(offset, row_of):
    # only one offset has a finite bias: each entry copies the token at that offset of its
    # window; the closing token of entry w's window is (w+1)m - 1 (offset L-1)
    S, m, L, C = 36, 4, 8, 3
    x = rng(6).standard_normal((1, S, C))
    bias = np.full(L, -np.inf)
    bias[offset] = 0.0
    pool = oracle.compress(x, rng(7).standard_normal(C), bias, m, L)
    for w in range(S // m):
        np.testing.assert_allclose(pool[0, w], x[0, row_of(w, m)], atol=1e-14)


def test_one_hot_bias_hca_first_token():
    S, m, C = 32, 8, 3
    x = rng(8).standard_normal((1, S, C))
    bias = np.full(m, -np.inf)
    bias[0] = 0.0
    pool = oracle.compress(x, rng(9).standard_normal(C), bias, m, m)
    for w in range(S // m):
        np.testing.assert_allclose(pool[0, w], x[0, w * m], atol=1e-14)


def test_rate_one_is_identity():
    x = rng(10).standard_normal((1, 9, 4))
    np.testing.assert_allclose(oracle.compress(x, rng(11).standard_normal(4), np.zeros(1), 1, 1),
                               x, atol=1e-14)


def test_pool_is_a_convex_combination():
    S, m, L, C = 24, 4, 8, 5
    c = rng(12).standard_normal(C)
    x = np.tile(c, (1, S, 1))
    pool = oracle.compress(x, rng(13).standard_normal(C), rng(14).standard_normal(L), m, L)
    np.testing.assert_allclose(pool[0], np.tile(c, (S // m, 1)), atol=1e-13)


def test_gate_concentrates_on_the_largest_projection():
    # a large gate along channel 0 puts (almost) all weight on the window's argmax of x[:,0]
    S, m, L, C = 32, 4, 8, 4
    x = rng(15).standard_normal((1, S, C))
    u = np.zeros(C)
    u[0] = 1e4
    pool = oracle.compress(x, u, np.zeros(L), m, L)
    for w in range(S // m):
        lo, hi = max(0, (w - 1) * m), (w + 1) * m
        j = lo + int(np.argmax(x[0, lo:hi, 0]))
        np.testing.assert_allclose(pool[0, w], x[0, j], atol=1e-9)


def test_entry_depends_only_on_its_closed_window():
    S, m, L, C = 32, 4, 8, 4
    r = rng(16)
    x = r.standard_normal((1, S, C))
    u, b = r.standard_normal(C), r.standard_normal(L)
    base = oracle.compress(x, u, b, m, L)
    for w in range(S // m):
        y = x.copy()
        y[0, (w + 1) * m:] += 5.0          # tokens after the window closed
        if (w - 1) * m > 0:
            y[0, :(w - 1) * m] -= 3.0      # tokens before the window opened
        np.testing.assert_allclose(oracle.compress(y, u, b, m, L)[0, w], base[0, w], atol=1e-14)
        y = x.copy()
        y[0, (w + 1) * m - 1] += 1.0       # the closing token is inside
        assert np.abs(oracle.compress(y, u, b, m, L)[0, w] - base[0, w]).max() > 1e-6


# ------------------------------------------------------------------------------------------------
# Indexer score and top-k
# ------------------------------------------------------------------------------------------------
def _ref_rank(scores, nvis, k):
    """Reference ranking with numpy: score descending, lower index first on ties."""
    idx = np.arange(nvis)
    order = np.lexsort((idx, -scores[:nvis]))
    out = np.full(k, -1, dtype=np.int32)
    out[:min(k, nvis)] = order[:k]
    return out


def test_single_head_positive_weight_ranks_by_dot_product():
    r = rng(20)
    N, cI, k = 200, 16, 30
    q = r.standard_normal((1, cI))
    K = r.standard_normal((N, cI))
    s = oracle.index_scores(q, np.array([1.0]), K, N)
    dots = K @ q[0]
    np.testing.assert_allclose(s, np.maximum(dots, 0.0), atol=1e-12)
    got = oracle.topk(s, N, k)
    np.testing.assert_array_equal(got, _ref_rank(np.maximum(dots, 0.0), N, k))
    # positives first, in decreasing dot order
    pos = np.argsort(-dots)[:min(k, int((dots > 0).sum()))]
    np.testing.assert_array_equal(got[:len(pos)], pos)


def test_negative_head_weight_flips_the_sign():
    r = rng(21)
    N, cI, k = 64, 8, 10
    q = r.standard_normal((1, cI))
    K = r.standard_normal((N, cI))
    s = oracle.index_scores(q, np.array([-1.0]), K, N)
    dots = K @ q[0]
    np.testing.assert_allclose(s, -np.maximum(dots, 0.0), atol=1e-12)
    # best are the entries with a non-positive dot (score 0), lowest index first
    zero = np.nonzero(dots <= 0)[0]
    np.testing.assert_array_equal(oracle.topk(s, N, k)[:min(k, len(zero))], zero[:k])


def test_heads_are_weighted_and_summed():
    r = rng(22)
    N, cI = 50, 8
    q = r.standard_normal((3, cI))
    K = r.standard_normal((N, cI))
    s01 = oracle.index_scores(q, np.array([1.0, 0.0, 0.0]), K, N)
    np.testing.assert_allclose(s01, oracle.index_scores(q[:1], np.array([1.0]), K, N),
                               atol=1e-12)
    w = np.array([0.5, -2.0, 3.0])
    parts = [oracle.index_scores(q[h:h + 1], np.array([w[h]]), K, N) for h in range(3)]
    np.testing.assert_allclose(oracle.index_scores(q, w, K, N), sum(parts), atol=1e-12)
    # positive homogeneity in the head weights keeps the ranking
    np.testing.assert_array_equal(oracle.topk(oracle.index_scores(q, 7.0 * w, K, N), N, 20),
                                  oracle.topk(oracle.index_scores(q, w, K, N), N, 20))


def test_topk_ties_go_to_the_lower_index_and_fill_with_sentinel():
    s = np.array([0.0, 1.0, 0.0, 1.0, 0.0, -1.0])
    np.testing.assert_array_equal(oracle.topk(s, 6, 4), [1, 3, 0, 2])
    np.testing.assert_array_equal(oracle.topk(s, 3, 5), [1, 0, 2, -1, -1])
    np.testing.assert_array_equal(oracle.topk(s, 0, 3), [-1, -1, -1])
    assert np.all(np.isneginf(oracle.index_scores(np.ones((1, 2)), np.ones(1), np.ones((5, 2)),
                                                  2)[2:]))


def test_topk_matches_numpy_on_random_rows():
    r = rng(23)
    for trial in range(20):
        n = int(r.integers(1, 300))
        s = np.round(r.standard_normal(n), 1)  # many exact ties
        k = int(r.integers(1, 40))
        np.testing.assert_array_equal(oracle.topk(s, n, k), _ref_rank(s, n, k))


# ------------------------------------------------------------------------------------------------
# Attention with the sink
# ------------------------------------------------------------------------------------------------
def test_attend_without_sink_is_plain_softmax_attention():
    r = rng(30)
    H, D, nk = 4, 16, 11
    q, keys = r.standard_normal((H, D)), r.standard_normal((nk, D))
    scale = 0.3
    o = oracle.attend(q, keys, np.full(H, NEG), scale)
    np.testing.assert_allclose(o, sdpa_explicit(q, keys, scale), atol=1e-13)


def test_sink_closed_form_on_identical_keys():
    # n identical keys k: o_h = n e^l / (e^s_h + n e^l) * k with l = scale <q_h, k>
    r = rng(31)
    H, D, n = 5, 8, 7
    k = r.standard_normal(D)
    q = r.standard_normal((H, D))
    sinks = r.standard_normal(H)
    scale = 1 / math.sqrt(D)
    o = oracle.attend(q, np.tile(k, (n, 1)), sinks, scale)
    for h in range(H):
        l = scale * q[h] @ k
        mass = n * math.exp(l) / (math.exp(sinks[h]) + n * math.exp(l))
        assert mass < 1.0
        np.testing.assert_allclose(o[h], mass * k, atol=1e-13)
    # an overwhelming sink takes all the mass
    np.testing.assert_allclose(oracle.attend(q, np.tile(k, (n, 1)), np.full(H, 1e300), scale),
                               0.0, atol=0)


def _tiny(kind, S=24, H=3, D=16, R=8, W=5, m=4, L=8, nI=2, cI=8, k=3, theta=10000.0, pos0=0):
    if kind == "swa":
        return OracleParams(1, S, H, D, R, theta, W, pos0=pos0)
    if kind == "hca":
        return OracleParams(1, S, H, D, R, theta, W, m=m, L=m, pos0=pos0)
    return OracleParams(1, S, H, D, R, theta, W, m=m, L=L, nI=nI, cI=cI, k=k, pos0=pos0)


def _inputs(p, seed):
    r = rng(seed)
    d = dict(q=r.standard_normal((1, p.S, p.H, p.D)), kv=r.standard_normal((1, p.S, p.D)),
             sinks=r.standard_normal(p.H), cmp_gate=r.standard_normal(p.D) / math.sqrt(p.D),
             cmp_bias=r.standard_normal(max(p.L, 1)))
    if p.k:
        d.update(q_idx=r.standard_normal((1, p.S, p.nI, p.cI)),
                 w_idx=r.standard_normal((1, p.S, p.nI)), k_idx=r.standard_normal((1, p.S, p.cI)),
                 idx_gate=r.standard_normal(p.cI), idx_bias=r.standard_normal(p.L))
    return d


def _run(kind, p, d, rows=None, topk_in=None):
    if kind == "swa":
        return oracle.swa_forward(p, d["q"] if rows is None else d["q"].reshape(-1, p.H, p.D)[rows],
                                  d["kv"], d["sinks"], rows=rows)
    q = d["q"] if rows is None else d["q"].reshape(-1, p.H, p.D)[rows]
    if kind == "hca":
        return oracle.hca_forward(p, q, d["kv"], d["cmp_gate"], d["cmp_bias"], d["sinks"],
                                  rows=rows)[0]
    sel = (lambda a: a if rows is None else a.reshape(p.B * p.S, *a.shape[2:])[rows])
    return oracle.csa_forward(p, q, d["kv"], d["cmp_gate"], d["cmp_bias"], sel(d["q_idx"]),
                              sel(d["w_idx"]), d["k_idx"], d["idx_gate"], d["idx_bias"],
                              d["sinks"], rows=rows, topk_in=topk_in)[0]


def test_single_key_output_is_the_unrotated_value():
    # W = 1 on a sliding layer: the only key is token t itself. The logit is rotation-invariant
    # and the output's rope slice is turned back by -P_t, so o = p * kv_t with the raw kv_t.
    p = _tiny("swa", W=1, pos0=1000)
    d = _inputs(p, 32)
    o = _run("swa", p, d).reshape(p.S, p.H, p.D)
    scale = 1 / math.sqrt(p.D)
    for t in range(p.S):
        for h in range(p.H):
            l = scale * d["q"][0, t, h] @ d["kv"][0, t]
            pm = 1.0 / (1.0 + math.exp(d["sinks"][h] - l))
            np.testing.assert_allclose(o[t, h], pm * d["kv"][0, t], atol=1e-12)


@pytest.mark.parametrize("kind", ["swa", "hca", "csa"])
def test_shifting_all_positions_leaves_the_output_unchanged(kind):
    p0 = _tiny(kind, pos0=0)
    p1 = _tiny(kind, pos0=12345)
    d = _inputs(p0, 33)
    np.testing.assert_allclose(_run(kind, p1, d), _run(kind, p0, d), atol=1e-11)


@pytest.mark.parametrize("kind", ["swa", "hca", "csa"])
def test_causality(kind):
    p = _tiny(kind)
    d = _inputs(p, 34)
    base = _run(kind, p, d).reshape(p.S, p.H, p.D)
    for t in [0, 3, 7, 15, 22]:
        e = {k: v.copy() for k, v in d.items()}
        e["kv"][0, t + 1:] += 3.0
        if "k_idx" in e:
            e["k_idx"][0, t + 1:] -= 2.0
        o = _run(kind, p, e).reshape(p.S, p.H, p.D)
        np.testing.assert_allclose(o[:t + 1], base[:t + 1], atol=1e-13)
        if t + 1 < p.S:
            assert np.abs(o[t + 1] - base[t + 1]).max() > 1e-6


def _window_keys(d, p, t, W):
    lo = max(0, t - W + 1)
    return np.stack([oracle.rope(d["kv"][0, j], p.R, p.theta, p.pos0 + j)
                     for j in range(lo, t + 1)])


def test_sliding_layer_is_softmax_over_the_window_without_sink():
    p = _tiny("swa", W=4)
    d = _inputs(p, 35)
    d["sinks"] = np.full(p.H, NEG)
    o = _run("swa", p, d).reshape(p.S, p.H, p.D)
    scale = 1 / math.sqrt(p.D)
    for t in range(p.S):
        qr = np.stack([oracle.rope(d["q"][0, t, h], p.R, p.theta, p.pos0 + t)
                       for h in range(p.H)])
        ref = sdpa_explicit(qr, _window_keys(d, p, t, p.W), scale)
        ref = np.stack([oracle.rope(ref[h], p.R, p.theta, -(p.pos0 + t)) for h in range(p.H)])
        np.testing.assert_allclose(o[t], ref, atol=1e-12)


def test_csa_attention_over_given_selection_is_softmax_over_window_and_entries():
    p = _tiny("csa", W=3, k=4)
    d = _inputs(p, 36)
    d["sinks"] = np.full(p.H, NEG)
    _, _, pool, _ = oracle.csa_forward(p, d["q"], d["kv"], d["cmp_gate"], d["cmp_bias"],
                                       d["q_idx"], d["w_idx"], d["k_idx"], d["idx_gate"],
                                       d["idx_bias"], d["sinks"])
    r = rng(37)
    sel = np.full((p.S, p.k), -1, dtype=np.int32)
    for t in range(p.S):
        nv = (t + 1) // p.m
        c = r.permutation(nv)[:p.k]
        sel[t, :len(c)] = c
    o = _run("csa", p, d, topk_in=sel).reshape(p.S, p.H, p.D)
    scale = 1 / math.sqrt(p.D)
    for t in range(p.S):
        keys = _window_keys(d, p, t, p.W)
        ent = [pool[0, w] for w in sel[t] if w >= 0]
        if ent:
            keys = np.concatenate([keys, np.stack(ent)])
        qr = np.stack([oracle.rope(d["q"][0, t, h], p.R, p.theta, p.pos0 + t)
                       for h in range(p.H)])
        ref = sdpa_explicit(qr, keys, scale)
        ref = np.stack([oracle.rope(ref[h], p.R, p.theta, -(p.pos0 + t)) for h in range(p.H)])
        np.testing.assert_allclose(o[t], ref, atol=1e-12)


def test_pool_entries_rotate_at_their_block_start():
    # HCA pool_out: entry w equals the un-rotated pool entry rotated at pos0 + w*m
    p = _tiny("hca", m=4, pos0=50)
    d = _inputs(p, 38)
    _, pool = oracle.hca_forward(p, d["q"], d["kv"], d["cmp_gate"], d["cmp_bias"], d["sinks"])
    raw = oracle.compress(d["kv"], d["cmp_gate"], d["cmp_bias"][:p.m], p.m, p.m)
    for w in range(p.S // p.m):
        np.testing.assert_allclose(pool[0, w], oracle.rope(raw[0, w], p.R, p.theta, 50 + w * p.m),
                                   atol=1e-13)


# ------------------------------------------------------------------------------------------------
# The page's worked mask example (16 tokens, sliding_window=8, CSA m=4, HCA m'=8, index_topk=2)
# ------------------------------------------------------------------------------------------------
@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_golden_sliding_window_cut(golden):
    # o_t with W = 8 equals softmax attention over keys (t-8, t]: key 0 is still in the window at
    # row 7 and cut at row 8 ("for i >= window the lower-left triangle is cut")
    cfg = golden["config"]
    p = OracleParams(1, cfg["S"], 2, 8, 0, 10000.0, cfg["sliding_window"])
    r = rng(40)
    q, kv = r.standard_normal((1, p.S, p.H, p.D)), r.standard_normal((1, p.S, p.D))
    o = oracle.swa_forward(p, q, kv, np.full(p.H, NEG)).reshape(p.S, p.H, p.D)
    scale = 1 / math.sqrt(p.D)
    g = golden["sliding"]
    for t, has_key0 in [(g["last_row_with_key0"], True), (g["first_row_without_key0"], False)]:
        lo = 0 if has_key0 else 1
        np.testing.assert_allclose(o[t], sdpa_explicit(q[0, t], kv[0, lo:t + 1], scale),
                                   atol=1e-13)
        # the other reading of the window (W+1 keys) would keep key 0 at row 8
        if not has_key0:
            assert np.abs(o[t] - sdpa_explicit(q[0, t], kv[0, 0:t + 1], scale)).max() > 1e-9


def test_golden_hca_entry_visibility(golden):
    cfg = golden["config"]
    g = golden["hca"]
    m = cfg["hca_m"]
    p = OracleParams(1, cfg["S"], 2, 8, 0, 10000.0, cfg["sliding_window"], m=m, L=m)
    r = rng(41)
    q, kv = r.standard_normal((1, p.S, p.H, p.D)), r.standard_normal((1, p.S, p.D))
    u, b = r.standard_normal(p.D), r.standard_normal(m)
    o, pool = oracle.hca_forward(p, q, kv, u, b, np.full(p.H, NEG))
    o = o.reshape(p.S, p.H, p.D)
    # entry w pools exactly the positions the page says it covers
    zero = oracle.compress(kv, np.zeros(p.D), np.zeros(m), m, m)
    for w, (a, z) in enumerate(g["entry_covers"]):
        np.testing.assert_allclose(zero[0, w], kv[0, a:z + 1].mean(0), atol=1e-14)
    scale = 1 / math.sqrt(p.D)
    first = g["entry_first_visible_row"]
    for t in range(p.S):
        nvis = sum(t >= f for f in first)
        keys = kv[0, max(0, t - p.W + 1):t + 1]
        if nvis:
            keys = np.concatenate([keys, pool[0, :nvis]])
        np.testing.assert_allclose(o[t], sdpa_explicit(q[0, t], keys, scale), atol=1e-12)
        # and not with one entry more or less
        for wrong in (nvis - 1, nvis + 1):
            if 0 <= wrong <= len(first):
                kw = kv[0, max(0, t - p.W + 1):t + 1]
                if wrong:
                    kw = np.concatenate([kw, pool[0, :wrong]])
                assert np.abs(o[t] - sdpa_explicit(q[0, t], kw, scale)).max() > 1e-9


def test_golden_csa_sentinel_rows(golden):
    cfg = golden["config"]
    g = golden["csa"]
    m, k = cfg["csa_m"], cfg["index_topk"]
    p = OracleParams(1, cfg["S"], 2, 8, 0, 10000.0, cfg["sliding_window"], m=m, L=2 * m, nI=2,
                     cI=4, k=k)
    d = _inputs(p, 42)
    _, tk, _, _ = oracle.csa_forward(p, d["q"], d["kv"], d["cmp_gate"], d["cmp_bias"][:2 * m],
                                     d["q_idx"], d["w_idx"], d["k_idx"], d["idx_gate"],
                                     d["idx_bias"][:2 * m], d["sinks"])
    for t in g["rows_with_no_entry"]:
        assert list(tk[t]) == [-1] * k
    assert (tk[g["first_row_with_an_entry"]] >= 0).sum() == 1
    # slots fill as t grows, up to k
    filled = (tk >= 0).sum(1)
    assert list(filled) == [min(k, (t + 1) // m) for t in range(p.S)]


def test_sentinel_count_on_the_tiny_workload():
    from sparse_attention_compressor_b200 import workloads as W
    wl = W.WORKLOADS["tiny_csa_f32"]
    x = W.prefill_inputs(wl)
    p = OracleParams(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, wl.W, m=wl.m, L=wl.L, nI=wl.nI,
                     cI=wl.cI, k=wl.k)
    _, tk, pool, kpool = oracle.csa_forward(p, x["q"], x["kv"], x["cmp_gate"], x["cmp_bias"],
                                            x["q_idx"], x["w_idx"], x["k_idx"], x["idx_gate"],
                                            x["idx_bias"], x["sinks"])
    assert pool.shape == (1, 64, wl.D) and kpool.shape == (1, 64, wl.cI)
    for t in range(wl.S):
        nvis = (t + 1) // wl.m
        assert (tk[t] == -1).sum() == max(0, wl.k - nvis)
        assert set(tk[t][tk[t] >= 0]) <= set(range(nvis))


# ------------------------------------------------------------------------------------------------
# Decode over a paged cache agrees with the prefill row of the same token
# ------------------------------------------------------------------------------------------------
def _paginate(rows, page_size, perm_seed):
    n = rows.shape[0]
    npg = (n + page_size - 1) // page_size
    perm = rng(perm_seed).permutation(npg + 3)[:npg]
    pages = np.zeros((npg + 3, page_size, rows.shape[1]))
    for lp in range(npg):
        chunk = rows[lp * page_size:(lp + 1) * page_size]
        pages[perm[lp], :len(chunk)] = chunk
    return pages, perm.astype(np.int32)


@pytest.mark.parametrize("kind", ["swa", "hca", "csa"])
def test_decode_equals_prefill_row(kind):
    p = _tiny(kind, S=29, W=6, k=3, pos0=7)
    d = _inputs(p, 43)
    kv_rot = np.stack([oracle.rope(d["kv"][0, j], p.R, p.theta, p.pos0 + j) for j in range(p.S)])
    ps = 4
    kvp, kvbt = _paginate(kv_rot, ps, 1)
    pool_pages = ipool_pages = pbt = None
    if kind == "hca":
        _, pool = oracle.hca_forward(p, d["q"], d["kv"], d["cmp_gate"], d["cmp_bias"], d["sinks"])
        pool_pages, pbt = _paginate(pool[0], ps, 2)
    if kind == "csa":
        _, _, pool, kpool = oracle.csa_forward(p, d["q"], d["kv"], d["cmp_gate"], d["cmp_bias"],
                                               d["q_idx"], d["w_idx"], d["k_idx"], d["idx_gate"],
                                               d["idx_bias"], d["sinks"])
        pool_pages, pbt = _paginate(pool[0], ps, 2)
        ipool_pages = np.zeros((pool_pages.shape[0], ps, p.cI))
        for lp in range(len(pbt)):
            chunk = kpool[0, lp * ps:(lp + 1) * ps]
            ipool_pages[pbt[lp], :len(chunk)] = chunk
    full = _run(kind, p, d).reshape(p.S, p.H, p.D)
    ts = [0, 3, 4, 11, 17, 28]
    ctx = np.array([t + 1 for t in ts], dtype=np.int32)
    nseq = len(ts)
    o, tk = oracle.decode(
        p, d["q"][0, ts], kvp, np.tile(kvbt, (nseq, 1)), ctx, ps,
        pool_pages=pool_pages, idx_pool_pages=ipool_pages,
        pool_block_table=None if pbt is None else np.tile(pbt, (nseq, 1)),
        q_idx=None if kind != "csa" else d["q_idx"][0, ts],
        w_idx=None if kind != "csa" else d["w_idx"][0, ts], sinks=d["sinks"])
    np.testing.assert_allclose(o, full[ts], atol=1e-12)


# ------------------------------------------------------------------------------------------------
# bf16 storage of the pools
# ------------------------------------------------------------------------------------------------
def test_round_bf16_matches_torch_conversion():
    r = rng(50)
    vals = np.concatenate([r.standard_normal(20000) * 10.0 ** r.integers(-6, 6, 20000),
                           [0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40]])
    # torch converts float32 -> bfloat16 with round-to-nearest-even
    ref = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).double().numpy()
    got = np.array([oracle.round_bf16(v) for v in vals])
    np.testing.assert_array_equal(got, ref)


def test_bf16_pools_round_the_stored_entries():
    p = _tiny("csa")
    d = _inputs(p, 51)
    args = (d["q"], d["kv"], d["cmp_gate"], d["cmp_bias"], d["q_idx"], d["w_idx"], d["k_idx"],
            d["idx_gate"], d["idx_bias"], d["sinks"])
    _, _, pool, kpool = oracle.csa_forward(p, *args)
    p.bf16_pools = True
    _, _, pool_r, kpool_r = oracle.csa_forward(p, *args)
    np.testing.assert_array_equal(pool_r, np.vectorize(oracle.round_bf16)(pool))
    np.testing.assert_array_equal(kpool_r, np.vectorize(oracle.round_bf16)(kpool))


# ---- grouped output projection ("Grouped Output Projection" bullet) --------------------------
def test_oproj_matches_numpy_matmul():
    rng = np.random.default_rng(3)
    o = rng.standard_normal((7, 6, 8))
    wa = rng.standard_normal((3, 5, 16))
    wb = rng.standard_normal((9, 15))
    mid, out = oracle.o_proj(o, wa, wb, 3)
    o2 = o.reshape(7, 48)
    ref_mid = np.concatenate([o2[:, g * 16:(g + 1) * 16] @ wa[g].T for g in range(3)], axis=1)
    assert np.allclose(mid, ref_mid, atol=1e-12)
    assert np.allclose(out, ref_mid @ wb.T, atol=1e-12)


def test_oproj_one_hot_selection_is_exact():
    # o_a_proj rows that pick single features and an o_b_proj permutation give the picked
    # features back, permuted, exactly
    rng = np.random.default_rng(4)
    G, rank, kg = 2, 3, 10
    o = rng.standard_normal((4, G * kg))
    wa = np.zeros((G, rank, kg))
    picks = [[0, 4, 9], [1, 2, 7]]
    for g in range(G):
        for i, c in enumerate(picks[g]):
            wa[g, i, c] = 1.0
    perm = rng.permutation(G * rank)
    wb = np.eye(G * rank)[perm]
    mid, out = oracle.o_proj(o, wa, wb, G)
    want = np.concatenate([o[:, g * kg + np.array(picks[g])] for g in range(G)], axis=1)
    assert np.array_equal(mid, want)
    assert np.array_equal(out, want[:, perm])


def test_oproj_groups_are_independent_and_rows_selectable():
    rng = np.random.default_rng(5)
    G, rank, kg = 4, 6, 8
    o = rng.standard_normal((5, G * kg))
    wa = rng.standard_normal((G, rank, kg))
    wb = rng.standard_normal((7, G * rank))
    mid, _ = oracle.o_proj(o, wa, wb, G)
    o2 = o.copy()
    o2[:, :kg] += 1.0  # only group 0's features
    mid2, _ = oracle.o_proj(o2, wa, wb, G)
    assert not np.allclose(mid2[:, :rank], mid[:, :rank])
    assert np.array_equal(mid2[:, rank:], mid[:, rank:])
    mid_r, out_r = oracle.o_proj(o, wa, wb, G, rows=[3, 1])
    _, out = oracle.o_proj(o, wa, wb, G)
    assert np.array_equal(out_r, out[[3, 1]])


def test_oproj_rounded_intermediate_is_bf16():
    rng = np.random.default_rng(6)
    o = rng.standard_normal((3, 16))
    wa = rng.standard_normal((2, 4, 8))
    wb = rng.standard_normal((5, 8))
    mid, _ = oracle.o_proj(o, wa, wb, 2, round_mid=True)
    as_bf16 = torch.from_numpy(mid).float().to(torch.bfloat16).double().numpy()
    assert np.array_equal(mid, as_bf16)


# ---- YaRN-scaled RoPE (the config pairs compress_rope_theta with a YaRN rope scaling) ---------
# Pair i of R rope channels turns r_i = L f_i / (2 pi) times over the original context L. YaRN
# keeps the pairs with r_i above beta_fast, interpolates those below beta_slow like position
# interpolation (position / s), and ramps between.
YARN = dict(theta=160000.0, R=64, factor=4.0, orig=4096, beta_fast=32.0, beta_slow=1.0)


def _turns(i, R, theta, orig):
    return orig * theta ** (-2.0 * i / R) / (2 * math.pi)


def _yarn(x, pos, **over):
    c = dict(YARN, **over)
    return oracle.rope_yarn(x, c["R"], c["theta"], pos, c["factor"], c["orig"], c["beta_fast"],
                            c["beta_slow"])


def test_yarn_with_factor_one_is_plain_rope():
    x = rng(80).standard_normal((5, 96))
    for pos in (0.0, 7.0, 123456.0, -99.0):
        np.testing.assert_array_equal(_yarn(x, pos, factor=1.0),
                                      oracle.rope(x, YARN["R"], YARN["theta"], pos))


def test_yarn_keeps_fast_pairs_and_interpolates_slow_pairs():
    R, D = YARN["R"], 96
    turns = [_turns(i, R, YARN["theta"], YARN["orig"]) for i in range(R // 2)]
    fast = [i for i, r in enumerate(turns) if r > YARN["beta_fast"]]
    slow = [i for i, r in enumerate(turns) if r < YARN["beta_slow"]]
    assert fast and slow  # the configuration exercises both ends of the ramp
    for i in fast + slow:
        x = np.zeros(D)
        x[D - R + 2 * i] = 1.0  # one-hot on pair i: the result is (cos phi, sin phi)
        for pos in (3.0, 1000.0, 77777.0):
            got = _yarn(x, pos)
            # fast pairs rotate like plain RoPE at pos; slow pairs like plain RoPE at pos / s
            ref_pos = pos if i in fast else pos / YARN["factor"]
            ref = oracle.rope(x, R, YARN["theta"], ref_pos)
            np.testing.assert_allclose(got, ref, atol=1e-9, err_msg=f"pair {i} pos {pos}")


def test_yarn_ramp_midpoint_is_the_mean_of_both_frequencies():
    # choose the original length so that pair 5 completes exactly (alpha + beta) / 2 turns:
    # its frequency is then halfway between f (kept) and f / s (interpolated)
    R, theta, i = 64, 10000.0, 5
    f = theta ** (-2.0 * i / R)
    mid = (YARN["beta_fast"] + YARN["beta_slow"]) / 2
    L_real = mid * 2 * math.pi / f
    L = int(round(L_real))
    r = L * f / (2 * math.pi)
    gamma = (r - YARN["beta_slow"]) / (YARN["beta_fast"] - YARN["beta_slow"])
    assert abs(gamma - 0.5) < 0.01
    got = oracle.rope_freq(i, R, theta, 4.0, L, YARN["beta_fast"], YARN["beta_slow"])
    np.testing.assert_allclose(got, (1 - gamma) * f / 4.0 + gamma * f, rtol=1e-14)
    assert f / 4.0 < got < f


def test_yarn_rotation_preserves_norm_and_inverts():
    x = rng(81).standard_normal((4, 96))
    y = _yarn(x, 4321.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(_yarn(y, -4321.0), x, atol=1e-12)


@pytest.mark.parametrize("kind", ["hca", "csa"])
def test_yarn_layers_stay_shift_invariant(kind):
    base = _tiny(kind, pos0=0)
    d = _inputs(base, 82)
    outs = []
    for pos0 in (0, 50000):
        p = _tiny(kind, pos0=pos0)
        p.yarn_factor, p.yarn_orig = 4.0, 64
        outs.append(_run(kind, p, d))
    np.testing.assert_allclose(outs[1], outs[0], atol=1e-11)
    plain = _run(kind, base, d)
    assert np.abs(outs[0] - plain).max() > 1e-6  # the scaling does change the output
