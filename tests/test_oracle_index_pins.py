"""Pins of the oracle's row-wise indexer scores (``oracle.csa_index_scores``) and of the bf16
storage of the pools, against parts of the oracle that do not share its code path.

``csa_index_scores`` builds its own indexer pool (compressor over k_idx, optional bf16 rounding)
and scores listed rows against it; the GPU parity tests take the top-k tie band from these scores.
It is pinned here by ``csa_forward`` (which selects through its own pool and loop), by the
single-query ``index_scores`` applied to the pool that ``csa_forward`` returns, by the visible
count of the page's rule w < (t+1)//m, and by batch isolation. A slip in any of its steps (a
missing rounding, the wrong pool stride for b > 0, a visible count off by one) fails one of them.

The bf16 pool storage ("Cache layers": pools are cached tensors of the layer's dtype) is checked
to move the attention output by less than the bf16 parity tolerance when the selection is held
fixed: the rounding only matters through the integer top-k decision, which the GPU parity tests
compare with a tie band.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import OracleParams
from sparse_attention_compressor_b200 import workloads as W


def _csa(B=2, S=67, H=2, D=16, R=8, W=6, m=4, L=8, nI=3, cI=8, k=5, bf16=False):
    return OracleParams(B, S, H, D, R, 10000.0, W, m=m, L=L, nI=nI, cI=cI, k=k, bf16_pools=bf16)


def _inputs(p, seed, bf16_values=False):
    r = np.random.default_rng(seed)
    d = dict(q=r.standard_normal((p.B, p.S, p.H, p.D)), kv=r.standard_normal((p.B, p.S, p.D)),
             sinks=r.standard_normal(p.H), cmp_gate=r.standard_normal(p.D) / math.sqrt(p.D),
             cmp_bias=r.standard_normal(p.L), q_idx=r.standard_normal((p.B, p.S, p.nI, p.cI)),
             w_idx=r.standard_normal((p.B, p.S, p.nI)) / math.sqrt(p.nI),
             k_idx=r.standard_normal((p.B, p.S, p.cI)),
             idx_gate=r.standard_normal(p.cI) / math.sqrt(p.cI), idx_bias=r.standard_normal(p.L))
    if bf16_values:  # values a bf16 layer would hold (exact in fp64)
        d = {k: torch.from_numpy(v).float().to(torch.bfloat16).double().numpy()
             for k, v in d.items()}
    return d


def _forward(p, d, topk_in=None):
    return oracle.csa_forward(p, d["q"], d["kv"], d["cmp_gate"], d["cmp_bias"], d["q_idx"],
                              d["w_idx"], d["k_idx"], d["idx_gate"], d["idx_bias"], d["sinks"],
                              topk_in=topk_in)


def _scores(p, d, rows):
    rows = np.asarray(rows, dtype=np.int64)
    qi = d["q_idx"].reshape(-1, p.nI, p.cI)[rows]
    wi = d["w_idx"].reshape(-1, p.nI)[rows]
    return oracle.csa_index_scores(p, qi, wi, d["k_idx"], d["idx_gate"], d["idx_bias"], rows)


@pytest.mark.parametrize("bf16", [False, True])
def test_top_k_of_row_scores_equals_the_forward_selection(bf16):
    # two sequences, so rows of the second one must use the second sequence's pool
    p = _csa(bf16=bf16)
    d = _inputs(p, 60, bf16_values=bf16)
    _, tk, _, _ = _forward(p, d)
    rows = np.arange(p.B * p.S)
    sc = _scores(p, d, rows)
    for i, r in enumerate(rows):
        nvis = (r % p.S + 1) // p.m
        np.testing.assert_array_equal(oracle.topk(sc[i], nvis, p.k), tk[i], err_msg=f"row {r}")


@pytest.mark.parametrize("bf16", [False, True])
def test_row_scores_equal_the_single_query_scores_over_the_returned_pool(bf16):
    p = _csa(bf16=bf16)
    d = _inputs(p, 61, bf16_values=bf16)
    _, _, _, kpool = _forward(p, d)
    rows = np.array([0, 3, 4, 17, 66, 67, 70, 99, 133])
    sc = _scores(p, d, rows)
    for i, r in enumerate(rows):
        b, t = divmod(int(r), p.S)
        ref = oracle.index_scores(d["q_idx"][b, t], d["w_idx"][b, t], kpool[b], (t + 1) // p.m)
        np.testing.assert_array_equal(sc[i], ref, err_msg=f"row {r}")


def test_row_scores_follow_the_visible_count():
    # entries w < (t+1)//m are scored, later ones are -inf ("Attention mask layout", HCA rule)
    p = _csa(B=1, S=40)
    d = _inputs(p, 62)
    rows = np.arange(p.S)
    sc = _scores(p, d, rows)
    for t in rows:
        nvis = (t + 1) // p.m
        assert np.isfinite(sc[t, :nvis]).all(), t
        assert np.isneginf(sc[t, nvis:]).all(), t


def test_row_scores_of_one_sequence_ignore_the_other_sequence():
    p = _csa()
    d = _inputs(p, 63)
    rows = np.arange(p.B * p.S)
    base = _scores(p, d, rows)
    e = {k: v.copy() for k, v in d.items()}
    e["k_idx"][0] += 1.5  # only the first sequence's indexer keys move
    moved = _scores(p, e, rows)
    np.testing.assert_array_equal(moved[p.S:], base[p.S:])
    first = np.isfinite(base[:p.S])
    assert np.abs(moved[:p.S][first] - base[:p.S][first]).max() > 1e-3


def test_rounded_pool_scores_are_the_scores_of_the_rounded_pool():
    # with bf16 pools the scores equal index_scores over the unrounded pool rounded to bf16
    p = _csa(bf16=False)
    d = _inputs(p, 64, bf16_values=True)
    _, _, _, kpool = _forward(p, d)
    kpool_r = torch.from_numpy(kpool).float().to(torch.bfloat16).double().numpy()
    p.bf16_pools = True
    rows = np.array([5, 20, 66, 90, 133])
    sc = _scores(p, d, rows)
    for i, r in enumerate(rows):
        b, t = divmod(int(r), p.S)
        ref = oracle.index_scores(d["q_idx"][b, t], d["w_idx"][b, t], kpool_r[b], (t + 1) // p.m)
        np.testing.assert_array_equal(sc[i], ref)


# ------------------------------------------------------------------------------------------------
# bf16 pool storage moves the attention output by less than the bf16 parity tolerance
# ------------------------------------------------------------------------------------------------
BF16_TOL = (2e-2, 2e-3)  # max and mean |error| of the bf16 parity tests


def _bf16_workload(kind):
    if kind == "csa":
        return W.Workload("csa_bf16_pool_rounding", "csa", "bf16", B=1, S=1030, m=4, L=8,
                          nI=64, cI=128, k=64, seed=70)
    return W.Workload("hca_bf16_pool_rounding", "hca", "bf16", B=1, S=1100, m=128, L=128,
                      seed=71)


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_bf16_pool_rounding_stays_inside_the_bf16_tolerance(kind):
    wl = _bf16_workload(kind)
    x = W.prefill_inputs(wl)
    rows = np.unique(np.concatenate([np.arange(0, wl.S, 37), [wl.S - 2, wl.S - 1]]))
    q = x["q"].reshape(-1, wl.H, wl.D)[torch.from_numpy(rows)]
    out = {}
    for rounded in (True, False):
        p = OracleParams(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, wl.W, m=wl.m, L=wl.L, nI=wl.nI,
                         cI=wl.cI, k=wl.k, bf16_pools=rounded)
        if kind == "hca":
            out[rounded] = oracle.hca_forward(p, q, x["kv"], x["cmp_gate"], x["cmp_bias"],
                                              x["sinks"], rows=rows)[0]
            continue
        qi = x["q_idx"].reshape(-1, wl.nI, wl.cI)[torch.from_numpy(rows)]
        wi = x["w_idx"].reshape(-1, wl.nI)[torch.from_numpy(rows)]
        # the selection of the rounded pool is held fixed for both runs
        sel = out.get("sel")
        o, tk, _, _ = oracle.csa_forward(p, q, x["kv"], x["cmp_gate"], x["cmp_bias"], qi, wi,
                                         x["k_idx"], x["idx_gate"], x["idx_bias"], x["sinks"],
                                         rows=rows, topk_in=sel)
        out[rounded] = o
        out["sel"] = tk
    err = np.abs(out[True] - out[False])
    assert err.max() > 0.0  # the rounding does change the pools
    assert err.max() <= BF16_TOL[0] and err.mean() <= BF16_TOL[1], (err.max(), err.mean())
