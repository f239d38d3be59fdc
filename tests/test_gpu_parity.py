"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Small shapes compare every output element; the full-size workloads compare sampled query rows
that the oracle computes one by one (plus the full pools). Edge cases: no visible entry (S < m),
fewer visible entries than index_topk (-1 fill), ragged tails (S not a multiple of m or of the
tiles), W = 1, W > S, batches, head counts that are not a multiple of the block's head group,
and shifted absolute positions."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from parity import (assert_close, check_topk_row, gpu_prefill, oracle_params)
from sparse_attention_compressor_b200 import workloads as W

pytestmark = pytest.mark.gpu


def wl_small(kind, dtype, **kw):
    base = dict(B=1, S=256, H=4, D=64, R=16, theta=10000.0, W=64, seed=7)
    if kind == "csa":
        base.update(m=4, L=8, nI=2, cI=32, k=8)
    if kind == "hca":
        base.update(m=16, L=16)
    base.update(kw)
    return W.Workload(f"{kind}_{dtype}_test", kind, dtype, **base)


SMALL = [
    ("tiny_config", W.WORKLOADS["tiny_csa_f32"], 0),
    ("csa_bf16_batch_ragged", wl_small("csa", "bf16", B=2, S=301, H=8, D=128, R=32, nI=4, cI=64,
                                       k=16, W=40, seed=11), 100),
    ("csa_bf16_heads64_d512", wl_small("csa", "bf16", S=1030, H=64, D=512, R=64, nI=64, cI=128,
                                       k=64, W=128, theta=160000.0, seed=12), 0),
    ("csa_f32_topk_exceeds_pool", wl_small("csa", "f32", S=64, k=32, seed=13), 3),
    ("csa_f32_no_entry", wl_small("csa", "f32", S=3, W=8, seed=14), 0),
    ("csa_f32_window1", wl_small("csa", "f32", S=97, W=1, seed=15), 0),
    ("hca_f32_ragged", wl_small("hca", "f32", S=333, H=6, D=64, R=16, W=50, seed=16), 5),
    ("hca_bf16_heads64_d512", wl_small("hca", "bf16", S=1100, H=64, D=512, R=64, m=128, L=128,
                                       W=128, theta=160000.0, seed=17), 0),
    ("hca_f32_no_entry", wl_small("hca", "f32", S=100, m=128, L=128, seed=18), 0),
    ("swa_f32_heads20_d256", wl_small("swa", "f32", B=2, S=200, H=20, D=256, R=64, W=33,
                                      seed=19), 0),
    ("swa_bf16_window_exceeds_S", wl_small("swa", "bf16", S=150, H=64, D=512, R=64, W=300,
                                           seed=20), 77),
]


def run_oracle(wl, x, pos0, topk_in=None):
    p = oracle_params(wl, pos0)
    if wl.kind == "swa":
        return dict(o=oracle.swa_forward(p, x["q"], x["kv"], x["sinks"]))
    if wl.kind == "hca":
        o, pool = oracle.hca_forward(p, x["q"], x["kv"], x["cmp_gate"], x["cmp_bias"], x["sinks"])
        return dict(o=o, pool=pool)
    o, tk, pool, kpool = oracle.csa_forward(p, x["q"], x["kv"], x["cmp_gate"], x["cmp_bias"],
                                            x["q_idx"], x["w_idx"], x["k_idx"], x["idx_gate"],
                                            x["idx_bias"], x["sinks"], topk_in=topk_in)
    return dict(o=o, topk=tk, pool=pool, idx_pool=kpool)


def check_csa_topk(wl, x, g, pos0, rows=None):
    """Compare the GPU's selections with the oracle's (tie band aware). Returns the GPU selection
    of the checked rows as [n, k]."""
    p = oracle_params(wl, pos0)
    rows = np.arange(wl.B * wl.S) if rows is None else np.asarray(rows)
    if "q_idx" in x:
        qi = x["q_idx"].reshape(-1, wl.nI, wl.cI)[torch.from_numpy(rows)]
        wi = x["w_idx"].reshape(-1, wl.nI)[torch.from_numpy(rows)]
    else:
        r = W.prefill_row_inputs(wl, rows)
        qi, wi = r["q_idx"], r["w_idx"]
    sc = oracle.csa_index_scores(p, qi, wi, x["k_idx"], x["idx_gate"], x["idx_bias"], rows)
    gsel = g["topk"].reshape(-1, wl.k).numpy()[rows]
    ndiff = 0
    for i, r in enumerate(rows):
        t = int(r % wl.S)
        nvis = (t + 1) // wl.m
        osel = oracle.topk(sc[i], nvis, wl.k)
        ndiff += check_topk_row(gsel[i], osel, sc[i], nvis, wl.k, f"row {r}")
    return gsel, ndiff


@pytest.mark.parametrize("name,wl,pos0", SMALL, ids=[s[0] for s in SMALL])
def test_small_full_parity(name, wl, pos0):
    x = W.prefill_inputs(wl)
    g = gpu_prefill(wl, x, pos0)
    topk_in = None
    if wl.kind == "csa":
        gsel, _ = check_csa_topk(wl, x, g, pos0)
        topk_in = gsel
    ref = run_oracle(wl, x, pos0, topk_in=topk_in)
    n = wl.B * wl.S
    assert_close(g["o"].reshape(n, wl.H, wl.D), ref["o"].reshape(n, wl.H, wl.D), wl.dtype, "o")
    if wl.kind in ("hca", "csa") and wl.N > 0:
        assert_close(g["pool"], ref["pool"], wl.dtype, "pool")
    if wl.kind == "csa" and wl.N > 0:
        assert_close(g["idx_pool"], ref["idx_pool"], wl.dtype, "indexer pool")


def test_tiny_topk_matches_oracle_exactly():
    # the tiny workload's selections (2 indexer heads, many exact zero ties) must be identical
    wl = W.WORKLOADS["tiny_csa_f32"]
    x = W.prefill_inputs(wl)
    g = gpu_prefill(wl, x)
    ref = run_oracle(wl, x, 0)
    for t in range(wl.S):
        gs = g["topk"][0, t].numpy()
        os_ = ref["topk"][t]
        assert sorted(gs[gs >= 0].tolist()) == sorted(os_[os_ >= 0].tolist()), t


def test_topk_all_scores_equal():
    # With q_idx = 0 every indexer score of a row is 0: ties are decided by the entry index alone,
    # so each row keeps its k lowest visible entries (then -1 fill).
    wl = SMALL[2][1]  # bf16, 64 indexer heads of 128: the tensor-core indexer
    x = W.prefill_inputs(wl)
    x["q_idx"] = torch.zeros_like(x["q_idx"])
    g = gpu_prefill(wl, x)
    for t in range(wl.S):
        nvis = (t + 1) // wl.m
        expect = np.arange(wl.k) if nvis >= wl.k else np.concatenate(
            [np.arange(nvis), -np.ones(wl.k - nvis, dtype=np.int64)])
        assert np.array_equal(g["topk"][0, t].numpy(), expect), t


@pytest.mark.parametrize("S", [8448, 33024])
def test_topk_ties_beyond_candidate_capacity(S):
    # All scores equal (q_idx = 0), on rows long enough that the threshold digit holds more keys
    # than the candidate list (2048): the top-k takes its whole-row fallback. S = 8448 keeps each
    # row's keys in shared memory (2112 entries), S = 33024 re-reads them from L2 (8256 entries).
    # Each row must keep its k lowest visible entries, in order.
    wl = wl_small("csa", "bf16", S=S, H=8, D=128, R=32, nI=64, cI=128, k=512, W=128,
                  theta=160000.0, seed=21)
    x = W.prefill_inputs(wl)
    x["q_idx"] = torch.zeros_like(x["q_idx"])
    g = gpu_prefill(wl, x, with_aux=False)
    sel = g["topk"][0].numpy()
    for t in list(range(0, S, 97)) + list(range(S - 64, S)):
        nvis = (t + 1) // wl.m
        expect = np.arange(wl.k) if nvis >= wl.k else np.concatenate(
            [np.arange(nvis), -np.ones(wl.k - nvis, dtype=np.int64)])
        assert np.array_equal(sel[t], expect), t


def test_relative_position_invariance_on_gpu():
    wl = SMALL[1][1]
    x = W.prefill_inputs(wl)
    a = gpu_prefill(wl, x, 0)["o"].float()
    b = gpu_prefill(wl, x, 4096)["o"].float()
    assert (a - b).abs().max().item() < 2e-2


# ------------------------------------------------------------------------------------------------
# Full-size workloads: sampled rows
# ------------------------------------------------------------------------------------------------
def sampled_rows(wl, fixed, n_random, seed):
    r = np.random.default_rng(seed)
    rows = set(int(v) for v in fixed if 0 <= v < wl.S)
    rows |= set(int(v) for v in r.integers(0, wl.S, n_random))
    return np.array(sorted(rows))


def full_size_check(wl, rows):
    x = W.prefill_inputs(wl)
    g = gpu_prefill(wl, x)
    p = oracle_params(wl)
    rq = W.prefill_row_inputs(wl, rows)
    assert torch.equal(rq["q"], x["q"].reshape(-1, wl.H, wl.D)[torch.from_numpy(rows)])
    if wl.kind == "hca":
        o, pool = oracle.hca_forward(p, rq["q"], x["kv"], x["cmp_gate"], x["cmp_bias"],
                                     x["sinks"], rows=rows)
    else:
        gsel, ndiff = check_csa_topk(wl, {k: v for k, v in x.items()
                                          if k not in ("q_idx", "w_idx")}, g, 0, rows)
        o, _, pool, kpool = oracle.csa_forward(p, rq["q"], x["kv"], x["cmp_gate"], x["cmp_bias"],
                                               rq["q_idx"], rq["w_idx"], x["k_idx"], x["idx_gate"],
                                               x["idx_bias"], x["sinks"], rows=rows, topk_in=gsel)
        assert_close(g["idx_pool"], kpool, wl.dtype, "indexer pool")
    assert_close(g["pool"], pool, wl.dtype, "pool")
    got = g["o"].reshape(-1, wl.H, wl.D)[torch.from_numpy(rows)]
    return assert_close(got, o, wl.dtype, "o (sampled rows)")


def test_csa_8k_sampled_rows():
    wl = W.WORKLOADS["csa_8k_bf16"]
    rows = sampled_rows(wl, [0, 1, 2, 3, 4, 127, 128, 129, 2046, 2047, 2048, 4095, 8190, 8191],
                        34, 1)
    full_size_check(wl, rows)


def test_hca_32k_sampled_rows():
    wl = W.WORKLOADS["hca_32k_bf16"]
    rows = sampled_rows(wl, [0, 1, 126, 127, 128, 255, 256, 16383, 32766, 32767], 22, 2)
    full_size_check(wl, rows)


@pytest.mark.slow
def test_csa_128k_sampled_rows():
    wl = W.WORKLOADS["csa_128k_bf16"]
    spiked = W.spiked_rows(wl)
    rows = sampled_rows(wl, [0, 3, 2047, 2048, 65535, 131071] + list(spiked[:8]), 10, 3)
    full_size_check(wl, rows)


# ------------------------------------------------------------------------------------------------
# Decode over the paged cache
# ------------------------------------------------------------------------------------------------
def logical(pages, bt, s, lo, hi):
    """Rows lo..hi-1 of sequence s of a paged cache (CPU tensors) -> float64 numpy."""
    ps = pages.shape[1]
    idx = np.arange(lo, hi)
    pg = bt[s, idx // ps].numpy()
    return pages[torch.from_numpy(pg).long(), torch.from_numpy(idx % ps)].double().numpy()


def oracle_decode(wl, d, layer, seqs, topk_in=None):
    """The oracle's decode of the listed sequences, on a page_size = 1 copy of the rows it reads
    (the window, the visible pool / indexer pool entries)."""
    m = d["m"]
    ctx = d["ctx_lens"].numpy()
    maxc = int(ctx[seqs].max())
    n = len(seqs)
    kv_rows, kv_bt = [], np.full((n, maxc), -1, dtype=np.int32)
    pool_rows, ipool_rows = [], []
    maxn = max(1, maxc // m)
    pbt = np.full((n, maxn), -1, dtype=np.int32)
    nk = npl = 0
    for i, s in enumerate(seqs):
        c = int(ctx[s])
        lo = max(0, c - wl.W)
        kv_rows.append(logical(d["kv_pages"], d["kv_block_table"], s, lo, c))
        kv_bt[i, lo:c] = np.arange(nk, nk + c - lo)
        nk += c - lo
        nv = c // m
        if nv:
            pool_rows.append(logical(d["pool_pages"], d["pool_block_table"], s, 0, nv))
            if layer == "csa":
                ipool_rows.append(logical(d["idx_pool_pages"], d["pool_block_table"], s, 0, nv))
            pbt[i, :nv] = np.arange(npl, npl + nv)
            npl += nv
    kvp = np.concatenate(kv_rows)[:, None, :]
    pp = np.concatenate(pool_rows)[:, None, :] if pool_rows else np.zeros((1, 1, wl.D))
    ipp = np.concatenate(ipool_rows)[:, None, :] if ipool_rows else None
    p = oracle.OracleParams(1, maxc, wl.H, wl.D, wl.R, wl.theta, wl.W, m=m,
                            L=wl.L if layer == "csa" else m, nI=wl.nI if layer == "csa" else 0,
                            cI=wl.cI if layer == "csa" else 0, k=wl.k if layer == "csa" else 0)
    return oracle.decode(p, d["q"][seqs], kvp, kv_bt, ctx[seqs], 1, pool_pages=pp,
                         idx_pool_pages=ipp, pool_block_table=pbt,
                         q_idx=None if layer != "csa" else d["q_idx"][seqs],
                         w_idx=None if layer != "csa" else d["w_idx"][seqs], sinks=d["sinks"],
                         topk_in=topk_in)


def gpu_decode(wl, d, layer, max_ctx):
    import sparse_attention_compressor_b200 as sac
    dev = torch.device("cuda", 0)
    m = d["m"]
    p = sac.make_params(1, max_ctx, wl.H, wl.D, wl.R, wl.theta, m=m,
                        win_len=wl.L if layer == "csa" else m, sliding_window=wl.W,
                        n_idx_heads=wl.nI if layer == "csa" else 0,
                        idx_dim=wl.cI if layer == "csa" else 0, topk=wl.k if layer == "csa" else 0,
                        dtype=wl.dtype)
    g = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in d.items()}
    nseq = g["q"].shape[0]
    o = torch.empty_like(g["q"])
    ps = wl.page_size
    kind = sac.SAC_KIND_HCA if layer == "hca" else sac.SAC_KIND_CSA
    ws = torch.empty(sac.sac_decode_workspace_size(p, kind, nseq), dtype=torch.uint8, device=dev)
    if layer == "hca":
        sac.hca_decode(p, nseq, g["q"], g["kv_pages"], g["kv_block_table"], g["ctx_lens"], ps,
                       g["pool_pages"], g["pool_block_table"], g["sinks"], o, ws)
        assert sac.sac_device_status(ws) == 0, "a kernel reported a device-side wait timeout"
        return o.cpu(), None
    tk = torch.empty((nseq, wl.k), dtype=torch.int32, device=dev)
    sac.csa_decode(p, nseq, g["q"], g["kv_pages"], g["kv_block_table"], g["ctx_lens"], ps,
                   g["pool_pages"], g["idx_pool_pages"], g["pool_block_table"], g["q_idx"],
                   g["w_idx"], g["sinks"], o, tk, ws)
    assert sac.sac_device_status(ws) == 0, "a kernel reported a device-side wait timeout"
    return o.cpu(), tk.cpu()


def small_decode_workload():
    return replace(W.WORKLOADS["decode_bf16"], nseq=6, ctx_lo=1, ctx_hi=3000, seed=99)


@pytest.mark.parametrize("layer", ["csa", "hca"])
@pytest.mark.parametrize("which", ["small", "full", "ps24", "ps12"])
def test_decode_parity(layer, which):
    """Decode of both layers against the oracle. The page sizes: 64 (the workload's), 24 (the
    paged indexer's box loads in runs of 8 rows) and 12 (not a multiple of 8: its row gathers)."""
    if which == "full":
        wl = W.WORKLOADS["decode_bf16"]
    elif which.startswith("ps"):
        wl = replace(small_decode_workload(), page_size=int(which[2:]))
    else:
        wl = small_decode_workload()
    d = W.decode_inputs(wl, layer)
    o, tk = gpu_decode(wl, d, layer, int(d["ctx_lens"].max()))
    nseq = wl.nseq
    seqs = np.arange(0, nseq, 8) if which == "full" else np.arange(nseq)
    gsel = None
    if layer == "csa":
        # oracle's own selections (via its decode) and the tie-band comparison on its scores
        ctx = d["ctx_lens"].numpy()
        _, osel = oracle_decode(wl, d, layer, seqs)
        for i, s in enumerate(seqs):
            nv = int(ctx[s]) // wl.m
            kp = logical(d["idx_pool_pages"], d["pool_block_table"], s, 0, nv) if nv else \
                np.zeros((0, wl.cI))
            sc = oracle.index_scores(d["q_idx"][s], d["w_idx"][s], kp, nv) if nv else np.zeros(0)
            check_topk_row(tk[s].numpy(), osel[i], sc, nv, wl.k, f"seq {s}")
        gsel = tk.numpy()[seqs]
    ref, _ = oracle_decode(wl, d, layer, seqs, topk_in=gsel)
    assert_close(o[torch.from_numpy(seqs)], ref, wl.dtype, f"{layer} decode o")
