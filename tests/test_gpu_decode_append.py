"""GPU parity of the decode cache append: tokens appended one by one through decode_append must
leave the same caches as the definitions applied to the whole token stream — each kv row rotated
at its position, and each closed pool entry the compressor's gated pool of its window, rotated at
its entry position (the indexer pool un-rotated). Sequences of different lengths, pages smaller
than a window, a shifted pos0 and a repeated append of the last token (idempotent) are covered."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_compressor_b200 as sac
from parity import KIND, assert_close
from sparse_attention_compressor_b200 import workloads as W

pytestmark = pytest.mark.gpu


def wl_case(kind, dtype):
    if dtype == "bf16":
        base = dict(H=64, D=512, R=64, theta=160000.0, W=128)
    else:
        base = dict(H=4, D=64, R=16, theta=10000.0, W=64)
    if kind == "csa":
        base.update(m=4, L=8, nI=4, cI=128 if dtype == "bf16" else 32, k=8)
    elif kind == "hca":
        base.update(m=128, L=128) if dtype == "bf16" else base.update(m=16, L=16)
    return W.Workload(f"append_{kind}_{dtype}", kind, dtype, B=3, S=300, seed=31, **base)


def paged(nseq, rows, width, page_size, dt, dev, seed):
    maxp = (rows + page_size - 1) // page_size
    perm = np.random.default_rng(seed).permutation(nseq * maxp).astype(np.int32)
    bt = torch.from_numpy(perm.reshape(nseq, maxp)).to(dev)
    pages = torch.zeros((nseq * maxp, page_size, width), dtype=dt, device=dev)
    return pages, bt


def logical(pages, bt, s, n):
    ps = pages.shape[1]
    return torch.stack([pages[int(bt[s, j // ps]), j % ps] for j in range(n)]) if n else None


@pytest.mark.parametrize("kind,dtype", [("csa", "bf16"), ("hca", "bf16"), ("csa", "f32"),
                                        ("hca", "f32"), ("swa", "f32")])
def test_decode_append_matches_definitions(kind, dtype):
    wl = wl_case(kind, dtype)
    dev = torch.device("cuda", 0)
    x = W.prefill_inputs(wl, with_queries=False)
    lens = [wl.S, 261, 1]
    pos0 = 5
    dt = wl.torch_dtype
    p = sac.make_params(1, wl.S, wl.H, wl.D, wl.R, wl.theta, m=wl.m, win_len=wl.L,
                        sliding_window=wl.W, n_idx_heads=wl.nI, idx_dim=wl.cI, topk=wl.k,
                        pos0=pos0, dtype=dtype)
    ps = 16
    kvp, kvbt = paged(wl.B, wl.S, wl.D, ps, dt, dev, 1)
    g = {k: v.to(dev).contiguous() for k, v in x.items()}
    extra = {}
    if kind != "swa":
        pp, pbt = paged(wl.B, max(wl.S // wl.m, 1), wl.D, ps, dt, dev, 2)
        extra.update(cmp_state=torch.zeros((wl.B, wl.L, wl.D), dtype=dt, device=dev),
                     cmp_gate=g["cmp_gate"], cmp_bias=g["cmp_bias"], pool_pages=pp,
                     pool_block_table=pbt)
    if kind == "csa":
        ipp = torch.zeros((pp.shape[0], ps, wl.cI), dtype=dt, device=dev)
        extra.update(idx_state=torch.zeros((wl.B, wl.L, wl.cI), dtype=dt, device=dev),
                     idx_gate=g["idx_gate"], idx_bias=g["idx_bias"], idx_pool_pages=ipp)
    for i in range(wl.S + 1):  # the last step repeats every sequence's last token
        t = [min(i, n - 1) for n in lens]
        ctx = torch.tensor([ti + 1 for ti in t], dtype=torch.int32, device=dev)
        kv_new = torch.stack([g["kv"][s, t[s]] for s in range(wl.B)]).contiguous()
        kw = dict(extra)
        if kind == "csa":
            kw["k_idx_new"] = torch.stack([g["k_idx"][s, t[s]] for s in range(wl.B)]).contiguous()
        sac.decode_append(p, KIND[kind], wl.B, ctx, kv_new, kvp, kvbt, ps, **kw)
    torch.cuda.synchronize()

    for s, n in enumerate(lens):
        kv = x["kv"][s, :n].double().numpy()
        ref = np.stack([oracle.rope(kv[j], wl.R, wl.theta, pos0 + j) for j in range(n)])
        if dtype == "bf16":  # the pages store bf16: compare with the rounded definition
            ref = np.vectorize(oracle.round_bf16)(ref)
        assert_close(logical(kvp, kvbt, s, n).cpu(), ref, dtype, f"seq {s} kv pages")
        if kind == "swa":
            continue
        nv = n // wl.m
        if nv == 0:
            continue
        pool = oracle.compress(kv[None], x["cmp_gate"].double().numpy(),
                               x["cmp_bias"].double().numpy(), wl.m, wl.L)[0]
        ref = np.stack([oracle.rope(pool[w], wl.R, wl.theta, pos0 + w * wl.m) for w in range(nv)])
        if dtype == "bf16":
            ref = np.vectorize(oracle.round_bf16)(ref)
        assert_close(logical(pp, pbt, s, nv).cpu(), ref, dtype, f"seq {s} pool pages")
        if kind == "csa":
            ki = x["k_idx"][s, :n].double().numpy()
            iref = oracle.compress(ki[None], x["idx_gate"].double().numpy(),
                                   x["idx_bias"].double().numpy(), wl.m, wl.L)[0]
            if dtype == "bf16":
                iref = np.vectorize(oracle.round_bf16)(iref)
            assert_close(logical(ipp, pbt, s, nv).cpu(), iref, dtype, f"seq {s} indexer pool")
        # the ring holds the last L un-rotated rows, row j in slot j mod L
        ring = extra["cmp_state"][s].cpu()
        for j in range(max(0, n - wl.L), n):
            assert torch.equal(ring[j % wl.L], x["kv"][s, j]), (s, j)
