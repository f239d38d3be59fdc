"""GPU parity of chunked prefill over the paged caches: a stream appended in chunks of varied
sizes (after a few single-token decode appends, so that sequences sit at different offsets)
through prefill_chunk_append must leave the caches the definitions give — kv rows rotated at their
positions, pool entries the compressor's gated pools of their windows (rotated; the indexer pool
un-rotated), the ring holding the last win_len rows — and the *_prefill_chunk attention of each
sequence's last chunk must match the oracle's decode of every chunk row at ctx = t + 1 (the
oracle's pin: a decode at ctx = t + 1 over a cache holding later tokens equals the prefill row t)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_compressor_b200 as sac
from parity import KIND, assert_close, check_topk_row
from sparse_attention_compressor_b200 import workloads as W

pytestmark = pytest.mark.gpu

OFFSETS = [0, 3, 11]               # tokens each sequence gets from decode_append first
CHUNKS = [1, 5, 37, 2, 130, 64]    # then chunks of these sizes (the last one is attended)
POS0 = 5


def wl_case(kind, dtype):
    if dtype == "bf16":
        base = dict(H=64, D=512, R=64, theta=160000.0, W=128)
    else:
        base = dict(H=4, D=64, R=16, theta=10000.0, W=64)
    if kind == "csa":
        base.update(m=4, L=8, nI=64 if dtype == "bf16" else 4, cI=128 if dtype == "bf16" else 32,
                    k=16 if dtype == "bf16" else 8)
    elif kind == "hca":
        base.update(m=128, L=128) if dtype == "bf16" else base.update(m=16, L=16)
    return W.Workload(f"chunk_{kind}_{dtype}", kind, dtype, B=3, S=300, seed=37, **base)


def paged(nseq, rows, width, page_size, dt, dev, seed):
    maxp = (rows + page_size - 1) // page_size
    perm = np.random.default_rng(seed).permutation(nseq * maxp).astype(np.int32)
    bt = torch.from_numpy(perm.reshape(nseq, maxp)).to(dev)
    pages = torch.zeros((nseq * maxp, page_size, width), dtype=dt, device=dev)
    return pages, bt


def logical(pages, bt, s, n):
    ps = pages.shape[1]
    return torch.stack([pages[int(bt[s, j // ps]), j % ps] for j in range(n)]) if n else None


def rounded(a, dtype):
    return np.vectorize(oracle.round_bf16)(a) if dtype == "bf16" else a


def build_caches(kind, dtype):
    """Append the stream through the GPU path; returns everything the checks need."""
    wl = wl_case(kind, dtype)
    dev = torch.device("cuda", 0)
    x = W.prefill_inputs(wl, with_queries=True)
    dt = wl.torch_dtype
    p = sac.make_params(1, wl.S, wl.H, wl.D, wl.R, wl.theta, m=wl.m, win_len=wl.L,
                        sliding_window=wl.W, n_idx_heads=wl.nI, idx_dim=wl.cI, topk=wl.k,
                        pos0=POS0, dtype=dtype)
    ps = 16
    g = {k: v.to(dev).contiguous() for k, v in x.items()}
    kvp, kvbt = paged(wl.B, wl.S, wl.D, ps, dt, dev, 1)
    c = dict(kv_pages=kvp, kv_block_table=kvbt)
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
    # single tokens first (a sequence at its offset re-appends its last token: idempotent)
    for i in range(1, max(OFFSETS) + 1):
        ctxl = [min(i, o) for o in OFFSETS]
        ctx = torch.tensor(ctxl, dtype=torch.int32, device=dev)
        rows = [max(cc - 1, 0) for cc in ctxl]
        kw = dict(extra)
        if kind == "csa":
            kw["k_idx_new"] = torch.stack([g["k_idx"][s, rows[s]] for s in range(wl.B)]).contiguous()
        kv_new = torch.stack([g["kv"][s, rows[s]] for s in range(wl.B)]).contiguous()
        sac.decode_append(p, KIND[kind], wl.B, ctx, kv_new, kvp, kvbt, ps, **kw)
    done = list(OFFSETS)
    for n in CHUNKS:
        ctxl = [d + n for d in done]
        ctx = torch.tensor(ctxl, dtype=torch.int32, device=dev)
        kv_new = torch.stack([g["kv"][s, ctxl[s] - n:ctxl[s]] for s in range(wl.B)]).contiguous()
        kw = dict(extra)
        if kind == "csa":
            kw["k_idx_new"] = torch.stack([g["k_idx"][s, ctxl[s] - n:ctxl[s]]
                                           for s in range(wl.B)]).contiguous()
        sac.prefill_chunk_append(p, KIND[kind], wl.B, n, ctx, kv_new, kvp, kvbt, ps, **kw)
        done = ctxl
    torch.cuda.synchronize()
    return wl, x, g, p, ps, c, extra, done


@pytest.mark.parametrize("kind,dtype", [("csa", "bf16"), ("hca", "bf16"), ("csa", "f32"),
                                        ("hca", "f32"), ("swa", "f32")])
def test_chunk_append_matches_definitions(kind, dtype):
    wl, x, g, p, ps, c, extra, lens = build_caches(kind, dtype)
    for s, n in enumerate(lens):
        kv = x["kv"][s, :n].double().numpy()
        ref = np.stack([oracle.rope(kv[j], wl.R, wl.theta, POS0 + j) for j in range(n)])
        assert_close(logical(c["kv_pages"], c["kv_block_table"], s, n).cpu(),
                     rounded(ref, dtype), dtype, f"seq {s} kv pages")
        if kind == "swa":
            continue
        nv = n // wl.m
        pool = oracle.compress(kv[None], x["cmp_gate"].double().numpy(),
                               x["cmp_bias"].double().numpy(), wl.m, wl.L)[0]
        ref = np.stack([oracle.rope(pool[w], wl.R, wl.theta, POS0 + w * wl.m) for w in range(nv)])
        got = logical(extra["pool_pages"], extra["pool_block_table"], s, nv).cpu()
        assert_close(got, rounded(ref, dtype), dtype, f"seq {s} pool pages")
        if kind == "csa":
            ki = x["k_idx"][s, :n].double().numpy()
            iref = oracle.compress(ki[None], x["idx_gate"].double().numpy(),
                                   x["idx_bias"].double().numpy(), wl.m, wl.L)[0]
            got = logical(extra["idx_pool_pages"], extra["pool_block_table"], s, nv).cpu()
            assert_close(got, rounded(iref, dtype), dtype, f"seq {s} indexer pool")
        ring = extra["cmp_state"][s].cpu()
        for j in range(max(0, n - wl.L), n):
            assert torch.equal(ring[j % wl.L], x["kv"][s, j]), (s, j)


def oracle_caches(wl, x, lens, dtype):
    """Caches from the definitions (page size 1, one block-table row per sequence)."""
    D = wl.D
    kv_rows, pool_rows, ipool_rows = [], [], []
    maxc = max(lens)
    maxn = max(1, maxc // wl.m) if wl.m else 1
    kbt = np.full((wl.B, maxc), -1, dtype=np.int32)
    pbt = np.full((wl.B, maxn), -1, dtype=np.int32)
    nk = npl = 0
    for s, n in enumerate(lens):
        kv = x["kv"][s, :n].double().numpy()
        kv_rows.append(rounded(np.stack([oracle.rope(kv[j], wl.R, wl.theta, POS0 + j)
                                         for j in range(n)]), dtype))
        kbt[s, :n] = np.arange(nk, nk + n)
        nk += n
        if wl.m:
            nv = n // wl.m
            pool = oracle.compress(kv[None], x["cmp_gate"].double().numpy(),
                                   x["cmp_bias"].double().numpy(), wl.m, wl.L)[0]
            pool_rows.append(rounded(np.stack([oracle.rope(pool[w], wl.R, wl.theta,
                                                           POS0 + w * wl.m)
                                               for w in range(nv)]), dtype))
            if wl.kind == "csa":
                ki = x["k_idx"][s, :n].double().numpy()
                ipool_rows.append(rounded(oracle.compress(
                    ki[None], x["idx_gate"].double().numpy(), x["idx_bias"].double().numpy(),
                    wl.m, wl.L)[0], dtype))
            pbt[s, :nv] = np.arange(npl, npl + nv)
            npl += nv
    out = {"kvp": np.concatenate(kv_rows)[:, None, :], "kbt": kbt, "pbt": pbt}
    if wl.m:
        out["pp"] = np.concatenate(pool_rows)[:, None, :]
    if wl.kind == "csa":
        out["ipp"] = np.concatenate(ipool_rows)[:, None, :]
    return out


@pytest.mark.parametrize("kind,dtype,n", [("csa", "bf16", 64), ("hca", "bf16", 64),
                                          ("swa", "bf16", 64), ("csa", "f32", 64),
                                          ("hca", "f32", 64), ("swa", "f32", 64),
                                          # 3 x 8 rows: each row's keys split over several CTAs
                                          ("csa", "bf16", 8), ("hca", "bf16", 8)])
def test_chunk_attention_matches_oracle(kind, dtype, n):
    """The last n tokens of each sequence (all in the caches) attended as one chunk."""
    wl, x, g, p, ps, c, extra, lens = build_caches(kind, dtype)
    dev = torch.device("cuda", 0)
    ctx = torch.tensor(lens, dtype=torch.int32, device=dev)
    rows = [(s, t) for s in range(wl.B) for t in range(lens[s] - n, lens[s])]
    q = torch.stack([g["q"][s, t] for s, t in rows]).reshape(wl.B, n, wl.H, wl.D).contiguous()
    o = torch.full_like(q, float("nan"))
    ws = torch.empty(sac.sac_chunk_workspace_size(p, KIND[kind], wl.B, n), dtype=torch.uint8,
                     device=dev)
    tk = None
    if kind == "swa":
        sac.swa_prefill_chunk(p, wl.B, n, q, c["kv_pages"], c["kv_block_table"], ctx, ps,
                              g["sinks"], o, ws)
    elif kind == "hca":
        sac.hca_prefill_chunk(p, wl.B, n, q, c["kv_pages"], c["kv_block_table"], ctx, ps,
                              extra["pool_pages"], extra["pool_block_table"], g["sinks"], o, ws)
    else:
        q_idx = torch.stack([g["q_idx"][s, t] for s, t in rows]).contiguous()
        w_idx = torch.stack([g["w_idx"][s, t] for s, t in rows]).contiguous()
        tk = torch.empty((wl.B * n, wl.k), dtype=torch.int32, device=dev)
        sac.csa_prefill_chunk(p, wl.B, n, q, c["kv_pages"], c["kv_block_table"], ctx, ps,
                              extra["pool_pages"], extra["idx_pool_pages"],
                              extra["pool_block_table"], q_idx, w_idx, g["sinks"], o, tk, ws)
    assert sac.sac_device_status(ws) == 0, "a kernel reported a device-side wait timeout"
    torch.cuda.synchronize()

    oc = oracle_caches(wl, x, lens, dtype)
    seq_of = np.array([s for s, _ in rows])
    op = oracle.OracleParams(1, wl.S, wl.H, wl.D, wl.R, wl.theta, wl.W, m=wl.m, L=wl.L,
                             nI=wl.nI, cI=wl.cI, k=wl.k, pos0=POS0)
    qo = torch.stack([x["q"][s, t] for s, t in rows]).double().numpy()
    kw = dict(pool_pages=oc.get("pp"), idx_pool_pages=oc.get("ipp"),
              pool_block_table=oc["pbt"][seq_of] if wl.m else None, sinks=x["sinks"])
    octx = np.array([t + 1 for _, t in rows], dtype=np.int32)
    gsel = None
    if kind == "csa":
        qI = torch.stack([x["q_idx"][s, t] for s, t in rows]).double().numpy()
        wI = torch.stack([x["w_idx"][s, t] for s, t in rows]).double().numpy()
        kw.update(q_idx=qI, w_idx=wI)
        _, osel = oracle.decode(op, qo, oc["kvp"], oc["kbt"][seq_of], octx, 1, **kw)
        gsel = tk.cpu().numpy()
        for i, (s, t) in enumerate(rows):
            nv = (t + 1) // wl.m
            kp = oc["ipp"][oc["pbt"][s, :nv], 0] if nv else np.zeros((0, wl.cI))
            sc = oracle.index_scores(qI[i], wI[i], kp, nv) if nv else np.zeros(0)
            check_topk_row(gsel[i], osel[i], sc, nv, wl.k, f"seq {s} t {t}")
    ref, _ = oracle.decode(op, qo, oc["kvp"], oc["kbt"][seq_of], octx, 1, topk_in=gsel, **kw)
    assert_close(o.reshape(wl.B * n, wl.H, wl.D).cpu(), ref, dtype, f"{kind} chunk o")


def test_decode_equals_chunk_of_one():
    """A one-token chunk is a decode step: same caches, same outputs, bit for bit."""
    wl, x, g, p, ps, c, extra, lens = build_caches("csa", "bf16")
    dev = torch.device("cuda", 0)
    ctx = torch.tensor(lens, dtype=torch.int32, device=dev)
    q = torch.stack([g["q"][s, lens[s] - 1] for s in range(wl.B)]).contiguous()
    q_idx = torch.stack([g["q_idx"][s, lens[s] - 1] for s in range(wl.B)]).contiguous()
    w_idx = torch.stack([g["w_idx"][s, lens[s] - 1] for s in range(wl.B)]).contiguous()
    outs = []
    for chunk in (False, True):
        o = torch.empty_like(q)
        tk = torch.empty((wl.B, wl.k), dtype=torch.int32, device=dev)
        args = (c["kv_pages"], c["kv_block_table"], ctx, ps, extra["pool_pages"],
                extra["idx_pool_pages"], extra["pool_block_table"], q_idx, w_idx, g["sinks"], o,
                tk)
        if chunk:
            ws = torch.empty(sac.sac_chunk_workspace_size(p, sac.SAC_KIND_CSA, wl.B, 1),
                             dtype=torch.uint8, device=dev)
            sac.csa_prefill_chunk(p, wl.B, 1, q, *args, ws)
        else:
            ws = torch.empty(sac.sac_decode_workspace_size(p, sac.SAC_KIND_CSA, wl.B),
                             dtype=torch.uint8, device=dev)
            sac.csa_decode(p, wl.B, q, *args, ws)
        torch.cuda.synchronize()
        outs.append((o.cpu(), tk.cpu()))
    assert torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][0], outs[1][0])
