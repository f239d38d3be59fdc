"""Query-sharded prefill (sparse_attention_compressor_b200.sharded).

CPU, gloo, world size 2: the plan, the halo exchange and the in-place pool all-gather of the
sharded step, driven on CPU tensors, with the fp64 oracle standing in for the per-rank kernels.
Each rank pools the entries whose windows close in its slice from its halo + slice rows only,
the all-gather assembles the pools, and each rank's query rows computed against the gathered
pools and its own window rows must equal the single-process oracle's rows exactly (the same fp64
arithmetic on the same values).

GPU, one device: the per-rank steps of the library (chunk append, pool all-gather, chunk
attention) for two ranks run one after the other on one GPU -- the all-gather done by copying
each rank's entries, since no kernel of one rank waits on another -- and their outputs match the
oracle row by row."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _wl(kind):
    from sparse_attention_compressor_b200 import workloads as W
    if kind == "csa":
        return W.Workload("csa_shard_test", "csa", "f32", B=1, S=512, H=4, D=64, R=16,
                          theta=10000.0, m=4, L=8, W=64, nI=2, cI=32, k=8, seed=210)
    return W.Workload("hca_shard_test", "hca", "f32", B=1, S=512, H=4, D=64, R=16,
                      theta=10000.0, m=32, L=32, W=64, seed=211)


def _oracle_params(wl):
    import oracle
    return oracle.OracleParams(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, wl.W, m=wl.m, L=wl.L,
                               nI=wl.nI, cI=wl.cI, k=wl.k)


def _entries(rows, t0, e0, e1, m, L, u, bias):
    """Entries w in [e0, e1) pooled (oracle compressor) from rows t0.. of the stream, each from
    its own window [(w+1)m - L, (w+1)m) clipped at 0."""
    import oracle
    out = []
    for w in range(e0, e1):
        hi = (w + 1) * m
        lo = max(0, hi - L)
        assert lo >= t0, "a window of the slice reaches past the halo"
        win = rows[lo - t0:hi - t0][None]
        out.append(oracle.compress(win, u, bias, m, L)[0, -1])
    return np.stack(out)


def _worker(rank, world, port, kind, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import oracle
    from sparse_attention_compressor_b200 import sharded
    from sparse_attention_compressor_b200 import workloads as W
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        wl = _wl(kind)
        x = W.prefill_inputs(wl)
        sp = sharded.plan(wl.S, world, rank, wl.m, wl.L, wl.W, page_size=64)
        kv = x["kv"][0].double()
        # 1. halo: the rows before the slice come from the left neighbour
        halo = sharded.exchange_halo(kv[sp.s0:sp.s1], sp.h)
        assert torch.equal(halo, kv[sp.t0:sp.s0])
        rows = torch.cat([halo, kv[sp.s0:sp.s1]]).numpy()
        # 2. the slice's entries from its own rows, rotated at their global positions
        p = _oracle_params(wl)
        N = wl.S // wl.m
        pool = torch.zeros((N, wl.D), dtype=torch.float64)
        ent = _entries(rows, sp.t0, sp.e0, sp.e1, wl.m, wl.L, x["cmp_gate"], x["cmp_bias"])
        for i, w in enumerate(range(sp.e0, sp.e1)):
            ent[i] = oracle.rope(ent[i], wl.R, wl.theta, w * wl.m)
        pool[sp.e0:sp.e1] = torch.from_numpy(ent)
        # 3. all-gather, in place
        sharded.gather_entries(pool, sp.e0, sp.e1)
        kw = {}
        if kind == "csa":
            ki = x["k_idx"][0].double()
            ihalo = sharded.exchange_halo(ki[sp.s0:sp.s1], sp.h)
            irows = torch.cat([ihalo, ki[sp.s0:sp.s1]]).numpy()
            ipool = torch.zeros((N, wl.cI), dtype=torch.float64)
            ipool[sp.e0:sp.e1] = torch.from_numpy(
                _entries(irows, sp.t0, sp.e0, sp.e1, wl.m, wl.L, x["idx_gate"], x["idx_bias"]))
            sharded.gather_entries(ipool, sp.e0, sp.e1)
            kw = dict(idx_pool_pages=ipool.numpy()[:, None, :],
                      q_idx=x["q_idx"][0, sp.s0:sp.s1], w_idx=x["w_idx"][0, sp.s0:sp.s1])
        # 4. this rank's rows: one query per row over a page-size-1 cache of its rotated rows
        rot = np.stack([oracle.rope(rows[j], wl.R, wl.theta, sp.t0 + j) for j in range(len(rows))])
        n = sp.n
        kbt = np.full((n, sp.s1), -1, dtype=np.int32)
        kbt[:, sp.t0:sp.s1] = np.arange(sp.s1 - sp.t0)
        ctx = np.arange(sp.s0, sp.s1, dtype=np.int32) + 1
        pbt = np.tile(np.arange(N, dtype=np.int32), (n, 1))
        o, _ = oracle.decode(p, x["q"][0, sp.s0:sp.s1], rot[:, None, :], kbt, ctx, 1,
                             pool_pages=pool.numpy()[:, None, :], pool_block_table=pbt,
                             sinks=x["sinks"], **kw)
        out.put((rank, pool.numpy(), o))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_sharded_decomposition_equals_single_process_oracle(kind):
    import oracle
    from sparse_attention_compressor_b200 import workloads as W
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, kind, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get() for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    wl = _wl(kind)
    x = W.prefill_inputs(wl)
    p = _oracle_params(wl)
    if kind == "csa":
        o, _, pool, _ = oracle.csa_forward(p, x["q"], x["kv"], x["cmp_gate"], x["cmp_bias"],
                                           x["q_idx"], x["w_idx"], x["k_idx"], x["idx_gate"],
                                           x["idx_bias"], x["sinks"])
    else:
        o, pool = oracle.hca_forward(p, x["q"], x["kv"], x["cmp_gate"], x["cmp_bias"], x["sinks"])
    o = o.reshape(wl.S, wl.H, wl.D)
    n = wl.S // world
    for rank, gathered, orow in res:
        np.testing.assert_array_equal(gathered, pool[0])  # every rank holds the whole pool
        np.testing.assert_allclose(orow, o[rank * n:(rank + 1) * n], rtol=0, atol=1e-12)


def test_plan_covers_the_sequence_with_page_aligned_slices():
    from sparse_attention_compressor_b200 import sharded
    S, world = 131072, 8
    plans = [sharded.plan(S, world, r, 4, 8, 128) for r in range(world)]
    assert plans[0].t0 == 0 and plans[-1].s1 == S
    for a, b in zip(plans, plans[1:]):
        assert a.s1 == b.s0 and a.e1 == b.e0
        assert b.s0 - b.t0 == b.h == 128 and b.t0 % 64 == 0
    assert sum(p.e1 - p.e0 for p in plans) == S // 4
    with pytest.raises(ValueError):
        sharded.plan(1000, 3, 0, 4, 8, 128)       # slices not whole pages
    with pytest.raises(ValueError):
        sharded.plan(512, 8, 0, 4, 8, 128)        # slices shorter than the halo


# ------------------------------------------------------------------------------------------------
# GPU: the library's per-rank steps for two emulated ranks on one device
# ------------------------------------------------------------------------------------------------
@pytest.mark.gpu
@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_sharded_steps_on_one_gpu_match_oracle(kind):
    import oracle
    import sparse_attention_compressor_b200 as sac
    from sparse_attention_compressor_b200 import sharded
    from sparse_attention_compressor_b200 import workloads as W
    from parity import assert_close, check_topk_row, oracle_params
    wl = (W.Workload("csa_shard_gpu", "csa", "bf16", B=1, S=2048, m=4, L=8, nI=64, cI=128,
                     k=64, seed=212) if kind == "csa" else
          W.Workload("hca_shard_gpu", "hca", "bf16", B=1, S=2048, m=128, L=128, seed=213))
    x = W.prefill_inputs(wl)
    dev = torch.device("cuda", 0)
    g = {k: v.to(dev) for k, v in x.items()}
    world = 2
    skind = sac.SAC_KIND_CSA if kind == "csa" else sac.SAC_KIND_HCA
    p = sac.make_params(1, wl.S, wl.H, wl.D, wl.R, wl.theta, m=wl.m, win_len=wl.L,
                        sliding_window=wl.W, n_idx_heads=wl.nI, idx_dim=wl.cI, topk=wl.k)
    plans = [sharded.plan(wl.S, world, r, wl.m, wl.L, wl.W) for r in range(world)]
    caches = []
    for sp in plans:  # local compress of each rank from its own halo + slice rows
        kv = g["kv"][0, sp.t0:sp.s1]
        ki = g["k_idx"][0, sp.t0:sp.s1] if kind == "csa" else None
        caches.append(sharded.local_caches(sp, skind, p, kv, g["cmp_gate"], g["cmp_bias"], ki,
                                           g.get("idx_gate"), g.get("idx_bias")))
    names = ["pool_pages"] + (["idx_pool_pages"] if kind == "csa" else [])
    for name in names:  # the all-gather: every rank's own entries into every rank's pool
        for src, sp in zip(caches, plans):
            for dst in caches:
                sharded.pool_rows(dst, name)[sp.e0:sp.e1] = sharded.pool_rows(src, name)[sp.e0:sp.e1]
    o = torch.empty_like(g["q"][0])
    tk = torch.empty((wl.S, wl.k), dtype=torch.int32, device=dev) if kind == "csa" else None
    for sp, c in zip(plans, caches):
        kw = {}
        if kind == "csa":
            kw = dict(q_idx=g["q_idx"][0, sp.s0:sp.s1][None].contiguous(),
                      w_idx=g["w_idx"][0, sp.s0:sp.s1][None].contiguous(),
                      topk_out=tk[sp.s0:sp.s1][None])
        sharded.local_attention(sp, skind, p, c, g["q"][0, sp.s0:sp.s1][None].contiguous(),
                                g["sinks"], o[sp.s0:sp.s1][None], **kw)
    torch.cuda.synchronize()
    po = oracle_params(wl)
    n = wl.S
    rows = np.arange(n)
    if kind == "csa":
        sc = oracle.csa_index_scores(po, x["q_idx"].reshape(n, wl.nI, wl.cI),
                                     x["w_idx"].reshape(n, wl.nI), x["k_idx"], x["idx_gate"],
                                     x["idx_bias"], rows)
        gsel = tk.cpu().numpy()
        for t in range(n):
            nvis = (t + 1) // wl.m
            check_topk_row(gsel[t], oracle.topk(sc[t], nvis, wl.k), sc[t], nvis, wl.k, f"row {t}")
        ref, _, pool, ipool = oracle.csa_forward(po, x["q"], x["kv"], x["cmp_gate"],
                                                 x["cmp_bias"], x["q_idx"], x["w_idx"],
                                                 x["k_idx"], x["idx_gate"], x["idx_bias"],
                                                 x["sinks"], topk_in=gsel)
        for c in caches:
            assert_close(sharded.pool_rows(c, "idx_pool_pages")[:n // wl.m].cpu(), ipool[0],
                         "bf16", "indexer pool")
    else:
        ref, pool = oracle.hca_forward(po, x["q"], x["kv"], x["cmp_gate"], x["cmp_bias"],
                                       x["sinks"])
    for c in caches:
        assert_close(sharded.pool_rows(c, "pool_pages")[:n // wl.m].cpu(), pool[0], "bf16", "pool")
    assert_close(o.cpu(), ref.reshape(n, wl.H, wl.D), "bf16", "o")
