"""A decode context length above p.S -- beyond the rows the block tables cover -- on the GPU.

Every kernel of a decode step reads the context length before any cache row, so a sequence with
ctx = S + 1 must read and write no cache row: its attention row is skipped (output undefined), its
top-k row is all -1, the cache append leaves its pages and ring untouched, and the call records
status 4 in the workspace's status word. The other sequences of the same call stay correct."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import sparse_attention_compressor_b200 as sac
from parity import assert_close
from sparse_attention_compressor_b200 import workloads as W
from test_gpu_parity import oracle_decode

pytestmark = pytest.mark.gpu

BAD_INPUT = 4  # status: a context length beyond the block tables


def _workload():
    return replace(W.WORKLOADS["decode_bf16"], nseq=5, ctx_lo=200, ctx_hi=2500, seed=123)


def _params(wl, layer, S, m):
    return sac.make_params(1, S, wl.H, wl.D, wl.R, wl.theta, m=m,
                           win_len=wl.L if layer == "csa" else m, sliding_window=wl.W,
                           n_idx_heads=wl.nI if layer == "csa" else 0,
                           idx_dim=wl.cI if layer == "csa" else 0,
                           topk=wl.k if layer == "csa" else 0, dtype=wl.dtype)


@pytest.mark.parametrize("layer", ["csa", "hca"])
def test_decode_skips_a_context_beyond_the_block_tables(layer):
    wl = _workload()
    d = W.decode_inputs(wl, layer)
    dev = torch.device("cuda", 0)
    S = int(d["ctx_lens"].max())  # the block tables cover S rows of every sequence
    bad = 2
    p = _params(wl, layer, S, d["m"])
    g = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in d.items()}
    g["ctx_lens"][bad] = S + 1
    nseq = wl.nseq
    o = torch.zeros_like(g["q"])
    kind = sac.SAC_KIND_CSA if layer == "csa" else sac.SAC_KIND_HCA
    ws = torch.empty(sac.sac_decode_workspace_size(p, kind, nseq), dtype=torch.uint8, device=dev)
    tk = None
    if layer == "csa":
        tk = torch.zeros((nseq, wl.k), dtype=torch.int32, device=dev)
        sac.csa_decode(p, nseq, g["q"], g["kv_pages"], g["kv_block_table"], g["ctx_lens"],
                       wl.page_size, g["pool_pages"], g["idx_pool_pages"],
                       g["pool_block_table"], g["q_idx"], g["w_idx"], g["sinks"], o, tk, ws)
    else:
        sac.hca_decode(p, nseq, g["q"], g["kv_pages"], g["kv_block_table"], g["ctx_lens"],
                       wl.page_size, g["pool_pages"], g["pool_block_table"], g["sinks"], o, ws)
    torch.cuda.synchronize()
    assert sac.sac_device_status(ws) == BAD_INPUT
    good = np.array([s for s in range(nseq) if s != bad])
    sel = None
    if tk is not None:
        assert (tk[bad].cpu() == -1).all()
        sel = tk.cpu().numpy()[good]
    ref, _ = oracle_decode(wl, d, layer, good, topk_in=sel)
    assert_close(o.cpu()[torch.from_numpy(good)], ref, wl.dtype, f"{layer} decode o")


def test_append_leaves_a_sequence_beyond_the_block_tables_untouched():
    wl = _workload()
    d = W.decode_inputs(wl, "csa")
    dev = torch.device("cuda", 0)
    S = int(d["ctx_lens"].max())
    bad = 3
    p = _params(wl, "csa", S, d["m"])
    g = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in d.items()}
    g["ctx_lens"][bad] = S + 1
    before = {k: g[k].clone() for k in ("kv_pages", "pool_pages", "idx_pool_pages", "cmp_state",
                                        "idx_state")}
    sac.decode_append(p, sac.SAC_KIND_CSA, wl.nseq, g["ctx_lens"], g["kv_new"], g["kv_pages"],
                      g["kv_block_table"], wl.page_size, cmp_state=g["cmp_state"],
                      cmp_gate=g["cmp_gate"], cmp_bias=g["cmp_bias"],
                      pool_pages=g["pool_pages"], pool_block_table=g["pool_block_table"],
                      k_idx_new=g["k_idx_new"], idx_state=g["idx_state"],
                      idx_gate=g["idx_gate"], idx_bias=g["idx_bias"],
                      idx_pool_pages=g["idx_pool_pages"])
    torch.cuda.synchronize()
    # the bad sequence's ring rows and pages are unchanged; every other sequence wrote its row
    assert torch.equal(g["cmp_state"][bad], before["cmp_state"][bad])
    assert torch.equal(g["idx_state"][bad], before["idx_state"][bad])
    bt = d["kv_block_table"]
    for pg in bt[bad][bt[bad] >= 0].tolist():
        assert torch.equal(g["kv_pages"][pg], before["kv_pages"][pg])
    pbt = d["pool_block_table"]
    for pg in pbt[bad][pbt[bad] >= 0].tolist():
        assert torch.equal(g["pool_pages"][pg], before["pool_pages"][pg])
        assert torch.equal(g["idx_pool_pages"][pg], before["idx_pool_pages"][pg])
    ctx = d["ctx_lens"].numpy()
    for s in range(wl.nseq):
        if s == bad:
            continue
        t = int(ctx[s]) - 1
        slot = t % wl.L
        assert torch.equal(g["cmp_state"][s, slot].cpu(), d["kv_new"][s])
