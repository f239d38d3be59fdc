"""Seeded synthetic workloads of the hybrid attention forward (shapes and value distributions only).

This module holds no step of the method: it only draws the inputs. Both the CUDA path's tests and
benchmark and the fp64 oracle read the same bytes from here. Every tensor is drawn on the CPU by
``torch.Generator`` streams seeded per (workload seed, tensor, row chunk), so any row range can be
regenerated on its own (the oracle checks sampled rows of the long workloads without holding the
whole fp64 query tensor).

Shapes follow the page's config defaults (head_dim 512, 64 query heads, one shared K=V head,
sliding_window 128, compress rates 4 / 128, index_n_heads 64, index_head_dim 128, index_topk 512).
Value distributions: activations ~N(0,1); compressor and indexer weights ~N(0, 1/fan_in); head
weights of the indexer ~N(0, 1/n_I); sinks ~N(0,1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

_TENSOR_IDS = {"q": 1, "kv": 2, "cmp_gate": 3, "cmp_bias": 4, "q_idx": 5, "w_idx": 6,
               "k_idx": 7, "idx_gate": 8, "idx_bias": 9, "sinks": 10, "spike": 11,
               "ctx": 12, "pages": 13, "kv_pages": 14, "pool_pages": 15, "idx_pool_pages": 16,
               "hca_kv_pages": 17, "hca_pool_pages": 18, "hca_page_perm": 19, "hca_sinks": 20,
               "kv_new": 21, "k_idx_new": 22, "cmp_state": 23, "idx_state": 24,
               "hca_cmp_gate": 25, "hca_cmp_bias": 26, "o_attn": 27, "o_a_proj": 28,
               "o_b_proj": 29}

ROW_CHUNK = 64  # rows per independently seeded chunk of a per-token tensor


@dataclass(frozen=True)
class Workload:
    """One synthetic workload. kind: 'csa' | 'hca' | 'swa' prefill, 'decode', or 'oproj'."""
    name: str
    kind: str
    dtype: str            # 'f32' or 'bf16'
    B: int = 1
    S: int = 0
    H: int = 64
    D: int = 512
    R: int = 64
    theta: float = 160000.0
    m: int = 0
    L: int = 0
    W: int = 128
    nI: int = 0
    cI: int = 0
    k: int = 0
    spike_frac: float = 0.0   # fraction of positions whose q / q_idx get a 4x component
    # decode only
    nseq: int = 0
    ctx_lo: int = 0
    ctx_hi: int = 0
    page_size: int = 64
    hca_m: int = 128
    chunk: int = 1            # query tokens per sequence and step (> 1: chunked prefill)
    # output projection only
    o_groups: int = 0
    o_rank: int = 0
    hidden: int = 0
    seed: int = 1234

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def N(self) -> int:
        return self.S // self.m if self.m else 0


WORKLOADS: Dict[str, Workload] = {
    # Tiny CSA fp32: every step at a size the oracle finishes in well under a second.
    "tiny_csa_f32": Workload("tiny_csa_f32", "csa", "f32", B=1, S=256, H=4, D=64, R=16,
                             theta=10000.0, m=4, L=8, W=64, nI=2, cI=32, k=8, seed=1234),
    "csa_8k_bf16": Workload("csa_8k_bf16", "csa", "bf16", B=1, S=8192, m=4, L=8, nI=64, cI=128,
                            k=512, seed=1235),
    "hca_32k_bf16": Workload("hca_32k_bf16", "hca", "bf16", B=1, S=32768, m=128, L=128,
                             seed=1236),
    "csa_128k_bf16": Workload("csa_128k_bf16", "csa", "bf16", B=1, S=131072, m=4, L=8, nI=64,
                              cI=128, k=512, spike_frac=0.05, seed=1237),
    "decode_bf16": Workload("decode_bf16", "decode", "bf16", nseq=64, ctx_lo=4096, ctx_hi=65536,
                            page_size=64, m=4, L=8, nI=64, cI=128, k=512, hca_m=128, seed=1238),
    # Chunked prefill: 8 sequences each take their next 1024 tokens against a cached prefix.
    "chunk_bf16": Workload("chunk_bf16", "decode", "bf16", nseq=8, ctx_lo=16384, ctx_hi=65536,
                           page_size=64, m=4, L=8, nI=64, cI=128, k=512, hca_m=128, chunk=1024,
                           seed=1240),
    # Grouped output projection of 8192 tokens: 64 heads of 512 in 8 groups of rank 1024 to 4096.
    "oproj_8k_bf16": Workload("oproj_8k_bf16", "oproj", "bf16", B=1, S=8192, o_groups=8,
                              o_rank=1024, hidden=4096, seed=1239),
}


def _gen(seed: int, tensor: str, chunk: int = 0) -> torch.Generator:
    s = (seed * 1000003 + _TENSOR_IDS[tensor] * 7919 + chunk * 104729) % (2 ** 62)
    return torch.Generator().manual_seed(s)


def _normal(shape, std, seed, tensor, chunk=0) -> torch.Tensor:
    return torch.randn(*shape, generator=_gen(seed, tensor, chunk)) * std


def _rows_tensor(wl: Workload, tensor: str, row_shape, std, rows: np.ndarray) -> torch.Tensor:
    """Per-token tensor [len(rows), *row_shape] (fp32) for flat rows b*S+t, chunk-seeded."""
    rows = np.asarray(rows, dtype=np.int64)
    out = torch.empty((len(rows),) + tuple(row_shape))
    if len(rows) == 0:
        return out
    chunks = rows // ROW_CHUNK
    for c in np.unique(chunks):
        blk = _normal((ROW_CHUNK,) + tuple(row_shape), std, wl.seed, tensor, int(c))
        sel = np.nonzero(chunks == c)[0]
        out[torch.from_numpy(sel)] = blk[torch.from_numpy(rows[sel] - c * ROW_CHUNK)]
    return out


def _all_rows_tensor(wl: Workload, tensor: str, row_shape, std, nrows: int) -> torch.Tensor:
    nchunk = (nrows + ROW_CHUNK - 1) // ROW_CHUNK
    out = torch.empty((nchunk * ROW_CHUNK,) + tuple(row_shape))
    for c in range(nchunk):
        out[c * ROW_CHUNK:(c + 1) * ROW_CHUNK] = _normal((ROW_CHUNK,) + tuple(row_shape), std,
                                                          wl.seed, tensor, c)
    return out[:nrows]


def _spike(wl: Workload, x: torch.Tensor, rows: np.ndarray, which: str) -> torch.Tensor:
    """Give spike_frac of the positions a 4x component along one seeded unit direction d:
    x <- x + 3 <x, d> d for every head vector of those rows (input shaping only)."""
    if wl.spike_frac <= 0:
        return x
    n_all = wl.B * wl.S
    g = _gen(wl.seed, "spike", 0)
    chosen = torch.rand(n_all, generator=g) < wl.spike_frac
    d_q = torch.randn(wl.D, generator=g)
    d_i = torch.randn(wl.cI, generator=g)
    d = d_q if which == "q" else d_i
    d = d / d.norm()
    mask = chosen[torch.from_numpy(np.asarray(rows, dtype=np.int64))]
    if mask.any():
        xs = x[mask]
        proj = (xs * d).sum(-1, keepdim=True)
        x[mask] = xs + 3.0 * proj * d
    return x


def spiked_rows(wl: Workload) -> np.ndarray:
    """Flat rows that carry the 4x component (empty unless spike_frac > 0)."""
    if wl.spike_frac <= 0:
        return np.zeros(0, dtype=np.int64)
    g = _gen(wl.seed, "spike", 0)
    chosen = torch.rand(wl.B * wl.S, generator=g) < wl.spike_frac
    return np.nonzero(chosen.numpy())[0]


def prefill_weights(wl: Workload) -> Dict[str, torch.Tensor]:
    """Compressor / indexer weights and sinks (CPU, workload dtype; biases and sinks fp32)."""
    dt = wl.torch_dtype
    out = {"sinks": _normal((wl.H,), 1.0, wl.seed, "sinks")}
    if wl.kind in ("csa", "hca"):
        out["cmp_gate"] = _normal((wl.D,), 1.0 / math.sqrt(wl.D), wl.seed, "cmp_gate").to(dt)
        out["cmp_bias"] = _normal((wl.L,), 1.0 / math.sqrt(wl.L), wl.seed, "cmp_bias")
    if wl.kind == "csa":
        out["idx_gate"] = _normal((wl.cI,), 1.0 / math.sqrt(wl.cI), wl.seed, "idx_gate").to(dt)
        out["idx_bias"] = _normal((wl.L,), 1.0 / math.sqrt(wl.L), wl.seed, "idx_bias")
    return out


def _q_rows(wl: Workload, rows: np.ndarray) -> torch.Tensor:
    return _spike(wl, _rows_tensor(wl, "q", (wl.H, wl.D), 1.0, rows), rows, "q").to(
        wl.torch_dtype)


def _qidx_rows(wl: Workload, rows: np.ndarray) -> torch.Tensor:
    qi = _rows_tensor(wl, "q_idx", (wl.nI, wl.cI), 1.0, rows)
    return _spike(wl, qi, rows, "qi").to(wl.torch_dtype)


def _widx_rows(wl: Workload, rows: np.ndarray) -> torch.Tensor:
    return _rows_tensor(wl, "w_idx", (wl.nI,), 1.0 / math.sqrt(wl.nI), rows)


def prefill_row_inputs(wl: Workload, rows) -> Dict[str, torch.Tensor]:
    """Per-query tensors of the listed flat rows: q [n,H,D], and for CSA q_idx [n,nI,cI],
    w_idx [n,nI] (fp32)."""
    rows = np.asarray(rows, dtype=np.int64)
    out = {"q": _q_rows(wl, rows)}
    if wl.kind == "csa":
        out["q_idx"] = _qidx_rows(wl, rows)
        out["w_idx"] = _widx_rows(wl, rows)
    return out


def prefill_inputs(wl: Workload, with_queries: bool = True) -> Dict[str, torch.Tensor]:
    """All prefill inputs on the CPU: q [B,S,H,D], kv [B,S,D], weights, and for CSA the indexer
    stream k_idx [B,S,cI], q_idx [B,S,nI,cI], w_idx [B,S,nI]."""
    dt = wl.torch_dtype
    n = wl.B * wl.S
    out = dict(prefill_weights(wl))
    out["kv"] = _all_rows_tensor(wl, "kv", (wl.D,), 1.0, n).to(dt).reshape(wl.B, wl.S, wl.D)
    if wl.kind == "csa":
        out["k_idx"] = _all_rows_tensor(wl, "k_idx", (wl.cI,), 1.0, n).to(dt).reshape(
            wl.B, wl.S, wl.cI)
    if with_queries:
        q = torch.empty((n, wl.H, wl.D), dtype=dt)
        step = ROW_CHUNK * 64
        for s0 in range(0, n, step):
            q[s0:s0 + step] = _q_rows(wl, np.arange(s0, min(n, s0 + step)))
        out["q"] = q.reshape(wl.B, wl.S, wl.H, wl.D)
        if wl.kind == "csa":
            rows = np.arange(n)
            out["q_idx"] = _qidx_rows(wl, rows).reshape(wl.B, wl.S, wl.nI, wl.cI)
            out["w_idx"] = _widx_rows(wl, rows).reshape(wl.B, wl.S, wl.nI)
    return out


def prefill_slice_inputs(wl: Workload, s0: int, s1: int) -> Dict[str, torch.Tensor]:
    """The inputs of tokens [s0, s1) of sequence 0 (the same bytes prefill_inputs draws for those
    rows), plus the weights: q [n,H,D], kv [n,D]; CSA: k_idx [n,cI], q_idx [n,nI,cI], w_idx
    [n,nI]. One rank's share of a query-sharded prefill."""
    rows = np.arange(s0, s1, dtype=np.int64)
    out = dict(prefill_weights(wl))
    out["kv"] = _rows_tensor(wl, "kv", (wl.D,), 1.0, rows).to(wl.torch_dtype)
    out.update(prefill_row_inputs(wl, rows))
    if wl.kind == "csa":
        out["k_idx"] = _rows_tensor(wl, "k_idx", (wl.cI,), 1.0, rows).to(wl.torch_dtype)
    return out


# ------------------------------------------------------------------------------------------------
# Decode: nseq sequences, one new token each, paged caches of page_size rows with physical pages
# shuffled through a pool. kv pages hold rotated kv, pool pages rotated entries, indexer pool pages
# un-rotated entries; here all cache values are drawn ~N(0,1) directly (the cache is an input of a
# decode step). kv pages outside a sequence's last W tokens are never read by a step: they are
# allocated at full size and left zero.
# ------------------------------------------------------------------------------------------------
@dataclass
class PagedCache:
    pages: torch.Tensor          # [num_pages, page_size, width]
    block_table: torch.Tensor    # [nseq, max_pages] int32 (-1 past the last page)


def _paged(wl: Workload, tensor: str, perm_tensor: str, lens: np.ndarray, width: int,
           fill_from: Optional[np.ndarray], dt) -> PagedCache:
    ps = wl.page_size
    npages = [(int(l) + ps - 1) // ps for l in lens]
    total = sum(npages)
    maxp = max(max(npages), 1)
    perm = torch.randperm(total, generator=_gen(wl.seed, perm_tensor, 0)).numpy()
    bt = np.full((len(lens), maxp), -1, dtype=np.int32)
    pages = torch.zeros((total, ps, width), dtype=dt)
    base = 0
    for s, n in enumerate(npages):
        bt[s, :n] = perm[base:base + n]
        first = 0 if fill_from is None else int(fill_from[s]) // ps
        for lp in range(first, n):
            pages[int(bt[s, lp])] = _normal((ps, width), 1.0, wl.seed, tensor,
                                            s * 1_000_000 + lp).to(dt)
        base += n
    return PagedCache(pages, torch.from_numpy(bt))


def decode_inputs(wl: Workload, layer: str) -> Dict[str, object]:
    """Inputs of one decode step of the CSA layer ('csa') or the HCA layer ('hca'); with
    wl.chunk = n > 1, of one prefill chunk: the per-token tensors gain an n axis after the
    sequence axis and ctx counts the chunk."""
    dt = wl.torch_dtype
    g = _gen(wl.seed, "ctx", 0)
    ctx = torch.randint(wl.ctx_lo, wl.ctx_hi + 1, (wl.nseq,), generator=g).to(torch.int32)
    lens = ctx.numpy()
    pfx = "" if layer == "csa" else "hca_"
    m = wl.m if layer == "csa" else wl.hca_m
    n = wl.chunk
    tok = (wl.nseq,) if n == 1 else (wl.nseq, n)  # leading shape of the per-token tensors
    win_start = np.maximum(lens - wl.W - (n - 1), 0)
    kv = _paged(wl, pfx + "kv_pages", "pages" if layer == "csa" else "hca_page_perm", lens,
                wl.D, win_start, dt)
    npool = lens // m
    pool = _paged(wl, pfx + "pool_pages", "pages" if layer == "csa" else "hca_page_perm",
                  np.maximum(npool, 1), wl.D, None, dt)
    out = {"ctx_lens": ctx, "kv_pages": kv.pages, "kv_block_table": kv.block_table,
           "pool_pages": pool.pages, "pool_block_table": pool.block_table, "m": m,
           "q": _normal(tok + (wl.H, wl.D), 1.0, wl.seed, "q", 10 ** 6 + (layer == "hca"))
           .to(dt),
           "sinks": _normal((wl.H,), 1.0, wl.seed, "sinks" if layer == "csa" else "hca_sinks")}
    # the step's cache append: the new token's un-rotated kv row, the compressor gate and ring
    L = wl.L if layer == "csa" else m
    out["kv_new"] = _normal(tok + (wl.D,), 1.0, wl.seed, "kv_new", layer == "hca").to(dt)
    out["cmp_gate"] = _normal((wl.D,), 1.0 / math.sqrt(wl.D), wl.seed,
                              "cmp_gate" if layer == "csa" else "hca_cmp_gate").to(dt)
    out["cmp_bias"] = _normal((L,), 1.0 / math.sqrt(L), wl.seed,
                              "cmp_bias" if layer == "csa" else "hca_cmp_bias")
    out["cmp_state"] = _normal((wl.nseq, L, wl.D), 1.0, wl.seed, "cmp_state",
                               layer == "hca").to(dt)
    if layer == "csa":
        out["k_idx_new"] = _normal(tok + (wl.cI,), 1.0, wl.seed, "k_idx_new").to(dt)
        out["idx_gate"] = _normal((wl.cI,), 1.0 / math.sqrt(wl.cI), wl.seed, "idx_gate").to(dt)
        out["idx_bias"] = _normal((L,), 1.0 / math.sqrt(L), wl.seed, "idx_bias")
        out["idx_state"] = _normal((wl.nseq, L, wl.cI), 1.0, wl.seed, "idx_state").to(dt)
        ipool = _paged(wl, "idx_pool_pages", "pages", np.maximum(npool, 1), wl.cI, None, dt)
        assert torch.equal(ipool.block_table, pool.block_table)
        out["idx_pool_pages"] = ipool.pages
        out["q_idx"] = _normal(tok + (wl.nI, wl.cI), 1.0, wl.seed, "q_idx", 10 ** 6).to(dt)
        out["w_idx"] = _normal(tok + (wl.nI,), 1.0 / math.sqrt(wl.nI), wl.seed, "w_idx",
                               10 ** 6)
    return out


# ------------------------------------------------------------------------------------------------
# Grouped output projection: an attention output o [T, H, D] ~ N(0, 1) and random-init weights
# (o_a_proj ~ N(0, 1/fan_in) per group, o_b_proj ~ N(0, 1/fan_in)) in the nn.Linear layout.
# ------------------------------------------------------------------------------------------------
def oproj_inputs(T: int, H: int, D: int, groups: int, rank: int, hidden: int, seed: int,
                 dtype=torch.bfloat16) -> Dict[str, torch.Tensor]:
    kg = H // groups * D
    o = torch.empty((T, H, D))
    for c0 in range(0, T, ROW_CHUNK):
        n = min(ROW_CHUNK, T - c0)
        o[c0:c0 + n] = _normal((ROW_CHUNK, H, D), 1.0, seed, "o_attn", c0 // ROW_CHUNK)[:n]
    return {"o": o.to(dtype),
            "w_a": _normal((groups, rank, kg), 1.0 / math.sqrt(kg), seed, "o_a_proj").to(dtype),
            "w_b": _normal((hidden, groups * rank), 1.0 / math.sqrt(groups * rank), seed,
                           "o_b_proj").to(dtype)}
