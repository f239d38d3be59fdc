"""Query-sharded prefill of one long sequence over several GPUs (one process per GPU).

Rank r of N owns the contiguous token slice [s0, s1) = [r S/N, (r+1) S/N): its queries, its kv
rows and its indexer key rows. Only the pools cross ranks ("Hybrid attention": every query of a
compressed layer sees the entries of all windows closed before it):

  1. halo: each rank receives from its left neighbour the last `halo` un-rotated kv rows (and
     indexer key rows) before its slice -- enough for the sliding window of its first query and
     for the compressor windows that close inside its slice (one send / recv per stream);
  2. local compress: the rank appends halo + slice to one-sequence paged caches with the chunk
     append kernels, which write the rotated window rows and pool every entry whose window closes
     in that range; the entries of its own slice, [s0/m, s1/m), are exact;
  3. pool all-gather: every rank contributes those entries to the full main and indexer pools,
     gathered in place into each GPU's own memory (NCCL all-gather over NVLink);
  4. local attention: the rank's queries run as one prefill chunk (indexer, top-k, attention) of
     the sequence, ctx = s1, against the gathered pools and its window rows.

No tile is ever read from another GPU's memory: remote data arrives only through the collectives.
The per-rank steps are split into `local_caches` / `local_attention` so that a caller can drive
them with any transport; `sharded_forward` drives them with torch.distributed.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import torch

from . import (SAC_KIND_CSA, SAC_KIND_HCA, csa_prefill_chunk, hca_prefill_chunk,
               prefill_chunk_append, sac_chunk_workspace_size)


@dataclass(frozen=True)
class ShardPlan:
    """Token ranges of one rank. Rows [t0, s1) are appended to its caches: the halo [t0, s0) and
    its own slice [s0, s1). Entries [e0, e1) are the ones whose windows close inside its slice.
    h is the halo every rank but the first receives (t0 = s0 - h there, 0 on rank 0)."""
    rank: int
    world: int
    S: int
    m: int
    page_size: int
    h: int
    s0: int
    s1: int
    t0: int
    e0: int
    e1: int

    @property
    def n(self) -> int:
        return self.s1 - self.s0

    @property
    def halo(self) -> int:
        return self.s0 - self.t0


def plan(S: int, world: int, rank: int, m: int, win_len: int, sliding_window: int,
         page_size: int = 64) -> ShardPlan:
    """Equal contiguous slices. Each slice is a whole number of pages and of compressor strides,
    so every rank owns whole entries and its rows start on a page; the halo h covers the W - 1
    window rows and the win_len - m older rows of a window that closes inside the slice, rounded
    up to whole pages, and comes whole from the left neighbour (a slice holds at least h rows)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    n = S // world
    unit = page_size * m // _gcd(page_size, m)
    if n * world != S or n % unit != 0:
        raise ValueError(f"S={S} must split into {world} slices of whole multiples of {unit} "
                         "(page size and compression rate)")
    need = max(sliding_window - 1, win_len - m, 0)
    h = -(-need // page_size) * page_size
    if world > 1 and n < h:
        raise ValueError(f"slices of {n} tokens are shorter than the {h}-row halo")
    s0, s1 = rank * n, (rank + 1) * n
    t0 = s0 - h if rank > 0 else 0
    return ShardPlan(rank, world, S, m, page_size, h, s0, s1, t0, s0 // m, s1 // m)


def _gcd(a: int, b: int) -> int:
    while b:
        a, b = b, a % b
    return a


# ------------------------------------------------------------------------------------------------
# collectives (torch.distributed: NCCL on GPUs, gloo on CPU)
# ------------------------------------------------------------------------------------------------
def exchange_halo(rows: torch.Tensor, h: int, group=None) -> torch.Tensor:
    """Send the last h rows of this rank's slice (rows [n >= h, C]) to rank + 1 and return the h
    rows rank - 1 sent; rank 0 has no left neighbour and gets an empty [0, C] tensor."""
    dist = torch.distributed
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    recv = torch.empty((h if rank > 0 else 0,) + tuple(rows.shape[1:]), dtype=rows.dtype,
                       device=rows.device)
    if h == 0 or world == 1:
        return recv
    send = rows[-h:].contiguous()
    ops = []
    if rank + 1 < world:
        ops.append(dist.P2POp(dist.isend, send, _global(rank + 1, group), group))
    if rank > 0:
        ops.append(dist.P2POp(dist.irecv, recv, _global(rank - 1, group), group))
    for req in dist.batch_isend_irecv(ops):
        req.wait()
    return recv


def _global(r: int, group) -> int:
    return r if group is None else torch.distributed.get_global_rank(group, r)


def gather_entries(full: torch.Tensor, e0: int, e1: int, group=None) -> None:
    """All-gather the pool: rank r's entries full[e0:e1] (equal counts on every rank, rank order)
    are copied into every rank's `full`, in place."""
    dist = torch.distributed
    world = dist.get_world_size(group)
    n = e1 - e0
    if world == 1:
        return
    if full.is_cuda:
        # in place: this rank's input is its own slot of the output buffer
        dist.all_gather_into_tensor(full[:world * n], full[e0:e1], group=group)
    else:
        parts = [torch.empty_like(full[e0:e1]) for _ in range(world)]
        dist.all_gather(parts, full[e0:e1].contiguous(), group=group)
        full[:world * n].copy_(torch.cat(parts))


# ------------------------------------------------------------------------------------------------
# per-rank steps on the GPU (the library's chunk kernels)
# ------------------------------------------------------------------------------------------------
def local_caches(sp: ShardPlan, kind: int, p, kv_rows: torch.Tensor, cmp_gate, cmp_bias,
                 k_idx_rows: Optional[torch.Tensor] = None, idx_gate=None,
                 idx_bias=None, stream=None) -> Dict[str, torch.Tensor]:
    """One-sequence paged caches of this rank, filled from its halo + slice rows.

    kv_rows [s1 - t0, D] (and k_idx_rows [s1 - t0, cI] for CSA) are the un-rotated rows t0..s1-1.
    The window pages hold those rows rotated; the pool pages hold, at entry w, every entry whose
    window closes in [t0, s1) -- exact for [e0, e1), while the entries the halo closes lack their
    older rows and are replaced by the all-gather. p.S must be the full sequence length."""
    dev = kv_rows.device
    ps, D = sp.page_size, kv_rows.shape[1]
    rows = sp.s1 - sp.t0
    kv_pages = torch.zeros((rows // ps, ps, D), dtype=kv_rows.dtype, device=dev)
    kv_bt = torch.full((1, sp.S // ps), -1, dtype=torch.int32, device=dev)
    kv_bt[0, sp.t0 // ps:sp.s1 // ps] = torch.arange(rows // ps, dtype=torch.int32, device=dev)
    N = sp.S // sp.m
    npp = -(-N // ps)
    pool_pages = torch.zeros((npp, ps, D), dtype=kv_rows.dtype, device=dev)
    pool_bt = torch.arange(npp, dtype=torch.int32, device=dev).reshape(1, npp)
    L = p.win_len
    c = {"kv_pages": kv_pages, "kv_block_table": kv_bt, "pool_pages": pool_pages,
         "pool_block_table": pool_bt,
         "ctx_lens": torch.tensor([sp.s1], dtype=torch.int32, device=dev),
         "cmp_state": torch.zeros((1, L, D), dtype=kv_rows.dtype, device=dev)}
    kw = {}
    if kind == SAC_KIND_CSA:
        cI = k_idx_rows.shape[1]
        c["idx_pool_pages"] = torch.zeros((npp, ps, cI), dtype=kv_rows.dtype, device=dev)
        c["idx_state"] = torch.zeros((1, L, cI), dtype=kv_rows.dtype, device=dev)
        kw = dict(k_idx_new=k_idx_rows.reshape(1, rows, cI).contiguous(),
                  idx_state=c["idx_state"], idx_gate=idx_gate, idx_bias=idx_bias,
                  idx_pool_pages=c["idx_pool_pages"])
    prefill_chunk_append(p, kind, 1, rows, c["ctx_lens"], kv_rows.reshape(1, rows, D).contiguous(),
                         kv_pages, kv_bt, ps, cmp_state=c["cmp_state"], cmp_gate=cmp_gate,
                         cmp_bias=cmp_bias, pool_pages=pool_pages, pool_block_table=pool_bt,
                         stream=stream, **kw)
    return c


def pool_rows(c: Dict[str, torch.Tensor], name: str) -> torch.Tensor:
    """The flat [entries, C] view of a pool page buffer (entry w at row w)."""
    pages = c[name]
    return pages.view(pages.shape[0] * pages.shape[1], pages.shape[2])


def local_attention(sp: ShardPlan, kind: int, p, c: Dict[str, torch.Tensor], q: torch.Tensor,
                    sinks, o: torch.Tensor, q_idx=None, w_idx=None, topk_out=None, ws=None,
                    stream=None) -> None:
    """This rank's queries (q [n, H, D], o [n, H, D]; CSA: q_idx [n, nI, cI], w_idx [n, nI]) as
    the last n tokens of a sequence of s1 tokens, over the caches (pools already gathered)."""
    n = sp.n
    if ws is None:
        ws = torch.empty(sac_chunk_workspace_size(p, kind, 1, n), dtype=torch.uint8,
                         device=q.device)
    if kind == SAC_KIND_HCA:
        hca_prefill_chunk(p, 1, n, q, c["kv_pages"], c["kv_block_table"], c["ctx_lens"],
                          sp.page_size, c["pool_pages"], c["pool_block_table"], sinks, o, ws,
                          stream)
    else:
        csa_prefill_chunk(p, 1, n, q, c["kv_pages"], c["kv_block_table"], c["ctx_lens"],
                          sp.page_size, c["pool_pages"], c["idx_pool_pages"],
                          c["pool_block_table"], q_idx, w_idx, sinks, o, topk_out, ws, stream)


def sharded_forward(sp: ShardPlan, kind: int, p, x: Dict[str, torch.Tensor], o: torch.Tensor,
                    topk_out=None, ws=None, group=None) -> Dict[str, torch.Tensor]:
    """The whole query-sharded step of one rank over torch.distributed (NCCL on GPUs).

    x holds this rank's slice: q [n,H,D], kv [n,D] and, for CSA, q_idx [n,nI,cI], w_idx [n,nI],
    k_idx [n,cI]; plus the layer's weights (cmp_gate, cmp_bias, sinks; CSA: idx_gate,
    idx_bias). Returns the caches (gathered pools included)."""
    kv_halo = exchange_halo(x["kv"], sp.h, group)
    kv_rows = torch.cat([kv_halo, x["kv"]])
    idx_rows = None
    if kind == SAC_KIND_CSA:
        idx_rows = torch.cat([exchange_halo(x["k_idx"], sp.h, group), x["k_idx"]])
    c = local_caches(sp, kind, p, kv_rows, x["cmp_gate"], x["cmp_bias"], idx_rows,
                     x.get("idx_gate"), x.get("idx_bias"))
    gather_entries(pool_rows(c, "pool_pages"), sp.e0, sp.e1, group)
    if kind == SAC_KIND_CSA:
        gather_entries(pool_rows(c, "idx_pool_pages"), sp.e0, sp.e1, group)
    local_attention(sp, kind, p, c, x["q"].reshape(1, sp.n, *x["q"].shape[1:]), x["sinks"],
                    o.reshape(1, sp.n, *o.shape[1:]),
                    q_idx=None if kind != SAC_KIND_CSA else
                    x["q_idx"].reshape(1, sp.n, *x["q_idx"].shape[1:]),
                    w_idx=None if kind != SAC_KIND_CSA else
                    x["w_idx"].reshape(1, sp.n, *x["w_idx"].shape[1:]),
                    topk_out=topk_out, ws=ws)
    return c
