"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI (via the binding)
and the fp64 oracle on the same seeded inputs, and compare with the tolerances of the spec:
  bf16 inputs: max |err| <= 2e-2 and mean |err| <= 2e-3;  fp32 inputs: max |err| <= 1e-4.
Top-k selections must match exactly, except inside the oracle's tie band at the k-th boundary
(|I_(k) - I_(k+1)| < 1e-3 relative), where any entry within that band of I_(k) is accepted."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_attention_compressor_b200 as sac
from sparse_attention_compressor_b200 import workloads as W

TOL = {"bf16": (2e-2, 2e-3), "f32": (1e-4, 1e-5)}
TIE_REL = 1e-3


def oracle_params(wl: W.Workload, pos0: int = 0, yarn=None) -> oracle.OracleParams:
    """yarn: None, or (factor, original context, beta_fast, beta_slow) of a YaRN-scaled RoPE."""
    p = oracle.OracleParams(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, wl.W, m=wl.m, L=wl.L,
                            nI=wl.nI, cI=wl.cI, k=wl.k, pos0=pos0, bf16_pools=wl.dtype == "bf16")
    if yarn is not None:
        p.yarn_factor, p.yarn_orig, p.yarn_beta_fast, p.yarn_beta_slow = yarn
    return p


def sac_params(wl: W.Workload, pos0: int = 0, yarn=None):
    kw = {}
    if yarn is not None:
        kw = dict(rope_factor=yarn[0], rope_orig_max_pos=yarn[1], yarn_beta_fast=yarn[2],
                  yarn_beta_slow=yarn[3])
    return sac.make_params(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, m=wl.m, win_len=wl.L,
                           sliding_window=wl.W, n_idx_heads=wl.nI, idx_dim=wl.cI, topk=wl.k,
                           pos0=pos0, dtype=wl.dtype, **kw)


KIND = {"swa": sac.SAC_KIND_SWA, "hca": sac.SAC_KIND_HCA, "csa": sac.SAC_KIND_CSA}


def gpu_prefill(wl: W.Workload, x: dict, pos0: int = 0, with_aux: bool = True,
                yarn=None) -> dict:
    """Run the layer's forward on cuda:0; returns CPU tensors o (and topk / pools)."""
    dev = torch.device("cuda", 0)
    p = sac_params(wl, pos0, yarn)
    g = {k: v.to(dev).contiguous() for k, v in x.items()}
    o = torch.empty_like(g["q"])
    ws = torch.empty(sac.sac_workspace_size(p, KIND[wl.kind]), dtype=torch.uint8, device=dev)
    out = {}
    if wl.kind == "swa":
        sac.swa_forward(p, g["q"], g["kv"], g["sinks"], o, ws)
    elif wl.kind == "hca":
        pool = torch.empty((wl.B, wl.N, wl.D), dtype=wl.torch_dtype, device=dev) if with_aux \
            else None
        sac.hca_forward(p, g["q"], g["kv"], g["cmp_gate"], g["cmp_bias"], g["sinks"], o, pool, ws)
        out["pool"] = pool
    else:
        tk = torch.empty((wl.B, wl.S, wl.k), dtype=torch.int32, device=dev)
        pool = torch.empty((wl.B, wl.N, wl.D), dtype=wl.torch_dtype, device=dev) if with_aux \
            else None
        ipool = torch.empty((wl.B, wl.N, wl.cI), dtype=wl.torch_dtype, device=dev) if with_aux \
            else None
        sac.csa_forward(p, g["q"], g["kv"], g["cmp_gate"], g["cmp_bias"], g["q_idx"], g["w_idx"],
                        g["k_idx"], g["idx_gate"], g["idx_bias"], g["sinks"], o, tk, pool, ipool,
                        ws)
        out.update(topk=tk, pool=pool, idx_pool=ipool)
    torch.cuda.synchronize()
    assert sac.sac_device_status(ws) == 0, "a kernel reported a device-side wait timeout"
    out["o"] = o
    return {k: (v.cpu() if v is not None else None) for k, v in out.items()}


def assert_close(got, ref, dtype: str, what: str):
    got = got.float().numpy().astype(np.float64) if hasattr(got, "numpy") else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    err = np.abs(got - ref)
    mx, mean = TOL[dtype]
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert err.max() <= mx, f"{what}: max |err| {err.max():.3e} > {mx:g}"
    assert err.mean() <= mean, f"{what}: mean |err| {err.mean():.3e} > {mean:g}"
    return float(err.max()), float(err.mean())


def check_topk_row(gpu_row, orc_row, orc_scores, nvis: int, k: int, what: str):
    """Selections of one query: same size, and equal as sets except inside the tie band."""
    gpu_row = np.asarray(gpu_row)
    n = min(k, nvis)
    g = gpu_row[gpu_row >= 0]
    assert len(g) == n and (gpu_row[n:] == -1).all(), f"{what}: {len(g)} selected, expect {n}"
    assert (g < nvis).all() and len(set(g.tolist())) == n, f"{what}: invalid entries"
    assert (np.diff(g) > 0).all(), f"{what}: not in ascending entry order"
    o = set(int(v) for v in orc_row[orc_row >= 0])
    gs = set(int(v) for v in g)
    if gs == o:
        return 0
    s = np.asarray(orc_scores[:nvis], dtype=np.float64)
    ranked = np.sort(s)[::-1]
    ik = ranked[n - 1]
    ik1 = ranked[n] if n < nvis else -np.inf
    scale = max(abs(ik), 1e-6 * float(np.abs(s).max()), 1e-30)
    assert ik - ik1 < TIE_REL * scale, f"{what}: sets differ outside a tie (gap {ik - ik1:.3e})"
    for w in gs ^ o:
        assert abs(s[w] - ik) <= TIE_REL * scale, f"{what}: entry {w} outside the tie band"
    return len(gs ^ o)
