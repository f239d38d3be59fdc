"""swa_forward_static: the sliding-window forward for callers that cannot allocate device memory
(a host framework's caching allocator owns all of it, or a serving loop forbids allocation after
start-up). Its scratch is a fixed array inside the library; this checks, through the C ABI, that
two calls in a row give the output of swa_forward (which takes a caller workspace) within the bf16
tolerance of the parity tests. This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import sparse_attention_compressor_b200 as sac
from sparse_attention_compressor_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3  # bf16 tolerance of the parity tests


def test_static_scratch_entry_matches_workspace_entry():
    wl = W.Workload("swa_static_test", "swa", "bf16", B=2, S=700, H=64, D=512, R=64, W=128,
                    theta=10000.0, seed=31)
    x = W.prefill_inputs(wl)
    dev = torch.device("cuda", 0)
    g = {k: v.to(dev) for k, v in x.items()}
    p = sac.make_params(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, sliding_window=wl.W,
                        dtype=wl.dtype)
    ref = torch.empty_like(g["q"])
    ws = torch.empty(sac.sac_workspace_size(p, sac.SAC_KIND_SWA), dtype=torch.uint8, device=dev)
    sac.swa_forward(p, g["q"], g["kv"], g["sinks"], ref, ws)
    outs = []
    for _ in range(2):
        o = torch.full_like(g["q"], float("nan"))
        sac.swa_forward_static(p, g["q"], g["kv"], g["sinks"], o)
        outs.append(o)
    torch.cuda.synchronize()
    r = ref.double().cpu().numpy()
    for o in outs:
        err = np.abs(o.double().cpu().numpy() - r)
        assert np.isfinite(err).all()
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS


def test_static_scratch_rejects_sizes_beyond_its_limit():
    cap = sac.sac_static_scratch_bytes()
    p = sac.make_params(1, cap // (512 * 2) + 1, 64, 512, 64, 1e4, sliding_window=128)
    dev = torch.device("cuda", 0)
    t = torch.empty(16, dtype=torch.bfloat16, device=dev)
    s = torch.empty(64, dtype=torch.float32, device=dev)
    with pytest.raises(sac.SacError) as ei:
        sac.swa_forward_static(p, t, t, s, t)
    assert ei.value.code == -2
