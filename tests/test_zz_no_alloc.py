"""swa_forward_static: the sliding-window forward for callers that cannot allocate device memory
(code inside a host framework whose caching allocator owns all of it, or a serving loop that
forbids allocation after start-up). Its scratch is a fixed array inside the library.

Through the C ABI, two calls in a row must give the output of swa_forward (which takes a caller
workspace and runs the same kernels) within the bf16 tolerance of the parity tests, and sampled
rows must match the fp64 oracle. The file name sorts last so that pytest collects it after every
other test: a run that stops at the first failure has then already run everything else. It holds
no state that other tests leave behind (each call writes every scratch byte it reads), so it
passes alone in a fresh process as well as after the rest of the suite."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_compressor_b200 as sac
from sparse_attention_compressor_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3  # bf16 tolerance of the parity tests
POS0 = 321


def _workload():
    return W.Workload("swa_static_test", "swa", "bf16", B=2, S=700, H=64, D=512, R=64, W=128,
                      theta=10000.0, seed=31)


def _close(got, ref):
    err = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))
    assert np.isfinite(err).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


def test_static_scratch_entry_matches_workspace_entry_and_oracle():
    wl = _workload()
    x = W.prefill_inputs(wl)
    dev = torch.device("cuda", 0)
    g = {k: v.to(dev) for k, v in x.items()}
    p = sac.make_params(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, sliding_window=wl.W,
                        pos0=POS0, dtype=wl.dtype)
    ref = torch.empty_like(g["q"])
    ws = torch.empty(sac.sac_workspace_size(p, sac.SAC_KIND_SWA), dtype=torch.uint8, device=dev)
    sac.swa_forward(p, g["q"], g["kv"], g["sinks"], ref, ws)
    outs = []
    for _ in range(2):  # two calls in a row share the one static array
        o = torch.full_like(g["q"], float("nan"))
        sac.swa_forward_static(p, g["q"], g["kv"], g["sinks"], o)
        outs.append(o)
    torch.cuda.synchronize()
    r = ref.double().cpu().numpy()
    for o in outs:
        _close(o.double().cpu().numpy(), r)
    # sampled rows of both sequences against the oracle
    rows = np.array([0, 1, 127, 128, 500, wl.S - 1, wl.S, wl.S + 130, 2 * wl.S - 1])
    po = oracle.OracleParams(wl.B, wl.S, wl.H, wl.D, wl.R, wl.theta, wl.W, pos0=POS0)
    q = x["q"].reshape(-1, wl.H, wl.D)[torch.from_numpy(rows)]
    want = oracle.swa_forward(po, q, x["kv"], x["sinks"], rows=rows)
    for o in outs:
        _close(o.reshape(-1, wl.H, wl.D)[torch.from_numpy(rows)].double().cpu().numpy(), want)


def test_static_scratch_rejects_sizes_beyond_its_limit():
    cap = sac.sac_static_scratch_bytes()
    p = sac.make_params(1, cap // (512 * 2) + 1, 64, 512, 64, 1e4, sliding_window=128)
    dev = torch.device("cuda", 0)
    t = torch.empty(16, dtype=torch.bfloat16, device=dev)
    s = torch.empty(64, dtype=torch.float32, device=dev)
    with pytest.raises(sac.SacError) as ei:
        sac.swa_forward_static(p, t, t, s, t)
    assert ei.value.code == -2
