"""GPU parity of the grouped low-rank output projection (o_proj_forward, the tcgen05 GEMM) against
the fp64 oracle, whose intermediate is rounded to bf16 as the kernel stores it: small cases with
several groups, row counts that are not a multiple of the 256-row tile, output widths that are not
a multiple of the 256-column tile and an o_b_proj contraction (G*rank = 120) that is not a
multiple of the 64-wide K step; and the page's configuration (64 heads of 512, 8 groups of rank
1024, hidden 4096) checked on all rows of a short run and on sampled rows of a long one."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_compressor_b200 as sac
from parity import assert_close
from sparse_attention_compressor_b200 import workloads as W

pytestmark = pytest.mark.gpu


def run(T, H, D, G, rank, hidden, seed):
    dev = torch.device("cuda", 0)
    x = W.oproj_inputs(T, H, D, G, rank, hidden, seed)
    g = {k: v.to(dev).contiguous() for k, v in x.items()}
    p = sac.make_params(1, max(T, 1), H, D, 0, 10000.0)
    ws = torch.empty(sac.sac_oproj_workspace_size(p, T, G, rank), dtype=torch.uint8, device=dev)
    out = torch.full((T, hidden), float("nan"), dtype=torch.bfloat16, device=dev)
    sac.o_proj_forward(p, T, G, rank, hidden, g["o"], g["w_a"], g["w_b"], out, ws)
    torch.cuda.synchronize()
    return x, out.cpu()


def f64(t):
    return t.double().numpy()


@pytest.mark.parametrize("T,H,D,G,rank,hidden", [(77, 8, 64, 4, 32, 96), (5, 4, 64, 1, 64, 64),
                                                 (200, 16, 128, 2, 256, 512),
                                                 (300, 6, 64, 3, 40, 72),
                                                 (513, 8, 128, 4, 264, 520)])
def test_oproj_small(T, H, D, G, rank, hidden):
    x, out = run(T, H, D, G, rank, hidden, 41)
    _, want = oracle.o_proj(f64(x["o"]), f64(x["w_a"]), f64(x["w_b"]), G, round_mid=True)
    assert_close(f64(out), want, "bf16", "o_proj small")


def test_oproj_page_config_all_rows():
    x, out = run(64, 64, 512, 8, 1024, 4096, 42)
    _, want = oracle.o_proj(f64(x["o"]), f64(x["w_a"]), f64(x["w_b"]), 8, round_mid=True)
    assert_close(f64(out), want, "bf16", "o_proj 64 rows")


def test_oproj_page_config_sampled_rows_long_run():
    T = 8192
    x, out = run(T, 64, 512, 8, 1024, 4096, 43)
    rows = np.random.default_rng(0).choice(T, 48, replace=False)
    rows = np.concatenate([rows, [0, T - 1]])
    _, want = oracle.o_proj(f64(x["o"]), f64(x["w_a"]), f64(x["w_b"]), 8, rows=rows,
                            round_mid=True)
    assert_close(f64(out[rows]), want, "bf16", "o_proj sampled rows")


def test_oproj_zero_rows_is_a_no_op():
    dev = torch.device("cuda", 0)
    p = sac.make_params(1, 1, 8, 64, 0, 10000.0)
    w_a = torch.zeros((4, 32, 128), dtype=torch.bfloat16, device=dev)
    w_b = torch.zeros((96, 128), dtype=torch.bfloat16, device=dev)
    o = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device=dev)
    out = torch.full((1, 96), 7.0, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(sac.sac_oproj_workspace_size(p, 1, 4, 32), dtype=torch.uint8, device=dev)
    sac.o_proj_forward(p, 0, 4, 32, 96, o, w_a, w_b, out, ws)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
