"""YaRN-scaled RoPE on the GPU (the rope scaling the config pairs with compress_rope_theta): the
CSA and HCA forwards with YaRN frequencies against the fp64 oracle, element by element. Every
rotation of the layer (queries, window keys, pool entries, the output's inverse turn) takes the
scaled frequencies, at absolute positions far past the original context."""
import numpy as np
import pytest

import oracle
from parity import assert_close, check_topk_row, gpu_prefill, oracle_params
from sparse_attention_compressor_b200 import workloads as W

pytestmark = pytest.mark.gpu

YARN = (4.0, 4096, 32.0, 1.0)  # factor, original context, beta_fast, beta_slow
POS0 = 20000


def _wl(kind):
    if kind == "csa":
        return W.Workload("csa_yarn_test", "csa", "bf16", B=1, S=700, m=4, L=8, nI=64, cI=128,
                          k=64, seed=90)
    return W.Workload("hca_yarn_test", "hca", "bf16", B=1, S=900, m=128, L=128, seed=91)


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_yarn_forward_matches_oracle(kind):
    wl = _wl(kind)
    x = W.prefill_inputs(wl)
    g = gpu_prefill(wl, x, POS0, yarn=YARN)
    p = oracle_params(wl, POS0, yarn=YARN)
    n = wl.B * wl.S
    if kind == "hca":
        o, pool = oracle.hca_forward(p, x["q"], x["kv"], x["cmp_gate"], x["cmp_bias"], x["sinks"])
        assert_close(g["pool"], pool, wl.dtype, "pool")
    else:
        rows = np.arange(n)
        sc = oracle.csa_index_scores(p, x["q_idx"].reshape(n, wl.nI, wl.cI),
                                     x["w_idx"].reshape(n, wl.nI), x["k_idx"], x["idx_gate"],
                                     x["idx_bias"], rows)
        gsel = g["topk"].reshape(n, wl.k).numpy()
        for t in range(n):
            nvis = (t + 1) // wl.m
            check_topk_row(gsel[t], oracle.topk(sc[t], nvis, wl.k), sc[t], nvis, wl.k, f"row {t}")
        o, _, pool, _ = oracle.csa_forward(p, x["q"], x["kv"], x["cmp_gate"], x["cmp_bias"],
                                           x["q_idx"], x["w_idx"], x["k_idx"], x["idx_gate"],
                                           x["idx_bias"], x["sinks"], topk_in=gsel)
        assert_close(g["pool"], pool, wl.dtype, "pool")
    assert_close(g["o"].reshape(n, wl.H, wl.D), o.reshape(n, wl.H, wl.D), wl.dtype, "o")
