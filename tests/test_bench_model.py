"""Host logic of bench.py: the algorithmic work each roofline divides by, against direct
per-query loops on small workloads (no GPU)."""
from dataclasses import replace

import numpy as np
import torch

import bench
from sparse_attention_compressor_b200 import workloads as W


def test_prefill_work_matches_per_query_counts():
    wl = W.Workload("t", "csa", "bf16", B=2, S=37, H=4, D=64, m=4, L=8, W=8, nI=3, cI=32, k=5)
    w = bench.work(wl)
    keys = sum(min(t + 1, wl.W) + min((t + 1) // wl.m, wl.k) for t in range(wl.S)) * wl.B
    assert w["attention"] == ("flops", keys * 4 * wl.H * wl.D)
    pairs = sum((t + 1) // wl.m for t in range(wl.S)) * wl.B
    assert w["indexer_score"] == ("flops", pairs * 2 * wl.nI * wl.cI)
    assert w["topk"] == ("bytes", float((pairs // wl.B * 4 + wl.S * wl.k * 4) * wl.B))
    # compressor: every token row read once, every entry written once (bf16)
    assert w["compress"] == ("bytes", float((wl.S + wl.S // wl.m) * wl.D * 2 * wl.B))
    hca = replace(wl, kind="hca", m=16, L=16)
    keys = sum(min(t + 1, wl.W) + (t + 1) // 16 for t in range(wl.S)) * wl.B
    assert bench.work(hca)["attention"] == ("flops", keys * 4 * wl.H * wl.D)


def _paged_ctx(ctx, m):
    return {"ctx_lens": torch.tensor(ctx, dtype=torch.int32), "m": m}


def test_chunk_work_matches_per_row_counts():
    wl = W.Workload("c", "decode", "bf16", nseq=2, H=4, D=64, m=4, L=8, W=8, nI=3, cI=32, k=5,
                    hca_m=16, chunk=6)
    dc, dh = _paged_ctx([20, 9], 4), _paged_ctx([33, 6], 16)
    w = bench.chunk_work(wl, dc, dh)
    rows = [(c, t) for c in (20, 9) for t in range(c - 6, c)]
    assert w["indexer_score"] == ("flops", float(sum((t + 1) // 4 for _, t in rows) * 2 * 3 * 32))
    csa_keys = sum(min((t + 1) // 4, wl.k) + min(t + 1, wl.W) for _, t in rows)
    assert w["csa_chunk_attention"] == ("flops", float(csa_keys * 4 * wl.H * wl.D))
    hrows = [t for c in (33, 6) for t in range(c - 6, c)]
    hca_keys = sum((t + 1) // 16 + min(t + 1, wl.W) for t in hrows)
    assert w["hca_chunk_attention"] == ("flops", float(hca_keys * 4 * wl.H * wl.D))
    # entries closing inside the chunks: CSA 20 -> 5 - 3 = 2, 9 -> 2 - 0 = 2; HCA 33 -> 2 - 1 = 1
    closing_csa = (20 // 4 - 14 // 4) + (9 // 4 - 3 // 4)
    assert w["chunk_append_index"][1] == float((12 + 2 * min(wl.L, 6)) * wl.cI * 2
                                               + closing_csa * (wl.L + 1) * wl.cI * 2)


def test_decode_bytes_fold_the_index_part_when_fused():
    wl = W.Workload("d", "decode", "bf16", nseq=3, H=4, D=64, m=4, L=8, W=8, nI=3, cI=32, k=5,
                    hca_m=16)
    dc, dh = _paged_ctx([8, 9, 40], 4), _paged_ctx([16, 17, 5], 16)
    db = bench.decode_bytes(wl, dc, dh)
    assert set(db) >= {"decode_append", "decode_append_index", "indexer_score", "topk",
                       "csa_decode_attention", "hca_decode_attention"}
    # closing windows: CSA ctx 8 and 40 (multiples of 4), HCA ctx 16
    app = 3 * 3 * wl.D * 2 + 2 * (wl.L + 1) * wl.D * 2 + 3 * 3 * wl.D * 2 + 1 * 17 * wl.D * 2
    assert db["decode_append"] == float(app)
    nv = np.array([8, 9, 40]) // 4
    assert db["topk"] == float((nv * 4).sum() + 3 * wl.k * 4)


def test_chunk_inputs_shapes_and_reproducibility():
    """A chunk workload's per-token tensors gain the chunk axis, the contexts hold the chunk, and
    the window pages cover the rows every chunk row can see; a decode workload keeps its shapes."""
    wl = W.Workload("c", "decode", "bf16", nseq=2, H=4, D=64, R=16, m=4, L=8, W=8, nI=3, cI=32,
                    k=5, hca_m=16, ctx_lo=40, ctx_hi=90, page_size=16, chunk=6, seed=5)
    d = W.decode_inputs(wl, "csa")
    assert d["q"].shape == (2, 6, 4, 64) and d["kv_new"].shape == (2, 6, 64)
    assert d["q_idx"].shape == (2, 6, 3, 32) and d["w_idx"].shape == (2, 6, 3)
    ctx = d["ctx_lens"].numpy()
    assert (ctx >= wl.chunk).all()
    for s in range(2):  # rows ctx - chunk - W + 1 .. ctx - 1 sit on filled pages
        lo = ctx[s] - wl.chunk - wl.W + 1
        for j in range(max(lo, 0), ctx[s]):
            page = int(d["kv_block_table"][s, j // wl.page_size])
            assert d["kv_pages"][page, j % wl.page_size].abs().sum() > 0, (s, j)
    d2 = W.decode_inputs(wl, "csa")
    assert torch.equal(d["q"], d2["q"]) and torch.equal(d["kv_pages"], d2["kv_pages"])
    dec = W.decode_inputs(replace(wl, chunk=1), "csa")
    assert dec["q"].shape == (2, 4, 64) and dec["q_idx"].shape == (2, 3, 32)


def test_traffic_record_reads_ncu_csv_and_goes_stale(tmp_path, monkeypatch):
    """A traffic record is the mean DRAM bytes of the matching captured launches (units taken from
    the CSV's unit row), scaled to the workload, and is dropped once the kernel's sources change."""
    raw = tmp_path / "raw.csv"
    raw.write_text('==PROF== log line\n'
                   '"ID","Kernel Name","dram__bytes_read.sum","dram__bytes_write.sum"\n'
                   '"","","Mbyte","Gbyte"\n'
                   '"0","void attention_tc_kernel<0>(...)","500","1.5"\n'
                   '"1","void other_kernel(...)","7","7"\n'
                   '"2","void attention_tc_kernel<0>(...)","1,500","0.5"\n')
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    rec = bench.record_traffic(str(raw), "csa_8k_bf16", "attention", r"attention_tc_kernel",
                               "attention.md", scale=2.0, scaled_from="x2")
    assert rec["launches_captured"] == 2
    assert rec["dram_bytes_per_launch"] == ((0.5e9 + 1.5e9) + (1.5e9 + 0.5e9)) / 2 * 2.0
    t, r = bench.ncu_traffic("csa_8k_bf16", "attention")
    assert t == rec["dram_bytes_per_launch"] and r["scaled_from"] == "x2"
    assert bench.ncu_traffic("csa_8k_bf16", "topk") == (None, None)
    monkeypatch.setattr(bench, "source_hash", lambda k, w="": "changed")
    assert bench.ncu_traffic("csa_8k_bf16", "attention") == (None, None)


def test_traffic_record_reads_the_metrics_launch_list(tmp_path, monkeypatch):
    """The `--metrics ... --csv` launch list (one row per launch and metric) gives the same sums."""
    raw = tmp_path / "list.csv"
    hdr = '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'
    raw.write_text('==PROF== x\n' + hdr +
                   '"0","attention_tc_kernel<0>","dram__bytes_read.sum","Gbyte","2.5"\n'
                   '"0","attention_tc_kernel<0>","dram__bytes_write.sum","Mbyte","500"\n'
                   '"0","attention_tc_kernel<0>","gpu__time_duration.sum","ms","30"\n'
                   '"1","topk_kernel","dram__bytes_read.sum","Gbyte","9"\n')
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    rec = bench.record_traffic(str(raw), "csa_128k_bf16", "attention", r"attention_tc", "x.md")
    assert rec["launches_captured"] == 1 and rec["dram_bytes_per_launch"] == 3.0e9
