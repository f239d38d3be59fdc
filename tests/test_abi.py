"""The C-ABI library loads, exports every entry point include/sac.h declares, and rejects bad
arguments on the host with the documented status codes (no GPU needed: validation runs before any
CUDA call)."""
import ctypes
import os
import re

import pytest

import sparse_attention_compressor_b200 as sac

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sac.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"SAC_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    return sac.load_library()


def test_header_declares_the_abi():
    assert set(declared_symbols()) == set(sac.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert sac.sac_version() == 200


def test_params_struct_layout_matches_header():
    # B,S,H,D,R ints (20) + pad (4) + double (8) + 6 ints (24) + float (4) + pad (4) + int64 (8)
    # + int (4) + pad (4) + double (8) + int (4) + pad (4) + 2 doubles (16)
    assert ctypes.sizeof(sac.sac_params) == 112
    assert sac.sac_params.rope_theta.offset == 24
    assert sac.sac_params.pos0.offset == 64
    assert sac.sac_params.rope_factor.offset == 80
    assert sac.sac_params.yarn_beta_slow.offset == 104


def p_csa(**kw):
    base = dict(B=1, S=8192, H=64, D=512, R=64, rope_theta=160000.0, m=4, win_len=8,
                sliding_window=128, n_idx_heads=64, idx_dim=128, topk=512)
    base.update(kw)
    return sac.make_params(**base)


def test_workspace_sizes():
    p = p_csa()
    n = 8192 // 4
    ws = sac.sac_workspace_size(p, sac.SAC_KIND_CSA)
    # status word + rotated kv + pool + indexer pool + scores + top-k, each 256-byte aligned
    expect = 256 + 8192 * 512 * 2 + n * 512 * 2 + n * 128 * 2 + 8192 * n * 4 + 8192 * 512 * 4
    assert ws == expect
    assert sac.sac_workspace_size(p, sac.SAC_KIND_SWA) == 256 + 8192 * 512 * 2
    assert sac.sac_workspace_size(p_csa(m=128, win_len=128), sac.SAC_KIND_HCA) == \
        256 + 8192 * 512 * 2 + 64 * 512 * 2
    assert sac.sac_workspace_size(p_csa(dtype="f32"), sac.SAC_KIND_SWA) == 256 + 8192 * 512 * 4
    # without a GPU the SM count defaults to 148: 16 sequences -> 8 splits (the cap) of fp32
    # partials, 37 -> 4; from 38 sequences on (fewer than 4 splits) the attention runs unsplit
    part = 16 * 8 * 64 * 512 * 4 + 16 * 8 * 64 * 2 * 4
    assert sac.sac_decode_workspace_size(p_csa(S=65536), sac.SAC_KIND_CSA, 16) == \
        256 + 16 * 16384 * 4 + 16 * 512 * 4 + part
    assert sac.sac_decode_workspace_size(p_csa(), sac.SAC_KIND_HCA, 16) == 256 + part
    assert sac.sac_decode_workspace_size(p_csa(), sac.SAC_KIND_SWA, 37) == \
        256 + 37 * 4 * 64 * 512 * 4 + (37 * 4 * 64 * 2 * 4 + 255) // 256 * 256
    assert sac.sac_decode_workspace_size(p_csa(S=65536), sac.SAC_KIND_CSA, 64) == \
        256 + 64 * 16384 * 4 + 64 * 512 * 4
    assert sac.sac_decode_workspace_size(p_csa(), sac.SAC_KIND_SWA, 38) == 256
    assert sac.sac_decode_workspace_size(p_csa(), sac.SAC_KIND_SWA, 200) == 256
    p32 = sac.make_params(1, 8192, 8, 128, 32, 1e4, sliding_window=16, dtype="f32")
    assert sac.sac_decode_workspace_size(p32, sac.SAC_KIND_SWA, 4) == 256  # CUDA-core path


@pytest.mark.parametrize("bad,code", [
    (dict(D=96), -2), (dict(D=1024), -2), (dict(R=63), -2), (dict(R=66 * 2), -2),
    (dict(dtype="f16"), None), (dict(S=0), -1), (dict(H=0), -1), (dict(sliding_window=0), -1),
    (dict(idx_dim=48), -2), (dict(topk=0), -1), (dict(m=0), -1), (dict(S=4 * (1 << 22) + 4), -2),
    (dict(softmax_scale=-1.0), -1), (dict(rope_theta=0.0), -1),
    (dict(rope_factor=4.0, rope_orig_max_pos=0), -1),
    (dict(rope_factor=4.0, rope_orig_max_pos=4096, yarn_beta_fast=1.0, yarn_beta_slow=32.0), -1),
])
def test_invalid_params_rejected_on_host(bad, code):
    kw = dict(bad)
    if kw.get("dtype") == "f16":
        p = p_csa()
        p.dtype = 7
        code = -2
    else:
        p = p_csa(**kw)
    assert sac.sac_workspace_size(p, sac.SAC_KIND_CSA) == 0
    lib = sac.load_library()
    fake = 1 << 20  # never dereferenced: validation fails first
    rc = lib.csa_forward(ctypes.byref(p), *([fake] * 11), None, None, None, fake, 1 << 40, None)
    assert rc == code
    assert lib.sac_last_error().decode() != ""


def test_null_and_misaligned_pointers_rejected():
    lib = sac.load_library()
    p = p_csa()
    fake = 1 << 20
    args = [fake] * 11
    args[0] = None
    rc = lib.csa_forward(ctypes.byref(p), *args, None, None, None, fake, 1 << 40, None)
    assert rc == -1
    assert "q must not be NULL" in lib.sac_last_error().decode()
    args = [fake] * 11
    args[1] = fake + 2
    rc = lib.csa_forward(ctypes.byref(p), *args, None, None, None, fake, 1 << 40, None)
    assert rc == -1 and "aligned" in lib.sac_last_error().decode()


def test_small_workspace_rejected():
    lib = sac.load_library()
    p = p_csa()
    fake = 1 << 20
    need = sac.sac_workspace_size(p, sac.SAC_KIND_CSA)
    rc = lib.csa_forward(ctypes.byref(p), *([fake] * 11), None, None, None, fake, need - 1, None)
    assert rc == -3 and "workspace" in lib.sac_last_error().decode()
    p2 = sac.make_params(1, 1024, 8, 128, 32, 1e4, sliding_window=16)
    rc = lib.swa_forward(ctypes.byref(p2), fake, fake, fake, fake, None, 0, None)
    assert rc == -3


def test_decode_validation():
    lib = sac.load_library()
    p = p_csa(S=65536, m=128, win_len=128)
    fake = 1 << 20
    # kv block table too short for contexts up to S
    rc = lib.hca_decode(ctypes.byref(p), 4, fake, fake, fake, 10, fake, 64, fake, fake, 8, fake,
                        fake, None, 0, None)
    assert rc == -1 and "block table" in lib.sac_last_error().decode()
    rc = lib.hca_decode(ctypes.byref(p), 0, fake, fake, fake, 1024, fake, 64, fake, fake, 8, fake,
                        fake, None, 0, None)
    assert rc == -1 and "nseq" in lib.sac_last_error().decode()


def test_decode_append_validation():
    lib = sac.load_library()
    fake = 1 << 20
    p = p_csa(S=4096)
    args = dict(kind=sac.SAC_KIND_CSA, nseq=2, ctx=fake, kv_new=fake, k_idx_new=fake,
                cmp_gate=fake, cmp_bias=fake, idx_gate=fake, idx_bias=fake, kv_pages=fake,
                kv_bt=fake, kv_max_pages=64, page_size=64, cmp_state=fake, idx_state=fake,
                pool_pages=fake, idx_pool_pages=fake, pool_bt=fake, pool_max_pages=16)

    def call(**kw):
        a = dict(args, **kw)
        return lib.decode_append(ctypes.byref(p), a["kind"], a["nseq"], a["ctx"], a["kv_new"],
                                 a["k_idx_new"], a["cmp_gate"], a["cmp_bias"], a["idx_gate"],
                                 a["idx_bias"], a["kv_pages"], a["kv_bt"], a["kv_max_pages"],
                                 a["page_size"], a["cmp_state"], a["idx_state"],
                                 a["pool_pages"], a["idx_pool_pages"], a["pool_bt"],
                                 a["pool_max_pages"], None)

    assert call(kind=7) == -1
    assert call(nseq=0) == -1
    assert call(kv_max_pages=63) == -1 and "block table" in lib.sac_last_error().decode()
    assert call(pool_max_pages=15) == -1 and "pool block table" in lib.sac_last_error().decode()
    assert call(idx_state=None) == -1 and "idx_state" in lib.sac_last_error().decode()
    assert call(cmp_state=fake + 8) == -1 and "aligned" in lib.sac_last_error().decode()
    # SWA needs no compressor state
    p_swa = sac.make_params(1, 4096, 64, 512, 64, 1e4, sliding_window=128)
    rc = lib.decode_append(ctypes.byref(p_swa), sac.SAC_KIND_SWA, 2, fake, fake, None, None, None,
                           None, None, fake, fake, 63, 64, None, None, None, None, None, 0, None)
    assert rc == -1 and "block table" in lib.sac_last_error().decode()


def test_oproj_validation_and_workspace():
    lib = sac.load_library()
    fake = 1 << 20
    p = sac.make_params(1, 64, 64, 512, 64, 1e4)
    need = sac.sac_oproj_workspace_size(p, 64, 8, 1024)
    # the status word, then the bf16 mid [64, 8*1024], each 256-byte aligned
    assert need == 256 + 64 * 8 * 1024 * 2
    assert sac.sac_oproj_workspace_size(p, -1, 8, 1024) == 0

    def call(T=64, groups=8, rank=1024, hidden=4096, ws=fake, ws_bytes=need, params=p):
        return lib.o_proj_forward(ctypes.byref(params), T, groups, rank, hidden, fake, fake, fake,
                                  fake, ws, ws_bytes, None)

    assert call(groups=3) == -2
    assert call(rank=1020) == -2
    assert call(hidden=4) == -2
    assert call(ws_bytes=need - 1) == -3
    assert call(ws=fake + 16) == -1 and "256-byte" in lib.sac_last_error().decode()
    p32 = sac.make_params(1, 64, 64, 512, 64, 1e4, dtype="f32")
    assert call(params=p32) == -2
    p_odd = sac.make_params(1, 64, 6, 40, 0, 1e4)  # groups of 3 heads x 40 = 120 features
    assert call(params=p_odd, groups=2, rank=64, hidden=64) == -2
    assert call(T=0) == 0  # nothing to do: no launch, no device touched


def test_chunk_validation_and_workspace():
    lib = sac.load_library()
    fake = 1 << 20
    p = p_csa(S=65536)
    # the decode layout for nseq * n rows: 4 * 16 = 64 rows -> no split; the CSA scores of all
    # 64 rows fit the 1 GiB budget
    assert sac.sac_chunk_workspace_size(p, sac.SAC_KIND_CSA, 4, 16) == \
        sac.sac_decode_workspace_size(p, sac.SAC_KIND_CSA, 64)
    assert sac.sac_chunk_workspace_size(p, sac.SAC_KIND_CSA, 4, 0) == 0
    # 16 Ki rows of 16 Ki entries: scores capped at 1 GiB (16 Ki rows x 64 KiB = 1 GiB exactly)
    big = sac.sac_chunk_workspace_size(p, sac.SAC_KIND_CSA, 8, 4096)
    assert big == 256 + (1 << 30) + 8 * 4096 * 512 * 4
    big2 = sac.sac_chunk_workspace_size(p, sac.SAC_KIND_CSA, 16, 4096)
    assert big2 == 256 + (1 << 30) + 16 * 4096 * 512 * 4
    # n < 1 is rejected before any device work
    rc = lib.swa_prefill_chunk(ctypes.byref(p), 2, 0, fake, fake, fake, 64, fake, 1024, fake,
                               fake, None, 0, None)
    assert rc == -1 and "query rows" in lib.sac_last_error().decode()
    rc = lib.prefill_chunk_append(ctypes.byref(p), sac.SAC_KIND_SWA, 2, 0, fake, fake, None, None,
                                  None, None, None, fake, fake, 64, 1024, None, None, None, None,
                                  None, 0, None)
    assert rc == -1 and "chunk tokens" in lib.sac_last_error().decode()
    rc = lib.hca_prefill_chunk(ctypes.byref(p), 2, 8, fake, fake, fake, 64, fake, 1024, None,
                               fake, 16, fake, fake, None, 0, None)
    assert rc == -1 and "pool_pages" in lib.sac_last_error().decode()
